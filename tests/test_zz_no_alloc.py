"""exl3_gemv_noalloc: the single-row product for callers that cannot allocate
device memory (no workspace argument; the library's own fixed scratch array
is used instead).  Checked through the C ABI against the fp64 oracle and
against exl3_gemv with a caller-allocated workspace (bitwise: the same
kernel and split), on two calls in a row (the scratch array keeps the
previous call's contents, so the second call checks that the entry point
clears what must start at zero).  Kept in a file of its own that pytest
collects last."""
import ctypes

import numpy as np
import pytest

from gemm_exl3_gemv_b200 import synth
from gpu_helpers import check_close, to_dev

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _noalloc(ex, x, packed, scale, su, sv, y, k, n, bits):
    import torch
    st = ex.lib.exl3_gemv_noalloc(P(x.data_ptr()), P(packed.data_ptr()), P(scale.data_ptr()),
                                  P(su.data_ptr()), P(sv.data_ptr()), P(y.data_ptr()), 1, k, n, bits,
                                  P(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("idx", [0, 1])
def test_noalloc_matches_oracle_and_workspace_gemv_twice(oracle_mod, idx):
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    spec = [synth.workload(2)[0], synth.workload(3)[2]][idx]          # o_proj 5120x5120; down 17408x5120
    inp = synth.make_inputs(spec)
    x, packed, scale, su, sv = (to_dev(a) for a in (inp.x[0], inp.packed, inp.scale, inp.su, inp.sv))
    ws_y = ex.gemm(x, packed, scale, su, sv, spec.bits, fp32=True).cpu().numpy()
    ref = oracle_mod.gemm(inp.x[:1], inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)[0]
    for call in range(2):
        y = torch.full((spec.n_out,), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc(ex, x, packed, scale, su, sv, y, spec.k_in, spec.n_out, spec.bits)
        assert st == ex.EXL3_OK, ex.lib.exl3_status_string(st)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        check_close(got, ref, f"noalloc call {call} vs oracle")
        assert np.array_equal(got, ws_y), f"noalloc call {call}: differs from exl3_gemv with a workspace"


def test_noalloc_rejects_problem_beyond_scratch():
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    # 8192 output blocks (the most one call takes): the partial sums alone
    # need more than the 4 MiB scratch.  The host check (the same workspace
    # size, host-only) must hold before the call, which then returns before
    # anything is enqueued, so small stand-in buffers are enough.
    k, n, bits = 128, 1 << 20, 2
    assert ex.workspace_bytes(1, k, n, bits) > 4 << 20
    buf = torch.zeros(64, dtype=torch.float16, device="cuda")
    assert _noalloc(ex, buf, buf, buf, buf, buf, buf, k, n, bits) == ex.EXL3_ERR_WORKSPACE
