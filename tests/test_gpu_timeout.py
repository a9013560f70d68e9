"""Failure detection without a GPU fault: the multi-row kernels' bounded waits
(the verify kernel and the many-row GEMM).
The test withholds the rotated input through the workspace's injection word
(a flag that nothing sets then), so every wait for it runs out after its 2 s
limit; the kernel winds down and the host reads EXL3_ERR_TIMEOUT from the
workspace status word.  The context stays usable: a normal call afterwards on
the same workspace is correct."""
import numpy as np
import pytest

from gemm_exl3_gemv_b200 import synth
from gpu_helpers import check_close, to_dev

pytestmark = pytest.mark.gpu


# (k, n, v): v = 1 withholds every rotated-input copy; v > 1 lets each CTA's
# first v - 1 through, so the CTAs with more units have MMAs issued (possibly
# still in flight) when their wait for the next runs out.  K_in a multiple of
# 256 takes 256-row units (two tile rows per warp), other K_in 128-row units.
@pytest.mark.parametrize("k,n,v", [(640, 256, 1),        # 128-row units, cluster cut, nothing issued
                                   (256, 65536, 1),      # 256-row units, stream-K cut, nothing issued
                                   (5120, 256, 2),       # 256-row units, cluster cut, 2 units per CTA
                                   (5248, 256, 3),       # 128-row units, 4-5 units per CTA
                                   (512, 65536, 3),      # 256-row units, stream-K cut, 3-4 units per CTA
                                   (384, 65536, 3)])     # 128-row units, stream-K cut, 5-6 units per CTA
def test_withheld_input_times_out_and_reports(oracle_mod, k, n, v):
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    m, bits = 8, 3
    spec = synth.MatrixSpec("to", k, n, bits, m, seed=71)
    inp = synth.make_inputs(spec)
    args = [to_dev(a) for a in (inp.x, inp.packed, inp.scale, inp.su, inp.sv)]
    ws = ex.alloc_workspace(m, k, n, bits)
    ws[4:8] = torch.tensor([v, 0, 0, 0], dtype=torch.uint8)   # inject: withhold the rotated input
    ex.gemm(*args, bits, fp32=True, workspace=ws)
    assert ex.workspace_status(ws) == ex.EXL3_ERR_TIMEOUT
    ws[4:8] = 0
    y = ex.gemm(*args, bits, fp32=True, workspace=ws)
    assert ex.workspace_status(ws) == ex.EXL3_OK
    blocks = [0, n // 128 - 1]
    ref = oracle_mod.gemm_sampled(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits, blocks)
    yv = y.cpu().numpy().astype(np.float64)
    check_close(np.concatenate([yv[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1), ref, "after timeout")


def test_many_row_withheld_operands_time_out_and_report(oracle_mod):
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    m, k, n, bits = 160, 256, 384, 3
    spec = synth.MatrixSpec("tl", k, n, bits, m, seed=73)
    inp = synth.make_inputs(spec)
    args = [to_dev(a) for a in (inp.x, inp.packed, inp.scale, inp.su, inp.sv)]
    ws = torch.zeros(int(ex.lib.exl3_large_m_workspace_bytes(m, k, n, bits)), dtype=torch.uint8, device="cuda")
    ws[4:8] = 1                                   # inject: the GEMM's producer issues no copy
    ex.gemm_large(*args, bits, fp32=True, workspace=ws)
    assert ex.workspace_status(ws) == ex.EXL3_ERR_TIMEOUT
    ws[4:8] = 0
    y = ex.gemm_large(*args, bits, fp32=True, workspace=ws)
    assert ex.workspace_status(ws) == ex.EXL3_OK
    ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits)
    check_close(y.cpu().numpy().astype(np.float64), ref, "many rows after timeout")
