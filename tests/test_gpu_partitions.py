"""GPU parity on shapes that drive the work partitions of both product
kernels into their corner cases, against the fp64 oracle:

* many output blocks per CTA (n_out = 65536: 512 blocks, more than one wave
  of CTAs holds) -- the M = 1 kernel's stream-K cut and the verify kernel's
  multi-segment stream-K path, whose CTAs span several output blocks;
* one output block and a deep input (17408 -> 128) -- every CTA shares the
  single block: many partial sums (M = 1) or one cluster reducing through
  distributed shared memory (verify kernel);
* bitwise repeatability on both."""
import numpy as np
import pytest

from gemm_exl3_gemv_b200 import synth
from gpu_helpers import check_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ex():
    import torch
    assert torch.cuda.is_available()
    from gemm_exl3_gemv_b200 import exl3
    return exl3


def _run(ex, inp, m, fp32=True):
    y = ex.gemm(to_dev(inp.x[:m]), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv),
                inp.spec.bits, fp32=fp32)
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("m", [1, 5, 32])
def test_wide_output_many_blocks_per_cta(ex, oracle_mod, m):
    spec = synth.MatrixSpec("wide", 256, 65536, 2, 32, seed=51)
    inp = synth.make_inputs(spec)
    blocks = [0, 1, 255, 256, 511]
    ref = oracle_mod.gemm_sampled(inp.x[:m], inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out,
                                  spec.bits, blocks)
    y = _run(ex, inp, m)
    got = np.concatenate([y[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1)
    check_close(got, ref, f"wide m={m}")


@pytest.mark.parametrize("m", [1, 2, 17, 32])
@pytest.mark.parametrize("bits", [3, 4])
def test_deep_input_single_block(ex, oracle_mod, m, bits):
    spec = synth.MatrixSpec("deep", 17408, 128, bits, 32, seed=52, index=bits)
    inp = synth.make_inputs(spec)
    ref = oracle_mod.gemm(inp.x[:m], inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
    check_close(_run(ex, inp, m, fp32=False), ref, f"deep m={m} bits={bits}")


@pytest.mark.parametrize("k,n", [(256, 65536), (17408, 128)])
@pytest.mark.parametrize("m", [1, 32])
def test_partitions_repeatable_bitwise(ex, k, n, m):
    import torch
    spec = synth.MatrixSpec("rep", k, n, 3, m, seed=53)
    inp = synth.make_inputs(spec)
    args = [to_dev(a) for a in (inp.x, inp.packed, inp.scale, inp.su, inp.sv)]
    ws = ex.alloc_workspace(m, k, n, 3)
    first = ex.gemm(*args, 3, workspace=ws).clone()
    for _ in range(4):
        assert torch.equal(ex.gemm(*args, 3, workspace=ws), first)
    assert ex.workspace_status(ws) == ex.EXL3_OK


@pytest.mark.parametrize("m", [1, 8, 32])
def test_shared_workspace_across_widths(m):
    """Calls of different output widths (and the grouped call) back to back on
    one workspace, sized for the largest: every output equals the same call on
    a fresh workspace, bit for bit.  (A call's partial sums or rotated input
    must never land on another call's arrival counters.)"""
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    shapes = [(5120, 1024), (5120, 17408), (17408, 5120), (5120, 1024), (256, 40960), (5120, 17408)]
    specs = [synth.MatrixSpec(f"sw{i}", k, n, 2, m, seed=150, index=i) for i, (k, n) in enumerate(shapes)]
    inps = [synth.make_inputs(s) for s in specs]
    dev = [[to_dev(a) for a in (i.x, i.packed, i.scale, i.su, i.sv)] for i in inps]
    fresh = [ex.gemm(*d, 2).clone() for d in dev]
    ws = torch.zeros(max(ex.workspace_bytes(m, k, n, 2) for k, n in shapes), dtype=torch.uint8, device="cuda")
    for rep in range(2):
        outs = [ex.gemm(*d, 2, workspace=ws) .clone() for d in dev]
        torch.cuda.synchronize()
        for s, f, o in zip(specs, fresh, outs):
            assert torch.equal(f, o), f"{s.name} m={m} pass {rep}"
    assert ex.workspace_status(ws) == ex.EXL3_OK
