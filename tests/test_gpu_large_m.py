"""exl3_gemm_large_m (the many-row path: decode once into the tensor-core
operand image, then a tcgen05 GEMM) against the fp64 oracle, against the
verify path at 32 rows, and for bitwise repeatability, through the C ABI."""
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


def _args(inp, m):
    return (to_dev(inp.x[:m]), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv))


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("m", [1, 33, 100, 256, 300])
@pytest.mark.parametrize("k,n", [(128, 128), (640, 384)])
def test_small_shapes_full_oracle(ex, oracle_mod, bits, m, k, n):
    spec = synth.MatrixSpec("lg", k, n, bits, 300, seed=81, layer=m, index=bits)
    inp = synth.make_inputs(spec)
    ref = oracle_mod.gemm(inp.x[:m], inp.packed, inp.scale, inp.su, inp.sv, k, n, bits)
    y = ex.gemm_large(*_args(inp, m), bits, fp32=True)
    check_close(y.cpu().numpy(), ref, f"m={m} k={k} n={n} bits={bits}")


@pytest.mark.parametrize("m,n", [(512, 5120), (256, 17408)])
def test_model_shapes_sampled(ex, oracle_mod, m, n):
    spec = synth.MatrixSpec("lgw", 5120, n, 3, m, seed=82)
    inp = synth.make_inputs(spec)
    blocks = sorted({0, n // 256, n // 128 - 1})
    rows = [0, m // 2, m - 1]
    ref = oracle_mod.gemm_sampled(inp.x[rows], inp.packed, inp.scale, inp.su, inp.sv, 5120, n, 3, blocks)
    y = ex.gemm_large(*_args(inp, m), 3, fp32=False).cpu().numpy().astype(np.float64)[rows]
    got = np.concatenate([y[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1)
    check_close(got, ref, f"m={m} n={n}")


@pytest.mark.parametrize("m,k,n,bits", [
    (1100, 256, 17408, 3),      # 680 tiles of 256 rows on 148 persistent CTAs; row-tile-fastest order
    (8192, 256, 1024, 2),       # 256 tiles; output-block-fastest order
])
def test_persistent_multi_tile_sampled(ex, oracle_mod, m, k, n, bits):
    """Several tiles per persistent CTA: both tensor-memory accumulators in
    turn, the ring running on across tiles, and each tile order."""
    spec = synth.MatrixSpec("lgp", k, n, bits, m, seed=85)
    inp = synth.make_inputs(spec)
    G = n // 128
    blocks = sorted({0, 1, G // 2, G - 1})
    rows = sorted({0, 255, 256, m // 2, m - 257, m - 1})
    ref = oracle_mod.gemm_sampled(inp.x[rows], inp.packed, inp.scale, inp.su, inp.sv, k, n, bits, blocks)
    y = ex.gemm_large(*_args(inp, m), bits, fp32=True).cpu().numpy().astype(np.float64)[rows]
    got = np.concatenate([y[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1)
    check_close(got, ref, f"m={m} k={k} n={n}")


def test_agrees_with_verify_path_at_32_rows(ex):
    spec = synth.MatrixSpec("lgv", 5120, 1024, 4, 32, seed=83)
    inp = synth.make_inputs(spec)
    a = _args(inp, 32)
    y_large = ex.gemm_large(*a, 4, fp32=True).cpu().numpy().astype(np.float64)
    y_small = ex.gemm(*a, 4, fp32=True).cpu().numpy().astype(np.float64)
    check_close(y_large, y_small, "large vs verify path")


def test_repeatable_bitwise(ex):
    import torch
    spec = synth.MatrixSpec("lgr", 1024, 2048, 2, 200, seed=84)
    inp = synth.make_inputs(spec)
    a = _args(inp, 200)
    n = ex.lib.exl3_large_m_workspace_bytes(200, 1024, 2048, 2)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    first = ex.gemm_large(*a, 2, workspace=ws).clone()
    for _ in range(3):
        assert torch.equal(ex.gemm_large(*a, 2, workspace=ws), first)
    assert ex.workspace_status(ws) == ex.EXL3_OK
