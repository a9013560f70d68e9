"""exl3_gemm_grouped (independent problems, each with its own input rows, signs,
weights and shape, in one pass) on the GPU through the C ABI: every member
against the fp64 oracle, against the separate products, and bitwise
repeatability of the grouped call."""
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


def _members(shapes, bits, m, seed):
    specs = [synth.MatrixSpec(f"grp{i}", k, n, bits, m, seed=seed, index=i) for i, (k, n) in enumerate(shapes)]
    return specs, [synth.make_inputs(s) for s in specs]


def _dev_problems(inps, fp32):
    import torch
    probs = []
    for inp in inps:
        s = inp.spec
        rows = inp.x.shape[0]
        y = torch.full((rows, s.n_out), float("nan"), dtype=torch.float32 if fp32 else torch.float16, device="cuda")
        probs.append((to_dev(inp.x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv), y))
    return probs


# member shapes with several k_in (several unit lengths per block) and widths
SHAPES = [(256, 384), (640, 128), (128, 256), (384, 512)]


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("m", [1, 3, 16, 32])
def test_grouped_members_match_oracle(ex, oracle_mod, bits, m):
    specs, inps = _members(SHAPES, bits, m, seed=81 + bits)
    probs = _dev_problems(inps, fp32=True)
    ex.gemm_grouped(probs, bits, fp32=True)
    for spec, inp, p in zip(specs, inps, probs):
        ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, bits)
        check_close(p[5].cpu().numpy(), ref, f"{spec.name} m={m} bits={bits}")


@pytest.mark.parametrize("m", [1, 32])
def test_grouped_single_member_and_eight_members(ex, oracle_mod, m):
    for shapes in ([(512, 256)], [(128 * (1 + i % 3), 128 * (1 + (i * 5) % 4)) for i in range(8)]):
        specs, inps = _members(shapes, 3, m, seed=90 + len(shapes))
        probs = _dev_problems(inps, fp32=True)
        ex.gemm_grouped(probs, 3, fp32=True)
        for spec, inp, p in zip(specs, inps, probs):
            ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, 3)
            check_close(p[5].cpu().numpy(), ref, f"{len(shapes)} members: {spec.name} m={m}")


@pytest.mark.parametrize("m", [1, 32])
def test_grouped_layer_full_outputs(ex, oracle_mod, m):
    """A whole layer of the 64-layer stack (q, k, v, o, gate, up, down) as one
    grouped call, every output of every member against the oracle."""
    specs = [s for s in synth.workload(5, m=32) if s.layer == 1]
    inps = [synth.make_inputs(s) for s in specs]
    for inp in inps:
        inp.x = inp.x[:m]
    probs = _dev_problems(inps, fp32=False)
    ex.gemm_grouped(probs, specs[0].bits)
    for spec, inp, p in zip(specs, inps, probs):
        ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
        check_close(p[5].cpu().numpy(), ref, f"{spec.name} m={m}")


@pytest.mark.parametrize("m", [1, 16, 32])
def test_grouped_repeatable_and_close_to_separate(ex, m):
    import torch
    specs, inps = _members([(5120, 1024), (17408, 512), (1024, 2048)], 3, m, seed=95)
    probs = _dev_problems(inps, fp32=True)
    n = ex.grouped_workspace_bytes(m, [(s.k_in, s.n_out) for s in specs], 3)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    ex.gemm_grouped(probs, 3, fp32=True, workspace=ws)
    first = [p[5].clone() for p in probs]
    for _ in range(5):
        ex.gemm_grouped(probs, 3, fp32=True, workspace=ws)
        for f, p in zip(first, probs):
            assert torch.equal(f, p[5])
    assert ex.workspace_status(ws) == ex.EXL3_OK
    for spec, p, f in zip(specs, probs, first):
        x, packed, scale, su, sv, _ = p
        sep = ex.gemm(x, packed, scale, su, sv, 3, fp32=True).cpu().numpy().astype(np.float64)
        check_close(f.cpu().numpy(), sep, f"grouped vs separate {spec.name}")


def test_grouped_rejects_bad_groups(ex):
    import ctypes
    import torch
    buf = torch.zeros(1 << 16, dtype=torch.float16, device="cuda")
    P = ex.Problem
    good = P(buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), 128, 128)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call(arr, n, m=1, bits=3, ws_bytes=1 << 20):
        return ex.lib.exl3_gemm_grouped(m, arr, n, 0, bits, ctypes.c_void_p(ws.data_ptr()), ws_bytes, stream)

    arr9 = (P * 9)(*([good] * 9))
    assert call(arr9, 9) == ex.EXL3_ERR_UNSUPPORTED                    # more than 8 members
    assert call(arr9, 0) == ex.EXL3_ERR_INVALID_ARG
    assert call(arr9, 2, m=33) == ex.EXL3_ERR_UNSUPPORTED
    assert call(arr9, 2, bits=5) == ex.EXL3_ERR_UNSUPPORTED
    bad = (P * 2)(good, P(buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(),
                          buf.data_ptr(), 130, 128))
    assert call(bad, 2) == ex.EXL3_ERR_UNSUPPORTED                     # k_in not a multiple of 128
    nul = (P * 2)(good, P(None, buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(),
                          128, 128))
    assert call(nul, 2) == ex.EXL3_ERR_INVALID_ARG
    mis = (P * 2)(good, P(buf.data_ptr() + 2, buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(),
                          buf.data_ptr(), 128, 128))
    assert call(mis, 2) == ex.EXL3_ERR_MISALIGNED
    assert call((P * 2)(good, good), 2, ws_bytes=16) == ex.EXL3_ERR_WORKSPACE
