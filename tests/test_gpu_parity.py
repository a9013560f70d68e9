"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on
the same seeded inputs.  Decode is bit-exact; products within rel-L2 1e-3 and
max-abs 1e-2 per matrix and per row."""
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


# ------------------------------------------------------------------ decode ---

@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("k,n", [(16, 16), (32, 48), (128, 128), (256, 384), (144, 80)])
def test_decode_tiles_bit_exact_small(ex, oracle_mod, bits, k, n):
    spec = synth.MatrixSpec("d", k, n, bits, 1, seed=21, index=bits)
    packed = synth.splitmix64_words_np(spec.stream_id, 0, spec.n_words)
    ref = oracle_mod.decode_tiles(packed, k, n, bits)
    got = ex.decode_tiles(to_dev(packed), k, n, bits).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("cfg", [1, 2])
def test_decode_tiles_bit_exact_workloads(ex, oracle_mod, cfg):
    for spec in synth.workload(cfg):
        packed = synth.splitmix64_words_np(spec.stream_id, 0, spec.n_words)
        ref = oracle_mod.decode_tiles(packed, spec.k_in, spec.n_out, spec.bits)
        got = ex.decode_tiles(to_dev(packed), spec.k_in, spec.n_out, spec.bits).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, ref), spec.name


def test_decode_tiles_full_size_mlp_bit_exact(ex, oracle_mod):
    spec = synth.workload(3)[2]           # down projection 17408 -> 5120, 4 bits
    packed = synth.splitmix64_words_np(spec.stream_id, 0, spec.n_words)
    ref = oracle_mod.decode_tiles(packed, spec.k_in, spec.n_out, spec.bits)
    got = ex.decode_tiles(to_dev(packed), spec.k_in, spec.n_out, spec.bits).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_decode_handles_all_ones_and_zero_streams(ex, oracle_mod):
    for fill in (0, 0xFFFFFFFF):
        packed = np.full(4 * 4 * 8 * 3, fill, dtype=np.uint32)
        ref = oracle_mod.decode_tiles(packed, 64, 64, 3)
        got = ex.decode_tiles(to_dev(packed), 64, 64, 3).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, ref)


# ---------------------------------------------------------------- Hadamard ---

@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("rows,n", [(1, 128), (3, 384), (32, 5120)])
def test_hadamard128_matches_oracle(ex, oracle_mod, mode, rows, n):
    rng = np.random.default_rng(rows * 1000 + n + mode)
    x = rng.standard_normal((rows, n)).astype(np.float16)
    s = np.where(rng.integers(0, 2, n) == 0, 1.0, -1.0).astype(np.float16)
    ref = oracle_mod.hadamard128(x, s, mode)
    got = ex.hadamard128(to_dev(x), to_dev(s), mode).cpu().numpy().astype(np.float64)
    # fp32 arithmetic, one fp16 rounding: within one fp16 ulp of the exact value
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(got - ref) <= ulp + 1e-7)


def test_hadamard128_in_place(ex):
    import torch
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 256)).astype(np.float16)
    s = np.where(rng.integers(0, 2, 256) == 0, 1.0, -1.0).astype(np.float16)
    t = to_dev(x)
    ref = ex.hadamard128(t.clone(), to_dev(s), 0)
    ex.hadamard128(t, to_dev(s), 0, out=t)
    torch.cuda.synchronize()
    assert torch.equal(t, ref)


# ---------------------------------------------------------------- products ---

def _run(ex, inp, m=None, fp32=True, ws=None):
    x = inp.x if m is None else inp.x[:m]
    y = ex.gemm(to_dev(x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv),
                inp.spec.bits, fp32=fp32, workspace=ws)
    return y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 8, 16, 17, 32])
@pytest.mark.parametrize("k,n", [(128, 128), (256, 384), (640, 256)])
def test_gemm_small_shapes(ex, oracle_mod, bits, m, k, n):
    spec = synth.MatrixSpec("g", k, n, bits, m, seed=31, layer=m, index=bits)
    inp = synth.make_inputs(spec)
    ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits)
    check_close(_run(ex, inp), ref, f"m={m} k={k} n={n} bits={bits}")


def test_gemm_fp16_output(ex, oracle_mod):
    spec = synth.MatrixSpec("h", 512, 512, 3, 4, seed=32)
    inp = synth.make_inputs(spec)
    ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, 512, 512, 3)
    check_close(_run(ex, inp, fp32=False), ref, "fp16 out")


def test_workload1_exact_oracle(ex, oracle_mod):
    (spec,) = synth.workload(1)
    inp = synth.make_inputs(spec)
    ref = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
    check_close(_run(ex, inp, fp32=False), ref, "workload 1")


def _sampled(ex, oracle_mod, spec, m, blocks):
    inp = synth.make_inputs(spec)
    x = inp.x[:m]
    ref = oracle_mod.gemm_sampled(x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out,
                                  spec.bits, blocks)
    y = _run(ex, inp, m=m, fp32=False)
    got = np.concatenate([y[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1)
    check_close(got, ref, f"{spec.name} m={m}")


def _blocks(n_out):
    nb = n_out // 128
    return sorted({0, 1, nb // 2, nb - 1})


def test_workload2_full_size(ex, oracle_mod):
    (spec,) = synth.workload(2)
    _sampled(ex, oracle_mod, spec, 1, _blocks(spec.n_out))


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_workload3_full_size(ex, oracle_mod, idx):
    spec = synth.workload(3)[idx]
    _sampled(ex, oracle_mod, spec, 1, _blocks(spec.n_out))


@pytest.mark.parametrize("m", [8, 16])
@pytest.mark.parametrize("idx", [0, 2])
def test_workload4_full_size(ex, oracle_mod, m, idx):
    spec = synth.workload(4)[idx]
    _sampled(ex, oracle_mod, spec, m, _blocks(spec.n_out))


@pytest.mark.parametrize("layer", [0, 63])
@pytest.mark.parametrize("m", [1, 32])
def test_workload5_layers(ex, oracle_mod, layer, m):
    specs = [s for s in synth.workload(5) if s.layer == layer]
    for spec in specs:
        _sampled(ex, oracle_mod, spec, m, _blocks(spec.n_out)[:2])


# ------------------------------------------------------------ determinism ---

@pytest.mark.parametrize("m", [1, 16, 32])
def test_repeatable_bitwise(ex, m):
    import torch
    spec = synth.MatrixSpec("r", 5120, 1024, 3, m, seed=41)
    inp = synth.make_inputs(spec)
    args = [to_dev(a) for a in (inp.x, inp.packed, inp.scale, inp.su, inp.sv)]
    ws = ex.alloc_workspace(m, 5120, 1024, 3)
    first = ex.gemm(*args, 3, workspace=ws).clone()
    for _ in range(9):
        y = ex.gemm(*args, 3, workspace=ws)
        assert torch.equal(y, first)
    assert ex.workspace_status(ws) == ex.EXL3_OK


def test_misaligned_device_pointer_rejected(ex):
    import torch
    spec = synth.MatrixSpec("a", 256, 256, 3, 1, seed=42)
    inp = synth.make_inputs(spec)
    xb = torch.zeros(256 + 8, dtype=torch.float16, device="cuda")
    with pytest.raises(ex.Exl3Error) as e:
        ex.gemm(xb[1:257], to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv), 3)
    assert e.value.status == ex.EXL3_ERR_MISALIGNED
