"""exl3_gemm_siblings (one pass over a group of matrices that share the input,
the sibling fusion of the MLP / attention projections) on the GPU, against
the fp64 oracle and against the separate products, through the C ABI."""
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


def _group(n_outs, k, bits, seed, m):
    """Matrices of a group: own packed words, scales and sv; x and su of member 0."""
    specs = [synth.MatrixSpec(f"sib{i}", k, n, bits, m, seed=seed, index=i) for i, n in enumerate(n_outs)]
    inps = [synth.make_inputs(s) for s in specs]
    return specs, inps


def _blocks(n_out):
    nb = n_out // 128
    return sorted({0, nb // 2, nb - 1})


@pytest.mark.parametrize("m", [1, 3, 16, 32])
def test_small_group_full_oracle(ex, oracle_mod, m):
    specs, inps = _group([128, 384, 256], 256, 3, 61, 32)
    x, su = inps[0].x[:m], inps[0].su
    mats = [(to_dev(i.packed), to_dev(i.scale), to_dev(i.sv)) for i in inps]
    ys = ex.gemm_siblings(to_dev(x), to_dev(su), mats, 3, fp32=True)
    for s, i, y in zip(specs, inps, ys):
        ref = oracle_mod.gemm(x, i.packed, i.scale, su, i.sv, s.k_in, s.n_out, s.bits)
        check_close(y.cpu().numpy(), ref, f"{s.name} m={m}")


@pytest.mark.parametrize("m", [1, 8, 32])
@pytest.mark.parametrize("group", ["gate_up", "qkv"])
def test_projection_groups_sampled(ex, oracle_mod, m, group):
    n_outs = [17408, 17408] if group == "gate_up" else [5120, 1024, 1024]
    bits = 4 if group == "gate_up" else 3
    specs, inps = _group(n_outs, 5120, bits, 62, 32)
    x, su = inps[0].x[:m], inps[0].su
    mats = [(to_dev(i.packed), to_dev(i.scale), to_dev(i.sv)) for i in inps]
    ys = ex.gemm_siblings(to_dev(x), to_dev(su), mats, bits, fp32=False)
    for s, i, y in zip(specs, inps, ys):
        blocks = _blocks(s.n_out)
        ref = oracle_mod.gemm_sampled(x, i.packed, i.scale, su, i.sv, s.k_in, s.n_out, s.bits, blocks)
        yv = y.cpu().numpy().astype(np.float64)
        got = np.concatenate([yv[:, 128 * b:128 * (b + 1)] for b in blocks], axis=1)
        check_close(got, ref, f"{group}/{s.name} m={m}")
        # and against the separate product of that matrix
        sep = ex.gemm(to_dev(x), mats[specs.index(s)][0], mats[specs.index(s)][1], to_dev(su),
                      mats[specs.index(s)][2], bits, fp32=False).cpu().numpy().astype(np.float64)
        check_close(yv, sep, f"{group}/{s.name} m={m} vs separate")


@pytest.mark.parametrize("m", [1, 32])
def test_group_repeatable_bitwise(ex, m):
    import torch
    specs, inps = _group([5120, 1024, 1024], 5120, 2, 63, m)
    x, su = to_dev(inps[0].x), to_dev(inps[0].su)
    mats = [(to_dev(i.packed), to_dev(i.scale), to_dev(i.sv)) for i in inps]
    ws = ex.alloc_workspace(m, 5120, 7168, 2)
    first = [y.clone() for y in ex.gemm_siblings(x, su, mats, 2, workspace=ws)]
    for _ in range(3):
        for a, b in zip(ex.gemm_siblings(x, su, mats, 2, workspace=ws), first):
            assert torch.equal(a, b)
    assert ex.workspace_status(ws) == ex.EXL3_OK
