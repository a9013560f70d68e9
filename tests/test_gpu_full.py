"""Every output of one full-size product per kernel path against the fp64
oracle: the MLP gate projection 5120 -> 17408 (136 output blocks, every
stream-K segment boundary and cluster rank of the full-size cut) through the
single-row GEMV, the 32-row tensor-core verify kernel, a 16-row verify batch,
and the many-row (prefill) GEMM."""
import pytest

from gemm_exl3_gemv_b200 import synth
from gpu_helpers import check_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gate():
    spec = synth.MatrixSpec("gate_full", 5120, 17408, 3, 256, seed=2, index=7)
    return spec, synth.make_inputs(spec)


@pytest.mark.parametrize("m", [1, 16, 32])
def test_full_size_gate_every_output(oracle_mod, gate, m):
    from gemm_exl3_gemv_b200 import exl3 as ex
    spec, inp = gate
    x = inp.x[:m]
    y = ex.gemm(to_dev(x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv), spec.bits)
    ref = oracle_mod.gemm(x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
    check_close(y.cpu().numpy(), ref, f"gate m={m}")


def test_full_size_gate_many_rows_every_output(oracle_mod, gate):
    from gemm_exl3_gemv_b200 import exl3 as ex
    spec, inp = gate
    x = inp.x[:256]
    y = ex.gemm_large(to_dev(x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv),
                      spec.bits)
    ref = oracle_mod.gemm(x, inp.packed, inp.scale, inp.su, inp.sv, spec.k_in, spec.n_out, spec.bits)
    check_close(y.cpu().numpy(), ref, "gate m=256 (many-row path)")
