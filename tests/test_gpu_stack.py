"""The benchmark's timed configuration, checked against the fp64 oracle.

bench.py times a stack of layers as ONE CUDA graph: every product launched
back to back with programmatic dependent launch (a kernel's prologue overlaps
the previous kernel's tail), all products sharing one workspace.  These tests
build a slice of that stack with the same runner (gemm_exl3_gemv_b200.stack),
capture and replay the graph, and compare every output of every product with
the oracle -- so an ordering fault between chained launches (a read of the
workspace or of x before the previous kernel has finished) cannot pass.

They also check the chained stack (a layer's output feeds the next layer) of
the layer-step graph against the oracle composed the same way."""
import numpy as np
import pytest

from gemm_exl3_gemv_b200 import synth
from gpu_helpers import check_close

pytestmark = pytest.mark.gpu


def _stack(m, layers, mode, grouped):
    import torch
    from gemm_exl3_gemv_b200 import exl3 as ex
    from gemm_exl3_gemv_b200.stack import Stack
    specs = [s for s in synth.workload(5, m=32) if s.layer < layers]
    weights = [synth.splitmix64_words_torch(s.stream_id, s.n_words, "cuda") for s in specs]
    st = Stack(ex, torch, torch.device("cuda"), m, specs, weights, mode=mode, grouped=grouped)
    st.run()                                   # the configuring first call, outside the capture
    torch.cuda.synchronize()
    return st


def _replay(st, times=2):
    import torch
    st.y_dev.fill_(float("nan"))
    g = st.capture()
    for _ in range(times):
        g.replay()
    torch.cuda.synchronize()
    from gemm_exl3_gemv_b200 import exl3 as ex
    assert ex.workspace_status(st.ws) == ex.EXL3_OK
    del g


@pytest.mark.parametrize("m", [32, 1])
@pytest.mark.parametrize("grouped", [True, False])
def test_graphed_stack_slice_matches_oracle(oracle_mod, m, grouped):
    st = _stack(m, 2, "sweep", grouped)
    _replay(st)
    for p in st.products:
        inp = synth.make_inputs(p.spec)
        x = inp.x[:m]
        ref = oracle_mod.gemm(x, inp.packed, inp.scale, inp.su, inp.sv, p.spec.k_in, p.spec.n_out, p.spec.bits)
        check_close(p.y.cpu().numpy(), ref, f"{p.spec.name} m={m} grouped={grouped}")


@pytest.mark.parametrize("m", [32, 1])
def test_graphed_end_to_end_matches_oracle(oracle_mod, m):
    """The bench's end-to-end step (inputs copied up from pinned host memory
    in chunks of layers, outputs copied down in chunks, as one CUDA graph):
    the device inputs and outputs are poisoned first, so every host output
    must come from this step's copies and products.  Five layers, so that
    both copy directions include a multi-layer chunk."""
    import torch
    st = _stack(m, 5, "sweep", True)
    assert any(b - a > 1 for a, b in st._copy_chunks())
    g = st.capture(st.run_e2e)
    st.x_dev.fill_(float("nan"))
    st.y_dev.fill_(float("nan"))
    st.y_pin.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    from gemm_exl3_gemv_b200 import exl3 as ex
    assert ex.workspace_status(st.ws) == ex.EXL3_OK
    del g
    for p in st.products:
        inp = synth.make_inputs(p.spec)
        ref = oracle_mod.gemm(inp.x[:m], inp.packed, inp.scale, inp.su, inp.sv, p.spec.k_in, p.spec.n_out, p.spec.bits)
        off = (p.y.data_ptr() - st.y_dev.data_ptr()) // 2
        host = st.y_pin[off:off + m * p.spec.n_out].view(m, p.spec.n_out).numpy()
        check_close(host, ref, f"end-to-end {p.spec.name} m={m}")


def _oracle_chain(oracle_mod, specs, m, layers):
    """The chained step composed from oracle products, with the activations
    rounded to fp16 between products (as the library stores them)."""
    byname = {s.name: s for s in specs}
    inp = {s.name: synth.make_inputs(s, chain=True) for s in specs}
    out = {}
    h = inp["l0.q"].x[:m]
    for l in range(layers):
        q = inp[f"l{l}.q"]
        su = q.su                                           # the sibling call takes q's sign vector
        for kind in ("q", "k", "v", "gate", "up"):
            s, i = byname[f"l{l}.{kind}"], inp[f"l{l}.{kind}"]
            out[s.name] = oracle_mod.gemm(h, i.packed, i.scale, su, i.sv, s.k_in, s.n_out, s.bits)
        for kind, src in (("o", "q"), ("down", "up")):
            s, i = byname[f"l{l}.{kind}"], inp[f"l{l}.{kind}"]
            xin = out[f"l{l}.{src}"].astype(np.float16)
            out[s.name] = oracle_mod.gemm(xin, i.packed, i.scale, i.su, i.sv, s.k_in, s.n_out, s.bits)
        h = out[f"l{l}.down"].astype(np.float16)
    return out


def _chain_depth(spec):
    """Products on the dependency path ending at this one: layer l's sibling
    call (q, k, v, gate, up) is product 2l + 1 of the chain, its o and down
    are product 2l + 2."""
    kind = spec.name.split(".")[1]
    return 2 * spec.layer + (2 if kind in ("o", "down") else 1)


@pytest.mark.parametrize("m", [1, 32])
@pytest.mark.parametrize("grouped", [True, False])
def test_graphed_chain_matches_composed_oracle(oracle_mod, m, grouped):
    """Tolerance: each product meets the per-product bound (rel-L2 1e-3,
    max-abs 1e-2) on its own inputs (the other tests).  In a chain the input
    of product d is the library's fp16 output of product d - 1, which already
    differs from the oracle's; the products are near norm-preserving (scales
    divided by their average gain), so a relative input error passes through
    at about its own size and the errors of the d products on the path add:
    rel-L2 <= d * 1e-3 and max-abs <= d * 1e-2 at depth d."""
    import gpu_helpers
    layers = 2
    st = _stack(m, layers, "chain", grouped)
    assert len(st._calls()) == layers * (2 if grouped else 3)
    _replay(st)
    ref = _oracle_chain(oracle_mod, st.specs, m, layers)
    for p in st.products:
        d = _chain_depth(p.spec)
        got = p.y.cpu().numpy().astype(np.float64)
        r = ref[p.spec.name]
        rel = np.linalg.norm(got - r) / np.linalg.norm(r)
        mx = np.abs(got - r).max()
        assert np.all(np.isfinite(got)), p.spec.name
        assert rel <= d * gpu_helpers.REL_L2, f"chain {p.spec.name} m={m} grouped={grouped} depth {d}: rel-L2 {rel:.3e}"
        assert mx <= d * gpu_helpers.MAX_ABS, f"chain {p.spec.name} m={m} grouped={grouped} depth {d}: max-abs {mx:.3e}"
    # the chain is carried: layer 1's input is layer 0's down output
    assert np.abs(ref["l1.down"]).max() > 0
