"""Run by tests/test_gpu_debug_bounds.py in a fresh process whose binding
loads the debug-bounds build (EXL3_LIBRARY=.../libexl3_debug.so): small
in-range calls of every product path, each checked against the fp64 oracle,
and every workspace status word checked clean (no index check failed)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import torch  # noqa: E402

import oracle  # noqa: E402
from gemm_exl3_gemv_b200 import exl3 as ex  # noqa: E402
from gemm_exl3_gemv_b200 import synth  # noqa: E402
from gpu_helpers import check_close, to_dev  # noqa: E402


def main():
    assert ex.LIB_PATH.endswith("libexl3_debug.so"), ex.LIB_PATH
    oracle.build()
    n = 0
    for m, k, n_out, bits in [(1, 640, 384, 3), (1, 256, 256, 2), (8, 384, 512, 4), (32, 640, 256, 3),
                              (16, 5120, 1024, 2)]:
        spec = synth.MatrixSpec("dbg", k, n_out, bits, m, seed=120 + m)
        inp = synth.make_inputs(spec)
        ws = ex.alloc_workspace(m, k, n_out, bits)
        y = ex.gemm(to_dev(inp.x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv), bits,
                    fp32=True, workspace=ws)
        assert ex.workspace_status(ws) == ex.EXL3_OK, (m, k, n_out, bits)
        check_close(y.cpu().numpy(), oracle.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n_out, bits),
                    f"debug m={m}")
        n += 1
    for m in (1, 8):
        specs = [synth.MatrixSpec(f"dg{i}", kk, nn, 3, m, seed=130, index=i)
                 for i, (kk, nn) in enumerate([(256, 384), (640, 128), (128, 256)])]
        inps = [synth.make_inputs(s) for s in specs]
        probs = [(to_dev(i.x), to_dev(i.packed), to_dev(i.scale), to_dev(i.su), to_dev(i.sv),
                  torch.empty((m, s.n_out), dtype=torch.float32, device="cuda")) for s, i in zip(specs, inps)]
        wsb = ex.grouped_workspace_bytes(m, [(s.k_in, s.n_out) for s in specs], 3)
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
        ex.gemm_grouped(probs, 3, fp32=True, workspace=ws)
        assert ex.workspace_status(ws) == ex.EXL3_OK
        for s, i, p in zip(specs, inps, probs):
            check_close(p[5].cpu().numpy(), oracle.gemm(i.x, i.packed, i.scale, i.su, i.sv, s.k_in, s.n_out, 3),
                        f"debug grouped m={m}")
        n += 1
    spec = synth.MatrixSpec("dbgl", 256, 384, 3, 160, seed=140)
    inp = synth.make_inputs(spec)
    wsb = int(ex.lib.exl3_large_m_workspace_bytes(160, 256, 384, 3))
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    y = ex.gemm_large(to_dev(inp.x), to_dev(inp.packed), to_dev(inp.scale), to_dev(inp.su), to_dev(inp.sv), 3,
                      fp32=True, workspace=ws)
    assert ex.workspace_status(ws) == ex.EXL3_OK
    check_close(y.cpu().numpy(), oracle.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, 256, 384, 3),
                "debug many rows")
    n += 1
    torch.cuda.synchronize()
    print(f"debug-bounds cases ok: {n}")


if __name__ == "__main__":
    main()
