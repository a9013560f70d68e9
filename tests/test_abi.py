"""Host-side checks of the C ABI (no GPU): the library loads, exports every
entry point include/exl3.h declares, and rejects invalid arguments with the
documented status codes before touching CUDA.  Only invalid calls are made
here, so nothing is ever launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ex():
    from gemm_exl3_gemv_b200 import build
    build.build()
    from gemm_exl3_gemv_b200 import exl3
    return exl3


def declared_entry_points():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"EXL3_API\s+[\w\s\*]*?\b(exl3_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(ex):
    names = declared_entry_points()
    assert len(names) >= 9
    for n in names:
        assert hasattr(ex.lib, n), n
    assert set(names) == set(ex.EXPORTS)


def test_debug_bounds_build_exports_the_same_symbols(ex):
    from gemm_exl3_gemv_b200 import build
    dbg = ctypes.CDLL(build.LIB_DEBUG)
    for n in declared_entry_points():
        assert hasattr(dbg, n), n
    dbg.exl3_status_string.restype = ctypes.c_char_p
    assert b"EXL3_ERR_BOUNDS" in dbg.exl3_status_string(ex.EXL3_ERR_BOUNDS)


def test_grouped_validation(ex):
    P = ex.Problem
    # size query: shapes only, pointers may be NULL
    two = (P * 2)(P(None, None, None, None, None, None, 5120, 1024), P(None, None, None, None, None, None, 17408, 5120))
    assert ex.lib.exl3_grouped_workspace_bytes(1, two, 2, 3) > 0
    assert ex.lib.exl3_grouped_workspace_bytes(32, two, 2, 3) > ex.lib.exl3_grouped_workspace_bytes(1, two, 2, 3)
    assert ex.lib.exl3_grouped_workspace_bytes(33, two, 2, 3) == 0
    assert ex.lib.exl3_grouped_workspace_bytes(1, two, 9, 3) == 0
    bad = (P * 1)(P(None, None, None, None, None, None, 130, 128))
    assert ex.lib.exl3_grouped_workspace_bytes(1, bad, 1, 3) == 0
    # the call itself: NULL pointers are rejected before anything runs
    st = ex.lib.exl3_gemm_grouped(1, two, 2, 0, 3, None, 0, None)
    assert st == ex.EXL3_ERR_INVALID_ARG
    assert ex.lib.exl3_gemm_grouped(1, two, 0, 0, 3, None, 0, None) == ex.EXL3_ERR_INVALID_ARG
    assert ex.lib.exl3_gemm_grouped(1, two, 2, 0, 5, None, 0, None) == ex.EXL3_ERR_UNSUPPORTED


def test_grouped_workspace_covers_separate_products(ex):
    """The grouped workspace holds at least the largest member's own needs."""
    P = ex.Problem
    shapes = [(5120, 5120), (5120, 1024), (5120, 1024), (5120, 5120), (5120, 17408), (5120, 17408), (17408, 5120)]
    arr = (P * 7)(*[P(None, None, None, None, None, None, k, n) for k, n in shapes])
    for m in (1, 8, 32):
        g = ex.lib.exl3_grouped_workspace_bytes(m, arr, 7, 3)
        assert g >= max(ex.workspace_bytes(m, k, n, 3) for k, n in shapes) // 2
        assert g % 16 == 0


def test_version_and_status_strings(ex):
    assert ex.lib.exl3_version() >= 100
    for st in range(8):
        s = ex.lib.exl3_status_string(st).decode()
        assert s.startswith("EXL3")
    assert "unknown" in ex.lib.exl3_status_string(99).decode()


def test_workspace_bytes(ex):
    assert ex.workspace_bytes(1, 5120, 5120, 3) > 0
    assert ex.workspace_bytes(32, 17408, 5120, 2) >= 32 * 5120 * 4
    for bad in [(0, 256, 256, 3), (33, 256, 256, 3), (1, 200, 256, 3), (1, 256, 100, 3),
                (1, 256, 256, 5), (1, 256, 256, 1), (1, -128, 256, 3)]:
        assert ex.workspace_bytes(*bad) == 0, bad


P = ctypes.c_void_p


def _gemv(ex, x=16, packed=16, scale=16, su=16, sv=16, y=16, k=256, n=256, bits=3, ws=256, ws_bytes=1 << 20):
    return ex.lib.exl3_gemv(P(x), P(packed), P(scale), P(su), P(sv), P(y), 0, k, n, bits, P(ws), ws_bytes, None)


def test_gemv_argument_validation(ex):
    assert _gemv(ex, x=0) == ex.EXL3_ERR_INVALID_ARG
    assert _gemv(ex, y=0) == ex.EXL3_ERR_INVALID_ARG
    assert _gemv(ex, k=0) == ex.EXL3_ERR_INVALID_ARG
    assert _gemv(ex, k=200) == ex.EXL3_ERR_UNSUPPORTED
    assert _gemv(ex, n=136) == ex.EXL3_ERR_UNSUPPORTED
    assert _gemv(ex, bits=5) == ex.EXL3_ERR_UNSUPPORTED
    assert _gemv(ex, x=18) == ex.EXL3_ERR_MISALIGNED
    assert _gemv(ex, packed=20) == ex.EXL3_ERR_MISALIGNED
    assert _gemv(ex, ws=0) == ex.EXL3_ERR_WORKSPACE
    assert _gemv(ex, ws_bytes=16) == ex.EXL3_ERR_WORKSPACE
    assert _gemv(ex, ws=16) == ex.EXL3_ERR_MISALIGNED


def test_small_m_validation(ex):
    f = ex.lib.exl3_gemm_small_m
    args = lambda m: (m, P(16), P(16), P(16), P(16), P(16), P(16), 0, 256, 256, 3, P(256), 1 << 24, None)
    assert f(*args(0)) == ex.EXL3_ERR_INVALID_ARG
    assert f(*args(33)) == ex.EXL3_ERR_UNSUPPORTED


def test_decode_and_hadamard_validation(ex):
    d = ex.lib.exl3_decode_tiles
    assert d(P(0), 16, 16, 3, P(16), None) == ex.EXL3_ERR_INVALID_ARG
    assert d(P(16), 24, 16, 3, P(16), None) == ex.EXL3_ERR_UNSUPPORTED
    assert d(P(16), 16, 16, 6, P(16), None) == ex.EXL3_ERR_UNSUPPORTED
    assert d(P(16), 16, 16, 3, P(8), None) == ex.EXL3_ERR_MISALIGNED
    h = ex.lib.exl3_hadamard128
    assert h(P(16), P(16), P(16), 1, 128, 2, None) == ex.EXL3_ERR_INVALID_ARG
    assert h(P(16), P(16), P(16), 0, 128, 0, None) == ex.EXL3_ERR_INVALID_ARG
    assert h(P(16), P(16), P(16), 1, 100, 0, None) == ex.EXL3_ERR_UNSUPPORTED
    assert h(P(16), P(4), P(16), 1, 128, 0, None) == ex.EXL3_ERR_MISALIGNED


def test_product_path_has_no_oracle_or_cpu_fallback():
    """The binding and the CUDA sources never reference the oracle."""
    pkg = os.path.join(ROOT, "gemm_exl3_gemv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")) and f != "synth.py":
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.lower() or f == "__init__.py", f


def test_siblings_validation(ex):
    f = ex.lib.exl3_gemm_siblings
    M = ex.Matrix

    def mats(*n_outs, ptr=16):
        arr = (M * max(1, len(n_outs)))()
        for i, n in enumerate(n_outs):
            arr[i] = M(ptr, ptr, ptr, ptr, n)
        return arr

    ws_ok = 1 << 26
    call = lambda m, arr, n, k=256, bits=3, ws=256, wsb=ws_ok: f(m, P(16), P(16), arr, n, 0, k, bits, P(ws), wsb, None)
    assert call(1, mats(256), 0) == ex.EXL3_ERR_INVALID_ARG                 # no matrices
    assert call(1, mats(*([128] * 9)), 9) == ex.EXL3_ERR_UNSUPPORTED       # more than 8
    assert call(1, mats(256, 200), 2) == ex.EXL3_ERR_UNSUPPORTED           # n_out not a multiple of 128
    assert call(1, mats(256, 0), 2) == ex.EXL3_ERR_INVALID_ARG             # empty member
    assert call(1, mats(256, 256, ptr=24), 2) == ex.EXL3_ERR_MISALIGNED    # member pointer misaligned
    assert call(1, mats(256, 256), 2, k=200) == ex.EXL3_ERR_UNSUPPORTED    # k_in not a multiple of 128
    assert call(33, mats(256), 1) == ex.EXL3_ERR_UNSUPPORTED               # too many rows
    assert call(1, mats(256, 256), 2, wsb=64) == ex.EXL3_ERR_WORKSPACE     # sized for the group's total width
    need = ex.workspace_bytes(32, 256, 512, 3)
    assert call(32, mats(256, 256), 2, wsb=need - 1) == ex.EXL3_ERR_WORKSPACE
    assert call(1, mats(256, 256), 2, ws=16) == ex.EXL3_ERR_MISALIGNED


def test_large_m_validation(ex):
    f = ex.lib.exl3_gemm_large_m
    need = ex.lib.exl3_large_m_workspace_bytes(300, 256, 256, 3)
    assert need >= 256 * 256 * 2 + 300 * 256 * 2
    assert ex.lib.exl3_large_m_workspace_bytes(0, 256, 256, 3) == 0
    assert ex.lib.exl3_large_m_workspace_bytes(300, 200, 256, 3) == 0
    args = lambda m=300, k=256, n=256, bits=3, x=16, ws=256, wsb=need: (
        m, P(x), P(16), P(16), P(16), P(16), P(16), 0, k, n, bits, P(ws), wsb, None)
    assert f(*args(m=0)) == ex.EXL3_ERR_INVALID_ARG
    assert f(*args(x=0)) == ex.EXL3_ERR_INVALID_ARG
    assert f(*args(m=(1 << 20) + 1)) == ex.EXL3_ERR_UNSUPPORTED
    assert f(*args(k=200)) == ex.EXL3_ERR_UNSUPPORTED
    assert f(*args(bits=1)) == ex.EXL3_ERR_UNSUPPORTED
    assert f(*args(x=8)) == ex.EXL3_ERR_MISALIGNED
    assert f(*args(wsb=need - 1)) == ex.EXL3_ERR_WORKSPACE
    assert f(*args(ws=0)) == ex.EXL3_ERR_WORKSPACE
    assert f(*args(ws=16)) == ex.EXL3_ERR_MISALIGNED


def test_large_m_workspace_layout(ex):
    """Header (256 bytes), the decoded image (2 bytes per weight) and the rotated
    input for m rows padded to the row tile: 256 rows when that gives 148 tiles,
    else 128, else 64."""
    def tile(m, n):
        g = n // 128
        for nb in (256, 128):
            if g * ((m + nb - 1) // nb) >= 148:
                return nb
        return 64
    for m, k, n in [(1, 128, 128), (300, 256, 256), (2048, 5120, 17408), (512, 5120, 5120), (8192, 5120, 5120)]:
        nb = tile(m, n)
        m_pad = (m + nb - 1) // nb * nb
        assert ex.lib.exl3_large_m_workspace_bytes(m, k, n, 3) == 256 + k * n * 2 + m_pad * k * 2, (m, k, n)
