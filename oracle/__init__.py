"""Plain fp64 CPU oracle for the EXL3 trellis GEMV -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path (the CUDA
library and its binding) never imports it, and it imports nothing from the
product.  The arithmetic lives in ``exl3_oracle.c`` (plain C, fp64); this
module compiles it with gcc and marshals numpy arrays through ctypes.

Inputs are fp16 / uint32 numpy arrays exactly as the library takes them; they
are widened to float64 here (an exact conversion) before the C code runs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "exl3_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) if the .so is missing or stale."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_double_to_half_rne.argtypes = [ctypes.c_double]
        lib.oracle_double_to_half_rne.restype = ctypes.c_uint16
        lib.oracle_3inst.argtypes = [ctypes.c_uint16]
        lib.oracle_3inst.restype = ctypes.c_uint16
        lib.oracle_state.argtypes = [P, ctypes.c_int, ctypes.c_int]
        lib.oracle_state.restype = ctypes.c_uint16
        lib.oracle_decode_tiles.argtypes = [P, L, L, ctypes.c_int, P]
        lib.oracle_decode_tiles.restype = None
        lib.oracle_hadamard128.argtypes = [P, P, P, L, L, ctypes.c_int]
        lib.oracle_hadamard128.restype = None
        lib.oracle_gemm.argtypes = [P, P, P, P, P, L, L, L, ctypes.c_int, P]
        lib.oracle_gemm.restype = None
        lib.oracle_gemm_sampled.argtypes = [P, P, P, P, P, L, L, L, ctypes.c_int, P, L, P]
        lib.oracle_gemm_sampled.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a).astype(np.float64))


def _check_shape(k_in, n_out, bits, mult=128):
    if k_in % mult or n_out % mult or k_in <= 0 or n_out <= 0:
        raise ValueError(f"k_in and n_out must be positive multiples of {mult}")
    if bits not in (1, 2, 3, 4, 5, 6, 7, 8):
        raise ValueError("bits out of range")


# ----------------------------------------------------------------- scalar ---

def half_to_double(h: int) -> float:
    return _load().oracle_half_to_double(int(h) & 0xFFFF)


def double_to_half(v: float) -> int:
    return int(_load().oracle_double_to_half_rne(float(v)))


def decode_state(state: int) -> int:
    """fp16 bit pattern of the weight that 16-bit trellis state `state` decodes to."""
    return int(_load().oracle_3inst(int(state) & 0xFFFF))


def tile_state(tile_words: np.ndarray, bits: int, i: int) -> int:
    w = np.ascontiguousarray(tile_words, dtype=np.uint32)
    assert w.size == 8 * bits
    return int(_load().oracle_state(_ptr(w), bits, i))


# ----------------------------------------------------------------- arrays ---

def decode_tiles(packed: np.ndarray, k_in: int, n_out: int, bits: int) -> np.ndarray:
    """Decoded fp16 bit patterns, K_in x N_out row-major (uint16)."""
    _check_shape(k_in, n_out, bits, mult=16)
    p = np.ascontiguousarray(packed, dtype=np.uint32)
    assert p.size == (k_in // 16) * (n_out // 16) * 8 * bits
    out = np.empty((k_in, n_out), dtype=np.uint16)
    _load().oracle_decode_tiles(_ptr(p), k_in, n_out, bits, _ptr(out))
    return out


def hadamard128(v, signs=None, mode: int = 0) -> np.ndarray:
    """mode 0: H(s*v); mode 1: s*(H v); rows of length n (n % 128 == 0), fp64."""
    a = _f64(v)
    if a.ndim == 1:
        a = a[None, :]
    rows, n = a.shape
    if n % 128:
        raise ValueError("n must be a multiple of 128")
    out = np.empty_like(a)
    s = None if signs is None else _f64(signs)
    _load().oracle_hadamard128(_ptr(a), _ptr(out), None if s is None else _ptr(s),
                               rows, n, int(mode))
    return out


def gemm(x, packed, scale, su, sv, k_in: int, n_out: int, bits: int) -> np.ndarray:
    """y (M x N_out, fp64) = sv * H(scale * ((H(su * x)) W))."""
    _check_shape(k_in, n_out, bits)
    xa = _f64(x)
    if xa.ndim == 1:
        xa = xa[None, :]
    M = xa.shape[0]
    assert xa.shape[1] == k_in
    p = np.ascontiguousarray(packed, dtype=np.uint32)
    assert p.size == (k_in // 16) * (n_out // 16) * 8 * bits
    sc, a_su, a_sv = _f64(scale), _f64(su), _f64(sv)
    assert sc.size == n_out and a_su.size == k_in and a_sv.size == n_out
    y = np.empty((M, n_out), dtype=np.float64)
    _load().oracle_gemm(_ptr(xa), _ptr(p), _ptr(sc), _ptr(a_su), _ptr(a_sv),
                        M, k_in, n_out, bits, _ptr(y))
    return y


def gemm_sampled(x, packed, scale, su, sv, k_in: int, n_out: int, bits: int,
                 blocks) -> np.ndarray:
    """The columns of `gemm` belonging to the listed 128-channel output blocks,
    concatenated in the order given (M x 128*len(blocks))."""
    _check_shape(k_in, n_out, bits)
    xa = _f64(x)
    if xa.ndim == 1:
        xa = xa[None, :]
    M = xa.shape[0]
    p = np.ascontiguousarray(packed, dtype=np.uint32)
    assert p.size == (k_in // 16) * (n_out // 16) * 8 * bits
    b = np.ascontiguousarray(np.asarray(blocks, dtype=np.int64))
    assert b.ndim == 1 and b.size > 0 and b.min() >= 0 and b.max() < n_out // 128
    y = np.empty((M, 128 * b.size), dtype=np.float64)
    _load().oracle_gemm_sampled(_ptr(xa), _ptr(p), _ptr(_f64(scale)), _ptr(_f64(su)),
                                _ptr(_f64(sv)), M, k_in, n_out, bits,
                                b.ctypes.data_as(ctypes.c_void_p), b.size, _ptr(y))
    return y
