"""ctypes binding of libexl3 (include/exl3.h).

Argument marshalling only: every step of the product runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
shared library is missing this module raises on import -- there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# EXL3_LIBRARY selects another build of the library, e.g. the debug-bounds
# build libexl3_debug.so next to this file.
LIB_PATH = os.environ.get("EXL3_LIBRARY") or os.path.join(_HERE, "libexl3.so")

EXL3_OK = 0
EXL3_ERR_INVALID_ARG = 1
EXL3_ERR_UNSUPPORTED = 2
EXL3_ERR_MISALIGNED = 3
EXL3_ERR_WORKSPACE = 4
EXL3_ERR_ARCH = 5
EXL3_ERR_CUDA = 6
EXL3_ERR_TIMEOUT = 7
EXL3_ERR_BOUNDS = 8

# every entry point include/exl3.h declares
EXPORTS = ("exl3_status_string", "exl3_last_cuda_error", "exl3_version", "exl3_workspace_bytes",
           "exl3_workspace_status", "exl3_kernel_launches", "exl3_decode_tiles", "exl3_hadamard128", "exl3_gemv",
           "exl3_gemm_small_m", "exl3_gemm_siblings", "exl3_large_m_workspace_bytes", "exl3_gemm_large_m",
           "exl3_gemv_noalloc", "exl3_grouped_workspace_bytes", "exl3_gemm_grouped")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libexl3.so not built ({LIB_PATH}); run `python -m gemm_exl3_gemv_b200.build`")

lib = ctypes.CDLL(LIB_PATH)
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
lib.exl3_status_string.argtypes = [_I]
lib.exl3_status_string.restype = ctypes.c_char_p
lib.exl3_last_cuda_error.argtypes = []
lib.exl3_last_cuda_error.restype = _I
lib.exl3_version.argtypes = []
lib.exl3_version.restype = _I
lib.exl3_workspace_bytes.argtypes = [_I, _I, _I, _I]
lib.exl3_workspace_bytes.restype = _Z
lib.exl3_kernel_launches.argtypes = [_I, _I, _I, _I]
lib.exl3_kernel_launches.restype = _I
lib.exl3_workspace_status.argtypes = [_P, _P]
lib.exl3_workspace_status.restype = _I
lib.exl3_decode_tiles.argtypes = [_P, _I, _I, _I, _P, _P]
lib.exl3_decode_tiles.restype = _I
lib.exl3_hadamard128.argtypes = [_P, _P, _P, _I, _I, _I, _P]
lib.exl3_hadamard128.restype = _I
lib.exl3_gemv.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]
lib.exl3_gemv.restype = _I
lib.exl3_gemm_small_m.argtypes = [_I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]
lib.exl3_gemm_small_m.restype = _I
lib.exl3_gemv_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]


class Matrix(ctypes.Structure):
    """exl3_matrix_t: one member of a sibling group (device pointers)."""
    _fields_ = [("packed", _P), ("scale", _P), ("sv", _P), ("y", _P), ("n_out", _I)]


lib.exl3_gemm_siblings.argtypes = [_I, _P, _P, ctypes.POINTER(Matrix), _I, _I, _I, _I, _P, _Z, _P]
lib.exl3_gemm_siblings.restype = _I
lib.exl3_large_m_workspace_bytes.argtypes = [_I, _I, _I, _I]
lib.exl3_large_m_workspace_bytes.restype = _Z
lib.exl3_gemm_large_m.argtypes = [_I, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]
lib.exl3_gemm_large_m.restype = _I
lib.exl3_gemv_noalloc.restype = _I


class Problem(ctypes.Structure):
    """exl3_problem_t: one member of a grouped call (device pointers)."""
    _fields_ = [("x", _P), ("su", _P), ("packed", _P), ("scale", _P), ("sv", _P), ("y", _P),
                ("k_in", _I), ("n_out", _I)]


lib.exl3_grouped_workspace_bytes.argtypes = [_I, ctypes.POINTER(Problem), _I, _I]
lib.exl3_grouped_workspace_bytes.restype = _Z
lib.exl3_gemm_grouped.argtypes = [_I, ctypes.POINTER(Problem), _I, _I, _I, _P, _Z, _P]
lib.exl3_gemm_grouped.restype = _I


class Exl3Error(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib.exl3_status_string(status).decode()
        if status == EXL3_ERR_CUDA:
            msg += f" (cudaError {lib.exl3_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")
        self.status = status


def _check(status: int, what: str):
    if status != EXL3_OK:
        raise Exl3Error(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_bytes(m: int, k_in: int, n_out: int, bits: int) -> int:
    return int(lib.exl3_workspace_bytes(m, k_in, n_out, bits))


def kernel_launches(m: int, k_in: int, n_out: int, bits: int) -> int:
    return int(lib.exl3_kernel_launches(m, k_in, n_out, bits))


def alloc_workspace(m: int, k_in: int, n_out: int, bits: int, device=None) -> torch.Tensor:
    """Zero-filled workspace (uint8) for problems up to this size."""
    n = workspace_bytes(m, k_in, n_out, bits)
    if n == 0:
        raise Exl3Error(EXL3_ERR_UNSUPPORTED, "workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib.exl3_workspace_status(_ptr(ws), _stream(stream)))


def decode_tiles(packed: torch.Tensor, k_in: int, n_out: int, bits: int,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decoded weights, k_in x n_out fp16."""
    if out is None:
        out = torch.empty((k_in, n_out), dtype=torch.float16, device=packed.device)
    _check(lib.exl3_decode_tiles(_ptr(packed), k_in, n_out, bits, _ptr(out), _stream(stream)),
           "exl3_decode_tiles")
    return out


def hadamard128(x: torch.Tensor, signs: torch.Tensor, mode: int = 0,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mode 0: H(signs*x); mode 1: signs*H(x); x is rows x n fp16."""
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    if out is None:
        out = torch.empty_like(x2)
    _check(lib.exl3_hadamard128(_ptr(x2), _ptr(out), _ptr(signs), x2.shape[0], x2.shape[1], mode,
                                _stream(stream)), "exl3_hadamard128")
    return out if x.dim() == 2 else out.reshape(x.shape)


def gemm(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, su: torch.Tensor,
         sv: torch.Tensor, bits: int, out: Optional[torch.Tensor] = None, fp32: bool = False,
         workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = sv*H(scale*(H(su*x) W)) for x of shape (m, k_in) (m <= 32) or (k_in,)."""
    squeeze = x.dim() == 1
    x2 = x.reshape(1, -1) if squeeze else x
    m, k_in = x2.shape
    n_out = scale.shape[0]
    if out is None:
        out = torch.empty((m, n_out), dtype=torch.float32 if fp32 else torch.float16, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(m, k_in, n_out, bits, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if m == 1:
        st = lib.exl3_gemv(_ptr(x2), _ptr(packed), _ptr(scale), _ptr(su), _ptr(sv), _ptr(out),
                           int(fp32), k_in, n_out, bits, _ptr(workspace), ws_bytes, _stream(stream))
        _check(st, "exl3_gemv")
    else:
        st = lib.exl3_gemm_small_m(m, _ptr(x2), _ptr(packed), _ptr(scale), _ptr(su), _ptr(sv),
                                   _ptr(out), int(fp32), k_in, n_out, bits, _ptr(workspace),
                                   ws_bytes, _stream(stream))
        _check(st, "exl3_gemm_small_m")
    return out.reshape(-1) if squeeze else out


def gemm_siblings(x: torch.Tensor, su: torch.Tensor, mats, bits: int, outs=None, fp32: bool = False,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """Products of one input with a group of matrices in one pass.  `mats` is a
    list of (packed, scale, sv); returns the list of outputs (m, n_out_i)."""
    squeeze = x.dim() == 1
    x2 = x.reshape(1, -1) if squeeze else x
    m, k_in = x2.shape
    if outs is None:
        outs = [torch.empty((m, sc.shape[0]), dtype=torch.float32 if fp32 else torch.float16, device=x.device)
                for (_, sc, _) in mats]
    n_total = sum(int(sc.shape[0]) for (_, sc, _) in mats)
    if workspace is None:
        workspace = alloc_workspace(m, k_in, n_total, bits, device=x.device)
    arr = (Matrix * len(mats))()
    for i, ((packed, scale, sv), y) in enumerate(zip(mats, outs)):
        arr[i] = Matrix(packed.data_ptr(), scale.data_ptr(), sv.data_ptr(), y.data_ptr(), int(scale.shape[0]))
    st = lib.exl3_gemm_siblings(m, _ptr(x2), _ptr(su), arr, len(mats), int(fp32), k_in, bits, _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "exl3_gemm_siblings")
    return [o.reshape(-1) for o in outs] if squeeze else outs


def gemm_large(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, su: torch.Tensor, sv: torch.Tensor,
               bits: int, out: Optional[torch.Tensor] = None, fp32: bool = False,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The product for many rows (x: m x k_in), decoding W once per call."""
    m, k_in = x.shape
    n_out = scale.shape[0]
    if out is None:
        out = torch.empty((m, n_out), dtype=torch.float32 if fp32 else torch.float16, device=x.device)
    if workspace is None:
        n = int(lib.exl3_large_m_workspace_bytes(m, k_in, n_out, bits))
        if n == 0:
            raise Exl3Error(EXL3_ERR_UNSUPPORTED, "exl3_large_m_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=x.device)
    st = lib.exl3_gemm_large_m(m, _ptr(x), _ptr(packed), _ptr(scale), _ptr(su), _ptr(sv), _ptr(out), int(fp32),
                               k_in, n_out, bits, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream))
    _check(st, "exl3_gemm_large_m")
    return out



def grouped_workspace_bytes(m: int, shapes, bits: int) -> int:
    """Workspace of a grouped call for members of shapes [(k_in, n_out), ...]."""
    arr = (Problem * len(shapes))()
    for i, (k, n) in enumerate(shapes):
        arr[i] = Problem(None, None, None, None, None, None, int(k), int(n))
    return int(lib.exl3_grouped_workspace_bytes(m, arr, len(shapes), bits))


def grouped_kernel_launches(m: int) -> int:
    """Kernel launches of one grouped call: the product (m = 1), or the
    rotation pre-pass and the product (m >= 2)."""
    return 1 if m == 1 else 2


def gemm_grouped(problems, bits: int, fp32: bool = False, workspace: Optional[torch.Tensor] = None,
                 stream=None):
    """Products of independent problems in one pass.  `problems` is a list of
    (x, packed, scale, su, sv, y) device tensors, x of shape (m, k_in) (or
    (k_in,) for m = 1) and y of shape (m, n_out); returns the list of y."""
    arr = (Problem * len(problems))()
    m = None
    shapes = []
    for i, (x, packed, scale, su, sv, y) in enumerate(problems):
        x2 = x.reshape(1, -1) if x.dim() == 1 else x
        if m is None:
            m = x2.shape[0]
        k_in, n_out = x2.shape[1], scale.shape[0]
        shapes.append((k_in, n_out))
        arr[i] = Problem(x2.data_ptr(), su.data_ptr(), packed.data_ptr(), scale.data_ptr(), sv.data_ptr(),
                         y.data_ptr(), int(k_in), int(n_out))
    if workspace is None:
        n = grouped_workspace_bytes(m, shapes, bits)
        if n == 0:
            raise Exl3Error(EXL3_ERR_UNSUPPORTED, "exl3_grouped_workspace_bytes")
        workspace = torch.zeros(n, dtype=torch.uint8, device=problems[0][0].device)
    st = lib.exl3_gemm_grouped(m, arr, len(problems), int(fp32), bits, _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "exl3_gemm_grouped")
    return [p[5] for p in problems]
