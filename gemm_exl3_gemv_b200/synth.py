"""Seeded synthetic inputs for the EXL3 trellis GEMV workloads.

This module only draws random inputs; it holds none of the method's
arithmetic (no decode, no Hadamard, no product).  Both the CUDA path (through
the tests and bench.py) and the CPU oracle take their inputs from here.

Recipe (one matrix, identified by (seed, layer, index)):

* packed trellis words: word j of the matrix is the high 32 bits of the
  SplitMix64 output for counter c = stream_id * 2**36 + j, where
  stream_id = (seed * 256 + layer) * 16 + index.  SplitMix64 (Steele, Lea &
  Flood, OOPSLA 2014; the constants of Vigna's public-domain splitmix64.c):
      z = (c + 1) * 0x9E3779B97F4A7C15
      z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
      z = (z ^ (z >> 27)) * 0x94D049BB133111EB
      z = z ^ (z >> 31)            (all mod 2**64)
  Counter-based, so any tile can be regenerated alone (numpy) and the
  full-size streams can be generated on the device (torch) bit-identically.
  The words are uniform random bits, as the workloads ask.
* scale, x, su, sv: numpy PCG64 seeded with [seed, layer, index], drawn in
  that order: scale = fp16(U(0.5, 1.5, N_out) / sqrt(K_in)); x = fp16(N(0,1))
  of shape (M, K_in); su, sv = +1 / -1 from integers(0, 2) (0 -> +1).
  fp16 conversions are numpy's (round to nearest even).

Workloads (sizes from the 27B-class decode / verify shapes):
  1  M=1, 256 -> 256, 3 bits, seed 0
  2  M=1, 5120 -> 5120 (attention o_proj), 3 bits, seed 1
  3  M=1, MLP gate 5120 -> 17408, up 5120 -> 17408, down 17408 -> 5120, 4 bits, seed 2
  4  the workload-3 shapes at 3 bits, M = 16 (the M = 8 case uses the first 8 rows), seed 3
  5  64 layers x {q, k, v, o, gate, up, down}; bits per layer drawn as
     default_rng(4).integers(2, 5, 64); M = 32 (M = 1 uses the first row), seed 4
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
_M64 = (1 << 64) - 1


def _signed64(v: int) -> int:
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


@dataclass(frozen=True)
class MatrixSpec:
    name: str
    k_in: int
    n_out: int
    bits: int
    m: int
    seed: int
    layer: int = 0
    index: int = 0

    @property
    def stream_id(self) -> int:
        return (self.seed * 256 + self.layer) * 16 + self.index

    @property
    def n_words(self) -> int:
        return (self.k_in // 16) * (self.n_out // 16) * 8 * self.bits

    @property
    def packed_bytes(self) -> int:
        return 4 * self.n_words

    @property
    def n_weights(self) -> int:
        return self.k_in * self.n_out


# --------------------------------------------------------------- SplitMix64 --

def splitmix64_words_np(stream_id: int, start: int, count: int) -> np.ndarray:
    """Words [start, start+count) of a matrix stream (uint32, numpy)."""
    c = (np.uint64(stream_id) << np.uint64(36)) + np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (c + np.uint64(1)) * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
        z = z ^ (z >> np.uint64(31))
    return (z >> np.uint64(32)).astype(np.uint32)


def _lsr(z, s: int):
    """Logical right shift of an int64 torch tensor (bit pattern as uint64)."""
    import torch
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64_words_torch(stream_id: int, count: int, device, chunk: int = 1 << 24):
    """All `count` words of a matrix stream as an int32 torch tensor (same bits
    as the numpy version), generated on `device` in chunks."""
    import torch
    out = torch.empty(count, dtype=torch.int32, device=device)
    base = stream_id << 36
    g, m1, m2 = _signed64(GAMMA), _signed64(MIX1), _signed64(MIX2)
    for s in range(0, count, chunk):
        e = min(count, s + chunk)
        z = torch.arange(base + s + 1, base + e + 1, dtype=torch.int64, device=device)
        z = z * g
        z = (z ^ _lsr(z, 30)) * m1
        z = (z ^ _lsr(z, 27)) * m2
        z = z ^ _lsr(z, 31)
        out[s:e] = (z >> 32).to(torch.int32)   # arithmetic shift: in int32 range, same bits
    return out


# ------------------------------------------------------------------ inputs ---

@dataclass
class MatrixInputs:
    spec: MatrixSpec
    packed: Optional[np.ndarray]   # uint32 words (None when generated on device only)
    scale: np.ndarray              # fp16, N_out
    x: np.ndarray                  # fp16, M x K_in
    su: np.ndarray                 # fp16 +-1, K_in
    sv: np.ndarray                 # fp16 +-1, N_out


# Chained runs (a layer's output is the next layer's input) divide the scales
# by this factor, so that activations stay near unit size along a deep chain
# instead of growing by about that factor per product.
CHAIN_SCALE_DIV = 1.3


def small_inputs(spec: MatrixSpec, chain: bool = False):
    """scale, x, su, sv for a matrix (numpy PCG64 seeded by [seed, layer, index]).
    chain=True: the scales of a chained run (same draw, divided by
    CHAIN_SCALE_DIV before the fp16 rounding)."""
    rng = np.random.default_rng([spec.seed, spec.layer, spec.index])
    div = np.sqrt(spec.k_in) * (CHAIN_SCALE_DIV if chain else 1.0)
    scale = (rng.uniform(0.5, 1.5, spec.n_out) / div).astype(np.float16)
    x = rng.standard_normal((spec.m, spec.k_in)).astype(np.float16)
    su = np.where(rng.integers(0, 2, spec.k_in) == 0, 1.0, -1.0).astype(np.float16)
    sv = np.where(rng.integers(0, 2, spec.n_out) == 0, 1.0, -1.0).astype(np.float16)
    return scale, x, su, sv


def make_inputs(spec: MatrixSpec, with_packed: bool = True, chain: bool = False) -> MatrixInputs:
    scale, x, su, sv = small_inputs(spec, chain)
    packed = splitmix64_words_np(spec.stream_id, 0, spec.n_words) if with_packed else None
    return MatrixInputs(spec, packed, scale, x, su, sv)


# --------------------------------------------------------------- workloads ---

LAYER_SHAPES = (("q", 5120, 5120), ("k", 5120, 1024), ("v", 5120, 1024),
                ("o", 5120, 5120), ("gate", 5120, 17408), ("up", 5120, 17408),
                ("down", 17408, 5120))
MLP_SHAPES = (("gate", 5120, 17408), ("up", 5120, 17408), ("down", 17408, 5120))


def stack_bits(n_layers: int = 64, seed: int = 4) -> np.ndarray:
    return np.random.default_rng(seed).integers(2, 5, n_layers)


def workload(cfg: int, m: Optional[int] = None, n_layers: int = 64) -> List[MatrixSpec]:
    """Matrix specs of a workload.  `m` overrides the row count where the
    workload has several (4: 8 or 16; 5: 1 or 32)."""
    if cfg == 1:
        return [MatrixSpec("w256", 256, 256, 3, m or 1, seed=0)]
    if cfg == 2:
        return [MatrixSpec("o_proj", 5120, 5120, 3, m or 1, seed=1)]
    if cfg == 3:
        return [MatrixSpec(n, k, o, 4, m or 1, seed=2, index=i)
                for i, (n, k, o) in enumerate(MLP_SHAPES)]
    if cfg == 4:
        return [MatrixSpec(n, k, o, 3, m or 16, seed=3, index=i)
                for i, (n, k, o) in enumerate(MLP_SHAPES)]
    if cfg == 5:
        bits = stack_bits(64, 4)
        return [MatrixSpec(f"l{l}.{n}", k, o, int(bits[l]), m or 32, seed=4, layer=l, index=i)
                for l in range(n_layers) for i, (n, k, o) in enumerate(LAYER_SHAPES)]
    raise ValueError(f"unknown workload {cfg}")


def rows_for(spec: MatrixSpec, x: np.ndarray, m: int) -> np.ndarray:
    """The first m activation rows (workload 4 at M=8, workload 5 at M=1)."""
    assert m <= x.shape[0]
    return x[:m]
