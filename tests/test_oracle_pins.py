"""Pins for the CPU oracle: each check compares the oracle with something other
than itself -- hand-derived values, numpy's / scipy's own routines, closed
forms, invariants and hand-built bitstreams -- chosen so that a plausible
mistake (bit order, window end, wrap, tile order, in-tile placement, scale
axis, Hadamard order or normalisation, sign placement, rounding mode) fails
at least one of them.  No GPU."""
import os

import numpy as np
import pytest
import scipy.linalg

from gemm_exl3_gemv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
HN = scipy.linalg.hadamard(128).astype(np.float64) / np.sqrt(128.0)   # Sylvester order


def _golden_3inst():
    rows = []
    with open(os.path.join(GOLDEN, "3inst_hand.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            s, x, m, w, v = line.split()
            rows.append((int(s, 16), int(x, 16), int(m, 16), int(w, 16), float(v)))
    return rows


def _h(bits16):
    return float(np.array([bits16], dtype=np.uint16).view(np.float16)[0])


# ------------------------------------------------------------------ fp16 ----

def test_half_decoder_matches_numpy_on_all_patterns(oracle_mod):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle_mod.half_to_double(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_rne_rounding_matches_numpy(oracle_mod):
    rng = np.random.default_rng(123)
    vals = list(rng.standard_normal(3000) * 4.0)
    vals += list(rng.uniform(-1e-4, 1e-4, 500))                  # subnormal range
    vals += list(rng.uniform(-65000, 65000, 300))                # large normals
    # exact midpoints between neighbouring fp16 values: ties must go to even
    pos = np.arange(0x0001, 0x7BFF, 37, dtype=np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).view(np.float16).astype(np.float64)
    mids = (lo + hi) / 2.0
    vals += list(mids) + list(-mids)
    vals += [0.0, -0.0, 65504.0, 65519.999, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26]
    for v in vals:
        ref = int(np.array([v]).astype(np.float16).view(np.uint16)[0])
        assert oracle_mod.double_to_half(v) == ref, (v, hex(ref))


# ----------------------------------------------------------------- 3INST ----

def test_3inst_hand_values(oracle_mod):
    for state, _x, _m, w_bits, w_val in _golden_3inst():
        assert oracle_mod.decode_state(state) == w_bits, hex(state)
        assert _h(w_bits) == w_val


def test_3inst_hand_intermediates_are_consistent():
    # the hand table's x and m columns reproduce its fp16 halves and sums
    for state, x, m, w_bits, _ in _golden_3inst():
        assert (x & 0x8FFF8FFF) ^ 0x3B603B60 == m
        lo, hi = _h(m & 0xFFFF), _h(m >> 16)
        s = np.float16(np.float32(lo) + np.float32(hi))   # numpy: fp32 sum then RNE to fp16
        assert int(np.array([s]).view(np.uint16)[0]) == w_bits


def test_3inst_table_against_numpy_binary16(oracle_mod):
    states = np.arange(65536, dtype=np.uint64)
    x = ((states * np.uint64(89226354) + np.uint64(64248484)) & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    m = (x & np.uint32(0x8FFF8FFF)) ^ np.uint32(0x3B603B60)
    lo = (m & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16).astype(np.float32)
    hi = (m >> np.uint32(16)).astype(np.uint16).view(np.float16).astype(np.float32)
    ref = (lo + hi).astype(np.float16).view(np.uint16)           # exact fp32 sum, RNE to fp16
    got = np.array([oracle_mod.decode_state(int(s)) for s in range(65536)], dtype=np.uint16)
    assert np.array_equal(got, ref)
    w = got.view(np.float16).astype(np.float64)
    assert np.all(np.isfinite(w))
    assert not np.any(got == 0x8000)                             # -0 cannot occur
    # ties occur, so the rounding mode matters (state 2 is one)
    exact = (lo.astype(np.float64) + hi.astype(np.float64))
    assert np.sum(exact != w) > 1000
    assert -4.0 < w.min() < -3.9 and 3.9 < w.max() < 4.0
    assert abs(w.mean()) < 1e-2 and 1.2 < w.std() < 1.3


# --------------------------------------------------------- bitstream pins ----

def test_window_msb_first_and_window_end(oracle_mod):
    tile = np.zeros(32, dtype=np.uint32)                         # K = 4: 8*4 words
    tile[0] = 0x12345678
    want = {0: 0x0001, 1: 0x0012, 2: 0x0123, 3: 0x1234, 4: 0x2345, 5: 0x3456,
            6: 0x4567, 7: 0x5678, 8: 0x6780, 9: 0x7800, 10: 0x8000}
    for i in range(256):
        assert oracle_mod.tile_state(tile, 4, i) == want.get(i, 0), i


def test_tail_biting_wrap(oracle_mod):
    tile = np.zeros(32, dtype=np.uint32)
    tile[31] = 0x0000ABCD                                        # the last 16 bits of the stream
    # a K=4 stream is 1024 bits: its last word feeds weights 252..255 and, by the
    # wrap, the first windows of weights 0..2
    want = {0: 0xBCD0, 1: 0xCD00, 2: 0xD000, 252: 0x000A, 253: 0x00AB, 254: 0x0ABC, 255: 0xABCD}
    for i in range(256):
        assert oracle_mod.tile_state(tile, 4, i) == want.get(i, 0), i


@pytest.mark.parametrize("p,affected", [(0, set(range(5))), (5, set(range(1, 7))),
                                        (767, set(range(5)) | {255})])
def test_one_hot_support_k3(oracle_mod, p, affected):
    tile = np.zeros(24, dtype=np.uint32)
    tile[p // 32] = np.uint32(1 << (31 - p % 32))
    hit = {i for i in range(256) if oracle_mod.tile_state(tile, 3, i) != 0}
    assert hit == affected


def test_tile_order_and_in_tile_placement(oracle_mod):
    k_in, n_out, bits = 32, 48, 4                                # 2 x 3 tiles
    packed = np.zeros(6 * 32, dtype=np.uint32)
    packed[3 * 32:4 * 32] = 0xFFFFFFFF                           # tile (tk=1, tn=0): states 0xFFFF
    packed[5 * 32 + 5] = 0x80000000                              # tile (1, 2): bit 160 set
    w = oracle_mod.decode_tiles(packed, k_in, n_out, bits)
    c0, cF, c8 = 0x3A25, 0xB110, 0xB7F8                          # hand values: 0x0000, 0xFFFF, 0x8000
    exp = np.full((k_in, n_out), c0, dtype=np.uint16)
    exp[16:32, 0:16] = cF
    # bit 160 of a K=4 stream is in the windows of weights 40..43 (states 0x0008,
    # 0x0080, 0x0800, 0x8000); weight 43 is row 2, column 11 of the tile
    exp[16 + 2, 32 + 8] = oracle_mod.decode_state(0x0008)
    exp[16 + 2, 32 + 9] = oracle_mod.decode_state(0x0080)
    exp[16 + 2, 32 + 10] = oracle_mod.decode_state(0x0800)
    exp[16 + 2, 32 + 11] = c8
    assert np.array_equal(w, exp)


def _bits_of(words):
    return "".join(format(int(v), "032b") for v in words)


def test_decode_against_pure_python_bitstring(oracle_mod):
    """Cross-check of the C decoder with a string-based restatement on random
    tiles (catches slips in the C code; shares the readings)."""
    rng = np.random.default_rng(5)
    for bits in (2, 3, 4):
        words = rng.integers(0, 2 ** 32, size=8 * bits, dtype=np.uint64).astype(np.uint32)
        s = _bits_of(words)
        n = 256 * bits
        for i in range(256):
            start = (i + 1) * bits - 16
            win = "".join(s[(start + j) % n] for j in range(16))
            assert oracle_mod.tile_state(words, bits, i) == int(win, 2)


# --------------------------------------------------------------- Hadamard ----

def test_hadamard_matches_scipy_sylvester(oracle_mod):
    rng = np.random.default_rng(7)
    v = rng.standard_normal((3, 256))
    s = np.where(rng.integers(0, 2, 256) == 0, 1.0, -1.0)
    got0 = oracle_mod.hadamard128(v, s, 0)
    got1 = oracle_mod.hadamard128(v, s, 1)
    for b in (0, 128):
        blk = slice(b, b + 128)
        np.testing.assert_allclose(got0[:, blk], (v[:, blk] * s[blk]) @ HN, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got1[:, blk], (v[:, blk] @ HN) * s[blk], rtol=0, atol=1e-12)


def test_hadamard_orthogonal_involution_and_ones(oracle_mod):
    eye = np.eye(128)
    H = oracle_mod.hadamard128(eye, None, 0)                     # rows: H e_i
    np.testing.assert_allclose(H @ H.T, eye, atol=1e-13)
    rng = np.random.default_rng(8)
    v = rng.standard_normal((4, 384))
    s = np.where(rng.integers(0, 2, 384) == 0, 1.0, -1.0)
    back = oracle_mod.hadamard128(oracle_mod.hadamard128(v, s, 0), s, 1)
    np.testing.assert_allclose(back, v, atol=1e-12)
    ones = oracle_mod.hadamard128(np.ones(128), None, 0)[0]
    np.testing.assert_allclose(ones, np.sqrt(128.0) * eye[0], atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(oracle_mod.hadamard128(v, s, 0), axis=1),
                               np.linalg.norm(v, axis=1), rtol=1e-13)


# ------------------------------------------------------------------- GEMM ----

def test_gemm_closed_form_all_zero_stream(oracle_mod):
    k, n, bits = 128, 128, 3
    packed = np.zeros((k // 16) * (n // 16) * 8 * bits, dtype=np.uint32)
    ones = np.ones(128)
    x = np.zeros(128)
    x[0] = 1.0
    y = oracle_mod.gemm(x, packed, ones, ones, ones, k, n, bits)[0]
    c = 0.76806640625
    np.testing.assert_allclose(y, 128 * c * np.eye(128)[0], atol=1e-12)
    assert abs(y[0] - 98.3125) < 1e-12
    # scale on channel 5 only: z = c*sqrt(128)*e_5, y_j = c * (-1)^popcount(j & 5)
    sc = np.zeros(128)
    sc[5] = 1.0
    y = oracle_mod.gemm(x, packed, sc, ones, ones, k, n, bits)[0]
    want = np.array([c * (-1) ** bin(j & 5).count("1") for j in range(128)])
    np.testing.assert_allclose(y, want, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gemm_recovers_scaled_weight_rows(oracle_mod, bits):
    """x = su * H[j] makes the rotated input sqrt(128) e_j, so undoing the output
    rotation must give sqrt(128) * scale * W[j, :] -- the decoded row j."""
    k, n = 256, 384
    spec = synth.MatrixSpec("t", k, n, bits, 1, seed=11, index=bits)
    inp = synth.make_inputs(spec)
    scale = inp.scale.astype(np.float64)
    su = inp.su.astype(np.float64)
    sv = inp.sv.astype(np.float64)
    W = oracle_mod.decode_tiles(inp.packed, k, n, bits).view(np.float16).astype(np.float64)
    H_un = scipy.linalg.hadamard(128).astype(np.float64)
    for j in (0, 37, 128 + 90):
        b, r = divmod(j, 128)
        x = np.zeros(k)
        x[b * 128:(b + 1) * 128] = H_un[r] * su[b * 128:(b + 1) * 128]
        y = oracle_mod.gemm(x, inp.packed, scale, su, sv, k, n, bits)[0]
        z = np.concatenate([(y[c:c + 128] * sv[c:c + 128]) @ HN for c in range(0, n, 128)])
        np.testing.assert_allclose(z, np.sqrt(128.0) * scale * W[j], rtol=1e-12, atol=1e-12)


def test_gemm_frobenius_invariant(oracle_mod):
    k, n, bits = 256, 256, 3
    inp = synth.make_inputs(synth.MatrixSpec("f", k, n, bits, 1, seed=12))
    scale = inp.scale.astype(np.float64)
    W = oracle_mod.decode_tiles(inp.packed, k, n, bits).view(np.float16).astype(np.float64)
    Y = oracle_mod.gemm(np.eye(k), inp.packed, scale, inp.su, inp.sv, k, n, bits)
    np.testing.assert_allclose(np.sum(Y ** 2), np.sum((W * scale) ** 2), rtol=1e-12)


def test_gemm_linearity(oracle_mod):
    k, n, bits = 256, 128, 2
    inp = synth.make_inputs(synth.MatrixSpec("l", k, n, bits, 2, seed=13))
    x1, x2 = inp.x.astype(np.float64)
    f = lambda v: oracle_mod.gemm(v, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits)[0]
    np.testing.assert_allclose(f(2.5 * x1 + x2), 2.5 * f(x1) + f(x2), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gemm_matches_library_composition(oracle_mod, bits):
    k, n, m = 256, 256, 3
    inp = synth.make_inputs(synth.MatrixSpec("c", k, n, bits, m, seed=14, index=bits))
    x = inp.x.astype(np.float64)
    su, sv, sc = (a.astype(np.float64) for a in (inp.su, inp.sv, inp.scale))
    W = oracle_mod.decode_tiles(inp.packed, k, n, bits).view(np.float16).astype(np.float64)
    xt = np.concatenate([(x[:, b:b + 128] * su[b:b + 128]) @ HN for b in range(0, k, 128)], axis=1)
    z = (xt @ W) * sc
    y = np.concatenate([(z[:, c:c + 128] @ HN) * sv[c:c + 128] for c in range(0, n, 128)], axis=1)
    got = oracle_mod.gemm(x, inp.packed, sc, su, sv, k, n, bits)
    np.testing.assert_allclose(got, y, rtol=1e-12, atol=1e-12)


def test_gemm_sampled_blocks_equal_full(oracle_mod):
    k, n, bits = 256, 512, 4
    inp = synth.make_inputs(synth.MatrixSpec("s", k, n, bits, 2, seed=15))
    full = oracle_mod.gemm(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits)
    part = oracle_mod.gemm_sampled(inp.x, inp.packed, inp.scale, inp.su, inp.sv, k, n, bits,
                                   [3, 1])
    np.testing.assert_array_equal(part, np.concatenate([full[:, 384:512], full[:, 128:256]], 1))


# -------------------------------------------------------------- generator ----

def test_splitmix64_published_vector():
    # first output of splitmix64 from state 0 (Vigna's reference implementation)
    z = (1 * synth.GAMMA) & ((1 << 64) - 1)
    z = ((z ^ (z >> 30)) * synth.MIX1) & ((1 << 64) - 1)
    z = ((z ^ (z >> 27)) * synth.MIX2) & ((1 << 64) - 1)
    z ^= z >> 31
    assert z == 0xE220A8397B1DCDAF
    assert int(synth.splitmix64_words_np(0, 0, 1)[0]) == 0xE220A839


def test_generator_numpy_torch_agree():
    import torch
    a = synth.splitmix64_words_np(12345, 0, 5000)
    b = synth.splitmix64_words_torch(12345, 5000, "cpu", chunk=777).numpy().view(np.uint32)
    assert np.array_equal(a, b)
    assert np.array_equal(synth.splitmix64_words_np(12345, 1000, 10), a[1000:1010])


def test_workload_shapes_and_bytes():
    assert synth.workload(2)[0].packed_bytes == 9_830_400
    assert [s.packed_bytes for s in synth.workload(3)] == [44_564_480] * 3
    assert [s.packed_bytes for s in synth.workload(4)] == [33_423_360] * 3
    w5 = synth.workload(5)
    assert len(w5) == 448
    assert sum(s.n_weights for s in w5[:7]) == 330_301_440
    assert set(synth.stack_bits()) <= {2, 3, 4}
