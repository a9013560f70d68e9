// exl3_decode.cuh -- device-side trellis decoding for the EXL3 format.
//
// The pages name the EXL3 trellis format (models at about 3 bits per weight:
// orcasaq2-rocm README and exl3-rdna4-recipe, opening paragraphs) without
// defining it.  The definition
// used here is the specification's: 16x16 tiles, each a tail-biting stream of
// 256*K bits; weight i of a tile is decoded from the 16-bit window that ends
// at stream bit (i+1)*K, through the 3INST map.  Readings where the
// definition is silent: bits are taken MSB-first from 32-bit words (stream
// bit j is bit 31-(j%32) of word j/32), window positions wrap modulo 256*K,
// and weight i sits at row i/16, column i%16 of its tile.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace exl3 {

// 3INST: x = state*89226354 + 64248484 (mod 2^32), then
// (x & 0x8FFF8FFF) ^ 0x3B603B60.  The result holds two fp16 values (low and
// high halves) whose sum is the weight.
// Written as one multiply-add and one three-input logic op (LUT 0x6A =
// (a & b) ^ c); left to itself the compiler spends an extra integer
// instruction on the two 32-bit constants.
__device__ __forceinline__ uint32_t inst3(uint32_t state)
{
    uint32_t m;
    asm("{\n\t.reg .b32 t;\n\t"
        "mad.lo.u32 t, %1, 89226354, 64248484;\n\t"
        "lop3.b32 %0, t, 0x8FFF8FFF, 0x3B603B60, 0x6A;\n\t}"
        : "=r"(m)
        : "r"(state));
    return m;
}

// State whose 16-bit window starts P bits after the most significant bit of
// buf[0]; buf holds consecutive stream words.  P is a compile-time constant
// in every caller, so the shifts below are immediates.
template <int P, int NW>
__device__ __forceinline__ uint32_t window16(const uint32_t (&buf)[NW])
{
    constexpr int wi = P >> 5;
    constexpr int off = P & 31;
    static_assert(wi + (off > 16 ? 1 : 0) < NW, "window outside the buffer");
    if constexpr (off <= 16) {
        return (buf[wi] >> (16 - off)) & 0xFFFFu;
    } else {
        return __funnelshift_r(buf[wi + 1], buf[wi], 48 - off) & 0xFFFFu;
    }
}

// Sum of the two fp16 halves of a 3INST result, rounded once to fp16
// (round-to-nearest-even): the decoded weight, bit-exact.
__device__ __forceinline__ __half weight_of(uint32_t m)
{
    __half2 h = *reinterpret_cast<__half2*>(&m);
    return __hadd(__low2half(h), __high2half(h));
}

// Two decoded weights packed as fp16 (w(ma) in the low half, w(mb) in the
// high half): the low halves and the high halves of the two 3INST words are
// gathered with byte permutes and added in one packed fp16 add (RNE), which
// gives the same bits as weight_of on each word.
// Same result, another instruction mix: each word's halves are added by one
// half-precision add (operand halves selected in the instruction), and the
// two sums are then packed -- more FMA-pipe and fewer integer-pipe work.
__device__ __forceinline__ uint32_t weight_pair_h(uint32_t ma, uint32_t mb)
{
    uint32_t r;
    asm("{\n\t.reg .f16 al, ah, bl, bh, wa, wb;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "add.rn.f16 wa, al, ah;\n\t"
        "add.rn.f16 wb, bl, bh;\n\t"
        "mov.b32 %0, {wa, wb};\n\t}"
        : "=r"(r)
        : "r"(ma), "r"(mb));
    return r;
}

__device__ __forceinline__ uint32_t weight_pair(uint32_t ma, uint32_t mb)
{
    const uint32_t lo = __byte_perm(ma, mb, 0x5410);   // (ma[15:0], mb[15:0])
    const uint32_t hi = __byte_perm(ma, mb, 0x7632);   // (ma[31:16], mb[31:16])
    __half2 s = __hadd2(*reinterpret_cast<const __half2*>(&lo), *reinterpret_cast<const __half2*>(&hi));
    return *reinterpret_cast<uint32_t*>(&s);
}

// Isolate the 16-bit window that starts P bits after the most significant bit
// of buf[0] (P a compile-time constant).  Windows at the top or bottom half
// of a word take one instruction.  Otherwise ALT selects the form:
//   ALT = false: shift right + mask (two integer-pipe instructions);
//   ALT = true : shift left so the window is the top half, then a high
//                multiply by 2^16 (`two16` is a runtime value, so the
//                multiply stays on the FMA pipe) -- one integer-pipe and one
//                FMA-pipe instruction.
template <int P, int NW, bool ALT>
__device__ __forceinline__ uint32_t window_of(const uint32_t (&buf)[NW], uint32_t two16)
{
    constexpr int wi = P >> 5, off = P & 31;
    static_assert(wi + (off > 16 ? 1 : 0) < NW, "window outside the buffer");
    if constexpr (off == 0) {
        return buf[wi] >> 16;
    } else if constexpr (off == 16) {
        return buf[wi] & 0xFFFFu;
    } else if constexpr (!ALT) {
        if constexpr (off < 16) return (buf[wi] >> (16 - off)) & 0xFFFFu;
        else return __funnelshift_r(buf[wi + 1], buf[wi], 48 - off) & 0xFFFFu;
    } else {
        uint32_t v;
        if constexpr (off < 16) v = buf[wi] << off;
        else v = __funnelshift_l(buf[wi + 1], buf[wi], off);
        return __umulhi(v, two16);
    }
}

// Byte-aligned variant for even bit widths: a window whose offset is r bits
// (r = off mod 8) past a byte boundary is read from the stream shifted left
// by r bits (one funnel shift per word, shared by every window of that word
// with the same r), where it sits at a byte boundary: top half (shift), bytes
// 1-2 (byte permute with zero fill) or bottom half (mask) -- one instruction.
// Windows that straddle the next word fall back to window_of.
template <int P, int NW>
__device__ __forceinline__ uint32_t window_bytes(const uint32_t (&buf)[NW], uint32_t two16)
{
    constexpr int wi = P >> 5, off = P & 31, r = off & 7, ob = off - r;
    if constexpr (ob == 24 || (r != 0 && wi + 1 >= NW)) {
        return window_of<P, NW, false>(buf, two16);
    } else {
        uint32_t w;
        if constexpr (r == 0) w = buf[wi];
        else w = __funnelshift_l(buf[wi + 1], buf[wi], r);
        if constexpr (ob == 0) return w >> 16;
        else if constexpr (ob == 8) return __byte_perm(w, 0u, 0x4421);
        else return w & 0xFFFFu;
    }
}


// Window isolation chosen per bit width (measured on B200): byte-aligned
// reads from shifted words for 2 and 4 bits; for 3 bits (windows at every
// bit offset) every third non-aligned window on the FMA pipe (every second:
// up to 2 % slower).  R is the weight's index in the run, P its window's
// start bit in `buf`.
template <int BITS, int R, int P, int NW>
__device__ __forceinline__ uint32_t window_auto(const uint32_t (&buf)[NW], uint32_t two16)
{
    if constexpr (BITS == 3) return window_of<P, NW, (R % 3) == 0>(buf, two16);
    else return window_bytes<P, NW>(buf, two16);
}

// A lane's share of one tile row of a 128-channel block: 2*BITS consecutive
// words at `src` (streaming loads: each word is read once).  K = 2, 4: 128-bit
// loads; K = 3: 64-bit loads (the lane's 24 bytes are 8-byte aligned).
// The later loads take their offset as an immediate in the instruction (no
// address arithmetic per load).
template <int BITS>
__device__ __forceinline__ void load_lane_words(uint32_t (&w)[2 * BITS], const uint32_t* src)
{
    if constexpr (BITS == 3) {
        asm volatile("ld.global.cs.v2.u32 {%0, %1}, [%6];\n\t"
                     "ld.global.cs.v2.u32 {%2, %3}, [%6+8];\n\t"
                     "ld.global.cs.v2.u32 {%4, %5}, [%6+16];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5])
                     : "l"(src));
    } else if constexpr (BITS == 4) {
        asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%8];\n\t"
                     "ld.global.cs.v4.u32 {%4, %5, %6, %7}, [%8+16];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                       "=r"(w[7])
                     : "l"(src));
    } else {
        static_assert(BITS == 2, "2, 3 or 4 bits");
        asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "l"(src));
    }
}

// load_lane_words, or zeros when the debug bounds check (the lane's words
// inside the matrix's n_words) fails.
template <int BITS>
__device__ __forceinline__ void load_lane_words_checked(uint32_t (&w)[2 * BITS], const uint32_t* src,
                                                        const uint32_t* base, size_t n_words, uint32_t* status)
{
    if (guard(src >= base && (size_t)(src - base) + 2 * BITS <= n_words, status)) {
        load_lane_words<BITS>(w, src);
    } else {
#pragma unroll
        for (int t = 0; t < 2 * BITS; ++t) w[t] = 0u;
    }
}

}  // namespace exl3
