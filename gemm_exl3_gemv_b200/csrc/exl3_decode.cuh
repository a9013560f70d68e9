// exl3_decode.cuh -- device-side trellis decoding for the EXL3 format.
//
// The pages name the EXL3 trellis format ("~3.2 bits/weight in the EXL3
// trellis format", orcasaq2-rocm README, opening paragraph; "EXL3, 3.0 bpw",
// exl3-rdna4-recipe, opening paragraph) without defining it.  The definition
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
__device__ __forceinline__ uint32_t weight_pair(uint32_t ma, uint32_t mb)
{
    const uint32_t lo = __byte_perm(ma, mb, 0x5410);   // (ma[15:0], mb[15:0])
    const uint32_t hi = __byte_perm(ma, mb, 0x7632);   // (ma[31:16], mb[31:16])
    __half2 s = __hadd2(*reinterpret_cast<const __half2*>(&lo), *reinterpret_cast<const __half2*>(&hi));
    return *reinterpret_cast<uint32_t*>(&s);
}

}  // namespace exl3
