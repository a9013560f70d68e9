// exl3_aop.cuh -- the tensor-core A operand of the trellis products: one
// tile row of a 128-channel output block (128 channels x 16 input rows, fp16,
// MN-major, 128-byte swizzle: 4 KB), written by the lanes of one warp straight
// from their decoded weights.  Used by the verify kernel (into shared memory)
// and by the large-M path (into a global image of the whole matrix).
#pragma once
#include <cstdint>
#include <utility>

#include "exl3_decode.cuh"

namespace exl3 {

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Row v of an accumulator (row v of A) holds output channel chan_of_row(v):
// tile j's 16 channels fill 16-byte chunks 4*(j&1) + 2*((j>>1)&1) + e of MN
// atom j/4 (e = channel/8), so that the 8 lanes of a store phase hit 8
// different banks.
__host__ __device__ constexpr int chunk_of_tile(int j4, int e) { return 4 * (j4 & 1) + 2 * ((j4 >> 1) & 1) + e; }
__device__ __forceinline__ int chan_of_row(int v)
{
    const int atom = v >> 6, chunk = (v >> 3) & 7, pos = v & 7;
    const int j4 = 2 * ((chunk >> 1) & 1) + ((chunk >> 2) & 1);
    return 16 * (4 * atom + j4) + 8 * (chunk & 1) + pos;
}

// Decode the 64 weights of quarter q of tile j (4 input rows x 16 channels)
// into fp16 (the two halves of each 3INST word added and rounded once, RNE:
// the exact decoded weight) and hand them to put(byte offset in the 4 KB tile
// row, four 32-bit words), two 16-byte chunks per row.  soff[rb][e]: per-lane
// byte offset of the chunk holding channels 8e..8e+7 of a row with
// (row & 1) == rb; row >> 1 selects the 8-row K group (+2048 bytes).
template <int BITS, int NW, typename Put>
__device__ __forceinline__ void decode_quarter_to_a(const uint32_t (&buf)[NW], const uint32_t (&soff)[2][2],
                                                    uint32_t two16, Put&& put)
{
    auto body = [&](auto R, auto E) {
        constexpr int r = decltype(R)::value, e = decltype(E)::value;
        // channels 8e + 2c, 8e + 2c + 1 of row r -> one fp16 pair
        auto pair = [&](auto Cc) -> uint32_t {
            constexpr int c = decltype(Cc)::value;
            constexpr int ia = 16 * r + 8 * e + 2 * c, ib = ia + 1;
            const uint32_t ma = inst3(window_auto<BITS, ia, (ia + 1) * BITS + 16>(buf, two16));
            const uint32_t mb = inst3(window_auto<BITS, ib, (ib + 1) * BITS + 16>(buf, two16));
            return weight_pair_h(ma, mb);
        };
        put(soff[r & 1][e] + (r >> 1) * 2048, pair(std::integral_constant<int, 0>{}),
            pair(std::integral_constant<int, 1>{}), pair(std::integral_constant<int, 2>{}),
            pair(std::integral_constant<int, 3>{}));
    };
    [&]<int... RE>(std::integer_sequence<int, RE...>) {
        (body(std::integral_constant<int, RE / 2>{}, std::integral_constant<int, RE % 2>{}), ...);
    }(std::make_integer_sequence<int, 8>{});
}

// Per-lane chunk offsets of the layout above for lane (tile j = lane/4,
// quarter q = lane%4).
__device__ __forceinline__ void lane_soff(int lane, uint32_t (&soff)[2][2])
{
    const int q = lane & 3, j = lane >> 2, atom = j >> 2, j4 = j & 3;
#pragma unroll
    for (int rb = 0; rb < 2; ++rb)
#pragma unroll
        for (int e = 0; e < 2; ++e)
            soff[rb][e] = atom * 1024 + (4 * rb + q) * 128 + ((uint32_t)(chunk_of_tile(j4, e) ^ (4 * rb + q)) << 4);
}

}  // namespace exl3
