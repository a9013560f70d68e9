// exl3_aop.cuh -- the tensor-core operands of the trellis products.
//   A: one tile row of a 128-channel output block (128 channels x 16 input
//      rows, fp16, MN-major, 128-byte swizzle: 4 KB), written by the lanes of
//      one warp straight from their decoded weights.  Used by the verify
//      kernel (into shared memory) and by the large-M path (into a global
//      image of the whole matrix).
//   B: the rotated input H(su .* x) in the matching K order (xt_rotate_item),
//      used by the large-M path's pre-pass.
#pragma once
#include <cstdint>
#include <utility>

#include <cuda_fp16.h>

#include "exl3_common.cuh"
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
// decode_quarter_chunks does chunks RE0 .. RE1 - 1 only (chunk RE = 2 r + e:
// row r of the quarter, channels 8e .. 8e + 7), with the same arithmetic and
// window forms per weight; decode_quarter_to_a does all eight.
template <int BITS, int RE0, int RE1, int NW, typename Put>
__device__ __forceinline__ void decode_quarter_chunks(const uint32_t (&buf)[NW], const uint32_t (&soff)[2][2],
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
        (body(std::integral_constant<int, (RE0 + RE) / 2>{}, std::integral_constant<int, (RE0 + RE) % 2>{}), ...);
    }(std::make_integer_sequence<int, RE1 - RE0>{});
}

template <int BITS, int NW, typename Put>
__device__ __forceinline__ void decode_quarter_to_a(const uint32_t (&buf)[NW], const uint32_t (&soff)[2][2],
                                                    uint32_t two16, Put&& put)
{
    decode_quarter_chunks<BITS, 0, 8>(buf, soff, two16, static_cast<Put&&>(put));
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


// xt = H(su .* x) / sqrt(128) as the MMA's B operand (K-major, 128-byte
// swizzle), for one warp item (row m, four 128-blocks of K_in): item
// < m_pad * ceil(K_in / 512).  Rows m_rows .. m_pad - 1 are written as zeros.
// Layout: per tile of nb rows and 64 k, nb x 128 contiguous bytes; row r of
// the tile at (r >> 3) * 1024 + (r & 7) * 128, its 16-byte pieces swizzled by
// (r & 7); inside each 16-row group of k, row k = 4q + s sits at position
// 4s + q (the A image's order).  One lane takes 16 consecutive inputs (one
// tile row), loaded and stored 16 bytes at a time; the transform runs over
// index bits 0-3 in registers and bits 4-6 across the eight lanes of a group.
__device__ __forceinline__ void xt_rotate_item(const __half* __restrict__ x, const __half* __restrict__ su,
                                               int m_rows, int k_in, int nb, uint8_t* __restrict__ xt,
                                               long long item)
{
    const int lane = threadIdx.x & 31;
    const int nblk = k_in / 128, nb4 = (nblk + 3) / 4;
    const int m = (int)(item / nb4), b = 4 * (int)(item % nb4) + (lane >> 3), l8 = lane & 7;
    const bool valid = b < nblk;                                // uniform per lane group
    const int k0 = 128 * b + 16 * l8;
    float v[16];
    if (valid && m < m_rows) {
        const uint4* xp = reinterpret_cast<const uint4*>(x + (size_t)m * k_in + k0);
        const uint4* sp = reinterpret_cast<const uint4*>(su + k0);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 xv = xp[h], sv = sp[h];
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&xw[t]));
                const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sw[t]));
                v[8 * h + 2 * t] = xf.x * sf.x;
                v[8 * h + 2 * t + 1] = xf.y * sf.y;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
    }
#pragma unroll
    for (int d = 1; d < 16; d <<= 1)                            // index bits 0-3: in registers
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i & d) == 0) {
                const float a0 = v[i], a1 = v[i + d];
                v[i] = a0 + a1;
                v[i + d] = a0 - a1;
            }
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {                           // index bits 4-6: lanes of the group
        const bool upper = (l8 & d) != 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float p = __shfl_xor_sync(0xffffffffu, v[i], d);
            v[i] = upper ? (p - v[i]) : (v[i] + p);
        }
    }
    if (valid) {
        // tile row tr = 8b + l8; inside it, position p holds row k16 = 4(p & 3) + (p >> 2)
        const int tr = 8 * b + l8;
        const int kchunk = tr >> 2, c16 = 2 * (tr & 3);
        const int j = m / nb, mr = m % nb;
        uint8_t* base = xt + ((size_t)j * (k_in / 64) + kchunk) * nb * 128 + (mr >> 3) * 1024 + (mr & 7) * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t o[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int p0 = 8 * h + 2 * t, p1 = p0 + 1;
                const float f0 = v[4 * (p0 & 3) + (p0 >> 2)] * kInvSqrt128;
                const float f1 = v[4 * (p1 & 3) + (p1 >> 2)] * kInvSqrt128;
                const __half2 hh = __floats2half2_rn(f0, f1);
                o[t] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(base + (((c16 + h) ^ (mr & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace exl3
