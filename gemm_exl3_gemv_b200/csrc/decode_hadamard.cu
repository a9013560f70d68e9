// decode_hadamard.cu -- exl3_decode_tiles and exl3_hadamard128 kernels.
//
// Decode: the trellis definition is the one in exl3_decode.cuh (EXL3 trellis
// format, named on the orcasaq2-rocm README, opening paragraph).  Each thread
// decodes a run of 32 consecutive weights of one tile (two tile rows); the
// run's bits start on a word boundary (32*K bits = K words), so every window
// position is a compile-time constant.
//
// Hadamard: normalised 128-point Hadamard with a +-1 sign vector on each
// contiguous 128-element block (the rotation the format applies on both
// sides of the product).
#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"

namespace exl3 {

template <int BITS, int R, int NW>
__device__ __forceinline__ void decode_run32(const uint32_t (&buf)[NW], uint32_t (&out)[16])
{
    if constexpr (R < 32) {
        // buf[0] is the word before the run; weight R's window starts at
        // bit 32 + (R+1)*BITS - 16 of buf.
        const uint32_t m0 = inst3(window16<(R + 1) * BITS + 16>(buf));
        const uint32_t m1 = inst3(window16<(R + 2) * BITS + 16>(buf));
        __half2 p = __halves2half2(weight_of(m0), weight_of(m1));
        out[R / 2] = *reinterpret_cast<uint32_t*>(&p);
        decode_run32<BITS, R + 2>(buf, out);
    }
}

template <int BITS>
__global__ void __launch_bounds__(256) decode_tiles_kernel(const uint32_t* __restrict__ packed, int k_in,
                                                           int n_out, uint16_t* __restrict__ w_out)
{
    constexpr int TW = 8 * BITS;                  // words per tile
    const long long tiles = (long long)(k_in / 16) * (n_out / 16);
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long tile = gid >> 3;
    const int run = (int)(gid & 7);               // 32-weight run: tile rows 2*run, 2*run+1
    if (tile >= tiles) return;
    const uint32_t* tw = packed + tile * TW;
    uint32_t buf[BITS + 1];
    buf[0] = __ldg(tw + ((run * BITS + TW - 1) % TW));   // word before the run (tail-biting)
#pragma unroll
    for (int j = 0; j < BITS; ++j) buf[1 + j] = __ldg(tw + run * BITS + j);
    uint32_t h[16];
    decode_run32<BITS, 0>(buf, h);
    const int tiles_n = n_out / 16;
    const long long tk = tile / tiles_n, tn = tile % tiles_n;
    uint16_t* row0 = w_out + (tk * 16 + 2 * run) * (long long)n_out + tn * 16;
    uint4* d0 = reinterpret_cast<uint4*>(row0);
    uint4* d1 = reinterpret_cast<uint4*>(row0 + n_out);
    d0[0] = make_uint4(h[0], h[1], h[2], h[3]);
    d0[1] = make_uint4(h[4], h[5], h[6], h[7]);
    d1[0] = make_uint4(h[8], h[9], h[10], h[11]);
    d1[1] = make_uint4(h[12], h[13], h[14], h[15]);
}

cudaError_t launch_decode_tiles(const uint32_t* packed, int k_in, int n_out, int bits, uint16_t* w_out,
                                cudaStream_t stream)
{
    const long long threads = (long long)(k_in / 16) * (n_out / 16) * 8;
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    switch (bits) {
        case 2: decode_tiles_kernel<2><<<blocks, 256, 0, stream>>>(packed, k_in, n_out, w_out); break;
        case 3: decode_tiles_kernel<3><<<blocks, 256, 0, stream>>>(packed, k_in, n_out, w_out); break;
        case 4: decode_tiles_kernel<4><<<blocks, 256, 0, stream>>>(packed, k_in, n_out, w_out); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// One warp per 128-element block; 8 warps per CTA.
__global__ void __launch_bounds__(256) hadamard128_kernel(const __half* in, __half* out,
                                                          const __half* __restrict__ signs, long long rows,
                                                          int n, int mode)
{
    const long long blocks_per_row = n / 128;
    const long long blk = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (blk >= rows * blocks_per_row) return;
    const int lane = threadIdx.x & 31;
    const long long row = blk / blocks_per_row;
    const int col = (int)(blk % blocks_per_row) * 128 + 4 * lane;
    const __half* src = in + row * n + col;
    uint2 raw = *reinterpret_cast<const uint2*>(src);
    uint2 sraw = *reinterpret_cast<const uint2*>(signs + col);
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
    const __half2* s = reinterpret_cast<const __half2*>(&sraw);
    float v[4], sg[4];
    float2 t0 = __half22float2(h[0]), t1 = __half22float2(h[1]);
    float2 u0 = __half22float2(s[0]), u1 = __half22float2(s[1]);
    v[0] = t0.x; v[1] = t0.y; v[2] = t1.x; v[3] = t1.y;
    sg[0] = u0.x; sg[1] = u0.y; sg[2] = u1.x; sg[3] = u1.y;
    if (mode == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] *= sg[e];
    }
    fwht128_warp(v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[e] *= kInvSqrt128;
        if (mode == 1) v[e] *= sg[e];
    }
    __half2 o[2] = {__floats2half2_rn(v[0], v[1]), __floats2half2_rn(v[2], v[3])};
    *reinterpret_cast<uint2*>(out + row * n + col) = *reinterpret_cast<uint2*>(o);
}

cudaError_t launch_hadamard128(const uint16_t* in, uint16_t* out, const uint16_t* signs, int rows, int n, int mode,
                               cudaStream_t stream)
{
    const long long nblk = (long long)rows * (n / 128);
    const unsigned grid = (unsigned)((nblk + 7) / 8);
    hadamard128_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const __half*>(in), reinterpret_cast<__half*>(out),
                                                 reinterpret_cast<const __half*>(signs), rows, n, mode);
    return cudaGetLastError();
}

}  // namespace exl3
