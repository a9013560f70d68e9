// gemv_cc.cu -- fused decode-and-dot product on CUDA cores for 1..4 input rows.
//
// The product (the decode-time matrix-vector step the pages' GEMV kernels
// serve: orcasaq2-rocm README, second paragraph, "EXL3 GEMM kernels were
// rewritten for RDNA's vector ALUs"):
//     y = sv .* H( scale .* ( H(su .* x) W ) )
// with W decoded on the fly from the trellis stream (exl3_decode.cuh).
//
// Work decomposition (B200: 148 SMs, bulk copies, warp shuffles):
//   * CTA (g, s): output channels [128g, 128g+128) -- one Hadamard block --
//     and the s-th of `splits` contiguous ranges of 128-row input blocks.
//   * The CTA rotates its slice of x (su, Hadamard-128) into shared memory.
//   * Each of the 8 warps streams whole tile rows (8 tiles = 16 input rows x
//     128 channels, 256*K contiguous bytes) through its own ring of shared
//     memory slots filled by 1-D bulk copies (cp.async.bulk + mbarrier).
//   * Lane l decodes the 64 consecutive weights of quarter l%4 of tile l/4:
//     4 input rows x 16 channels.  The quarter's bits start on a word
//     boundary (64*K bits = 2K words); the 16-bit look-back comes from the
//     neighbouring lane by a shuffle (the tail-biting wrap for quarter 0).
//   * Split-K partial sums go to the workspace; the last CTA of a channel
//     block (atomic arrival counter) adds them in split order -- fixed, so
//     results are bitwise repeatable -- scales, rotates and writes y.
#include <atomic>

#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"

namespace exl3 {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 4;   // ring slots per warp

template <int MR>
struct Acc {
    float v[MR][16];
};

// Decode the 64 weights of a quarter tile and accumulate w * xt.
template <int BITS, int MR, int R, int NW>
__device__ __forceinline__ void quarter_mac(const uint32_t (&buf)[NW], const float (&xv)[MR][4], Acc<MR>& acc)
{
    if constexpr (R < 64) {
        const uint32_t m = inst3(window16<(R + 1) * BITS + 16>(buf));
        const float w = __half2float(weight_of(m));
#pragma unroll
        for (int mr = 0; mr < MR; ++mr) acc.v[mr][R & 15] = fmaf(w, xv[mr][R >> 4], acc.v[mr][R & 15]);
        quarter_mac<BITS, MR, R + 1>(buf, xv, acc);
    }
}

struct SmemPlan {
    size_t bars, ring, xt, red, flag, total;
};

template <int BITS, int MR>
__host__ __device__ inline SmemPlan smem_plan(int krange_max)
{
    SmemPlan p;
    p.bars = 0;
    p.ring = align_up(sizeof(uint64_t) * kWarps * kStages, 128);
    const size_t slot = 256 * BITS;                               // one tile row of a 128-channel block
    p.xt = align_up(p.ring + slot * kWarps * kStages, 128);
    p.red = align_up(p.xt + sizeof(float) * MR * (size_t)krange_max, 128);
    p.flag = align_up(p.red + sizeof(float) * kWarps * MR * 128, 16);
    p.total = p.flag + 16;
    return p;
}

template <int BITS, int MR>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_cc_kernel(GemmArgs a, int splits, int krange_max, int row0, int rows)
{
    constexpr int TW = 8 * BITS;        // words per tile
    constexpr int QW = 2 * BITS;        // words per quarter tile
    constexpr int ROWW = 8 * TW;        // words per tile row of the channel block
    extern __shared__ __align__(1024) unsigned char smem[];
    const SmemPlan plan = smem_plan<BITS, MR>(krange_max);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + plan.bars);
    uint32_t* ring = reinterpret_cast<uint32_t*>(smem + plan.ring);
    float* xt = reinterpret_cast<float*>(smem + plan.xt);
    float* red = reinterpret_cast<float*>(smem + plan.red);
    int* flag = reinterpret_cast<int*>(smem + plan.flag);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x, s = blockIdx.y;
    const int kb_total = a.k_in / 128;
    const int kb0 = (int)((long long)s * kb_total / splits);
    const int kb1 = (int)((long long)(s + 1) * kb_total / splits);
    const int tk0 = kb0 * 8, ntk = (kb1 - kb0) * 8;      // tile rows of this split
    const int tiles_n = a.n_out / 16;
    const uint32_t* base = a.packed + ((size_t)tk0 * tiles_n + 8 * (size_t)g) * TW;
    const size_t row_stride = (size_t)tiles_n * TW;      // words between consecutive tile rows
    const int nmine = ntk > warp ? (ntk - warp + kWarps - 1) / kWarps : 0;   // rows warp, warp+8, ...
    uint64_t* mybars = bars + warp * kStages;
    uint32_t* myring = ring + (size_t)warp * kStages * ROWW;

    if (threadIdx.x == 0) flag[0] = 0;
    if (lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&mybars[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (lane == 0) {
        for (int u = 0; u < kStages && u < nmine; ++u) {
            mbar_arrive_expect_tx(&mybars[u], ROWW * 4);
            bulk_g2s(myring + u * ROWW, base + (size_t)(warp + u * kWarps) * row_stride, ROWW * 4, &mybars[u]);
        }
    }

    // ---- input rotation of this split's slice: xt[mr][k] = H(su .* x) ----
    const int nkb = kb1 - kb0;
    for (int item = warp; item < MR * nkb; item += kWarps) {
        const int mr = item / nkb, kb = item % nkb;
        const int col = (kb0 + kb) * 128 + 4 * lane;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (mr < rows) {
            const uint2 raw = *reinterpret_cast<const uint2*>(a.x + (size_t)(row0 + mr) * a.k_in + col);
            const uint2 sraw = *reinterpret_cast<const uint2*>(a.su + col);
            const float2 x0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 x1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            const float2 s0 = __half22float2(*reinterpret_cast<const __half2*>(&sraw.x));
            const float2 s1 = __half22float2(*reinterpret_cast<const __half2*>(&sraw.y));
            v[0] = x0.x * s0.x; v[1] = x0.y * s0.y; v[2] = x1.x * s1.x; v[3] = x1.y * s1.y;
        }
        fwht128_warp(v);
        float4 o = make_float4(v[0] * kInvSqrt128, v[1] * kInvSqrt128, v[2] * kInvSqrt128, v[3] * kInvSqrt128);
        *reinterpret_cast<float4*>(xt + (size_t)mr * krange_max + kb * 128 + 4 * lane) = o;
    }
    __syncthreads();

    // ---- main loop: this warp's tile rows ----
    const int j = lane >> 2, q = lane & 3;
    const int src_prev = (lane & ~3) | ((q + 3) & 3);
    Acc<MR> acc;
#pragma unroll
    for (int mr = 0; mr < MR; ++mr)
#pragma unroll
        for (int c = 0; c < 16; ++c) acc.v[mr][c] = 0.f;
    bool timed_out = false;
    int u = 0;
    for (; u < nmine; ++u) {
        const int slot = u % kStages;
        const uint32_t par = (uint32_t)(u / kStages) & 1u;
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&mybars[slot], par));
        if (!ok) { timed_out = true; break; }
        const uint32_t* sw = myring + slot * ROWW + j * TW + q * QW;
        uint32_t buf[QW + 1];
        if constexpr (QW % 4 == 0) {
#pragma unroll
            for (int t = 0; t < QW / 4; ++t) {
                const uint4 v = reinterpret_cast<const uint4*>(sw)[t];
                buf[1 + 4 * t] = v.x; buf[2 + 4 * t] = v.y; buf[3 + 4 * t] = v.z; buf[4 + 4 * t] = v.w;
            }
        } else {
#pragma unroll
            for (int t = 0; t < QW / 2; ++t) {
                const uint2 v = reinterpret_cast<const uint2*>(sw)[t];
                buf[1 + 2 * t] = v.x; buf[2 + 2 * t] = v.y;
            }
        }
        buf[0] = __shfl_sync(0xffffffffu, buf[QW], src_prev);
        __syncwarp();
        if (lane == 0 && u + kStages < nmine) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&mybars[slot], ROWW * 4);
            bulk_g2s(myring + slot * ROWW, base + (size_t)(warp + (u + kStages) * kWarps) * row_stride, ROWW * 4,
                     &mybars[slot]);
        }
        const int krel = (warp + u * kWarps) * 16 + 4 * q;
        float xv[MR][4];
#pragma unroll
        for (int mr = 0; mr < MR; ++mr) {
            const float4 t = *reinterpret_cast<const float4*>(xt + (size_t)mr * krange_max + krel);
            xv[mr][0] = t.x; xv[mr][1] = t.y; xv[mr][2] = t.z; xv[mr][3] = t.w;
        }
        quarter_mac<BITS, MR, 0>(buf, xv, acc);
    }
    if (timed_out) {
        // let copies already issued into this warp's ring land (bounded) before the CTA can exit
        for (int v = u; v < nmine && v < u + kStages; ++v)
            (void)mbar_wait_bounded(&mybars[v % kStages], (uint32_t)(v / kStages) & 1u, 100000000ull);
        if (lane == 0) atomicOr(flag, 1);
    }

    // ---- reduce: the 4 quarters of a tile, then the 8 warps (fixed order) ----
#pragma unroll
    for (int mr = 0; mr < MR; ++mr)
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float t = acc.v[mr][c];
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            acc.v[mr][c] = t;
        }
    if (q == 0) {
#pragma unroll
        for (int mr = 0; mr < MR; ++mr) {
            float4* d = reinterpret_cast<float4*>(red + ((size_t)warp * MR + mr) * 128 + 16 * j);
#pragma unroll
            for (int t = 0; t < 4; ++t)
                d[t] = make_float4(acc.v[mr][4 * t], acc.v[mr][4 * t + 1], acc.v[mr][4 * t + 2], acc.v[mr][4 * t + 3]);
        }
    }
    __syncthreads();
    float zpart[MR > 1 ? (MR * 128 + kThreads - 1) / kThreads : 1];
#pragma unroll
    for (int t = 0; t < (MR * 128 + kThreads - 1) / kThreads; ++t) {
        const int o = threadIdx.x + t * kThreads;
        float z = 0.f;
        if (o < MR * 128) {
#pragma unroll
            for (int w = 0; w < kWarps; ++w) z += red[(size_t)w * MR * 128 + o];
        }
        zpart[t] = z;
    }

    // ---- split-K: last-arriving CTA of this channel block finishes ----
    float* part = reinterpret_cast<float*>(a.ws + ws_part_off(a.n_out));
    uint32_t* counters = reinterpret_cast<uint32_t*>(a.ws + ws_counter_off());
    __syncthreads();   // everyone done reading `red`
    if (splits > 1) {
#pragma unroll
        for (int t = 0; t < (MR * 128 + kThreads - 1) / kThreads; ++t) {
            const int o = threadIdx.x + t * kThreads;
            if (o < MR * 128) {
                const int mr = o / 128, n = o % 128;
                if (mr < rows)
                    __stcg(part + ((size_t)s * a.m + row0 + mr) * a.n_out + 128 * g + n, zpart[t]);
            }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const uint32_t prev = atomicAdd(&counters[g], 1u);
            flag[1] = (prev == (uint32_t)splits - 1) ? 1 : 0;
        }
        __syncthreads();
        if (!flag[1]) {
            if (threadIdx.x == 0 && flag[0]) atomicOr(reinterpret_cast<uint32_t*>(a.ws), kStatusTimeout);
            return;
        }
        __threadfence();
        // sum the partials in split order into `red` (as z[mr][n]); loads are
        // issued 8 splits at a time so that they are in flight together
#pragma unroll
        for (int t = 0; t < (MR * 128 + kThreads - 1) / kThreads; ++t) {
            const int o = threadIdx.x + t * kThreads;
            if (o < MR * 128) {
                const int mr = o / 128, n = o % 128;
                float z = 0.f;
                if (mr < rows) {
                    const float* src = part + ((size_t)row0 + mr) * a.n_out + 128 * g + n;
                    const size_t stride = (size_t)a.m * a.n_out;
                    int ss = 0;
                    for (; ss + 8 <= splits; ss += 8) {
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] = __ldcg(src + (size_t)(ss + e) * stride);
#pragma unroll
                        for (int e = 0; e < 8; ++e) z += v[e];
                    }
                    for (; ss < splits; ++ss) z += __ldcg(src + (size_t)ss * stride);
                }
                red[o] = z;
            }
        }
        if (threadIdx.x == 0) counters[g] = 0u;   // ready for the next call on this stream
    } else {
#pragma unroll
        for (int t = 0; t < (MR * 128 + kThreads - 1) / kThreads; ++t) {
            const int o = threadIdx.x + t * kThreads;
            if (o < MR * 128) red[o] = zpart[t];
        }
    }
    if (threadIdx.x == 0 && flag[0]) atomicOr(reinterpret_cast<uint32_t*>(a.ws), kStatusTimeout);
    __syncthreads();

    // ---- epilogue: scale, output rotation, signs, store ----
    if (warp < MR && warp < rows) {
        const int mr = warp;
        const int n0 = 128 * g + 4 * lane;
        const float4 z4 = *reinterpret_cast<const float4*>(red + mr * 128 + 4 * lane);
        const uint2 sc = *reinterpret_cast<const uint2*>(a.scale + n0);
        const uint2 sg = *reinterpret_cast<const uint2*>(a.sv + n0);
        const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&sc.x));
        const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&sc.y));
        const float2 sg0 = __half22float2(*reinterpret_cast<const __half2*>(&sg.x));
        const float2 sg1 = __half22float2(*reinterpret_cast<const __half2*>(&sg.y));
        float v[4] = {z4.x * sc0.x, z4.y * sc0.y, z4.z * sc1.x, z4.w * sc1.y};
        fwht128_warp(v);
        v[0] *= kInvSqrt128 * sg0.x;
        v[1] *= kInvSqrt128 * sg0.y;
        v[2] *= kInvSqrt128 * sg1.x;
        v[3] *= kInvSqrt128 * sg1.y;
        const size_t yo = (size_t)(row0 + mr) * a.n_out + n0;
        if (a.y_fp32) {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.y) + yo) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            __half2 h[2] = {__floats2half2_rn(v[0], v[1]), __floats2half2_rn(v[2], v[3])};
            *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(a.y) + yo) = *reinterpret_cast<uint2*>(h);
        }
    }
}

template <int BITS, int MR>
cudaError_t launch_t(const GemmArgs& a, int splits, int row0, int rows, cudaStream_t stream)
{
    const int kb_total = a.k_in / 128;
    const int krange_max = ((kb_total + splits - 1) / splits) * 128;
    const SmemPlan plan = smem_plan<BITS, MR>(krange_max);
    auto kern = gemv_cc_kernel<BITS, MR>;
    // raise the dynamic shared-memory limit once per kernel (not per launch, so
    // launches can be captured in a CUDA graph after the first call)
    static std::atomic<int> configured{0};
    if ((int)plan.total > configured.load()) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        configured.store(200 * 1024);
    }
    dim3 grid(a.n_out / 128, splits);
    kern<<<grid, kThreads, plan.total, stream>>>(a, splits, krange_max, row0, rows);
    return cudaGetLastError();
}

template <int MR>
cudaError_t launch_bits(const GemmArgs& a, int splits, int row0, int rows, cudaStream_t stream)
{
    switch (a.bits) {
        case 2: return launch_t<2, MR>(a, splits, row0, rows, stream);
        case 3: return launch_t<3, MR>(a, splits, row0, rows, stream);
        case 4: return launch_t<4, MR>(a, splits, row0, rows, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

int cc_splits(int m, int k_in, int n_out, int bits)
{
    (void)bits;
    const int groups = n_out / 128, kb = k_in / 128;
    const int target = 2 * 148;                      // two CTAs per SM on B200
    int s = (target + groups - 1) / groups;
    if (s > kb) s = kb;
    // keep the rotated input slice within a comfortable shared-memory budget
    const int mr = m < 4 ? m : 4;
    while (s < kb && (size_t)((kb + s - 1) / s) * 128 * mr * 4 > 96 * 1024) ++s;
    return s < 1 ? 1 : s;
}

size_t cc_workspace_bytes(int m, int k_in, int n_out, int bits)
{
    const int s = cc_splits(m, k_in, n_out, bits);
    return ws_part_off(n_out) + (size_t)s * m * n_out * sizeof(float);
}

int cc_launches(int m) { return (m + 3) / 4; }

cudaError_t launch_gemv_cc(const GemmArgs& a, cudaStream_t stream)
{
    const int splits = cc_splits(a.m, a.k_in, a.n_out, a.bits);
    for (int r0 = 0; r0 < a.m; r0 += 4) {
        const int rows = a.m - r0 < 4 ? a.m - r0 : 4;
        cudaError_t e;
        switch (rows) {
            case 1: e = launch_bits<1>(a, splits, r0, rows, stream); break;
            case 2: e = launch_bits<2>(a, splits, r0, rows, stream); break;
            default: e = launch_bits<4>(a, splits, r0, rows, stream); break;
        }
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace exl3
