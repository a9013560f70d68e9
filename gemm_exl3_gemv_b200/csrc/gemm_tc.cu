// gemm_tc.cu -- the verify-batch product (2..32 input rows) on the 5th-generation
// tensor cores (tcgen05), with the trellis decode on the CUDA cores.
//
// What is computed (the "WMMA GEMV for draft verification" / "batched
// verification up to 32 rows" the exl3-rdna4-recipe page describes in "What we
// added on top of upstream", here on B200):
//     y = sv .* H( scale .* ( H(su .* x) W ) ),   x: m x K_in, y: m x N_out
//
// Design:
//   * A pre-pass writes xt = H(su .* x) once per call, fp16, already laid out
//     as the MMA's B operand (K-major, 128-byte swizzle), m padded to NT = 16
//     or 32 rows with zeros.
//   * Persistent stream-K grid (at most one CTA per SM): the G x TR work units
//     (128-channel output block g, 16-row tile row tr) are cut into equal
//     contiguous ranges, one per CTA.  A range may cover the end of one block
//     and the start of the next; each (CTA, block) piece is a segment.
//   * Warp roles.  warp 0: 1-D bulk copies of packed tile rows (256*K bytes)
//     and xt chunks into shared-memory rings.  warp 1: allocates tensor memory
//     and issues the MMAs (one thread).  warps 2-5: drain the accumulators.
//     warps 6-13: decode.
//   * Decode straight into the A operand: the two fp16 halves of each 3INST
//     word are kept as two adjacent A rows (lo, hi) of the same input row k,
//     so the decoded 32-bit word is stored as is and the tensor core adds the
//     halves.  A is M = 128 rows (64 channels x lo/hi) by K = 16, MN-major with
//     the 128-byte swizzle; one tile row gives two such MMAs (channels 0-63,
//     64-127).  The order of the 16 k inside a tile row is permuted (the same
//     permutation is applied to xt) so that the 16-byte stores of the 32 lanes
//     are free of bank conflicts.
//   * Accumulators: two buffers x two channel halves x NT fp32 columns in
//     tensor memory; a segment's result is drained while the next segment
//     accumulates.  Segments of a block are combined by the last CTA to finish
//     (arrival counter) in segment order -- a fixed order, so results are
//     bitwise repeatable -- which then scales, rotates and writes y.
#include <atomic>
#include <utility>

#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"
#include "exl3_tc.cuh"

namespace exl3 {

namespace {

constexpr int kDecWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kTcWarps = 2 + kEpiWarps + kDecWarps;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kSP = 32;     // packed ring slots (one tile row each)
constexpr int kSA = 8;      // A stages (one tile row each)
constexpr int kSB = 4;      // xt stages (one 64-row chunk each)
constexpr int kABytes = 8192;
constexpr int kMaxCtas = 148;
constexpr int kMinUnitsPerCta = 24;

template <int BITS, int NT>
struct TcLayout {
    static constexpr int ROWB = 256 * BITS;                 // packed bytes per tile row
    static constexpr int BBYTES = NT * 128;                 // xt bytes per 64-row chunk
    static constexpr int TMEM_COLS = 4 * NT;                // 2 buffers x 2 halves x NT
    static constexpr int off_a = 0;
    static constexpr int off_b = off_a + kSA * kABytes;
    static constexpr int off_p = off_b + kSB * BBYTES;
    static constexpr int off_z = off_p + kSP * ROWB;
    static constexpr int off_bar = off_z + NT * 128 * 4;
    static constexpr int nbar = 2 * kSP + 2 * kSA + 2 * kSB + 4;
    static constexpr int off_misc = off_bar + nbar * 8;
    static constexpr int total = off_misc + 64 + 1024;      // + slack to align the base to 1024
    static_assert(off_b % 1024 == 0 && off_p % 16 == 0 && off_z % 16 == 0 && off_bar % 8 == 0, "layout");
};

struct TcParams {
    GemmArgs a;
    const uint8_t* xt;      // rotated input, B-operand layout
    float* part;            // segment partial sums, [slot][NT][128]
    uint32_t* counters;     // per output block
    uint32_t* status;       // workspace status word
    int G, TR, P;
    long long U;
};

__host__ __device__ inline int cta_of_unit(long long x, int P, long long U)
{
    return (int)(((x + 1) * P - 1) / U);
}

// Bounded wait; also gives up early once another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > 2000000000ull) {
            atomicExch((int*)abort_flag, 1);
            return false;
        }
    }
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Decode the 64 weights of quarter q of tile j (4 input rows x 16 channels)
// and store the raw 3INST words into the A stage at `ast` (see the layout in
// the file comment).  soff[rb][t]: per-lane byte offsets of the 16-byte chunk
// holding channels 4t..4t+3 of a row with (row & 1) == rb; row >> 1 selects
// the 8-row K group (+2048 bytes).
template <int BITS, int NW>
__device__ __forceinline__ void decode_quarter_to_a(const uint32_t (&buf)[NW], uint32_t ast, const uint32_t (&soff)[2][4])
{
    // fully unrolled over (row r, chunk t): every window position is a compile-time constant
    auto body = [&](auto R, auto T) {
        constexpr int r = decltype(R)::value, t = decltype(T)::value;
        const uint32_t m0 = inst3(window16<(16 * r + 4 * t + 1) * BITS + 16>(buf));
        const uint32_t m1 = inst3(window16<(16 * r + 4 * t + 2) * BITS + 16>(buf));
        const uint32_t m2 = inst3(window16<(16 * r + 4 * t + 3) * BITS + 16>(buf));
        const uint32_t m3 = inst3(window16<(16 * r + 4 * t + 4) * BITS + 16>(buf));
        sts128(ast + soff[r & 1][t] + (r >> 1) * 2048, m0, m1, m2, m3);
    };
    [&]<int... RT>(std::integer_sequence<int, RT...>) {
        (body(std::integral_constant<int, RT / 4>{}, std::integral_constant<int, RT % 4>{}), ...);
    }(std::make_integer_sequence<int, 16>{});
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(TcParams prm)
{
    using L = TcLayout<BITS, NT>;
    constexpr int TW = 8 * BITS, QW = 2 * BITS, ROWW = 8 * TW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::off_bar);
    uint64_t* pfull = bar;
    uint64_t* pempty = pfull + kSP;
    uint64_t* afull = pempty + kSP;
    uint64_t* aempty = afull + kSA;
    uint64_t* bfull = aempty + kSA;
    uint64_t* bempty = bfull + kSB;
    uint64_t* dfull = bempty + kSB;
    uint64_t* dempty = dfull + 2;
    int* misc = reinterpret_cast<int*>(smem + L::off_misc);   // [0] tmem base, [1] abort, [2] last-CTA flag
    volatile int* abort_flag = misc + 1;
    float* zsm = reinterpret_cast<float*>(smem + L::off_z);

    const GemmArgs& a = prm.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = blockIdx.x;
    const long long b0 = (long long)p * prm.U / prm.P;
    const long long b1 = (long long)(p + 1) * prm.U / prm.P;
    const int n = (int)(b1 - b0);
    const int TR = prm.TR;
    const int tiles_n = a.n_out / 16;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSP; ++i) { mbar_init(&pfull[i], 1); mbar_init(&pempty[i], 1); }
        for (int i = 0; i < kSA; ++i) { mbar_init(&afull[i], 1); mbar_init(&aempty[i], 1); }
        for (int i = 0; i < kSB; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&dfull[i], 1); mbar_init(&dempty[i], kEpiWarps); }
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(reinterpret_cast<uint32_t*>(&misc[0]), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];

    if (warp == 0) {
        // ------------------------------------------------------ producer ---
        if (lane == 0) {
            int bcount = 0;
            for (int u = 0; u < n; ++u) {
                const long long unit = b0 + u;
                const int g = (int)(unit / TR), tr = (int)(unit % TR);
                if (u == 0 || (tr & 3) == 0) {
                    const int bs = bcount % kSB;
                    if (!wait_or_abort(&bempty[bs], ((bcount / kSB) & 1) ^ 1, abort_flag)) break;
                    mbar_arrive_expect_tx(&bfull[bs], L::BBYTES);
                    bulk_g2s(smem + L::off_b + bs * L::BBYTES, prm.xt + (size_t)(tr >> 2) * L::BBYTES, L::BBYTES,
                             &bfull[bs]);
                    ++bcount;
                }
                const int s = u % kSP;
                if (!wait_or_abort(&pempty[s], ((u / kSP) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&pfull[s], L::ROWB);
                bulk_g2s(smem + L::off_p + s * L::ROWB, a.packed + ((size_t)tr * tiles_n + 8 * (size_t)g) * TW,
                         L::ROWB, &pfull[s]);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_amn(128, NT);
            int bcount = 0, seg = 0, cur_b = 0;
            for (int u = 0; u < n; ++u) {
                const long long unit = b0 + u;
                const int tr = (int)(unit % TR);
                const bool first = (u == 0) || (tr == 0);
                const bool last = (u == n - 1) || (tr == TR - 1);
                if (u == 0 || (tr & 3) == 0) {
                    cur_b = bcount % kSB;
                    if (!wait_or_abort(&bfull[cur_b], (bcount / kSB) & 1, abort_flag)) break;
                    ++bcount;
                }
                const int db = seg & 1;
                if (first && !wait_or_abort(&dempty[db], ((seg >> 1) & 1) ^ 1, abort_flag)) break;
                const int as = u % kSA;
                if (!wait_or_abort(&afull[as], (u / kSA) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t abase = smem_u32(smem + L::off_a + as * kABytes);
                const uint32_t bbase = smem_u32(smem + L::off_b + cur_b * L::BBYTES) + (tr & 3) * 32;
                const uint64_t bdesc = sdesc_sw128(bbase, 16, 1024);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    mma_f16_ss(tmem + db * 2 * NT + h * NT, sdesc_sw128(abase + h * 4096, 1024, 2048), bdesc, idesc,
                               first ? 0u : 1u);
                mma_commit(&aempty[as]);
                if ((tr & 3) == 3 || last) mma_commit(&bempty[cur_b]);
                if (last) {
                    mma_commit(&dfull[db]);
                    ++seg;
                }
            }
        }
    } else if (warp < 2 + kEpiWarps) {
        // ----------------------------------------------------- epilogue ---
        const int ew = warp - 2;            // 0..3
        const int quad = warp & 3;          // tensor-memory lanes 32*quad .. 32*quad+31
        const int et = threadIdx.x - 64;    // 0..127
        int seg = 0;
        for (long long u0 = 0; u0 < n; ++seg) {
            const long long unit = b0 + u0;
            const int g = (int)(unit / TR), tr0 = (int)(unit % TR);
            const long long len = (n - u0) < (TR - tr0) ? (n - u0) : (TR - tr0);
            u0 += len;
            const int db = seg & 1;
            if (!__all_sync(0xffffffffu, wait_or_abort(&dfull[db], (seg >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            uint32_t r[2][NT];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int c = 0; c < NT / 16; ++c) {
                    uint32_t t16[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + db * 2 * NT + h * NT + 16 * c, t16);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[h][16 * c + i] = t16[i];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dempty[db]);
            // rows 2c (lo) and 2c+1 (hi) of the accumulator belong to channel c
            const int v = 32 * quad + lane;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int mm = 0; mm < NT; ++mm) {
                    float s = __uint_as_float(r[h][mm]);
                    s += __shfl_xor_sync(0xffffffffu, s, 1);
                    if ((lane & 1) == 0) zsm[mm * 128 + 64 * h + (v >> 1)] = s;
                }
            }
            named_bar(1, 128);
            const int p_first = cta_of_unit((long long)g * TR, prm.P, prm.U);
            const int p_last = cta_of_unit((long long)(g + 1) * TR - 1, prm.P, prm.U);
            if (p_last > p_first) {
                float* myslot = prm.part + (size_t)(p + g) * NT * 128;
                for (int o = et; o < a.m * 128; o += 128) __stcg(myslot + o, zsm[o]);
                __threadfence();
                named_bar(1, 128);
                if (et == 0) {
                    const uint32_t prev = atomicAdd(&prm.counters[g], 1u);
                    misc[2] = (prev == (uint32_t)(p_last - p_first)) ? 1 : 0;
                }
                named_bar(1, 128);
                if (!misc[2]) continue;
                __threadfence();
                for (int o = et; o < a.m * 128; o += 128) {
                    float z = 0.f;
                    for (int q = p_first; q <= p_last; ++q) z += __ldcg(prm.part + (size_t)(q + g) * NT * 128 + o);
                    zsm[o] = z;
                }
                if (et == 0) prm.counters[g] = 0u;
                named_bar(1, 128);
            }
            // final epilogue for block g: scale, output rotation, signs, store
            for (int mm = ew; mm < a.m; mm += kEpiWarps) {
                const int n0 = 128 * g + 4 * lane;
                const float4 z4 = *reinterpret_cast<const float4*>(zsm + mm * 128 + 4 * lane);
                const uint2 sc = *reinterpret_cast<const uint2*>(a.scale + n0);
                const uint2 sg = *reinterpret_cast<const uint2*>(a.sv + n0);
                const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&sc.x));
                const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&sc.y));
                const float2 sg0 = __half22float2(*reinterpret_cast<const __half2*>(&sg.x));
                const float2 sg1 = __half22float2(*reinterpret_cast<const __half2*>(&sg.y));
                float vv[4] = {z4.x * sc0.x, z4.y * sc0.y, z4.z * sc1.x, z4.w * sc1.y};
                fwht128_warp(vv);
                vv[0] *= kInvSqrt128 * sg0.x;
                vv[1] *= kInvSqrt128 * sg0.y;
                vv[2] *= kInvSqrt128 * sg1.x;
                vv[3] *= kInvSqrt128 * sg1.y;
                const size_t yo = (size_t)mm * a.n_out + n0;
                if (a.y_fp32) {
                    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.y) + yo) =
                        make_float4(vv[0], vv[1], vv[2], vv[3]);
                } else {
                    __half2 hh[2] = {__floats2half2_rn(vv[0], vv[1]), __floats2half2_rn(vv[2], vv[3])};
                    *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(a.y) + yo) = *reinterpret_cast<uint2*>(hh);
                }
            }
            named_bar(1, 128);
        }
    } else {
        // ------------------------------------------------------ decoders ---
        const int d = warp - 2 - kEpiWarps;
        const int j = lane >> 2, q = lane & 3;
        const int src_prev = (lane & ~3) | ((q + 3) & 3);
        // per-lane store offsets inside an A stage (see decode_quarter_to_a)
        uint32_t soff[2][4];
        {
            const int hh = j >> 2, vgrp = (j >> 1) & 1;
#pragma unroll
            for (int rb = 0; rb < 2; ++rb)
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    soff[rb][t] = hh * 4096 + vgrp * 1024 + (4 * rb + q) * 128 +
                                  ((uint32_t)(4 * ((j & 1) ^ rb) + (t ^ q)) << 4);
        }
        const uint32_t* pring = reinterpret_cast<const uint32_t*>(smem + L::off_p);
        const uint32_t abase0 = smem_u32(smem + L::off_a);
        for (int u = d; u < n; u += kDecWarps) {
            const int s = u % kSP;
            if (!__all_sync(0xffffffffu, wait_or_abort(&pfull[s], (u / kSP) & 1, abort_flag))) break;
            const uint32_t* sw = pring + s * ROWW + j * TW + q * QW;
            uint32_t buf[QW + 1];
            if constexpr (QW % 4 == 0) {
#pragma unroll
                for (int t = 0; t < QW / 4; ++t) {
                    const uint4 vv = reinterpret_cast<const uint4*>(sw)[t];
                    buf[1 + 4 * t] = vv.x; buf[2 + 4 * t] = vv.y; buf[3 + 4 * t] = vv.z; buf[4 + 4 * t] = vv.w;
                }
            } else {
#pragma unroll
                for (int t = 0; t < QW / 2; ++t) {
                    const uint2 vv = reinterpret_cast<const uint2*>(sw)[t];
                    buf[1 + 2 * t] = vv.x; buf[2 + 2 * t] = vv.y;
                }
            }
            buf[0] = __shfl_sync(0xffffffffu, buf[QW], src_prev);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[s]);
            const int as = u % kSA;
            if (!__all_sync(0xffffffffu, wait_or_abort(&aempty[as], ((u / kSA) & 1) ^ 1, abort_flag))) break;
            decode_quarter_to_a<BITS>(buf, abase0 + as * kABytes, soff);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[as]);
        }
    }

    // ------------------------------------------------------------ teardown ---
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    if (threadIdx.x == 0 && misc[1]) atomicOr(prm.status, kStatusTimeout);
}

// xt = H(su .* x) / sqrt(128) for rows 0..NT-1 (zero rows past m), written in
// the B-operand layout: 64-row chunks of NT x 128 bytes, rows of 8 x 16-byte
// pieces swizzled by (row & 7), and inside each 16-row group k = 4q + r
// placed at position 8(r >> 1) + 4(r & 1) + q.
template <int NT>
__global__ void __launch_bounds__(256) xt_prepass_kernel(const __half* __restrict__ x, const __half* __restrict__ su,
                                                         int m_rows, int k_in, uint8_t* __restrict__ xt)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = k_in / 128;
    const long long item = (long long)blockIdx.x * 8 + warp;
    if (item >= (long long)NT * nblk) return;
    const int m = (int)(item / nblk), b = (int)(item % nblk);
    // lane holds elements i = (lane & 3) | (e << 2) | ((lane >> 2) << 4)
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int k = 128 * b + ((lane & 3) | (e << 2) | ((lane >> 2) << 4));
        v[e] = (m < m_rows) ? __half2float(x[(size_t)m * k_in + k]) * __half2float(su[k]) : 0.f;
    }
    fwht128_warp(v);   // the transform factors over index bits: any bit-to-(lane, e) map works
    const int tr = 8 * b + (lane >> 2);
    const int pk0 = 16 * tr + 8 * ((lane >> 1) & 1) + 4 * (lane & 1);
    const int kchunk = pk0 >> 6, o = pk0 & 63, c16 = o >> 3, pos = o & 7;
    uint8_t* dst = xt + (size_t)kchunk * NT * 128 + (m >> 3) * 1024 + (m & 7) * 128 + ((c16 ^ (m & 7)) << 4) + pos * 2;
    __half2 h2[2] = {__floats2half2_rn(v[0] * kInvSqrt128, v[1] * kInvSqrt128),
                     __floats2half2_rn(v[2] * kInvSqrt128, v[3] * kInvSqrt128)};
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<uint2*>(h2);
}

int nt_for(int m) { return m <= 16 ? 16 : 32; }

template <int BITS, int NT>
cudaError_t launch_tc_t(const GemmArgs& a, cudaStream_t stream)
{
    using L = TcLayout<BITS, NT>;
    TcParams prm;
    prm.a = a;
    prm.G = a.n_out / 128;
    prm.TR = a.k_in / 16;
    prm.U = (long long)prm.G * prm.TR;
    prm.P = tc_ctas(a.m, a.k_in, a.n_out, a.bits);
    uint8_t* ws = a.ws;
    prm.status = reinterpret_cast<uint32_t*>(ws);
    prm.counters = reinterpret_cast<uint32_t*>(ws + ws_counter_off());
    const size_t xt_off = align_up(ws_counter_off() + 4 * (size_t)prm.G, 1024);
    prm.xt = ws + xt_off;
    prm.part = reinterpret_cast<float*>(ws + align_up(xt_off + (size_t)a.k_in * NT * 2, 256));

    const long long items = (long long)NT * (a.k_in / 128);
    xt_prepass_kernel<NT><<<(unsigned)((items + 7) / 8), 256, 0, stream>>>(
        reinterpret_cast<const __half*>(a.x), reinterpret_cast<const __half*>(a.su), a.m, a.k_in, ws + xt_off);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    auto kern = gemm_tc_kernel<BITS, NT>;
    static std::atomic<int> configured{0};
    if (!configured.load()) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::total);
        if (e != cudaSuccess) return e;
        configured.store(1);
    }
    kern<<<prm.P, kTcThreads, L::total, stream>>>(prm);
    return cudaGetLastError();
}

}  // namespace

int tc_ctas(int m, int k_in, int n_out, int bits)
{
    (void)m;
    (void)bits;
    const long long U = (long long)(n_out / 128) * (k_in / 16);
    long long p = U / kMinUnitsPerCta;
    if (p > kMaxCtas) p = kMaxCtas;
    if (p < 1) p = 1;
    return (int)p;
}

size_t tc_workspace_bytes(int m, int k_in, int n_out, int bits)
{
    const int NT = nt_for(m);
    const int G = n_out / 128;
    const size_t xt_off = align_up(ws_counter_off() + 4 * (size_t)G, 1024);
    const size_t part_off = align_up(xt_off + (size_t)k_in * NT * 2, 256);
    return part_off + (size_t)(tc_ctas(m, k_in, n_out, bits) + G) * NT * 128 * sizeof(float);
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream)
{
    const bool wide = nt_for(a.m) == 32;
    switch (a.bits) {
        case 2: return wide ? launch_tc_t<2, 32>(a, stream) : launch_tc_t<2, 16>(a, stream);
        case 3: return wide ? launch_tc_t<3, 32>(a, stream) : launch_tc_t<3, 16>(a, stream);
        case 4: return wide ? launch_tc_t<4, 32>(a, stream) : launch_tc_t<4, 16>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace exl3
