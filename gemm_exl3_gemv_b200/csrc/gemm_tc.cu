// gemm_tc.cu -- the verify-batch product (2..32 input rows) on the 5th-generation
// tensor cores (tcgen05), with the trellis decode on the CUDA cores.
//
// What is computed (the "WMMA GEMV for draft verification" / "batched
// verification up to 32 rows" the exl3-rdna4-recipe page describes in "What we
// added on top of upstream", here on B200):
//     y = sv .* H( scale .* ( H(su .* x) W ) ),   x: m x K_in, y: m x N_out
//
// Design (each choice measured on B200):
//   * A pre-pass writes xt = H(su .* x) once per call, fp16, already laid out
//     as the MMA's B operand (K-major, 128-byte swizzle), m padded to NT = 16
//     or 32 rows with zeros.
//   * Work unit = one 64-row chunk of K_in for one 128-channel output block
//     (4 tile rows, 8192 weights).  Persistent stream-K grid: the G x C units
//     are cut into equal contiguous ranges, at most one CTA per SM.  A range
//     may cover the end of one block and the start of the next; each
//     (CTA, block) piece is a segment.
//   * Decode straight into the A operand: the two fp16 halves of each 3INST
//     word are kept as two adjacent A rows (lo, hi) of the same input row k,
//     so the decoded 32-bit word is stored as is and the tensor core adds the
//     halves.  A is M = 128 rows (64 channels x lo/hi) by K = 16, MN-major with
//     the 128-byte swizzle; one tile row gives two MMAs (channels 0-63,
//     64-127).  The 16 k of a tile row are permuted (the same permutation is
//     applied to xt) so that the 16-byte stores of a warp hit distinct banks.
//   * 16 decoder warps (4 per scheduler, enough to keep the integer pipes
//     busy); decoder d always decodes tile row d%4 of the units u = d/4
//     (mod 4) into its own A stage and fetches its own packed words with 1-D bulk copies into a
//     private 3-slot ring -- bulk-copy issue costs ~85 ns per copy per thread,
//     so it is spread over 16 threads.
//   * 4 MMA-issuing threads (one per warp).  A thread that waits on a barrier
//     right after issuing MMAs stalls until they drain (~0.1 us), so a single
//     issuer cannot keep the tensor core busy; issuer i takes every unit
//     u = i (mod 4) (8 MMAs per barrier wait) into its own accumulator, the
//     four interleave on the tensor core, and the epilogue adds the four
//     accumulators in a fixed order.
//   * Accumulators in tensor memory: 4 issuers x 2 buffers x 2 channel halves
//     x NT fp32 columns; a segment is drained while the next accumulates.
//     Segments of a block are combined by the last CTA to finish (arrival
//     counter) in segment order -- fixed, so results are bitwise repeatable --
//     which then scales, rotates and writes y.
//   * Every wait is bounded (2 s); on expiry the CTA records a timeout in the
//     workspace status word and winds down.
#include <atomic>
#include <utility>

#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"
#include "exl3_tc.cuh"

namespace exl3 {

namespace {

constexpr int kDecWarps = 16;
constexpr int kIssuers = 4;
constexpr int kEpiWarps = 4;
constexpr int kWarpProd0 = 0;                         // warps 0..3 issue the bulk copies of slots 0..3
constexpr int kWarpIss0 = 4;                          // warps 4..7 issue MMAs
constexpr int kWarpEpi0 = kWarpIss0 + kIssuers;       // warps 8..11 drain accumulators
constexpr int kWarpDec0 = kWarpEpi0 + kEpiWarps;      // warps 12..27 decode
constexpr int kTcWarps = kWarpDec0 + kDecWarps;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kRing = 3;      // packed-word slots per decoder
constexpr int kSB = 2;        // xt chunk stages per slot
constexpr int kABytes = 4096; // one tile row of A (128 channels x 16 k, fp16)
constexpr int kABuf = 2;      // A stages per decoder (double buffered)
constexpr int kMaxCtas = 148;
constexpr int kMinUnitsPerCta = 10;
// Suspend hints for barrier waits (ns): waiting threads are parked in
// hardware instead of polling, leaving the issue slots to the decoders.
constexpr uint32_t kSleepNs = 2000;
constexpr uint32_t kIssSleepNs = 1000;
constexpr uint32_t kEpiSleepNs = 20000;

template <int BITS, int NT>
struct TcLayout {
    static constexpr int ROWB = 256 * BITS;                 // packed bytes per tile row
    static constexpr int BBYTES = NT * 128;                 // xt bytes per 64-row chunk
    static constexpr int TMEM_COLS = kIssuers * 2 * NT;     // issuers x buffers x NT columns
    static constexpr int off_a = 0;                          // kABuf x kDecWarps A stages
    static constexpr int off_b = off_a + kABuf * kDecWarps * kABytes;
    static constexpr int off_p = off_b + kIssuers * kSB * BBYTES;
    static constexpr int off_z = off_p + kDecWarps * kRing * ROWB;
    static constexpr int off_bar = off_z + NT * 128 * 4;
    // pfull[dec][ring], pempty[dec][ring], afull[slot][buf], aempty[slot][buf], bfull[slot][SB],
    // bempty[slot][SB], dfull[iss][2], dempty[iss][2]
    static constexpr int nbar = 2 * kDecWarps * kRing + 2 * kIssuers * kABuf + 2 * kIssuers * kSB + 4 * kIssuers;
    static constexpr int off_misc = off_bar + nbar * 8;
    static constexpr int total = off_misc + 64 + 1024;      // + slack to align the base to 1024
    static_assert(off_b % 1024 == 0 && off_p % 16 == 0 && off_z % 16 == 0 && off_bar % 8 == 0, "layout");
    static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512, "tensor memory");
    static_assert(total <= 227 * 1024, "shared memory");
};

struct TcParams {
    GemmArgs a;
    const uint8_t* xt;      // rotated input, B-operand layout
    float* part;            // segment partial sums, [slot][NT][128]
    uint32_t* counters;     // per output block
    uint32_t* status;       // workspace status word
    int G, C, P;            // output blocks, 64-row chunks per block, CTAs
    long long U;            // units = G * C
};

__host__ __device__ inline int cta_of_unit(long long x, int P, long long U)
{
    return (int)(((x + 1) * P - 1) / U);
}

// Bounded wait; also gives up early once another role has aborted.  With
// sleep_ns > 0 the thread may be suspended in hardware between checks (it is
// resumed when the phase completes).
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              uint32_t sleep_ns = 0)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 8; ++i) {
            if (sleep_ns ? mbar_try_wait_sleep(bar, parity, sleep_ns) : mbar_try_wait(bar, parity)) return true;
        }
        if (*abort_flag) return false;
        if (global_ns() - t0 > 2000000000ull) {
            atomicExch((int*)abort_flag, 1);
            return false;
        }
    }
}

// Warp-wide wait: lane 0 polls, the outcome is broadcast, then every lane
// observes the completed phase once itself (acquire for each thread).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t sleep_ns = 0)
{
    // fast path: the phase is usually complete already -- one check per lane
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, abort_flag, sleep_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
        // the phase has completed and cannot advance again before this warp
        // acts on it, so this succeeds at once; bounded all the same
        int tries = 0;
        while (!mbar_try_wait(bar, parity) && ++tries < (1 << 20)) {
        }
        ok = __all_sync(0xffffffffu, tries < (1 << 20)) ? 1 : 0;
        if (!ok && (threadIdx.x & 31) == 0) atomicExch((int*)abort_flag, 1);
    }
    return ok != 0;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Decode the 64 weights of quarter q of tile j (4 input rows x 16 channels)
// into fp16 (the two halves of each 3INST word added and rounded once, RNE:
// the exact decoded weight) and store them into the A stage at `ast`, two
// 16-byte chunks per row.  soff[rb][e]: per-lane byte offset of the chunk
// holding channels 8e..8e+7 of a row with (row & 1) == rb; row >> 1 selects
// the 8-row K group (+2048 bytes).
template <int BITS, int NW>
__device__ __forceinline__ void decode_quarter_to_a(const uint32_t (&buf)[NW], uint32_t ast, const uint32_t (&soff)[2][2])
{
    // fully unrolled over (row r, chunk e): every window position is a compile-time constant
    auto body = [&](auto R, auto E) {
        constexpr int r = decltype(R)::value, e = decltype(E)::value;
        // channels 8e + 2c, 8e + 2c + 1 of row r -> one fp16 pair
        auto pair = [&](auto Cc) -> uint32_t {
            constexpr int c = decltype(Cc)::value;
            const uint32_t ma = inst3(window16<(16 * r + 8 * e + 2 * c + 1) * BITS + 16>(buf));
            const uint32_t mb = inst3(window16<(16 * r + 8 * e + 2 * c + 2) * BITS + 16>(buf));
            return weight_pair(ma, mb);
        };
        sts128(ast + soff[r & 1][e] + (r >> 1) * 2048, pair(std::integral_constant<int, 0>{}),
               pair(std::integral_constant<int, 1>{}), pair(std::integral_constant<int, 2>{}),
               pair(std::integral_constant<int, 3>{}));
    };
    [&]<int... RE>(std::integer_sequence<int, RE...>) {
        (body(std::integral_constant<int, RE / 2>{}, std::integral_constant<int, RE % 2>{}), ...);
    }(std::make_integer_sequence<int, 8>{});
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

// zsm[0 .. m*128) = sum of the partial slots (q + g) for q = p_first..p_last,
// added in that order.  128 threads; each owns up to NT/4 float4 outputs and
// keeps 2 x NT/4 independent loads in flight (a dependent chain of L2 loads
// would take ~0.4 us per partial).
template <int NT>
__device__ __forceinline__ void reduce_segments(const float* part, int g, int p_first, int p_last, int m, int et,
                                                float* zsm)
{
    constexpr int F = NT / 4;                  // float4 outputs per thread, at most
    float4 acc[F];
    const int nf = m * 32;                     // float4 outputs in use
#pragma unroll
    for (int r = 0; r < F; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    int qq = p_first;
    for (; qq + 1 <= p_last; qq += 2) {
        const float4* s0 = reinterpret_cast<const float4*>(part + (size_t)(qq + g) * NT * 128);
        const float4* s1 = reinterpret_cast<const float4*>(part + (size_t)(qq + 1 + g) * NT * 128);
        float4 v0[F], v1[F];
#pragma unroll
        for (int r = 0; r < F; ++r) {
            const int f = et + 128 * r;
            v0[r] = f < nf ? __ldcg(s0 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            v1[r] = f < nf ? __ldcg(s1 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < F; ++r) {
            acc[r].x += v0[r].x; acc[r].y += v0[r].y; acc[r].z += v0[r].z; acc[r].w += v0[r].w;
            acc[r].x += v1[r].x; acc[r].y += v1[r].y; acc[r].z += v1[r].z; acc[r].w += v1[r].w;
        }
    }
    if (qq <= p_last) {
        const float4* s0 = reinterpret_cast<const float4*>(part + (size_t)(qq + g) * NT * 128);
#pragma unroll
        for (int r = 0; r < F; ++r) {
            const int f = et + 128 * r;
            if (f < nf) {
                const float4 v = __ldcg(s0 + f);
                acc[r].x += v.x; acc[r].y += v.y; acc[r].z += v.z; acc[r].w += v.w;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < F; ++r) {
        const int f = et + 128 * r;
        if (f < nf) reinterpret_cast<float4*>(zsm)[f] = acc[r];
    }
}

template <int BITS, int NT>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(TcParams prm)
{
    using L = TcLayout<BITS, NT>;
    constexpr int TW = 8 * BITS, QW = 2 * BITS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::off_bar);
    uint64_t* pfull = bar;                                   // [kDecWarps][kRing]: packed words landed
    uint64_t* pempty = pfull + kDecWarps * kRing;            // [kDecWarps][kRing]: decoder has read them
    uint64_t* afull = pempty + kDecWarps * kRing;            // [slot][buf]: the 4 decoders of a slot arrive
    uint64_t* aempty = afull + kIssuers * kABuf;             // [slot][buf]: the slot's issuer commits
    uint64_t* bfull = aempty + kIssuers * kABuf;             // [slot][kSB]
    uint64_t* bempty = bfull + kIssuers * kSB;               // [slot][kSB]
    uint64_t* dfull = bempty + kIssuers * kSB;               // [kIssuers][2]
    uint64_t* dempty = dfull + 2 * kIssuers;                 // [kIssuers][2]
    int* misc = reinterpret_cast<int*>(smem + L::off_misc);   // [0] tmem base, [1] abort, [2] last-CTA flag
    volatile int* abort_flag = misc + 1;
    float* zsm = reinterpret_cast<float*>(smem + L::off_z);

    const GemmArgs& a = prm.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = blockIdx.x;
    const long long b0 = (long long)p * prm.U / prm.P;
    const long long b1 = (long long)(p + 1) * prm.U / prm.P;
    const int n = (int)(b1 - b0);                            // units of this CTA
    const int C = prm.C;
    const int tiles_n = a.n_out / 16;
    const int g_first = (int)(b0 / C), c_first = (int)(b0 % C);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecWarps * kRing; ++i) { mbar_init(&pfull[i], 1); mbar_init(&pempty[i], 1); }
        for (int i = 0; i < kIssuers * kABuf; ++i) { mbar_init(&afull[i], 4); mbar_init(&aempty[i], 1); }
        for (int i = 0; i < kIssuers * kSB; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
        for (int i = 0; i < 2 * kIssuers; ++i) { mbar_init(&dfull[i], 1); mbar_init(&dempty[i], kEpiWarps); }
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
    }
    if (warp == kWarpIss0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(&misc[0]), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];

    if (warp < kWarpIss0) {
        // ------------------------------------------------------ producers ---
        // Producer s issues, for each unit u = s (mod 4) of this CTA, the
        // packed words of its 4 tile rows (one bulk copy into the ring of each
        // decoder of slot s) and its xt chunk (into the slot's xt ring).
        if (lane == 0) {
            const int sl = warp - kWarpProd0;
            int g = g_first, c = c_first + sl;
            while (c >= C) { c -= C; ++g; }
            for (int u = sl, k = 0; u < n; u += 4, ++k) {
                const int rs = k % kRing;
                const uint32_t rpar = ((k / kRing) & 1) ^ 1;
                bool ok = true;
#pragma unroll
                for (int t = 0; t < 4 && ok; ++t) {
                    const int d = sl * 4 + t;
                    ok = wait_or_abort(&pempty[d * kRing + rs], rpar, abort_flag, kSleepNs);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&pfull[d * kRing + rs], L::ROWB);
                    bulk_g2s(smem + L::off_p + (size_t)(d * kRing + rs) * L::ROWB,
                             a.packed + ((size_t)(4 * c + t) * tiles_n + 8 * (size_t)g) * TW, L::ROWB,
                             &pfull[d * kRing + rs]);
                }
                if (!ok) break;
                const int bs = sl * kSB + k % kSB;
                if (!wait_or_abort(&bempty[bs], ((k / kSB) & 1) ^ 1, abort_flag, kSleepNs)) break;
                mbar_arrive_expect_tx(&bfull[bs], L::BBYTES);
                bulk_g2s(smem + L::off_b + bs * L::BBYTES, prm.xt + (size_t)c * L::BBYTES, L::BBYTES, &bfull[bs]);
                c += 4;
                while (c >= C) { c -= C; ++g; }
            }
        }
    } else if (warp < kWarpEpi0) {
        // --------------------------------------------------- MMA issuers ---
        // Issuer i takes the units u = i (mod 4) -- all 4 tile rows, 8 MMAs per
        // barrier wait -- into its own accumulator.  It takes part in every
        // segment (waits for its buffer, commits it) even when it has no unit
        // there, so that every barrier sees one phase per segment.
        if (lane == 0) {
            const int i = warp - kWarpIss0;
            constexpr uint32_t idesc = idesc_f16_amn(128, NT);
            int seg = 0, u0 = 0, c0 = c_first;
            bool ok = true;
            while (ok && u0 < n) {
                const int len = (n - u0) < (C - c0) ? (n - u0) : (C - c0);
                const int db = seg & 1;
                if (!wait_or_abort(&dempty[2 * i + db], ((seg >> 1) & 1) ^ 1, abort_flag, kIssSleepNs)) break;
                const uint32_t dcol = tmem + (uint32_t)((i * 2 + db) * NT);
                bool first = true;
                for (int u = u0 + ((i - u0) & 3); u < u0 + len; u += 4) {
                    const int k = u >> 2, ab = k & 1;            // k-th unit of slot i, A buffer
                    if (!wait_or_abort(&afull[i * kABuf + ab], (k >> 1) & 1, abort_flag, kIssSleepNs)) { ok = false; break; }
                    tc_fence_after();
                    const int bs = i * kSB + k % kSB;
                    const uint32_t bbase = smem_u32(smem + L::off_b + bs * L::BBYTES);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint32_t abase = smem_u32(smem + L::off_a + (ab * kDecWarps + i * 4 + t) * kABytes);
                        mma_f16_ss(dcol, sdesc_sw128(abase, 1024, 2048), sdesc_sw128(bbase + t * 32, 16, 1024), idesc,
                                   (first && t == 0) ? 0u : 1u);
                    }
                    first = false;
                    mma_commit(&aempty[i * kABuf + ab]);
                    mma_commit(&bempty[bs]);
                }
                mma_commit(&dfull[2 * i + db]);
                ++seg;
                u0 += len;
                c0 = 0;
            }
        }
    } else if (warp < kWarpDec0) {
        // ----------------------------------------------------- epilogue ---
        const int ew = warp - kWarpEpi0;    // 0..3
        const int quad = warp & 3;          // tensor-memory lanes 32*quad .. 32*quad+31
        const int et = threadIdx.x - 32 * kWarpEpi0;   // 0..127
        int seg = 0;
        int u0 = 0, g = g_first, c0 = c_first;
        while (u0 < n) {
            const int len = (n - u0) < (C - c0) ? (n - u0) : (C - c0);
            const int db = seg & 1;
            bool ok = true;
            for (int i = 0; i < kIssuers && ok; ++i)
                ok = warp_wait(&dfull[2 * i + db], (seg >> 1) & 1, abort_flag, kEpiSleepNs);
            if (!ok) break;
            tc_fence_after();
            {
                const int v = 32 * quad + lane;
                float acc[NT];
#pragma unroll
                for (int mm = 0; mm < NT; ++mm) acc[mm] = 0.f;
#pragma unroll
                for (int i = 0; i < kIssuers; ++i) {
                    if (len < 4 && ((i - u0) & 3) >= len) continue;   // issuer i had no unit here
#pragma unroll
                    for (int cc = 0; cc < NT / 16; ++cc) {
                        uint32_t t16[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)((i * 2 + db) * NT + 16 * cc), t16);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e) acc[16 * cc + e] += __uint_as_float(t16[e]);
                    }
                }
                const int ch = chan_of_row(v);
#pragma unroll
                for (int mm = 0; mm < NT; ++mm) zsm[mm * 128 + ch] = acc[mm];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int i = 0; i < kIssuers; ++i) mbar_arrive(&dempty[2 * i + db]);
            named_bar(1, 128);
            const int p_first = cta_of_unit((long long)g * C, prm.P, prm.U);
            const int p_last = cta_of_unit((long long)(g + 1) * C - 1, prm.P, prm.U);
            bool finish = true;
            if (p_last > p_first) {
                float4* myslot = reinterpret_cast<float4*>(prm.part + (size_t)(p + g) * NT * 128);
                const float4* z4s = reinterpret_cast<const float4*>(zsm);
                for (int f = et; f < a.m * 32; f += 128) __stcg(myslot + f, z4s[f]);
                __threadfence();
                named_bar(1, 128);
                if (et == 0) {
                    const uint32_t prev = atomicAdd(&prm.counters[g], 1u);
                    misc[2] = (prev == (uint32_t)(p_last - p_first)) ? 1 : 0;
                }
                named_bar(1, 128);
                finish = misc[2] != 0;
                if (finish) {
                    __threadfence();
                    reduce_segments<NT>(prm.part, g, p_first, p_last, a.m, et, zsm);
                    if (et == 0) prm.counters[g] = 0u;
                    named_bar(1, 128);
                }
            }
            if (finish) {
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
                        *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(a.y) + yo) =
                            *reinterpret_cast<uint2*>(hh);
                    }
                }
            }
            named_bar(1, 128);
            ++seg;
            u0 += len;
            c0 = 0;
            ++g;
        }
    } else {
        // ------------------------------------------------------ decoders ---
        const int d = warp - kWarpDec0;           // 0..15
        const int slot = d >> 2;                  // units u = slot (mod 4); tile row d % 4 of each
        const int j = lane >> 2, q = lane & 3;
        const int src_prev = (lane & ~3) | ((q + 3) & 3);
        uint32_t soff[2][2];
        {
            const int atom = j >> 2, j4 = j & 3;
#pragma unroll
            for (int rb = 0; rb < 2; ++rb)
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    soff[rb][e] = atom * 1024 + (4 * rb + q) * 128 + ((uint32_t)(chunk_of_tile(j4, e) ^ (4 * rb + q)) << 4);
        }
        const uint8_t* ring = smem + L::off_p + (size_t)d * kRing * L::ROWB;
        const uint32_t ast0 = smem_u32(smem + L::off_a + d * kABytes);  // stage d (+ kDecWarps for buffer 1)
        const int nk = n > slot ? (n - slot + 3) / 4 : 0;      // units this decoder handles
        for (int k = 0; k < nk; ++k) {
            const int rs = k % kRing;
            if (!warp_wait(&pfull[d * kRing + rs], (k / kRing) & 1, abort_flag, kSleepNs)) break;
            const uint32_t* sw = reinterpret_cast<const uint32_t*>(ring + rs * L::ROWB) + j * TW + q * QW;
            uint32_t buf[QW + 1];
            if constexpr (QW % 4 == 0) {
#pragma unroll
                for (int w = 0; w < QW / 4; ++w) {
                    const uint4 vv = reinterpret_cast<const uint4*>(sw)[w];
                    buf[1 + 4 * w] = vv.x; buf[2 + 4 * w] = vv.y; buf[3 + 4 * w] = vv.z; buf[4 + 4 * w] = vv.w;
                }
            } else {
#pragma unroll
                for (int w = 0; w < QW / 2; ++w) {
                    const uint2 vv = reinterpret_cast<const uint2*>(sw)[w];
                    buf[1 + 2 * w] = vv.x; buf[2 + 2 * w] = vv.y;
                }
            }
            buf[0] = __shfl_sync(0xffffffffu, buf[QW], src_prev);
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[d * kRing + rs]);      // slot free for the producer
            const int ab = k & 1;
            if (!warp_wait(&aempty[slot * kABuf + ab], ((k >> 1) & 1) ^ 1, abort_flag, kSleepNs)) break;
            decode_quarter_to_a<BITS>(buf, ast0 + ab * kDecWarps * kABytes, soff);
            fence_proxy_async_smem();
            // the unit's xt chunk must have landed before its MMAs are issued;
            // the decoder checks it here so that the issuer waits only on afull
            if (!warp_wait(&bfull[slot * kSB + k % kSB], (k / kSB) & 1, abort_flag, kSleepNs)) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[slot * kABuf + ab]);
        }
    }

    // ------------------------------------------------------------ teardown ---
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpIss0) {
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
    prm.C = a.k_in / 64;
    prm.U = (long long)prm.G * prm.C;
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
    const long long U = (long long)(n_out / 128) * (k_in / 64);
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
