// gemm_tc.cu -- the verify-batch product (2..32 input rows) on the 5th-generation
// tensor cores (tcgen05), with the trellis decode on the CUDA cores.
//
// What is computed (the exl3-rdna4-recipe page verifies drafted tokens with a
// tensor-core GEMV and keeps verify batches of up to 32 rows on its fast
// kernel, section "What we added on top of upstream"; here on B200):
//     y = sv .* H( scale .* ( H(su .* x) W ) ),   x: m x K_in, y: m x N_out
//
// Design:
//   * A pre-pass writes xt = H(su .* x) once per call into the workspace, fp16,
//     laid out as the MMA's B operand (K-major, 128-byte swizzle), m padded to
//     NT = 16 or 32 rows with zeros.
//   * Unit = one block of 128 RPW rows of K_in for one 128-channel output
//     block: 8 RPW tile rows.  RPW = 2 (256-row units) when every K_in of the
//     call is a multiple of 256, else 1.  Two ways to cut the units over the
//     CTAs (two per SM), chosen per shape by a small cost model (see
//     TcParams): clusters of S CTAs per output block that add their partial
//     sums through distributed shared memory, or a stream-K cut with
//     workspace partials.
//   * Eight decoder warps.  Warp w decodes tile rows w (and w + 8) of every
//     unit: lane l takes quarter l%4 of tile l/4 (64 consecutive weights) from
//     its words, loaded straight from HBM into registers one tile row ahead
//     (coalesced: the warp reads the tile row's 256*K contiguous bytes).  The
//     two fp16 halves of each 3INST word are added once (RNE: the exact
//     decoded weight) and stored into the warp's own A stage (128 channels x
//     16 k per tile row, MN-major, 128-byte swizzle).  The warp then issues
//     the unit's MMAs itself (one elected lane, from converged code) --
//     tcgen05.mma kind::f16, M = 128 channels, N = NT rows, K = 16 -- into its
//     own tensor-memory accumulator (so the accumulation order is fixed), and
//     commits them to the stage's barrier.  A warp waits only for its own
//     stage and for the unit's xt; with two tile rows per unit it hands off
//     half as often (measured: 3 % off a grouped layer call).
//   * A ninth warp streams each unit's xt (1-D bulk copies + mbarrier) into a
//     ring shared by the eight decoders (four stages of 128 rows, or two of
//     256).
//   * End of a block's share: the CTA reads all eight accumulators
//     (tcgen05.ld) and adds them in a fixed order; the partial sums of a block
//     split over several CTAs meet in rank / CTA order -- fixed, so results
//     are bitwise repeatable -- then the finishing warps scale, rotate and
//     write y.
//   * Launched with programmatic dependent launch: set-up and the first word
//     loads overlap the previous kernel; xt, y and the workspace are touched
//     only after griddepcontrol.wait.
//   * Every mbarrier wait is bounded (2 s); on expiry the CTA records a
//     timeout in the workspace status word and winds down through the same
//     barriers (tested by withholding xt: see the workspace injection word).
#include <atomic>
#include <mutex>
#include <utility>

#include <cooperative_groups.h>

#include "exl3_aop.cuh"
#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"
#include "exl3_tc.cuh"

namespace exl3 {

namespace cg = cooperative_groups;

namespace {

constexpr int kDec = 8;                        // decoder warps (one accumulator each)
constexpr int kProdWarp = kDec;                // warp 8: xt chunk producer
constexpr int kTcThreads = 32 * (kDec + 1);
constexpr int kATile = 4096;                   // one tile row of A: 128 channels x 16 k, fp16
constexpr int kCtasPerSm = 2;
constexpr int kSms = 148;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// RPW tile rows per decoder warp per unit: a unit is 128 * RPW input rows.
// RPW = 1: two A stages of one tile row per warp, four xt stages; RPW = 2:
// one A stage of two tile rows per warp (the first half tile row is decoded
// into registers while the previous unit's MMAs finish), two xt stages.
template <int NT, int RPW>
struct TcLayout {
    static constexpr int AST = RPW == 1 ? 2 : 1;              // A stages per decoder warp
    static constexpr int BST = RPW == 1 ? 4 : 2;              // xt unit stages (shared by the decoders)
    static constexpr int ABYTES = RPW * kATile;               // one A stage
    static constexpr int CHUNK = NT * 128;                    // xt bytes per 64 input rows
    static constexpr int BUNIT = 2 * RPW * CHUNK;             // xt bytes per unit
    static constexpr int TMEM_COLS = kDec * NT;               // one NT-column accumulator per decoder
    static constexpr int off_a = 0;                           // [kDec][AST] A stages
    static constexpr int off_z = off_a;                       // z [NT][128] fp32, over the A stages (segment end)
    static constexpr int off_b = off_a + kDec * AST * ABYTES;
    static constexpr int off_bar = off_b + BST * BUNIT;
    // aempty[kDec][AST], bfull[BST], bempty[BST], segdone, lastbar
    static constexpr int nbar = kDec * AST + 2 * BST + 2;
    static constexpr int off_misc = off_bar + nbar * 8;
    static constexpr int total = off_misc + 64 + 1024;       // + slack to align the base to 1024
    static_assert(off_b % 1024 == 0 && off_z % 16 == 0 && off_bar % 8 == 0, "layout");
    static_assert(NT * 128 * 4 <= kDec * AST * ABYTES, "z fits over the A stages");
    static_assert((BST & (BST - 1)) == 0, "power of two");
    static_assert(TMEM_COLS == 128 || TMEM_COLS == 256, "tensor memory (power of two, two CTAs per SM)");
    // at most two CTAs fit on an SM, so their accumulators always fit in its 512 columns
    static_assert(3 * total > 227 * 1024, "a third CTA per SM must not fit");
    // 228 KB of shared memory per SM, 1 KB of it reserved per resident CTA
    static_assert(kCtasPerSm * (total + 1024) <= 228 * 1024, "two CTAs per SM");
};

// Two ways to cut the G x C units (output block g, 128-row input block c):
//   cluster (S > 0): S CTAs per output block, launched as one cluster; CTA r
//     takes units [rC/S, (r+1)C/S) of its block; the S partial sums meet in
//     distributed shared memory.  Best when few CTAs per block fill the GPU
//     poorly otherwise, or when many would have to share a block.
//   stream-K (S == 0): P equal contiguous ranges of the block-major unit
//     order, one per CTA; partial sums of blocks cut between CTAs go through
//     the workspace and the last CTA to arrive adds them.  Best balance when
//     a block is shared by only a few CTAs.
struct TcParams {
    GemmArgs a;
    const uint8_t* xt;      // rotated input, B-operand layout
    float* part;            // stream-K partial sums, [slot][NT][128]
    uint32_t* counters;     // stream-K arrival counters, per output block
    uint32_t* status;       // workspace status word
    size_t xt_bytes;        // size of the rotated-input region (debug-bounds checks)
    int nslots;             // partial-sum slots in the workspace (debug-bounds checks)
    int S;                  // cluster size (CTAs per output block), 0: stream-K
    int P;                  // stream-K CTAs
    long long U;            // units: sum over members of blocks x 128-row input blocks
    uint32_t two16;         // 2^16, passed at run time (keeps a multiply on the FMA pipe)
};

__host__ __device__ inline int cta_of_unit(long long x, int P, long long U)
{
    return (int)(((x + 1) * P - 1) / U);
}

// Bounded wait on one thread; gives up early once another thread has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait_sleep(bar, parity, 1000)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicExch((int*)abort_flag, 1);
            return false;
        }
    }
}

// Warp-wide wait: every lane tries the phase once (one instruction for the
// warp) and the warp votes; only if the phase is not complete yet does lane 0
// run the bounded wait and broadcast the outcome.  Nearly nine waits in ten
// find the phase complete, and this fast path spares them the lane-0 branch,
// its reconvergence and the broadcast (measured: 0.24 fewer instructions per
// weight, 3 % faster).  Returns the same value on every lane.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int lane)
{
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    int ok = 1;
    if (lane == 0) ok = wait_or_abort(bar, parity, abort_flag) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// zsm[0 .. m*128) = sum of the partial slots (q + g) for q = p_first..p_last,
// added in that order, by the 256 decoder threads.
template <int NT>
__device__ __forceinline__ void reduce_segments(const float* part, int g, int p_first, int p_last, int m, int et,
                                                float* zsm)
{
    // thread et owns float4 outputs et + 256 i (i < NI); per step it loads one
    // float4 of each of its outputs from two partials: 2 * NI loads in flight
    constexpr int NI = NT / 8;                 // NT * 32 float4 outputs / 256 threads
    const int nf = m * 32;                     // float4 outputs in use
    float4 acc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    int qq = p_first;
    for (; qq + 1 <= p_last; qq += 2) {
        const float4* s0 = reinterpret_cast<const float4*>(part + (size_t)(qq + g) * NT * 128);
        const float4* s1 = reinterpret_cast<const float4*>(part + (size_t)(qq + 1 + g) * NT * 128);
        float4 v0[NI], v1[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int f = et + 32 * kDec * i;
            v0[i] = f < nf ? __ldcg(s0 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            v1[i] = f < nf ? __ldcg(s1 + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            acc[i].x += v0[i].x; acc[i].y += v0[i].y; acc[i].z += v0[i].z; acc[i].w += v0[i].w;
            acc[i].x += v1[i].x; acc[i].y += v1[i].y; acc[i].z += v1[i].z; acc[i].w += v1[i].w;
        }
    }
    if (qq <= p_last) {
        const float4* s0 = reinterpret_cast<const float4*>(part + (size_t)(qq + g) * NT * 128);
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int f = et + 32 * kDec * i;
            if (f < nf) {
                const float4 v = __ldcg(s0 + f);
                acc[i].x += v.x; acc[i].y += v.y; acc[i].z += v.z; acc[i].w += v.w;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int f = et + 32 * kDec * i;
        if (f < nf) reinterpret_cast<float4*>(zsm)[f] = acc[i];
    }
}

// Final epilogue of one output row mm of block g, by one warp: z (this lane's
// channels 4*lane .. +3) times scale, output rotation, signs, store.
__device__ __forceinline__ void finish_row_regs(const GemmArgs& a, int g, int mm, const float (&z)[4], int lane)
{
    const MemView sib = member_of_block(a, g);            // the matrix holding block g
    const int n0 = 128 * sib.gl + 4 * lane;
    // warp-uniform (the rotation below shuffles across the warp)
    if (!guard(mm < a.m && 128 * sib.gl + 128 <= sib.n_out, reinterpret_cast<uint32_t*>(a.ws))) return;
    const uint2 sc = *reinterpret_cast<const uint2*>(sib.scale + n0);
    const uint2 sg = *reinterpret_cast<const uint2*>(sib.sv + n0);
    const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&sc.x));
    const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&sc.y));
    const float2 sg0 = __half22float2(*reinterpret_cast<const __half2*>(&sg.x));
    const float2 sg1 = __half22float2(*reinterpret_cast<const __half2*>(&sg.y));
    float vv[4] = {z[0] * sc0.x, z[1] * sc0.y, z[2] * sc1.x, z[3] * sc1.y};
    fwht128_warp(vv);
    vv[0] *= kInvSqrt128 * sg0.x;
    vv[1] *= kInvSqrt128 * sg0.y;
    vv[2] *= kInvSqrt128 * sg1.x;
    vv[3] *= kInvSqrt128 * sg1.y;
    const size_t yo = (size_t)mm * sib.n_out + n0;
    if (a.y_fp32) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(sib.y) + yo) = make_float4(vv[0], vv[1], vv[2], vv[3]);
    } else {
        __half2 hh[2] = {__floats2half2_rn(vv[0], vv[1]), __floats2half2_rn(vv[2], vv[3])};
        *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(sib.y) + yo) = *reinterpret_cast<uint2*>(hh);
    }
}

__device__ __forceinline__ void finish_row(const GemmArgs& a, int g, int mm, const float* zrow, int lane)
{
    const float4 z4 = *reinterpret_cast<const float4*>(zrow + 4 * lane);
    const float z[4] = {z4.x, z4.y, z4.z, z4.w};
    finish_row_regs(a, g, mm, z, lane);
}

// Two MMAs into one accumulator (the second always accumulating) and two
// commits, issued by one elected lane under a single election.
__device__ __forceinline__ void mma2_f16_ss_commit2_elect(uint32_t d_tmem, uint64_t adesc0, uint64_t bdesc0,
                                                          uint64_t adesc1, uint64_t bdesc1, uint32_t idesc,
                                                          uint32_t accumulate, uint64_t* bar0, uint64_t* bar1)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %5, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %4, %5, 1;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%8];\n\t}" ::"r"(d_tmem),
        "l"(adesc0), "l"(bdesc0), "l"(adesc1), "l"(bdesc1), "r"(idesc), "r"(accumulate), "r"(smem_u32(bar0)),
        "r"(smem_u32(bar1))
        : "memory");
}

template <int BITS, int NT, int RPW>
__global__ void __launch_bounds__(kTcThreads, kCtasPerSm) gemm_tc_kernel(TcParams prm)
{
    using L = TcLayout<NT, RPW>;
    constexpr int AST = L::AST, BST = L::BST;
    constexpr int KU = 128 * RPW;                             // input rows per unit
    constexpr int TW = 8 * BITS, QW = 2 * BITS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::off_bar);
    uint64_t* aempty = bar;                                   // [kDec][AST]: the stage's MMAs completed
    uint64_t* bfull = aempty + kDec * AST;                    // [BST]: xt unit landed
    uint64_t* bempty = bfull + BST;                           // [BST]: all 8 warps' MMAs on it completed
    uint64_t* segdone = bempty + BST;                         // every accumulator final
    uint64_t* lastbar = segdone + 1;                          // every MMA of the CTA completed
    int* misc = reinterpret_cast<int*>(smem + L::off_misc);   // [0] tmem base, [1] abort
    volatile int* abort_flag = misc + 1;
    float* zsm = reinterpret_cast<float*>(smem + L::off_z);

    const GemmArgs& a = prm.a;
    // the warp index broadcast from lane 0: provably warp-uniform, so the values
    // derived from it (shared-memory descriptors, tensor-memory columns) can stay
    // in uniform registers, where the tcgen05 instructions take them (measured:
    // 0.1 fewer instructions per weight, 1-2 % faster)
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
    const int S = prm.S;
    const int p = blockIdx.x;
    // this CTA's units [b0, b1) in the group's block-major order
    long long b0, b1;
    if (S > 0) {
        const int gc = p / S, rc = p % S;
        const MemView cm = member_of_block(a, gc);
        const int C = cm.k_in / KU;
        const long long ublk = cm.u0 + (long long)cm.gl * C;
        b0 = ublk + (long long)rc * C / S;
        b1 = ublk + (long long)(rc + 1) * C / S;
    } else {
        b0 = (long long)p * prm.U / prm.P;
        b1 = (long long)(p + 1) * prm.U / prm.P;
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < kDec * AST; ++i) mbar_init(&aempty[i], 1);
        for (int i = 0; i < BST; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], kDec); }
        mbar_init(segdone, kDec);
        mbar_init(lastbar, kDec);
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(reinterpret_cast<uint32_t*>(&misc[0]), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    grid_dep_launch();                 // the next kernel may start launching

    if (warp == kProdWarp) {
        grid_dep_wait();               // xt is written by the pre-pass
        // ------------------------------------------------- xt producer ---
        // xt of unit (g, c) is chunks 2 RPW c .. 2 RPW c + 2 RPW - 1: BUNIT contiguous bytes.
        // A nonzero injection word v (tests of the timeout path) lets only the
        // CTA's first v - 1 xt copies through, so the decoders' wait for the
        // next one runs out (with MMAs of the earlier units possibly in flight).
        const uint32_t inject = *reinterpret_cast<const volatile uint32_t*>(a.ws + kWsInjectOff);
        const long long allowed = inject ? (long long)inject - 1 : (b1 - b0);
        if (lane == 0) {
            int kk = 0;
            for (long long u = b0; u < b1 && kk < allowed; ++u, ++kk) {
                const int s = kk & (BST - 1);
                if (kk >= BST && !wait_or_abort(&bempty[s], (uint32_t)(kk / BST - 1) & 1u, abort_flag)) break;
                const MemView um = member_of_unit(a, u);
                const int c = (int)((u - um.u0) % (um.k_in / KU));
                if (!guard(um.xt0 + (size_t)(c + 1) * L::BUNIT <= prm.xt_bytes, prm.status)) break;
                mbar_arrive_expect_tx(&bfull[s], L::BUNIT);
                bulk_g2s(smem + L::off_b + s * L::BUNIT, prm.xt + um.xt0 + (size_t)c * L::BUNIT, L::BUNIT, &bfull[s]);
            }
            // every issued copy lands before the CTA can exit (a no-op wait in
            // a normal run: the decoders have consumed them)
            const int issued = kk;
            for (int v = issued > BST ? issued - BST : 0; v < issued; ++v)
                (void)mbar_wait_bounded(&bfull[v & (BST - 1)], (uint32_t)(v / BST) & 1u, 100000000ull);
        }
    } else {
        // --------------------------------------------- decoder warps ---
        // Segment loop: the CTA's units grouped by output block (one segment
        // in cluster mode).  The producer never joins these warps' barriers
        // (the 256-thread named barrier 1).
        const int q = lane & 3;
        const int src_prev = (lane & ~3) | ((q + 3) & 3);
        uint32_t soff[2][2];
        lane_soff(lane, soff);
        constexpr uint32_t idesc = idesc_f16_amn(128, NT);
        const uint32_t ast0 = smem_u32(smem + L::off_a + (warp * AST + 0) * L::ABYTES);
        // RPW = 1: the second A stage; RPW = 2: the stage's second tile row
        const uint32_t ast1 = RPW == 1 ? smem_u32(smem + L::off_a + (warp * AST + 1) * L::ABYTES) : ast0 + kATile;
        const uint64_t adesc0 = sdesc_sw128(ast0, 1024, 2048), adesc1 = sdesc_sw128(ast1, 1024, 2048);
        // this warp's tile rows are rows 16 (warp + 8 j) .. +15 of a unit (j < RPW): chunk warp/4 + 2 j,
        // 32 bytes per 16 rows; stage bs adds bs * BUNIT to the start address (no carry out of its
        // 14-bit field: smem < 256 KB)
        const uint32_t bw = (uint32_t)((warp >> 2) * L::CHUNK + (warp & 3) * 32);
        const uint64_t bdesc0 = sdesc_sw128(smem_u32(smem + L::off_b) + bw, 16, 1024);
        const uint32_t dcol = tmem + (uint32_t)(warp * NT);
        bool fail0 = false;                                      // a wait gave up (warp-uniform)
        int kk = 0;                                              // CTA unit counter (stages, parities)
        int seg = 0;
        for (long long u0 = b0; u0 < b1; ++seg) {
            const MemView sib = member_of_unit(a, u0);                 // the matrix holding unit u0
            const int C = sib.k_in / KU;                               // units per block of this matrix
            const int gl = (int)((u0 - sib.u0) / C);
            const int g = sib.g0 + gl;                                 // group block index
            const long long ublk = sib.u0 + (long long)gl * C;         // the block's first unit
            const int c0 = (int)(u0 - ublk);
            const long long u1 = (ublk + C < b1) ? ublk + C : b1;
            const int nseg = (int)(u1 - u0);
            const int tiles_n = sib.n_out / 16;
            const size_t rstep = (size_t)8 * tiles_n * TW;        // words between tile rows w and w + 8
            const uint32_t* src =
                sib.packed + ((size_t)(8 * RPW * c0 + warp) * tiles_n + 8 * (size_t)gl) * TW + (size_t)lane * QW;
            const size_t unit_step = (size_t)RPW * rstep;        // words between consecutive units
            const size_t n_words = (size_t)C * unit_step;
            bool ok = true;                                      // warp-uniform
            uint32_t wa[QW], wb[QW];
            // RPW = 1: decode the segment's unit k (the CTA's kk-th) from `wds`
            // into A stage kk & 1, then one elected lane issues its MMA into
            // this warp's accumulator
            auto unit = [&](const uint32_t (&wds)[QW], int k, int kq) {
                const int s = kq & (AST - 1), bs = kq & (BST - 1);
                const uint32_t ph = (uint32_t)(kq / AST) & 1u, bph = (uint32_t)(kq / BST) & 1u;
                // every lane sees the MMA that last read this stage complete before
                // it stores into the stage
                if (fail0 || !(kq < AST || warp_wait(&aempty[warp * AST + s], ph ^ 1u, abort_flag, lane)))
                    ok = false;
                if (!ok) return;
                uint32_t buf[QW + 1];
                buf[0] = __shfl_sync(0xffffffffu, wds[QW - 1], src_prev);
#pragma unroll
                for (int t = 0; t < QW; ++t) buf[t + 1] = wds[t];
                const uint32_t ast = s ? ast1 : ast0;
                decode_quarter_to_a<BITS>(buf, soff, prm.two16, [&](uint32_t off, uint32_t w0, uint32_t w1,
                                                                    uint32_t w2, uint32_t w3) {
                    sts128(ast + off, w0, w1, w2, w3);
                });
                fence_proxy_async_smem();          // generic-proxy stores -> visible to the tensor core
                __syncwarp();
                if (warp_wait(&bfull[bs], bph, abort_flag, lane)) {
                    tc_fence_after();
                    const uint64_t bdesc = bdesc0 + (uint64_t)((bs * L::BUNIT) >> 4);
                    mma_f16_ss_commit2_elect(dcol, s ? adesc1 : adesc0, bdesc, idesc, k > 0 ? 1u : 0u,
                                             &aempty[warp * AST + s], &bempty[bs]);
                } else {
                    fail0 = true;                        // warp-uniform: ends the warp's units
                }
            };
            // RPW = 2: unit k's tile row 0 (words in wa) and tile row 1 (words in
            // wb) into the warp's one A stage, then both MMAs and the commits
            // under one election.  The first half of tile row 0 is decoded into
            // registers before the wait for the previous unit's MMAs.
            auto unit2 = [&](int k, int kq) {
                const int bs = kq & (BST - 1);
                const uint32_t ph = (uint32_t)kq & 1u, bph = (uint32_t)(kq / BST) & 1u;
                if (fail0) ok = false;
                if (!ok) return;
                load_lane_words_checked<BITS>(wb, src + (size_t)k * unit_step + rstep, sib.packed, n_words,
                                              prm.status);
                uint32_t buf[QW + 1];
                buf[0] = __shfl_sync(0xffffffffu, wa[QW - 1], src_prev);
#pragma unroll
                for (int t = 0; t < QW; ++t) buf[t + 1] = wa[t];
                uint32_t stg[4][4], stg_off[4];
                int n = 0;
                decode_quarter_chunks<BITS, 0, 4>(buf, soff, prm.two16, [&](uint32_t off, uint32_t w0, uint32_t w1,
                                                                            uint32_t w2, uint32_t w3) {
                    stg[n][0] = w0;
                    stg[n][1] = w1;
                    stg[n][2] = w2;
                    stg[n][3] = w3;
                    stg_off[n] = off;
                    ++n;
                });
                // every lane sees the MMAs that last read the stage complete before it stores
                if (!(kq < 1 || warp_wait(&aempty[warp], ph ^ 1u, abort_flag, lane))) {
                    ok = false;
                    return;
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) sts128(ast0 + stg_off[t], stg[t][0], stg[t][1], stg[t][2], stg[t][3]);
                decode_quarter_chunks<BITS, 4, 8>(buf, soff, prm.two16, [&](uint32_t off, uint32_t w0, uint32_t w1,
                                                                            uint32_t w2, uint32_t w3) {
                    sts128(ast0 + off, w0, w1, w2, w3);
                });
                if (k + 1 < nseg)
                    load_lane_words_checked<BITS>(wa, src + (size_t)(k + 1) * unit_step, sib.packed, n_words,
                                                  prm.status);
                buf[0] = __shfl_sync(0xffffffffu, wb[QW - 1], src_prev);
#pragma unroll
                for (int t = 0; t < QW; ++t) buf[t + 1] = wb[t];
                decode_quarter_chunks<BITS, 0, 8>(buf, soff, prm.two16, [&](uint32_t off, uint32_t w0, uint32_t w1,
                                                                            uint32_t w2, uint32_t w3) {
                    sts128(ast1 + off, w0, w1, w2, w3);
                });
                fence_proxy_async_smem();          // generic-proxy stores -> visible to the tensor core
                __syncwarp();
                if (warp_wait(&bfull[bs], bph, abort_flag, lane)) {
                    tc_fence_after();
                    const uint64_t bdesc = bdesc0 + (uint64_t)((bs * L::BUNIT) >> 4);
                    mma2_f16_ss_commit2_elect(dcol, adesc0, bdesc, adesc1, bdesc + (uint64_t)((2 * L::CHUNK) >> 4),
                                              idesc, k > 0 ? 1u : 0u, &aempty[warp], &bempty[bs]);
                } else {
                    fail0 = true;                        // warp-uniform: ends the warp's units
                }
            };
            load_lane_words_checked<BITS>(wa, src, sib.packed, n_words, prm.status);
            if (seg == 0) grid_dep_wait();     // weights are never written; y and the workspace after this
            if constexpr (RPW == 1) {
                (void)unit2;
                int k = 0;
                for (; k + 2 <= nseg; k += 2) {
                    load_lane_words_checked<BITS>(wb, src + (size_t)(k + 1) * unit_step, sib.packed, n_words,
                                                  prm.status);
                    unit(wa, k, kk + k);
                    if (k + 2 < nseg)
                        load_lane_words_checked<BITS>(wa, src + (size_t)(k + 2) * unit_step, sib.packed, n_words,
                                                      prm.status);
                    unit(wb, k + 1, kk + k + 1);
                }
                if (k < nseg) unit(wa, k, kk + k);
            } else {
                static_assert(RPW == 2, "one or two tile rows per warp");
                (void)unit;
                for (int k = 0; k < nseg; ++k) unit2(k, kk + k);
            }
            kk += nseg;
            // arrives once every MMA this warp issued has completed -- also after a
            // wait gave up part-way (then it covers the MMAs already in flight)
            mma_commit_elect(segdone);

            // ---- accumulators -> zsm[NT][128] (the eight summed in a fixed order) ----
            int okd = 1;
            if (lane == 0) okd = wait_or_abort(segdone, (uint32_t)(seg & 1), abort_flag) ? 1 : 0;
            okd = __shfl_sync(0xffffffffu, okd, 0);
            tc_fence_after();
            constexpr int kReaders = NT == 32 ? 8 : 4;     // warps reading the accumulators
            if (warp < kReaders) {
                const int quad = warp & 3;                   // tensor-memory lanes 32*quad .. +31
                const int tok0 = (warp >> 2) * 16;           // 16 rows (accumulator columns) per warp
                float acc[16];
#pragma unroll
                for (int t = 0; t < 16; ++t) acc[t] = 0.f;
                if (okd) {
#pragma unroll
                    for (int w = 0; w < kDec; ++w) {
                        uint32_t t16[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(w * NT + tok0), t16);
                        tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 16; ++t) acc[t] += __uint_as_float(t16[t]);
                    }
                }
                const int ch = chan_of_row(32 * quad + lane);
#pragma unroll
                for (int t = 0; t < 16; ++t) zsm[(tok0 + t) * 128 + ch] = acc[t];
            }
            tc_fence_before();
            if (S > 0) break;                                // cluster mode: one segment, finished below

            // ---- stream-K: a block cut over several CTAs, the last to arrive finishes it ----
            named_bar(1, 32 * kDec);
            bool finish = true;
            if (nseg < C) {
                const int p_first = cta_of_unit(ublk, prm.P, prm.U);
                const int p_last = cta_of_unit(ublk + C - 1, prm.P, prm.U);
                float4* myslot = reinterpret_cast<float4*>(prm.part + (size_t)(p + g) * NT * 128);
                const float4* z4s = reinterpret_cast<const float4*>(zsm);
                if (guard(p + g < prm.nslots, prm.status))
                    for (int f = threadIdx.x; f < a.m * 32; f += 32 * kDec) __stcg(myslot + f, z4s[f]);
                __threadfence();
                named_bar(1, 32 * kDec);
                if (threadIdx.x == 0) {
                    const uint32_t prev = atomicAdd(&prm.counters[g], 1u);
                    misc[2] = (prev == (uint32_t)(p_last - p_first)) ? 1 : 0;
                }
                named_bar(1, 32 * kDec);
                finish = misc[2] != 0;
                if (finish) {
                    __threadfence();
                    if (guard(p_first + g >= 0 && p_last + g < prm.nslots, prm.status))
                        reduce_segments<NT>(prm.part, g, p_first, p_last, a.m, threadIdx.x, zsm);
                    if (threadIdx.x == 0) prm.counters[g] = 0u;      // ready for the next call on this stream
                    named_bar(1, 32 * kDec);
                }
            }
            if (finish)
                for (int mm = warp; mm < a.m; mm += kDec) finish_row(a, g, mm, zsm + mm * 128, lane);
            named_bar(1, 32 * kDec);                         // zsm and the accumulators free for the next segment
            tc_fence_after();
            u0 = u1;
        }
        mma_commit_elect(lastbar);                           // arrives once this warp's last MMA completed
    }

    // ---- cluster mode: the cluster's CTAs add their z in rank order
    // (distributed shared memory) and each finishes every S-th row ----
    if (S > 0) {
        cg::cluster_group cluster = cg::this_cluster();
        const int g = p / S, r = p % S;
        cluster.sync();                                      // every z of the cluster written
        if (warp < kDec) {
            for (int mm = r + S * warp; mm < a.m; mm += S * kDec) {
                // all S loads in flight first, then added in rank order
                float4 v[16];
#pragma unroll
                for (int qr = 0; qr < 16; ++qr) {
                    v[qr] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (qr < S) {
                        const float* peer = cluster.map_shared_rank(zsm, qr);
                        v[qr] = *reinterpret_cast<const float4*>(peer + mm * 128 + 4 * lane);
                    }
                }
                float4 z4 = v[0];
#pragma unroll
                for (int qr = 1; qr < 16; ++qr) {
                    if (qr < S) {
                        z4.x += v[qr].x; z4.y += v[qr].y; z4.z += v[qr].z; z4.w += v[qr].w;
                    }
                }
                float zr[4] = {z4.x, z4.y, z4.z, z4.w};
                finish_row_regs(a, g, mm, zr, lane);
            }
        }
        cluster.sync();                                      // no CTA leaves while its z is being read
    }

    // ------------------------------------------------------------ teardown ---
    // Every issued MMA completes (its operands are in shared memory already),
    // so this wait ends even after an aborted run; only then may the tensor
    // memory and the barriers its commits arrive on go away.
    if (threadIdx.x == 0) (void)mbar_wait_bounded(lastbar, 0u, 100000000ull);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    if (threadIdx.x == 0 && misc[1]) atomicOr(prm.status, kStatusTimeout);
}

// xt = H(su .* x) / sqrt(128) for rows 0..NT-1 (zero rows past m), written in
// the B-operand layout: 64-row chunks of NT x 128 bytes, rows of 8 x 16-byte
// pieces swizzled by (row & 7), and inside each 16-row group k = 4q + r
// placed at position 8(r >> 1) + 4(r & 1) + q.  One warp item = (member,
// row, 128-block); a sibling group (shared x) rotates member 0's x only.
template <int NT>
__global__ void __launch_bounds__(256) xt_prepass_kernel(GemmArgs a, const uint8_t* __restrict__ xt_base,
                                                         size_t xt_bytes)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_launch();                 // the product kernel may start its prologue
    grid_dep_wait();                   // x and the workspace only after the previous kernel
    long long item = (long long)blockIdx.x * 8 + warp;
    // the member of this item: members in order, NT * (k_in / 128) items each
    const __half* x = reinterpret_cast<const __half*>(a.mem[0].x);
    const __half* su = reinterpret_cast<const __half*>(a.mem[0].su);
    int k_in = a.mem[0].k_in;
    long long xt0 = a.mem[0].xt0;
    bool found = false;
    const int nm = a.shared_x ? 1 : a.nmem;
#pragma unroll
    for (int t = 0; t < kMaxMembers; ++t) {
        if (t < nm && !found) {
            const long long cnt = (long long)NT * (a.mem[t].k_in / 128);
            if (item < cnt) {
                found = true;
                x = reinterpret_cast<const __half*>(a.mem[t].x);
                su = reinterpret_cast<const __half*>(a.mem[t].su);
                k_in = a.mem[t].k_in;
                xt0 = a.mem[t].xt0;
            } else {
                item -= cnt;
            }
        }
    }
    if (!found) return;
    const int nblk = k_in / 128;
    const int m = (int)(item / nblk), b = (int)(item % nblk);
    // lane holds elements i = (lane & 3) | (e << 2) | ((lane >> 2) << 4)
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int k = 128 * b + ((lane & 3) | (e << 2) | ((lane >> 2) << 4));
        v[e] = (m < a.m) ? __half2float(x[(size_t)m * k_in + k]) * __half2float(su[k]) : 0.f;
    }
    fwht128_warp(v);   // the transform factors over index bits: any bit-to-(lane, e) map works
    const int tr = 8 * b + (lane >> 2);
    const int pk0 = 16 * tr + 8 * ((lane >> 1) & 1) + 4 * (lane & 1);
    const int kchunk = pk0 >> 6, o = pk0 & 63, c16 = o >> 3, pos = o & 7;
    const size_t doff = (size_t)xt0 + (size_t)kchunk * NT * 128 + (m >> 3) * 1024 + (m & 7) * 128 +
                        ((c16 ^ (m & 7)) << 4) + pos * 2;
    if (!guard(doff + 8 <= xt_bytes, reinterpret_cast<uint32_t*>(a.ws))) return;
    uint8_t* dst = const_cast<uint8_t*>(xt_base) + doff;
    __half2 h2[2] = {__floats2half2_rn(v[0] * kInvSqrt128, v[1] * kInvSqrt128),
                     __floats2half2_rn(v[2] * kInvSqrt128, v[3] * kInvSqrt128)};
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<uint2*>(h2);
}

int nt_for(int m) { return m <= 16 ? 16 : 32; }

size_t xt_offset(int G) { (void)G; return align_up(ws_data_off(), 1024); }

// Units of the group (sum over members of blocks x 128-row input blocks).
// Units of the group at RPW tile rows per warp (128 RPW input rows each).
long long group_units(const GemmArgs& a, int rpw = 1)
{
    long long U = 0;
    for (int i = 0; i < a.nmem; ++i) U += (long long)(a.mem[i].n_out / 128) * (a.mem[i].k_in / (128 * rpw));
    return U;
}

// Two tile rows per warp when every member's K_in allows 256-row units.
int rpw_for(const GemmArgs& a)
{
    for (int i = 0; i < a.nmem; ++i)
        if (a.mem[i].k_in % 256 != 0) return 1;
    return 2;
}

// Bytes of rotated input: one k_in x NT fp16 operand per distinct input.
size_t xt_bytes(const GemmArgs& a, int NT)
{
    if (a.shared_x) return (size_t)a.mem[0].k_in * NT * 2;
    size_t b = 0;
    for (int i = 0; i < a.nmem; ++i) b += (size_t)a.mem[i].k_in * NT * 2;
    return b;
}

// stream-K CTA count: one wave (two CTAs per SM), at most 8 CTAs per output
// block on average (the last CTA of a block reads every partial of it), at
// most one CTA per unit
int sk_ctas(int G, long long U)
{
    long long p = (long long)kSms * kCtasPerSm;
    if (p > 8LL * G) p = 8LL * G;
    if (p > U) p = U;
    if (p < 1) p = 1;
    return (int)p;
}

size_t part_offset(const GemmArgs& a, int NT) { return align_up(xt_offset(a.n_out / 128) + xt_bytes(a, NT), 256); }

size_t group_ws_bytes(const GemmArgs& a, int NT)
{
    // the stream-K partial slots are always reserved (either cut may be chosen;
    // counted on 128-row units, the most CTAs any unit size gives)
    const int G = a.n_out / 128;
    return part_offset(a, NT) + (size_t)(sk_ctas(G, group_units(a)) + G) * NT * 128 * sizeof(float);
}

// Stand-in with the product kernel's block size and shared memory but
// nothing else, for the cluster-occupancy query: for the product kernel
// itself (which uses tensor memory) the query reports one CTA per SM,
// although two run (its registers, threads and shared memory fit twice).
__global__ void __launch_bounds__(kTcThreads) cluster_fit_probe_kernel(int* never)
{
    extern __shared__ int probe_smem[];
    if (never) never[0] = probe_smem[threadIdx.x];
}

struct TcPlan {
    int S;   // > 0: cluster mode with S CTAs per block; 0: stream-K
    int P;   // CTAs launched
};

// Pick the cut of the units for this shape.  Cost, in unit-decode times, of
// the busiest CTA:
//   * its units;
//   * kSegCost per segment (the accumulator read-out and partial exchange that
//     ends each block share).  The busiest CTA of an unaligned stream-K cut
//     has two segments, because ranges straddle blocks; an aligned cut (P a
//     multiple of G) or a cluster has one;
//   * the reduction.  Stream-K: the finishing CTA reads P/G partials, about
//     0.3 unit-times each, plus kGlobalRed for going through global memory.
//     Cluster: one pass over distributed shared memory.
// The constants fit measured B200 times at M = 32:
//   * 5120 -> 17408: clusters of 2, 39.4 us; aligned stream-K, 41.3 us;
//     stream-K over 296 CTAs, 43.4 us;
//   * 17408 -> 5120: aligned stream-K over 280 CTAs, 42.3 us; stream-K over
//     296 CTAs, 43.6 us; clusters of 6, 44.2 us.
// A cluster size is used only if all G clusters fit at once.
constexpr double kSegCost = 3.0;
constexpr double kGlobalRed = 1.2;
TcPlan choose_plan(int k_in, int n_out, size_t smem, int rpw)
{
    auto kern = cluster_fit_probe_kernel;
    const int G = n_out / 128, C = k_in / (128 * rpw);
    const long long U = (long long)G * C;
    // costs in 128-row unit decode times
    auto cost_sk = [&](long long P) {
        const long long per = (U + P - 1) / P;
        const double segs = (P % G == 0) ? 1.0 : (double)((per - 1) / C + 2);
        return (double)(per * rpw) + 0.3 * (double)P / G + kSegCost * segs + kGlobalRed;
    };
    TcPlan best{0, sk_ctas(G, U)};
    double best_cost = cost_sk(best.P);
    // aligned stream-K: S' CTAs per block (S' <= 8 keeps P within the workspace's partial slots)
    for (int s2 = 2; s2 <= 8 && (long long)s2 * G <= (long long)kSms * kCtasPerSm && s2 <= C; ++s2) {
        const double c = cost_sk((long long)s2 * G);
        if (c < best_cost) {
            best_cost = c;
            best = TcPlan{0, s2 * G};
        }
    }
    int Smax = (kSms * kCtasPerSm) / G;
    if (Smax > 10) Smax = 10;          // measured: 16-CTA clusters were slower than 10 (k/v shapes)
    if (Smax > C) Smax = C;
    for (int S = Smax; S >= 1; --S) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(G * S), 1, 1);
        cfg.blockDim = dim3(kTcThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            continue;
        }
        if (nclusters >= G) {
            const double cost_cl = (double)((C + S - 1) / S * rpw) + 0.2 + 0.05 * S + kSegCost;
            if (cost_cl < best_cost) best = TcPlan{S, G * S};
            break;
        }
    }
    return best;
}

template <int BITS, int NT, int RPW>
cudaError_t launch_tc_r(GemmArgs a, cudaStream_t stream)
{
    using L = TcLayout<NT, RPW>;
    // member units and rotated-input offsets of the group
    {
        long long U = 0, xo = 0;
        for (int i = 0; i < a.nmem; ++i) {
            a.mem[i].u0 = U;
            U += (long long)(a.mem[i].n_out / 128) * (a.mem[i].k_in / (128 * RPW));
            a.mem[i].xt0 = a.shared_x ? 0 : xo;
            xo += (long long)a.mem[i].k_in * NT * 2;
        }
    }
    TcParams prm;
    prm.a = a;
    const int G = a.n_out / 128;
    prm.U = group_units(a, RPW);
    prm.two16 = 0x10000u;
    uint8_t* ws = a.ws;
    prm.status = reinterpret_cast<uint32_t*>(ws);
    prm.counters = reinterpret_cast<uint32_t*>(ws + ws_counter_off());
    const size_t xt_off = xt_offset(G);
    prm.xt = ws + xt_off;
    prm.part = reinterpret_cast<float*>(ws + part_offset(a, NT));
    prm.xt_bytes = xt_bytes(a, NT);
    prm.nslots = sk_ctas(G, prm.U) + G;

    long long items = 0;
    for (int i = 0; i < (a.shared_x ? 1 : a.nmem); ++i) items += (long long)NT * (a.mem[i].k_in / 128);
    cudaLaunchAttribute pdl_attr;
    pdl_attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr.val.programmaticStreamSerializationAllowed = 1;
    {
        cudaLaunchConfig_t pcfg = {};
        pcfg.gridDim = dim3((unsigned)((items + 7) / 8), 1, 1);
        pcfg.blockDim = dim3(256, 1, 1);
        pcfg.stream = stream;
        pcfg.attrs = &pdl_attr;
        pcfg.numAttrs = a.pdl ? 1 : 0;
        cudaError_t e = cudaLaunchKernelEx(&pcfg, xt_prepass_kernel<NT>, a, (const uint8_t*)(ws + xt_off),
                                           xt_bytes(a, NT));
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    auto kern = gemm_tc_kernel<BITS, NT, RPW>;
    static std::atomic<int> configured[kMaxDevices];
    e = once_per_device(configured, [&] {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::total);
        if (r == cudaSuccess) r = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(cluster_fit_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     TcLayout<32, 1>::total);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(cluster_fit_probe_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        return r;
    });
    if (e != cudaSuccess) return e;

    TcPlan pl{0, sk_ctas(G, prm.U)};
    if (a.same_k) {
        // one block length: plan decided once per shape (host-side occupancy
        // queries), then cached.  Groups of several lengths take stream-K.
        static std::mutex mu;
        static long long cache_key[32] = {};
        static TcPlan cache_val[32];
        static int cache_next = 0;
        const int k_in = a.mem[0].k_in;
        const long long key = (long long)k_in * 1000003LL + a.n_out;
        bool hit = false;
        {
            std::lock_guard<std::mutex> lock(mu);
            for (int i = 0; i < 32; ++i)
                if (cache_key[i] == key) {
                    pl = cache_val[i];
                    hit = true;
                }
        }
        if (!hit) {
            pl = choose_plan(k_in, a.n_out, L::total, RPW);
            std::lock_guard<std::mutex> lock(mu);
            cache_key[cache_next] = key;
            cache_val[cache_next] = pl;
            cache_next = (cache_next + 1) % 32;
        }
    }
    prm.S = pl.S;
    prm.P = pl.S > 0 ? 0 : pl.P;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.S > 0 ? pl.S : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl_attr;
    cfg.gridDim = dim3((unsigned)pl.P, 1, 1);
    cfg.blockDim = dim3(kTcThreads, 1, 1);
    cfg.dynamicSmemBytes = L::total;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, kern, prm);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BITS, int NT>
cudaError_t launch_tc_t(const GemmArgs& a, cudaStream_t stream)
{
    return rpw_for(a) == 2 ? launch_tc_r<BITS, NT, 2>(a, stream) : launch_tc_r<BITS, NT, 1>(a, stream);
}

}  // namespace

int tc_ctas(int m, int k_in, int n_out, int bits)
{
    (void)m;
    (void)bits;
    return sk_ctas(n_out / 128, (long long)(n_out / 128) * (k_in / 128));
}

size_t tc_group_workspace_bytes(const GemmArgs& a) { return group_ws_bytes(a, nt_for(a.m)); }

size_t tc_workspace_bytes(int m, int k_in, int n_out, int bits)
{
    GemmArgs a = {};
    a.m = m;
    a.bits = bits;
    a.nmem = 1;
    a.shared_x = 1;
    a.mem[0].k_in = k_in;
    a.mem[0].n_out = n_out;
    finish_group(a);
    return group_ws_bytes(a, nt_for(m));
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
