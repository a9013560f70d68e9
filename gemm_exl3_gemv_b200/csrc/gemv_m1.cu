// gemv_m1.cu -- the single-row product (the decode-time GEMV) on CUDA cores.
//
// What is computed (the matrix-vector step behind the decode speeds of the
// orcasaq2-rocm README, whose second paragraph moves the EXL3 products onto
// the GPU's vector ALUs):
//     y = sv .* H( scale .* ( H(su .* x) W ) ),   x: 1 x K_in,  y: 1 x N_out
// with W decoded on the fly from the trellis stream (exl3_decode.cuh).
//
// At one input row the product does 2 flops per weight, so the decode sets
// the pace: the kernel is built to spend as few issue slots per weight as
// the format allows, spread over the integer (ALU) and FMA pipes.
//   * Per weight: isolate the 16-bit window (1-2 instructions, immediates
//     only), 3INST (IMAD + LOP3), and one packed fp16 FMA that multiplies
//     BOTH fp16 halves of the 3INST word by the activation at once:
//     acc2 += (lo, hi) * (x, x).  The two halves are never added to each
//     other per weight; their sum appears in the accumulators.
//   * The fp16 accumulators take 8 input rows (two tile rows), then are added
//     into fp32 (mixed-precision f16 + f32 adds, sm_100).  Rounding budget:
//     x~ and the short fp16 sums each round at 2^-11 relative; against an
//     fp64 evaluation of the definition the relative L2 error stays near
//     6e-4 (the acceptance bound is 1e-3).
//   * Work: unit = one tile row of one 128-channel output block (one
//     Hadamard block): 8 tiles = 256*K contiguous bytes.  Stream-K: the units
//     are cut into equal contiguous ranges, one per CTA, one wave of CTAs,
//     so every SM decodes the same number of weights.  Within a segment (the
//     part of a range inside one block) warp w takes tile rows w, w+8, ...
//     and lane l decodes quarter l%4 of
//     tile l/4 (4 input rows x 16 channels, 64 consecutive weights whose bits
//     start on a word boundary).  Lane l's words are bytes [8K*l, 8K*l + 8K)
//     of the tile row, so the warp's loads are contiguous 128-bit (K = 2, 4)
//     or 64-bit (K = 3) global loads straight into registers, one tile row
//     ahead of the decode; no shared-memory staging.  The 16 look-back bits
//     come from the neighbouring lane by a shuffle (the tail-biting wrap for
//     quarter 0 comes from quarter 3 of the same tile).
//   * A block cut over several CTAs: each writes its partial sum to the
//     workspace; the last CTA to arrive (atomic counter, no waiting) adds
//     them in CTA order -- fixed, so results are bitwise repeatable -- then
//     scales, rotates and writes y.
#include <atomic>

#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"

namespace exl3 {

namespace {

constexpr int kM1Warps = 8;
constexpr int kM1Threads = 32 * kM1Warps;
// resident CTAs per SM the register budget is set for (80 registers a thread;
// at 64 the accumulators, two tile rows of words and the segment state spill)
template <int BITS>
constexpr int kM1MinBlocks = 3;
constexpr int kSms = 148;

__device__ __forceinline__ __half2 as_h2(uint32_t u)
{
    return *reinterpret_cast<const __half2*>(&u);
}

// acc += lo + hi of a packed fp16 pair, in fp32 (two mixed-precision adds)
__device__ __forceinline__ float add_pair_f32(float acc, __half2 p)
{
    const uint32_t u = *reinterpret_cast<const uint32_t*>(&p);
    float r;
    asm("{\n\t.reg .f16 l, h;\n\t"
        "mov.b32 {l, h}, %1;\n\t"
        "add.f32.f16 %0, l, %2;\n\t"
        "add.f32.f16 %0, h, %0;\n\t}"
        : "=f"(r)
        : "r"(u), "f"(acc));
    return r;
}

// Decode one quarter tile (weights R = 0..63: input row R/16 of the quarter,
// channel R%16 of the tile) and accumulate (lo, hi) * (x, x).  FIRST: the
// accumulators start from this quarter (multiply instead of FMA on row 0).
// ALT_EVERY: every ALT_EVERY-th non-aligned window uses the FMA-pipe form;
// ALT_EVERY < 0: byte-aligned windows from shifted words (even bit widths).
template <int BITS, int R, bool FIRST, int ALT_EVERY, int NW>
__device__ __forceinline__ void quarter_hfma(const uint32_t (&buf)[NW], const __half2 (&xx)[4], __half2 (&acc)[16],
                                             uint32_t two16)
{
    if constexpr (R < 64) {
        constexpr bool alt = ALT_EVERY > 0 && (R % (ALT_EVERY > 0 ? ALT_EVERY : 1)) == 0;
        uint32_t st;
        if constexpr (ALT_EVERY < 0) st = window_bytes<(R + 1) * BITS + 16, NW>(buf, two16);
        else st = window_of<(R + 1) * BITS + 16, NW, alt>(buf, two16);
        const uint32_t m = inst3(st);
        if constexpr (FIRST && R < 16) acc[R & 15] = __hmul2(as_h2(m), xx[R >> 4]);
        else acc[R & 15] = __hfma2(as_h2(m), xx[R >> 4], acc[R & 15]);
        quarter_hfma<BITS, R + 1, FIRST, ALT_EVERY>(buf, xx, acc, two16);
    }
}

template <int BITS, bool FIRST, int ALT_EVERY>
__device__ __forceinline__ void tile_row(const uint32_t (&w)[2 * BITS], const uint32_t* xxs, int krow, int src_prev,
                                         __half2 (&acc)[16], uint32_t two16)
{
    constexpr int QW = 2 * BITS;
    uint32_t buf[QW + 1];
    buf[0] = __shfl_sync(0xffffffffu, w[QW - 1], src_prev);
#pragma unroll
    for (int t = 0; t < QW; ++t) buf[t + 1] = w[t];
    const uint4 xv = *reinterpret_cast<const uint4*>(xxs + krow);
    const __half2 xx[4] = {as_h2(xv.x), as_h2(xv.y), as_h2(xv.z), as_h2(xv.w)};
    quarter_hfma<BITS, 0, FIRST, ALT_EVERY>(buf, xx, acc, two16);
}

// Stream-K partition: the G x T units (channel block g, tile row r; block
// major) are cut into P equal contiguous ranges, one per CTA, P = SMs x
// resident CTAs, so every SM gets the same amount of decode work.  A range
// may cover the end of one block and the start of the next; each (CTA,
// block) piece is a segment, whose partial sum goes to workspace slot
// p + g (unique: ranges are monotone).
struct M1Plan {
    int P;            // CTAs
    long long U;      // units: sum over the group's members of blocks x tile rows
    int kb_max;       // 128-row input blocks one segment can touch
};

__host__ __device__ inline int m1_cta_of_unit(long long x, int P, long long U)
{
    return (int)(((x + 1) * P - 1) / U);
}

template <int BITS, int ALT_EVERY>
__global__ void __launch_bounds__(kM1Threads, kM1MinBlocks<BITS>)
    gemv_m1_kernel(GemmArgs a, M1Plan pl, uint32_t two16)
{
    constexpr int QW = 2 * BITS;       // words per lane per tile row
    constexpr int TW = 8 * BITS;       // words per tile
    extern __shared__ __align__(16) unsigned char smem[];
    float* red = reinterpret_cast<float*>(smem);                              // [warps][128]
    int* flag = reinterpret_cast<int*>(smem + sizeof(float) * kM1Warps * 128); // last-CTA flag
    uint32_t* xxs = reinterpret_cast<uint32_t*>(smem + sizeof(float) * kM1Warps * 128 + 16);   // (x, x) per row

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = blockIdx.x;
    const long long b0 = (long long)p * pl.U / pl.P, b1 = (long long)(p + 1) * pl.U / pl.P;
    const int q = lane & 3;
    const int src_prev = (lane & ~3) | ((q + 3) & 3);
    float* part = reinterpret_cast<float*>(a.ws + ws_data_off());
    uint32_t* counters = reinterpret_cast<uint32_t*>(a.ws + ws_counter_off());
    uint32_t* status = reinterpret_cast<uint32_t*>(a.ws);
    const int G = a.n_out / 128;
    // partial slot s is in bounds (debug builds)
    auto slot_ok = [&](long long s) {
        return guard(s >= 0 && s < (long long)pl.P + G &&
                         ws_data_off() + (size_t)(s + 1) * 128 * sizeof(float) <= a.ws_bytes,
                     status);
    };
    grid_dep_launch();                     // the next product may start loading its weights
    bool first_seg = true;
    // the first words of this warp's next segment, loaded before the current
    // segment's reduction and epilogue so that their latency hides behind them
    // (measured: 2.4 % off the single-row layer call)
    uint32_t wa[QW];
    auto seg_load = [&](long long us) {
        const MemView mv = member_of_unit(a, us);
        const int T = mv.k_in / 16;
        const int gl = (int)((us - mv.u0) / T);
        const long long ublk = mv.u0 + (long long)gl * T;
        const int rs = (int)(us - ublk);
        const int re = (int)((ublk + T < b1 ? ublk + T : b1) - ublk);
        if (re - rs > warp) {
            const int tiles_n = mv.n_out / 16;
            const uint32_t* s0 = mv.packed + ((size_t)(rs + warp) * tiles_n + 8 * (size_t)gl) * TW + (size_t)lane * QW;
            load_lane_words_checked<BITS>(wa, s0, mv.packed, (size_t)T * tiles_n * TW, status);
        }
    };
    if (b0 < b1) seg_load(b0);

    for (long long u = b0; u < b1;) {
        // ---- segment: block g (group numbering), tile rows [r0, r1) of its member ----
        // (the member view is looked up again after the main loop, from g, so
        // that nothing of it stays live in registers across the decode)
        int g, r0, r1;
        const uint32_t* src;
        const uint32_t* wbase;                                         // the member's packed words
        size_t row_step, n_words;                                      // words between a warp's rows; matrix size
        {
            const MemView mv = member_of_unit(a, u);
            const int T = mv.k_in / 16;                                // tile rows per block of this member
            const int gl = (int)((u - mv.u0) / T);
            g = mv.g0 + gl;
            const long long ublk = mv.u0 + (long long)gl * T;          // the block's first unit
            r0 = (int)(u - ublk);
            r1 = (int)((ublk + T < b1 ? ublk + T : b1) - ublk);
            const int tiles_n = mv.n_out / 16;
            row_step = (size_t)kM1Warps * tiles_n * TW;
            n_words = (size_t)T * tiles_n * TW;
            wbase = mv.packed;
            src = mv.packed + ((size_t)(r0 + warp) * tiles_n + 8 * (size_t)gl) * TW + (size_t)lane * QW;
        }
        u += r1 - r0;
        const int kb_lo = r0 >> 3, kb_hi = (r1 + 7) >> 3;             // 128-row input blocks touched
        const int nrow = r1 - r0;
        const int nw = nrow > warp ? (nrow - warp + kM1Warps - 1) / kM1Warps : 0;
        uint32_t wb[QW];
        if (first_seg) grid_dep_wait();    // weights are never written; x, y, workspace only after this
        first_seg = false;

        __syncthreads();                                               // previous segment done with smem
        // input rotation of the touched blocks: xxs[k - 128 kb_lo] = (xt, xt)
        for (int kb = kb_lo + warp; kb < kb_hi; kb += kM1Warps) {
            const MemView mv = member_of_block(a, g);
            const int col = kb * 128 + 4 * lane;
            const bool in = guard(col + 4 <= mv.k_in && kb - kb_lo < pl.kb_max, status);
            const uint2 raw = in ? *reinterpret_cast<const uint2*>(mv.x + col) : make_uint2(0u, 0u);
            const uint2 sraw = in ? *reinterpret_cast<const uint2*>(mv.su + col) : make_uint2(0u, 0u);
            const float2 x0 = __half22float2(as_h2(raw.x)), x1 = __half22float2(as_h2(raw.y));
            const float2 s0 = __half22float2(as_h2(sraw.x)), s1 = __half22float2(as_h2(sraw.y));
            float v[4] = {x0.x * s0.x, x0.y * s0.y, x1.x * s1.x, x1.y * s1.y};
            fwht128_warp(v);
            uint4 o;
            __half2 h;
            h = __float2half2_rn(v[0] * kInvSqrt128); o.x = *reinterpret_cast<uint32_t*>(&h);
            h = __float2half2_rn(v[1] * kInvSqrt128); o.y = *reinterpret_cast<uint32_t*>(&h);
            h = __float2half2_rn(v[2] * kInvSqrt128); o.z = *reinterpret_cast<uint32_t*>(&h);
            h = __float2half2_rn(v[3] * kInvSqrt128); o.w = *reinterpret_cast<uint32_t*>(&h);
            if (in) *reinterpret_cast<uint4*>(xxs + (kb - kb_lo) * 128 + 4 * lane) = o;
        }
        __syncthreads();

        // ---- main loop: tile rows r0 + warp + 8 i of the segment ----
        const int kx0 = (r0 + warp) * 16 - kb_lo * 128 + 4 * q;         // xxs index of this lane's first row
        constexpr int kx_step = kM1Warps * 16;

        float accf[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) accf[c] = 0.f;
        __half2 acc[16];
        int i = 0;
        for (; i + 2 <= nw; i += 2) {
            load_lane_words_checked<BITS>(wb, src + (size_t)(i + 1) * row_step, wbase, n_words, status);
            tile_row<BITS, true, ALT_EVERY>(wa, xxs, kx0 + i * kx_step, src_prev, acc, two16);
            if (i + 2 < nw) load_lane_words_checked<BITS>(wa, src + (size_t)(i + 2) * row_step, wbase, n_words, status);
            tile_row<BITS, false, ALT_EVERY>(wb, xxs, kx0 + (i + 1) * kx_step, src_prev, acc, two16);
#pragma unroll
            for (int c = 0; c < 16; ++c) accf[c] = add_pair_f32(accf[c], acc[c]);
        }
        if (i < nw) {
            tile_row<BITS, true, ALT_EVERY>(wa, xxs, kx0 + i * kx_step, src_prev, acc, two16);
#pragma unroll
            for (int c = 0; c < 16; ++c) accf[c] = add_pair_f32(accf[c], acc[c]);
        }

        if (u < b1) seg_load(u);                                       // in flight during the reduction
        // ---- reduce: the 4 quarters of a tile, then the 8 warps (fixed order) ----
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float t = accf[c];
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            accf[c] = t;
        }
        if (q == 0) {
            float4* d = reinterpret_cast<float4*>(red + warp * 128 + 16 * (lane >> 2));
#pragma unroll
            for (int t = 0; t < 4; ++t)
                d[t] = make_float4(accf[4 * t], accf[4 * t + 1], accf[4 * t + 2], accf[4 * t + 3]);
        }
        __syncthreads();
        float z = 0.f;
        if (threadIdx.x < 128) {
#pragma unroll
            for (int w = 0; w < kM1Warps; ++w) z += red[w * 128 + threadIdx.x];
        }

        // ---- a block split over several CTAs: the last to arrive finishes it ----
        const MemView mv = member_of_block(a, g);
        const int T = mv.k_in / 16;
        const long long ublk = mv.u0 + (long long)mv.gl * T;
        if (nrow < T) {
            const int p_first = m1_cta_of_unit(ublk, pl.P, pl.U);
            const int p_last = m1_cta_of_unit(ublk + T - 1, pl.P, pl.U);
            if (threadIdx.x < 128 && slot_ok(p + g)) __stcg(part + (size_t)(p + g) * 128 + threadIdx.x, z);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) {
                const uint32_t prev = atomicAdd(&counters[g], 1u);
                flag[0] = (prev == (uint32_t)(p_last - p_first)) ? 1 : 0;
            }
            __syncthreads();
            if (!flag[0]) continue;                                    // uniform across the CTA
            __threadfence();
            {
                // all 256 threads: channel t % 128 over every second partial
                // (t / 128 picks the parity), eight independent loads in flight,
                // then the two parities added -- a fixed order
                const int c = threadIdx.x & 127, h = threadIdx.x >> 7;
                const float* pp = part + (size_t)g * 128 + c;
                float zz = 0.f;
                int qq = p_first + h;
                for (; qq + 14 <= p_last; qq += 16) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        v[e] = slot_ok(qq + 2 * e + g) ? __ldcg(pp + (size_t)(qq + 2 * e) * 128) : 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) zz += v[e];
                }
                for (; qq <= p_last; qq += 2) zz += slot_ok(qq + g) ? __ldcg(pp + (size_t)qq * 128) : 0.f;
                red[threadIdx.x] = zz;
                __syncthreads();
                if (threadIdx.x < 128) z = red[threadIdx.x] + red[128 + threadIdx.x];
            }
            if (threadIdx.x == 0) counters[g] = 0u;                    // ready for the next call on this stream
        }
        __syncthreads();                                               // all reads of `red` done
        if (threadIdx.x < 128) red[threadIdx.x] = z;
        __syncthreads();

        // ---- epilogue (warp 0): scale, output rotation, signs, store ----
        if (warp == 0 && guard(128 * mv.gl + 128 <= mv.n_out, status)) {
            const MemView sib = mv;
            const int n0 = 128 * mv.gl + 4 * lane;
            const float4 z4 = *reinterpret_cast<const float4*>(red + 4 * lane);
            const uint2 sc = *reinterpret_cast<const uint2*>(sib.scale + n0);
            const uint2 sg = *reinterpret_cast<const uint2*>(sib.sv + n0);
            const float2 sc0 = __half22float2(as_h2(sc.x)), sc1 = __half22float2(as_h2(sc.y));
            const float2 sg0 = __half22float2(as_h2(sg.x)), sg1 = __half22float2(as_h2(sg.y));
            float v[4] = {z4.x * sc0.x, z4.y * sc0.y, z4.z * sc1.x, z4.w * sc1.y};
            fwht128_warp(v);
            v[0] *= kInvSqrt128 * sg0.x;
            v[1] *= kInvSqrt128 * sg0.y;
            v[2] *= kInvSqrt128 * sg1.x;
            v[3] *= kInvSqrt128 * sg1.y;
            if (a.y_fp32) {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(sib.y) + n0) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                __half2 h[2] = {__floats2half2_rn(v[0], v[1]), __floats2half2_rn(v[2], v[3])};
                *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(sib.y) + n0) = *reinterpret_cast<uint2*>(h);
            }
        }
    }
}

// Units of member i start at u0 = the tile rows of the members before it.
// Sets a.mem[i].u0 (host side) and returns the plan.
M1Plan m1_plan(GemmArgs& a)
{
    const int per_sm = kM1MinBlocks<3>;
    long long U = 0;
    for (int i = 0; i < a.nmem; ++i) {
        a.mem[i].u0 = U;
        U += (long long)(a.mem[i].n_out / 128) * (a.mem[i].k_in / 16);
    }
    const int G = a.n_out / 128;
    M1Plan pl;
    pl.U = U;
    const long long slots = (long long)kSms * per_sm;   // one wave of resident CTAs
    // When every block has the same length (one k_in), give every block the
    // same whole number of CTAs, so that no range straddles two blocks (one
    // segment per CTA: the per-segment costs -- input rotation, reduction,
    // arrival -- are paid once), unless that leaves more than 15 % of the
    // slots idle; then, and for groups of several lengths, cut evenly across
    // blocks (stream-K).
    long long P = (a.same_k && G <= slots) ? (long long)G * (slots / G) : slots;
    if (20 * P < 17 * slots) P = slots;                 // whole-block split would idle >15 % of the slots
    if (P > pl.U / kM1Warps) P = pl.U / kM1Warps;       // at least one tile row per warp
    const long long rows_cap = 1024;                    // bounds the rotated input kept in shared memory
    if (P < (pl.U + rows_cap - 1) / rows_cap) P = (pl.U + rows_cap - 1) / rows_cap;
    if (P < 1) P = 1;
    pl.P = (int)P;
    const long long rows_max = (pl.U + P - 1) / P;
    pl.kb_max = (int)((rows_max + 7) / 8 + 1);
    return pl;
}

size_t m1_smem_bytes(const M1Plan& pl)
{
    return sizeof(float) * kM1Warps * 128 + 16 + sizeof(uint32_t) * 128 * (size_t)pl.kb_max;
}

// Form of the window isolation per bit width (measured on B200): 2 and 4
// bits read byte-aligned windows from shifted words; 3 bits (windows at
// every bit offset) puts every third non-aligned window on the FMA pipe
// (every second: 2-4 % slower; every one: 15 % slower).
#ifndef EXL3_M1_ALT3
#define EXL3_M1_ALT3 3
#endif
#ifndef EXL3_M1_ALT24
#define EXL3_M1_ALT24 (-1)
#endif
template <int BITS>
constexpr int kAltEvery = BITS == 3 ? EXL3_M1_ALT3 : EXL3_M1_ALT24;

template <int BITS>
cudaError_t launch_m1_t(GemmArgs a, cudaStream_t stream)
{
    const M1Plan pl = m1_plan(a);
    const size_t smem = m1_smem_bytes(pl);
    auto kern = gemv_m1_kernel<BITS, kAltEvery<BITS>>;
    static std::atomic<int> configured[kMaxDevices];
    if ((int)smem > 200 * 1024) return cudaErrorInvalidValue;
    cudaError_t ce = once_per_device(configured, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    });
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)pl.P, 1, 1);
    cfg.blockDim = dim3(kM1Threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, pl, 0x10000u);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

size_t m1_group_workspace_bytes(const GemmArgs& a0)
{
    GemmArgs a = a0;
    const M1Plan pl = m1_plan(a);
    return ws_data_off() + (size_t)(pl.P + a.n_out / 128) * 128 * sizeof(float);
}

size_t m1_workspace_bytes(int k_in, int n_out, int bits)
{
    GemmArgs a = {};
    a.m = 1;
    a.bits = bits;
    a.nmem = 1;
    a.mem[0].k_in = k_in;
    a.mem[0].n_out = n_out;
    finish_group(a);
    return m1_group_workspace_bytes(a);
}

cudaError_t launch_gemv_m1(const GemmArgs& a, cudaStream_t stream)
{
    switch (a.bits) {
        case 2: return launch_m1_t<2>(a, stream);
        case 3: return launch_m1_t<3>(a, stream);
        case 4: return launch_m1_t<4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace exl3
