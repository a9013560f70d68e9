// gemm_large.cu -- the product for many input rows (prompt prefill): decode the
// whole matrix once into the tensor-core operand layout, then a tcgen05 GEMM.
//
// What is computed (the prompt-processing side of the decode speeds on the
// orcasaq2-rocm README -- the prefill rates given below its speed table -- and
// of the exl3-rdna4-recipe page, "What you get"):
//     y = sv .* H( scale .* ( H(su .* x) W ) ),   x: m x K_in, y: m x N_out
// At large m each decoded weight feeds 2m flops, so the decode is paid once per
// call and the contraction runs as a dense tensor-core GEMM:
//   1. decode_aimage_kernel: every warp decodes one tile row of one 128-channel
//      output block (as the verify kernel's decoders do) and writes it as the
//      4 KB MN-major, 128-byte-swizzled A operand image the MMA reads, into the
//      workspace: image (g, 64-row chunk c) = 16 KB = 4 tile rows, contiguous.
//   2. xt_tiled_prepass_kernel: xt = H(su .* x) in fp16, laid out as the B
//      operand (K-major, 128-byte swizzle) per tile of NB input rows:
//      xt (j, c) = NB rows x 64 k = NB * 128 contiguous bytes, rows past m zero.
//   3. gemm_large_kernel<NB>: persistent CTAs (one wave), each taking every
//      gridDim-th tile (output block g, row tile j).  Warp 0 streams A and B
//      chunks with 1-D bulk copies (cp.async.bulk + mbarrier) into a 3- or
//      4-stage ring that runs on across tiles; one thread of warp 1 issues
//      tcgen05.mma kind::f16 (M = 128 channels, N = NB rows, K = 16; four per
//      64-row chunk) into one of two tensor-memory accumulators, alternating
//      per tile; warps 4-7 drain the other one 16 rows at a time (tcgen05.ld),
//      scale, rotate and store y -- the epilogue of a tile overlaps the
//      mainloop of the next.
//   No split-K: each output element is one accumulator's fixed-order sum, so
//   results are bitwise repeatable.  Every wait is bounded (2 s).
#include <atomic>

#include "exl3_aop.cuh"
#include "exl3_common.cuh"
#include "exl3_decode.cuh"
#include "exl3_internal.h"
#include "exl3_tc.cuh"

namespace exl3 {

namespace {

constexpr int kLgThreads = 256;                // warp 0 producer, warp 1 MMA issuer, warps 4-7 epilogue
constexpr int kLgEpiWarp0 = 4;
constexpr int kAChunk = 16384;                 // A image of one 64-row chunk of one output block
constexpr uint64_t kLgWaitNs = 2000000000ull;

// ------------------------------------------------------------- 1. decode ---
template <int BITS>
__global__ void __launch_bounds__(256) decode_aimage_kernel(const uint32_t* __restrict__ packed, int k_in, int n_out,
                                                            uint8_t* __restrict__ image, uint32_t two16,
                                                            uint32_t* status)
{
    constexpr int TW = 8 * BITS, QW = 2 * BITS;
    grid_dep_wait();                                  // the image is read by the previous call's GEMM
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = k_in / 16, tiles_n = n_out / 16;
    const long long item = (long long)blockIdx.x * 8 + warp;   // (block g, tile row tr)
    if (item >= (long long)(n_out / 128) * T) return;
    const int g = (int)(item / T), tr = (int)(item % T);
    uint32_t w[QW];
    load_lane_words_checked<BITS>(w, packed + ((size_t)tr * tiles_n + 8 * (size_t)g) * TW + (size_t)lane * QW, packed,
                                  (size_t)T * tiles_n * TW, status);
    const int q = lane & 3;
    uint32_t buf[QW + 1];
    buf[0] = __shfl_sync(0xffffffffu, w[QW - 1], (lane & ~3) | ((q + 3) & 3));
#pragma unroll
    for (int t = 0; t < QW; ++t) buf[t + 1] = w[t];
    uint32_t soff[2][2];
    lane_soff(lane, soff);
    uint8_t* dst = image + ((size_t)g * T + tr) * 4096;
    const bool in = guard(((size_t)g * T + tr + 1) * 4096 <= (size_t)k_in * n_out * 2, status);
    decode_quarter_to_a<BITS>(buf, soff, two16, [&](uint32_t off, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
        if (in) *reinterpret_cast<uint4*>(dst + off) = make_uint4(w0, w1, w2, w3);
    });
    grid_dep_launch();
}

// ---------------------------------------------------------- 2. pre-pass ---
// Same rotation and in-chunk layout as the verify kernel's pre-pass (within
// each 16-row group, k = 4q + r sits at position 8(r >> 1) + 4(r & 1) + q, to
// match the A image), tiled by NB input rows.
__global__ void __launch_bounds__(256) xt_tiled_prepass_kernel(const __half* __restrict__ x,
                                                               const __half* __restrict__ su, int m_rows,
                                                               int m_pad, int k_in, int nb, uint8_t* __restrict__ xt)
{
    grid_dep_wait();
    const long long item = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (item < (long long)m_pad * ((k_in / 128 + 3) / 4)) xt_rotate_item(x, su, m_rows, k_in, nb, xt, item);
    grid_dep_launch();
}

// --------------------------------------------------------------- 3. GEMM ---
template <int NB>
struct LgLayout {
    static constexpr int BCHUNK = NB * 128;                 // B bytes per 64-row chunk
    static constexpr int STAGE = kAChunk + BCHUNK;
    // ring depth: a 256-row tile runs one CTA per SM and takes four stages (the
    // bulk-copy latency of three left the tensor pipe half idle, measured);
    // smaller tiles run two CTAs per SM with three stages each
    static constexpr int STAGES = NB == 256 ? 4 : 3;
    static constexpr int off_stage = 0;
    static constexpr int off_z = off_stage + STAGES * STAGE;   // z [16][128] fp32
    static constexpr int off_bar = off_z + 16 * 128 * 4;
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], last
    static constexpr int nbar = 2 * STAGES + 5;
    static constexpr int off_misc = off_bar + nbar * 8;
    static constexpr int total = off_misc + 64 + 1024;      // + slack to align the base to 1024
    // two accumulators of NB columns (the epilogue of one tile overlaps the
    // mainloop of the next); CTAS_PER_SM resident CTAs fill tensor memory exactly
    static constexpr int TMEM_COLS = 2 * NB;
    static constexpr int CTAS_PER_SM = NB == 256 ? 1 : 2;
    static_assert(STAGE % 1024 == 0 && off_z % 1024 == 0, "layout");
    static_assert(total <= 227 * 1024, "shared memory");
    static_assert(NB == 64 || NB == 128 || NB == 256, "tensor memory columns");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "tensor memory");
    // no further CTA fits on an SM (shared memory), so allocations never wait
    static_assert((CTAS_PER_SM + 1) * (total + 1024) > 228 * 1024, "CTAs per SM");
};

struct LgParams {
    const uint8_t* image;     // decoded A images
    const uint8_t* xt;        // B images
    const uint16_t* scale;
    const uint16_t* sv;
    void* y;
    uint32_t* status;
    int y_fp32, m, k_in, n_out;
    int J;                    // row tiles (m_pad / NB)
    int jfast;                // tile order: 1 = row tile fastest, 0 = output block fastest
};

__device__ __forceinline__ bool lg_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait_sleep(bar, parity, 1000)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kLgWaitNs) {
            atomicExch((int*)abort_flag, 1);
            return false;
        }
    }
}

// Tile t of the persistent order.  A wave of resident CTAs covers consecutive
// tiles, so the order decides what must stay in L2: output-block fastest keeps
// the whole A image and a few row tiles of xt; row-tile fastest keeps the
// whole xt and a few output blocks of the image.  The launcher picks the
// smaller set.
__device__ __forceinline__ void tile_of(const LgParams& prm, int G, int t, int& g, int& j)
{
    if (prm.jfast) {
        j = t % prm.J;
        g = t / prm.J;
    } else {
        g = t % G;
        j = t / G;
    }
}

template <int NB>
__global__ void __launch_bounds__(kLgThreads, 1) gemm_large_kernel(LgParams prm)
{
    using L = LgLayout<NB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::off_bar);
    uint64_t* empty = full + L::STAGES;
    uint64_t* acc_full = empty + L::STAGES;      // [2]: the tile's MMAs into accumulator a completed
    uint64_t* acc_empty = acc_full + 2;          // [2]: the epilogue has read accumulator a
    uint64_t* lastbar = acc_empty + 2;           // every MMA of the CTA completed
    int* misc = reinterpret_cast<int*>(smem + L::off_misc);   // [0] tmem base, [1] abort
    volatile int* abort_flag = misc + 1;
    float* zsm = reinterpret_cast<float*>(smem + L::off_z);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = prm.n_out / 128;
    const int tiles = G * prm.J;                 // tile t -> (g, j): see tile_of
    const int C64 = prm.k_in / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < L::STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
        mbar_init(lastbar, 1);
        misc[1] = 0;
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
    grid_dep_wait();                                   // A and B images are the pre-passes' output

    if (warp == 0 && lane == 0) {
        // ---- producer: A and B chunks of this CTA's tiles into the stage ring ----
        int q = 0;                                     // chunks issued (ring position)
        // a nonzero injection word (tests of the timeout path) withholds every copy
        bool ok = *reinterpret_cast<const volatile uint32_t*>(reinterpret_cast<const uint8_t*>(prm.status) +
                                                               kWsInjectOff) == 0u;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            int g, j;
            tile_of(prm, G, t, g, j);
            const uint8_t* a_src = prm.image + (size_t)g * C64 * kAChunk;
            const uint8_t* b_src = prm.xt + (size_t)j * C64 * L::BCHUNK;
            if (!guard((size_t)(g + 1) * C64 * kAChunk <= (size_t)prm.k_in * prm.n_out * 2 &&
                           (size_t)(j + 1) * C64 * L::BCHUNK <= (size_t)prm.J * NB * prm.k_in * 2,
                       prm.status)) {
                ok = false;
                break;
            }
            for (int c = 0; c < C64; ++c, ++q) {
                const int s = q % L::STAGES;
                if (q >= L::STAGES && !lg_wait(&empty[s], (uint32_t)(q / L::STAGES - 1) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full[s], L::STAGE);
                uint8_t* st = smem + L::off_stage + s * L::STAGE;
                bulk_g2s(st, a_src + (size_t)c * kAChunk, kAChunk, &full[s]);
                bulk_g2s(st + kAChunk, b_src + (size_t)c * L::BCHUNK, L::BCHUNK, &full[s]);
            }
        }
        // on abort, let every issued copy land before the CTA can exit
        if (*abort_flag)
            for (int v = q > L::STAGES ? q - L::STAGES : 0; v < q; ++v)
                (void)mbar_wait_bounded(&full[v % L::STAGES], (uint32_t)(v / L::STAGES) & 1u, 100000000ull);
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: per tile, four K = 16 steps per chunk into accumulator it & 1 ----
        constexpr uint32_t idesc = idesc_f16_amn(128, NB);
        bool ok = true;
        int q = 0, it = 0;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t d = tmem + (uint32_t)(acc * NB);
            if (it >= 2 && !lg_wait(&acc_empty[acc], (uint32_t)((it >> 1) - 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int c = 0; c < C64; ++c, ++q) {
                const int s = q % L::STAGES;
                if (!lg_wait(&full[s], (uint32_t)(q / L::STAGES) & 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + L::off_stage + s * L::STAGE);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ss(d, sdesc_sw128(st + k * 4096, 1024, 2048), sdesc_sw128(st + kAChunk + k * 32, 16, 1024),
                               idesc, (c > 0 || k > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(&acc_full[acc]);
        }
        // every MMA issued here completes before the CTA may free tensor memory
        mma_commit(lastbar);
        (void)mbar_wait_bounded(lastbar, 0u, 100000000ull);
    } else if (warp >= kLgEpiWarp0) {
        // ---- epilogue warps (tensor-memory lanes 32 * (warp % 4)): accumulator -> z -> y,
        // 16 rows at a time, while the next tile's MMAs run into the other accumulator ----
        const int ew = warp - kLgEpiWarp0;                         // == warp % 4
        const int ch = chan_of_row(32 * ew + lane);
        int it = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
            const int acc = it & 1;
            int g, j;
            tile_of(prm, G, t, g, j);
            // this lane's four output channels of block g: scale and signs
            const int n0 = 128 * g + 4 * lane;
            float osc[4], osg[4];
            {
                const uint2 sc = *reinterpret_cast<const uint2*>(prm.scale + n0);
                const uint2 sg = *reinterpret_cast<const uint2*>(prm.sv + n0);
                const float2 sc0 = __half22float2(*reinterpret_cast<const __half2*>(&sc.x));
                const float2 sc1 = __half22float2(*reinterpret_cast<const __half2*>(&sc.y));
                const float2 sg0 = __half22float2(*reinterpret_cast<const __half2*>(&sg.x));
                const float2 sg1 = __half22float2(*reinterpret_cast<const __half2*>(&sg.y));
                osc[0] = sc0.x; osc[1] = sc0.y; osc[2] = sc1.x; osc[3] = sc1.y;
                osg[0] = kInvSqrt128 * sg0.x; osg[1] = kInvSqrt128 * sg0.y;
                osg[2] = kInvSqrt128 * sg1.x; osg[3] = kInvSqrt128 * sg1.y;
            }
            int okd = 1;
            if (lane == 0) okd = lg_wait(&acc_full[acc], (uint32_t)(it >> 1) & 1u, abort_flag) ? 1 : 0;
            okd = __shfl_sync(0xffffffffu, okd, 0);
            tc_fence_after();
            for (int t0 = 0; t0 < NB; t0 += 16) {
                if (j * NB + t0 >= prm.m) break;              // uniform: rows past m are padding
                uint32_t t16[16];
                if (okd) {
                    tmem_ld16(tmem + ((uint32_t)(32 * ew) << 16) + (uint32_t)(acc * NB + t0), t16);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) t16[u] = 0u;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) zsm[u * 128 + ch] = __uint_as_float(t16[u]);
                named_bar(1, 128);
                // this warp's four rows together (independent shuffle chains)
                float vv[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 z4 = *reinterpret_cast<const float4*>(zsm + (4 * ew + i) * 128 + 4 * lane);
                    vv[i][0] = z4.x * osc[0];
                    vv[i][1] = z4.y * osc[1];
                    vv[i][2] = z4.z * osc[2];
                    vv[i][3] = z4.w * osc[3];
                }
                fwht128_warp_rows<4>(vv);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int mm = j * NB + t0 + 4 * ew + i;
                    if (mm >= prm.m) break;
                    const size_t yo = (size_t)mm * prm.n_out + n0;
                    const float o0 = vv[i][0] * osg[0], o1 = vv[i][1] * osg[1];
                    const float o2 = vv[i][2] * osg[2], o3 = vv[i][3] * osg[3];
                    if (prm.y_fp32) {
                        *reinterpret_cast<float4*>(reinterpret_cast<float*>(prm.y) + yo) = make_float4(o0, o1, o2, o3);
                    } else {
                        __half2 hh[2] = {__floats2half2_rn(o0, o1), __floats2half2_rn(o2, o3)};
                        *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(prm.y) + yo) = *reinterpret_cast<uint2*>(hh);
                    }
                }
                named_bar(1, 128);
            }
            // accumulator read out: the MMA issuer may reuse it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
        }
    }
    grid_dep_launch();

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
    if (threadIdx.x == 0 && misc[1]) atomicOr(prm.status, kStatusTimeout);
}

}  // namespace

// ------------------------------------------------------------------ host ---

int large_tile_rows(int m, int n_out)
{
    const long long G = n_out / 128;
    for (int nb : {256, 128}) {
        if (G * ((m + nb - 1) / nb) >= kLargeMinCtas) return nb;
    }
    return 64;
}

size_t large_workspace_bytes(int m, int k_in, int n_out)
{
    const int nb = large_tile_rows(m, n_out);
    const size_t m_pad = (size_t)((m + nb - 1) / nb) * nb;
    return kWsHeader + (size_t)k_in * n_out * 2 + m_pad * k_in * 2;
}

namespace {

template <int NB>
cudaError_t launch_gemm_large_nb(const LgParams& prm, cudaStream_t stream, int pdl)
{
    using L = LgLayout<NB>;
    auto kern = gemm_large_kernel<NB>;
    static std::atomic<int> configured[kMaxDevices];
    cudaError_t e = once_per_device(configured, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::total);
    });
    if (e != cudaSuccess) return e;
    const int G = prm.n_out / 128;
    // persistent: at most one wave of resident CTAs, each taking every gridDim-th tile
    int sms = 0, dev = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)G * prm.J;
    const long long slots = (long long)sms * L::CTAS_PER_SM;
    const int grid = (int)(tiles < slots ? tiles : slots);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kLgThreads, 1, 1);
    cfg.dynamicSmemBytes = L::total;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int BITS>
cudaError_t launch_decode_image(const uint32_t* packed, int k_in, int n_out, uint8_t* image, cudaStream_t stream,
                                int pdl, uint32_t* status)
{
    const long long items = (long long)(n_out / 128) * (k_in / 16);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)((items + 7) / 8), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, decode_aimage_kernel<BITS>, packed, k_in, n_out, image, 0x10000u, status);
}

}  // namespace

cudaError_t launch_gemm_large(const GemmArgs& a, cudaStream_t stream)
{
    const Member& sb = a.mem[0];                 // one product per call
    const int k_in = sb.k_in;
    const int nb = large_tile_rows(a.m, a.n_out);
    const int m_pad = (a.m + nb - 1) / nb * nb;
    uint8_t* image = a.ws + kWsHeader;
    uint8_t* xt = image + (size_t)k_in * a.n_out * 2;

    cudaError_t e = cudaErrorInvalidValue;
    switch (a.bits) {
        case 2: e = launch_decode_image<2>(sb.packed, k_in, a.n_out, image, stream, a.pdl, reinterpret_cast<uint32_t*>(a.ws)); break;
        case 3: e = launch_decode_image<3>(sb.packed, k_in, a.n_out, image, stream, a.pdl, reinterpret_cast<uint32_t*>(a.ws)); break;
        case 4: e = launch_decode_image<4>(sb.packed, k_in, a.n_out, image, stream, a.pdl, reinterpret_cast<uint32_t*>(a.ws)); break;
    }
    if (e != cudaSuccess) return e;
    {
        const long long items = (long long)m_pad * ((k_in / 128 + 3) / 4);
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.gridDim = dim3((unsigned)((items + 7) / 8), 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = a.pdl ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, xt_tiled_prepass_kernel, reinterpret_cast<const __half*>(sb.x),
                               reinterpret_cast<const __half*>(sb.su), a.m, m_pad, k_in, nb, xt);
        if (e != cudaSuccess) return e;
    }
    LgParams prm;
    prm.image = image;
    prm.xt = xt;
    prm.scale = sb.scale;
    prm.sv = sb.sv;
    prm.y = sb.y;
    prm.status = reinterpret_cast<uint32_t*>(a.ws);
    prm.y_fp32 = a.y_fp32;
    prm.m = a.m;
    prm.k_in = k_in;
    prm.n_out = a.n_out;
    prm.J = m_pad / nb;
    {
        // L2 working set of a wave of tiles in each order (bytes): keep the smaller
        const double image = 2.0 * k_in * a.n_out, xtb = 2.0 * m_pad * k_in;
        const double wave = 148.0;                 // about one tile per SM in flight
        const double G = a.n_out / 128, J = prm.J;
        const double g_fast = image + xtb * (wave / G < J ? wave / G : J) / J;
        const double j_fast = xtb + image * (wave / J < G ? wave / J : G) / G;
        prm.jfast = j_fast < g_fast ? 1 : 0;
    }
    switch (nb) {
        case 256: e = launch_gemm_large_nb<256>(prm, stream, a.pdl); break;
        case 128: e = launch_gemm_large_nb<128>(prm, stream, a.pdl); break;
        default: e = launch_gemm_large_nb<64>(prm, stream, a.pdl); break;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace exl3
