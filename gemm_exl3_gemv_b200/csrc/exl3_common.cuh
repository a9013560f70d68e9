// exl3_common.cuh -- helpers shared by the libexl3 kernels: shared-memory
// barriers and bulk copies (sm_90+ PTX), the warp-level Hadamard-128, and the
// workspace layout.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace exl3 {

// ------------------------------------------------------------ workspace ---
// [0, 256)            status word (uint32 at 0): nonzero after a timed-out wait;
//                     word 1 (uint32 at 4): timeout injection for tests -- while
//                     it is nonzero (value v) each verify-kernel CTA issues only
//                     its first v - 1 copies of the rotated input, so the wait
//                     for the next one runs out (zero in normal use: the
//                     workspace is zero-filled)
// [256, 256 + 4*kMaxBlocks)  one arrival counter per 128-channel output block;
//                     a FIXED region, so that no call's partial sums or rotated
//                     input ever land on another call's counters when calls of
//                     different widths share a workspace (every call leaves the
//                     counters it used at zero)
// [ws_data_off(), ...) the call's own data: split-K partial sums, rotated input
constexpr size_t kWsHeader = 256;
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;     // debug builds: an index check failed
constexpr size_t kWsInjectOff = 4;

// Debug builds (compiled with -DEXL3_DEBUG_BOUNDS): the kernels check the
// index of every global access to the packed words, the workspace and the
// outputs against the size of the array it touches.  guard(ok, status)
// returns ok; a failed check also records kStatusBounds in the workspace
// status word, and the caller skips the access (a load gives zeros) -- never a
// trap, so the context stays usable.  Release builds compile the checks away.
#ifdef EXL3_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
#ifdef __CUDACC__
__device__ __forceinline__ bool guard(bool ok, uint32_t* status)
{
    if constexpr (kDebugBounds) {
        if (!ok) atomicOr(status, kStatusBounds);
        return ok;
    } else {
        return true;
    }
}
#endif

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
// output blocks (128 channels) of one call, summed over a group: at most
// kMaxBlocks (1,048,576 output channels)
constexpr int kMaxBlocks = 8192;
__host__ __device__ inline size_t ws_counter_off() { return kWsHeader; }
__host__ __device__ inline size_t ws_data_off() { return align_up(kWsHeader + 4 * (size_t)kMaxBlocks, 256); }

// ------------------------------------------------------------ addressing ---
__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------- mbarrier ---
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// make barrier initialisation visible to the async (bulk-copy) proxy
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended in hardware for up to
// `hint_ns` nanoseconds while the phase is incomplete (no polling traffic).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after ~`limit_ns`
// nanoseconds.  Returns false on timeout (the caller records it and skips
// its work; nothing spins forever).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns = 2000000000ull)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// 1-D bulk copy global -> shared, completion reported on `bar` (tx bytes).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------- programmatic dependent launch ---
// A kernel launched with programmatic stream serialization may start while
// the previous kernel of its stream is still running.  grid_dep_wait():
// block until that kernel has completed and its writes are visible (returns
// at once for an ordinary launch); every thread that touches memory the
// previous kernel may read or write calls it first.  grid_dep_launch(): let
// the next kernel of the stream begin launching its CTAs.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------ Hadamard ---
// Unnormalised Walsh-Hadamard transform of one 128-element block held by a
// warp, 4 consecutive elements per lane (element 4*lane + e in v[e]).  Natural
// (Sylvester) order: butterflies (a, b) -> (a + b, a - b) with `a` the element
// whose index has the stage bit clear.
__device__ __forceinline__ void fwht128_warp(float (&v)[4])
{
    // stage bits 0 and 1 are inside the lane
    float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2;
    v[1] = a1 + a3;
    v[2] = a0 - a2;
    v[3] = a1 - a3;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {      // stage bits 2..6 live in the lane index
        const bool upper = (lane & d) != 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float p = __shfl_xor_sync(0xffffffffu, v[e], d);
            v[e] = upper ? (p - v[e]) : (v[e] + p);
        }
    }
}

// fwht128_warp on R independent rows at once (same arithmetic per row): each
// shuffle stage issues R*4 independent shuffles, so one warp hides the
// shuffle latency that a row-by-row loop exposes.
template <int R>
__device__ __forceinline__ void fwht128_warp_rows(float (&v)[R][4])
{
#pragma unroll
    for (int r = 0; r < R; ++r) {
        float a0 = v[r][0] + v[r][1], a1 = v[r][0] - v[r][1], a2 = v[r][2] + v[r][3], a3 = v[r][2] - v[r][3];
        v[r][0] = a0 + a2;
        v[r][1] = a1 + a3;
        v[r][2] = a0 - a2;
        v[r][3] = a1 - a3;
    }
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const bool upper = (lane & d) != 0;
        float p[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < 4; ++e) p[r][e] = __shfl_xor_sync(0xffffffffu, v[r][e], d);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < 4; ++e) v[r][e] = upper ? (p[r][e] - v[r][e]) : (v[r][e] + p[r][e]);
    }
}

constexpr float kInvSqrt128 = 0.08838834764831845f;

}  // namespace exl3
