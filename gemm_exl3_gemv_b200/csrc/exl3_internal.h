// exl3_internal.h -- launchers shared between the libexl3 translation units.
#pragma once
#include <cstddef>
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

namespace exl3 {

cudaError_t launch_decode_tiles(const uint32_t* packed, int k_in, int n_out, int bits, uint16_t* w_out,
                                cudaStream_t stream);
cudaError_t launch_hadamard128(const uint16_t* in, uint16_t* out, const uint16_t* signs, int rows, int n, int mode,
                               cudaStream_t stream);

// One product of a sibling group: the matrices that share the input x (and
// its sign vector su), e.g. the gate and up projections of an MLP, or q, k
// and v.  Output blocks of the group are numbered consecutively: sibling i
// owns blocks [g0, g0 + n_out / 128).
constexpr int kMaxSiblings = 8;
struct Sibling {
    const uint32_t* packed;   // trellis words (k_in x n_out)
    const uint16_t* scale;    // n_out fp16
    const uint16_t* sv;       // n_out fp16 +-1
    void* y;                  // m x n_out, fp16 or fp32
    int n_out;
    int g0;                   // first output block of this sibling
};

// Problem description shared by the product kernels.
struct GemmArgs {
    const uint16_t* x;        // m x k_in fp16
    const uint16_t* su;       // k_in fp16 +-1
    int y_fp32;
    int m, k_in, bits;
    int n_out;                // total output width of the group (sum over siblings)
    int nsib;                 // 1 .. kMaxSiblings
    Sibling sib[kMaxSiblings];
    unsigned char* ws;        // workspace base
    int pdl;                  // launch with programmatic dependent launch (overlap the previous kernel's tail)
};

#ifdef __CUDACC__
// The sibling holding group output block g, and g's block index inside it.
// Unrolled over the fixed-size table (no dynamically indexed parameters).
struct SibView {
    const uint32_t* packed;
    const uint16_t* scale;
    const uint16_t* sv;
    void* y;
    int n_out;
    int gl;
};
__device__ __forceinline__ SibView sibling_of(const GemmArgs& a, int g)
{
    SibView v{a.sib[0].packed, a.sib[0].scale, a.sib[0].sv, a.sib[0].y, a.sib[0].n_out, g};
#pragma unroll
    for (int t = 1; t < kMaxSiblings; ++t) {
        if (t < a.nsib && g >= a.sib[t].g0) {
            v = SibView{a.sib[t].packed, a.sib[t].scale, a.sib[t].sv, a.sib[t].y, a.sib[t].n_out, g - a.sib[t].g0};
        }
    }
    return v;
}
#endif

// Kernel attributes (shared-memory limit, cluster size) are per device: a
// process that drives several GPUs sets them once on each.  `done` is a
// per-kernel table indexed by device; returns the first error.
constexpr int kMaxDevices = 64;
template <typename F>
cudaError_t once_per_device(std::atomic<int> (&done)[kMaxDevices], F&& setup)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = setup();                                     // idempotent: a race only repeats it
    if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
    return e;
}

// Single-row product on CUDA cores (gemv_m1.cu).
size_t m1_workspace_bytes(int k_in, int n_out, int bits);
cudaError_t launch_gemv_m1(const GemmArgs& a, cudaStream_t stream);

// Tensor-core path (2..32 rows): CTA count (planned), workspace size,
// launcher (two launches per call: input rotation pre-pass and the product
// kernel, launched as clusters of the CTAs that share an output block).
int tc_ctas(int m, int k_in, int n_out, int bits);
size_t tc_workspace_bytes(int m, int k_in, int n_out, int bits);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream);

// Many-row path (gemm_large.cu): decode once into the tensor-core operand
// image, then a tcgen05 GEMM.  Rows per tile (256, 128 or 64: the largest that
// still gives kLargeMinCtas tiles), workspace size, launcher (three launches).
constexpr int kLargeMinCtas = 148;
int large_tile_rows(int m, int n_out);
size_t large_workspace_bytes(int m, int k_in, int n_out);
cudaError_t launch_gemm_large(const GemmArgs& a, cudaStream_t stream);

}  // namespace exl3
