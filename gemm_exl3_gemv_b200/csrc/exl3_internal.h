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

// A launch covers a group of 1..kMaxMembers products.  Member i has its own
// weights (packed, scale, sv), output y and shape; its input rows x and sign
// vector su are either its own (a grouped call: independent problems, e.g.
// the seven matrices of a layer in a verify sweep) or shared by every member
// (a sibling group: the gate and up projections of an MLP, or q, k and v).
// Output blocks (128 channels) and work units of the group are numbered
// member after member: member i owns blocks [g0, g0 + n_out/128) and units
// [u0, u0 + units of member i) of the launching kernel.
constexpr int kMaxMembers = 8;
struct Member {
    const uint16_t* x;        // m x k_in fp16 input rows
    const uint16_t* su;       // k_in fp16 +-1
    const uint32_t* packed;   // trellis words (k_in x n_out)
    const uint16_t* scale;    // n_out fp16
    const uint16_t* sv;       // n_out fp16 +-1
    void* y;                  // m x n_out, fp16 or fp32
    int k_in, n_out;
    int g0;                   // first output block of this member
    int pad_;
    long long u0;             // first work unit of this member (set by the launching path)
    long long xt0;            // verify path: byte offset of this member's rotated input in the x~ region
};

// Problem description shared by the product kernels.
struct GemmArgs {
    int y_fp32;
    int m, bits;
    int n_out;                // total output width of the group (sum over members)
    int k_max;                // largest k_in of the group
    int nmem;                 // 1 .. kMaxMembers
    int same_k;               // every member has the same k_in
    int shared_x;             // every member takes the same x and su (sibling group)
    Member mem[kMaxMembers];
    unsigned char* ws;        // workspace base
    size_t ws_bytes;          // workspace size (checked by the debug-bounds build)
    int pdl;                  // launch with programmatic dependent launch (overlap the previous kernel's tail)
};

// Fill the group numbering (g0) and n_out / k_max / same_k of `a` from its
// members' shapes.  Host side.
inline void finish_group(GemmArgs& a)
{
    int g = 0, kmax = 0, same = 1;
    for (int i = 0; i < a.nmem; ++i) {
        a.mem[i].g0 = g;
        g += a.mem[i].n_out / 128;
        if (a.mem[i].k_in > kmax) kmax = a.mem[i].k_in;
        if (a.mem[i].k_in != a.mem[0].k_in) same = 0;
    }
    a.n_out = 128 * g;
    a.k_max = kmax;
    a.same_k = same;
}

#ifdef __CUDACC__
// The member holding a group output block or work unit, with the block's
// index inside it.  Selected by unrolled compares over the fixed-size table
// (no dynamically indexed kernel parameters).
struct MemView {
    const uint16_t* x;
    const uint16_t* su;
    const uint32_t* packed;
    const uint16_t* scale;
    const uint16_t* sv;
    void* y;
    int k_in, n_out;
    int g0;
    long long u0;
    long long xt0;
    int gl;                   // block index inside the member (member_of_block)
};
__device__ __forceinline__ MemView view_of(const Member& t)
{
    return MemView{t.x, t.su, t.packed, t.scale, t.sv, t.y, t.k_in, t.n_out, t.g0, t.u0, t.xt0, 0};
}
__device__ __forceinline__ MemView member_of_block(const GemmArgs& a, int g)
{
    MemView v = view_of(a.mem[0]);
#pragma unroll
    for (int t = 1; t < kMaxMembers; ++t)
        if (t < a.nmem && g >= a.mem[t].g0) v = view_of(a.mem[t]);
    v.gl = g - v.g0;
    return v;
}
__device__ __forceinline__ MemView member_of_unit(const GemmArgs& a, long long u)
{
    MemView v = view_of(a.mem[0]);
#pragma unroll
    for (int t = 1; t < kMaxMembers; ++t)
        if (t < a.nmem && u >= a.mem[t].u0) v = view_of(a.mem[t]);
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

// Single-row product on CUDA cores (gemv_m1.cu).  The workspace of a group
// depends on its total width and its total work (tile rows).
size_t m1_workspace_bytes(int k_in, int n_out, int bits);
size_t m1_group_workspace_bytes(const GemmArgs& a);
cudaError_t launch_gemv_m1(const GemmArgs& a, cudaStream_t stream);

// Tensor-core path (2..32 rows): CTA count (planned), workspace size,
// launcher (two launches per call: input rotation pre-pass and the product
// kernel, launched as clusters of the CTAs that share an output block).
int tc_ctas(int m, int k_in, int n_out, int bits);
size_t tc_workspace_bytes(int m, int k_in, int n_out, int bits);
size_t tc_group_workspace_bytes(const GemmArgs& a);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream);

// Many-row path (gemm_large.cu): decode once into the tensor-core operand
// image, then a tcgen05 GEMM.  Rows per tile (256, 128 or 64: the largest that
// still gives kLargeMinCtas tiles), workspace size, launcher (three launches).
constexpr int kLargeMinCtas = 148;
int large_tile_rows(int m, int n_out);
size_t large_workspace_bytes(int m, int k_in, int n_out);
cudaError_t launch_gemm_large(const GemmArgs& a, cudaStream_t stream);

}  // namespace exl3
