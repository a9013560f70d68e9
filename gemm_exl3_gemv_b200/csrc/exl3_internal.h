// exl3_internal.h -- launchers shared between the libexl3 translation units.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace exl3 {

cudaError_t launch_decode_tiles(const uint32_t* packed, int k_in, int n_out, int bits, uint16_t* w_out,
                                cudaStream_t stream);
cudaError_t launch_hadamard128(const uint16_t* in, uint16_t* out, const uint16_t* signs, int rows, int n, int mode,
                               cudaStream_t stream);

// Problem description shared by the product kernels.
struct GemmArgs {
    const uint16_t* x;        // m x k_in fp16
    const uint32_t* packed;   // trellis words
    const uint16_t* scale;    // n_out fp16
    const uint16_t* su;       // k_in fp16 +-1
    const uint16_t* sv;       // n_out fp16 +-1
    void* y;                  // m x n_out, fp16 or fp32
    int y_fp32;
    int m, k_in, n_out, bits;
    unsigned char* ws;        // workspace base
    int pdl;                  // launch with programmatic dependent launch (overlap the previous kernel's tail)
};

// Single-row product on CUDA cores (gemv_m1.cu).
size_t m1_workspace_bytes(int k_in, int n_out, int bits);
cudaError_t launch_gemv_m1(const GemmArgs& a, cudaStream_t stream);

// Tensor-core path (2..32 rows): CTA count (planned), workspace size,
// launcher (two launches per call: input rotation pre-pass and the product
// kernel, launched as clusters of the CTAs that share an output block).
int tc_ctas(int m, int k_in, int n_out, int bits);
size_t tc_workspace_bytes(int m, int k_in, int n_out, int bits);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream);

}  // namespace exl3
