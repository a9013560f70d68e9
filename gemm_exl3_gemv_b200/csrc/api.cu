// api.cu -- the extern "C" entry points of libexl3 (declared in include/exl3.h):
// argument validation on the host, architecture check, dispatch to kernels.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/exl3.h"
#include "exl3_common.cuh"
#include "exl3_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e)
{
    g_last_cuda_error = (int)e;
    return EXL3_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4; }

// The kernels are built for sm_100a only; check the current device once per
// call (cheap: cached attribute queries in the runtime).
int check_arch()
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    return (major == 10 && minor == 0) ? EXL3_OK : EXL3_ERR_ARCH;
}

int validate_gemm(int m, const uint16_t* x, const uint32_t* packed, const uint16_t* scale, const uint16_t* su,
                  const uint16_t* sv, const void* y, int k_in, int n_out, int bits, const void* ws, size_t ws_bytes)
{
    if (!x || !packed || !scale || !su || !sv || !y) return EXL3_ERR_INVALID_ARG;
    if (m <= 0 || k_in <= 0 || n_out <= 0) return EXL3_ERR_INVALID_ARG;
    if (m > 32 || !bits_ok(bits) || k_in % 128 || n_out % 128 || n_out / 128 > exl3::kMaxBlocks)
        return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scale) || !aligned16(su) || !aligned16(sv) ||
        !aligned16(y))
        return EXL3_ERR_MISALIGNED;
    if (!ws || ws_bytes < exl3_workspace_bytes(m, k_in, n_out, bits)) return EXL3_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return EXL3_ERR_MISALIGNED;
    return EXL3_OK;
}

// Problem description of a single product (a group of one member).
exl3::GemmArgs single_args(int m, const uint16_t* x, const uint32_t* packed, const uint16_t* scale,
                           const uint16_t* su, const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out,
                           int bits, void* ws, size_t ws_bytes)
{
    exl3::GemmArgs a = {};
    a.y_fp32 = y_fp32 ? 1 : 0;
    a.m = m;
    a.bits = bits;
    a.nmem = 1;
    a.shared_x = 1;
    a.mem[0] = exl3::Member{x, su, packed, scale, sv, y, k_in, n_out, 0, 0, 0, 0};
    exl3::finish_group(a);
    a.ws = static_cast<unsigned char*>(ws);
    a.ws_bytes = ws_bytes;
    a.pdl = 1;
    return a;
}

cudaError_t launch_product(const exl3::GemmArgs& a, cudaStream_t s)
{
    return a.m == 1 ? exl3::launch_gemv_m1(a, s) : exl3::launch_gemm_tc(a, s);
}

int run_gemm(int m, const uint16_t* x, const uint32_t* packed, const uint16_t* scale, const uint16_t* su,
             const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out, int bits, void* ws, size_t ws_bytes,
             void* stream)
{
    int st = validate_gemm(m, x, packed, scale, su, sv, y, k_in, n_out, bits, ws, ws_bytes);
    if (st != EXL3_OK) return st;
    st = check_arch();
    if (st != EXL3_OK) return st;
    exl3::GemmArgs a = single_args(m, x, packed, scale, su, sv, y, y_fp32, k_in, n_out, bits, ws, ws_bytes);
    cudaError_t e = launch_product(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

const char* exl3_status_string(int status)
{
    switch (status) {
        case EXL3_OK: return "EXL3_OK";
        case EXL3_ERR_INVALID_ARG: return "EXL3_ERR_INVALID_ARG: null pointer, non-positive size or bad mode";
        case EXL3_ERR_UNSUPPORTED: return "EXL3_ERR_UNSUPPORTED: bits, shape or row count not supported";
        case EXL3_ERR_MISALIGNED: return "EXL3_ERR_MISALIGNED: pointer not 16-byte (workspace: 256-byte) aligned";
        case EXL3_ERR_WORKSPACE: return "EXL3_ERR_WORKSPACE: workspace missing or too small";
        case EXL3_ERR_ARCH: return "EXL3_ERR_ARCH: current device is not a compute capability 10.0 GPU";
        case EXL3_ERR_CUDA: return "EXL3_ERR_CUDA: a CUDA runtime call failed (see exl3_last_cuda_error)";
        case EXL3_ERR_TIMEOUT: return "EXL3_ERR_TIMEOUT: a kernel gave up a bounded wait; output invalid";
        case EXL3_ERR_BOUNDS: return "EXL3_ERR_BOUNDS: a debug-build index check failed; output invalid";
    }
    return "EXL3: unknown status";
}

int exl3_last_cuda_error(void) { return g_last_cuda_error; }

int exl3_version(void) { return 100; }

size_t exl3_workspace_bytes(int m, int k_in, int n_out, int bits)
{
    if (m <= 0 || m > 32 || k_in <= 0 || n_out <= 0 || k_in % 128 || n_out % 128 || !bits_ok(bits) ||
        n_out / 128 > exl3::kMaxBlocks)
        return 0;
    return m == 1 ? exl3::m1_workspace_bytes(k_in, n_out, bits) : exl3::tc_workspace_bytes(m, k_in, n_out, bits);
}

int exl3_kernel_launches(int m, int k_in, int n_out, int bits)
{
    if (m <= 0 || m > 32 || k_in <= 0 || n_out <= 0 || k_in % 128 || n_out % 128 || !bits_ok(bits) ||
        n_out / 128 > exl3::kMaxBlocks)
        return 0;
    return m == 1 ? 1 : 2;
}

int exl3_workspace_status(void* workspace, void* stream)
{
    if (!workspace) return EXL3_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (word == 0) return EXL3_OK;
    e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    return (word & exl3::kStatusBounds) ? EXL3_ERR_BOUNDS : EXL3_ERR_TIMEOUT;
}

int exl3_decode_tiles(const uint32_t* packed, int k_in, int n_out, int bits, uint16_t* w_out, void* stream)
{
    if (!packed || !w_out || k_in <= 0 || n_out <= 0) return EXL3_ERR_INVALID_ARG;
    if (!bits_ok(bits) || k_in % 16 || n_out % 16) return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(packed) || !aligned16(w_out)) return EXL3_ERR_MISALIGNED;
    int st = check_arch();
    if (st != EXL3_OK) return st;
    cudaError_t e = exl3::launch_decode_tiles(packed, k_in, n_out, bits, w_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

int exl3_hadamard128(const uint16_t* in, uint16_t* out, const uint16_t* signs, int rows, int n, int mode,
                     void* stream)
{
    if (!in || !out || !signs || rows <= 0 || n <= 0 || (mode != 0 && mode != 1)) return EXL3_ERR_INVALID_ARG;
    if (n % 128) return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(in) || !aligned16(out) || !aligned16(signs)) return EXL3_ERR_MISALIGNED;
    int st = check_arch();
    if (st != EXL3_OK) return st;
    cudaError_t e = exl3::launch_hadamard128(in, out, signs, rows, n, mode, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

int exl3_gemv(const uint16_t* x, const uint32_t* packed, const uint16_t* scale, const uint16_t* su,
              const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out, int bits, void* workspace,
              size_t ws_bytes, void* stream)
{
    return run_gemm(1, x, packed, scale, su, sv, y, y_fp32, k_in, n_out, bits, workspace, ws_bytes, stream);
}

int exl3_gemm_small_m(int m, const uint16_t* x, const uint32_t* packed, const uint16_t* scale, const uint16_t* su,
                      const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out, int bits, void* workspace,
                      size_t ws_bytes, void* stream)
{
    return run_gemm(m, x, packed, scale, su, sv, y, y_fp32, k_in, n_out, bits, workspace, ws_bytes, stream);
}

}  // extern "C"

// ----------------------------------------------------------------- large m ---

extern "C" size_t exl3_large_m_workspace_bytes(int m, int k_in, int n_out, int bits)
{
    if (m <= 0 || m > (1 << 20) || k_in <= 0 || n_out <= 0 || k_in % 128 || n_out % 128 || !bits_ok(bits)) return 0;
    return exl3::large_workspace_bytes(m, k_in, n_out);
}

extern "C" int exl3_gemm_large_m(int m, const uint16_t* x, const uint32_t* packed, const uint16_t* scale,
                                 const uint16_t* su, const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out,
                                 int bits, void* workspace, size_t ws_bytes, void* stream)
{
    if (!x || !packed || !scale || !su || !sv || !y) return EXL3_ERR_INVALID_ARG;
    if (m <= 0 || k_in <= 0 || n_out <= 0) return EXL3_ERR_INVALID_ARG;
    if (m > (1 << 20) || !bits_ok(bits) || k_in % 128 || n_out % 128) return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scale) || !aligned16(su) || !aligned16(sv) ||
        !aligned16(y))
        return EXL3_ERR_MISALIGNED;
    if (!workspace || ws_bytes < exl3_large_m_workspace_bytes(m, k_in, n_out, bits)) return EXL3_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return EXL3_ERR_MISALIGNED;
    int st = check_arch();
    if (st != EXL3_OK) return st;
    exl3::GemmArgs a = single_args(m, x, packed, scale, su, sv, y, y_fp32, k_in, n_out, bits, workspace, ws_bytes);
    cudaError_t e = exl3::launch_gemm_large(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

// ------------------------------------------------------------- siblings ---

extern "C" int exl3_gemm_siblings(int m, const uint16_t* x, const uint16_t* su, const exl3_matrix_t* mats,
                                  int n_mats, int y_fp32, int k_in, int bits, void* workspace, size_t ws_bytes,
                                  void* stream)
{
    if (!x || !su || !mats) return EXL3_ERR_INVALID_ARG;
    if (m <= 0 || k_in <= 0 || n_mats <= 0) return EXL3_ERR_INVALID_ARG;
    if (n_mats > exl3::kMaxMembers || m > 32 || !bits_ok(bits) || k_in % 128) return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(su)) return EXL3_ERR_MISALIGNED;
    exl3::GemmArgs a = {};
    long long total = 0;
    for (int i = 0; i < n_mats; ++i) {
        const exl3_matrix_t& t = mats[i];
        if (!t.packed || !t.scale || !t.sv || !t.y) return EXL3_ERR_INVALID_ARG;
        if (t.n_out <= 0) return EXL3_ERR_INVALID_ARG;
        if (t.n_out % 128) return EXL3_ERR_UNSUPPORTED;
        if (!aligned16(t.packed) || !aligned16(t.scale) || !aligned16(t.sv) || !aligned16(t.y))
            return EXL3_ERR_MISALIGNED;
        a.mem[i] = exl3::Member{x, su, t.packed, t.scale, t.sv, t.y, k_in, t.n_out, 0, 0, 0, 0};
        total += t.n_out;
    }
    if (total / 128 > exl3::kMaxBlocks) return EXL3_ERR_UNSUPPORTED;
    const int n_total = (int)total;
    if (!workspace || ws_bytes < exl3_workspace_bytes(m, k_in, n_total, bits)) return EXL3_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return EXL3_ERR_MISALIGNED;
    int st = check_arch();
    if (st != EXL3_OK) return st;
    a.y_fp32 = y_fp32 ? 1 : 0;
    a.m = m;
    a.bits = bits;
    a.nmem = n_mats;
    a.shared_x = 1;
    exl3::finish_group(a);
    a.ws = static_cast<unsigned char*>(workspace);
    a.ws_bytes = ws_bytes;
    a.pdl = 1;
    cudaError_t e = launch_product(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

// ---------------------------------------------------------------- grouped ---

namespace {

// Validate a grouped call's problem list and fill the group description
// (everything but the workspace).  Host only, no CUDA call.
int grouped_args(int m, const exl3_problem_t* probs, int n_probs, int y_fp32, int bits, exl3::GemmArgs& a,
                 bool check_ptrs)
{
    if (!probs || m <= 0 || n_probs <= 0) return EXL3_ERR_INVALID_ARG;
    if (n_probs > exl3::kMaxMembers || m > 32 || !bits_ok(bits)) return EXL3_ERR_UNSUPPORTED;
    a = exl3::GemmArgs{};
    long long total = 0;
    for (int i = 0; i < n_probs; ++i) {
        const exl3_problem_t& t = probs[i];
        if (check_ptrs && (!t.x || !t.su || !t.packed || !t.scale || !t.sv || !t.y)) return EXL3_ERR_INVALID_ARG;
        if (t.k_in <= 0 || t.n_out <= 0) return EXL3_ERR_INVALID_ARG;
        if (t.k_in % 128 || t.n_out % 128) return EXL3_ERR_UNSUPPORTED;
        if (check_ptrs && (!aligned16(t.x) || !aligned16(t.su) || !aligned16(t.packed) || !aligned16(t.scale) ||
                           !aligned16(t.sv) || !aligned16(t.y)))
            return EXL3_ERR_MISALIGNED;
        a.mem[i] = exl3::Member{t.x, t.su, t.packed, t.scale, t.sv, t.y, t.k_in, t.n_out, 0, 0, 0, 0};
        total += t.n_out;
    }
    if (total / 128 > exl3::kMaxBlocks) return EXL3_ERR_UNSUPPORTED;
    a.y_fp32 = y_fp32 ? 1 : 0;
    a.m = m;
    a.bits = bits;
    a.nmem = n_probs;
    a.shared_x = 0;
    exl3::finish_group(a);
    a.pdl = 1;
    return EXL3_OK;
}

size_t grouped_ws(const exl3::GemmArgs& a)
{
    return a.m == 1 ? exl3::m1_group_workspace_bytes(a) : exl3::tc_group_workspace_bytes(a);
}

}  // namespace

extern "C" size_t exl3_grouped_workspace_bytes(int m, const exl3_problem_t* probs, int n_probs, int bits)
{
    exl3::GemmArgs a;
    if (grouped_args(m, probs, n_probs, 0, bits, a, false) != EXL3_OK) return 0;
    return grouped_ws(a);
}

extern "C" int exl3_gemm_grouped(int m, const exl3_problem_t* probs, int n_probs, int y_fp32, int bits,
                                 void* workspace, size_t ws_bytes, void* stream)
{
    exl3::GemmArgs a;
    int st = grouped_args(m, probs, n_probs, y_fp32, bits, a, true);
    if (st != EXL3_OK) return st;
    if (!workspace || ws_bytes < grouped_ws(a)) return EXL3_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return EXL3_ERR_MISALIGNED;
    st = check_arch();
    if (st != EXL3_OK) return st;
    a.ws = static_cast<unsigned char*>(workspace);
    a.ws_bytes = ws_bytes;
    cudaError_t e = launch_product(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}

// ------------------------------------------------------ no-allocation GEMV ---
//
// exl3_gemv_noalloc: the single-row product without a caller workspace, for
// callers that cannot allocate device memory (see include/exl3.h).  Its
// split-K scratch is this file-scope device array.  In host code the name
// g_noalloc_scratch is only a host-side stand-in, so its device address is
// looked up once per device (cudaGetSymbolAddress, with that device current)
// and passed to the kernel as the workspace pointer.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // held by every device that loads the library

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
int noalloc_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return EXL3_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return EXL3_OK;
}

}  // namespace

extern "C" int exl3_gemv_noalloc(const uint16_t* x, const uint32_t* packed, const uint16_t* scale,
                                 const uint16_t* su, const uint16_t* sv, void* y, int y_fp32, int k_in, int n_out,
                                 int bits, void* stream)
{
    if (!x || !packed || !scale || !su || !sv || !y) return EXL3_ERR_INVALID_ARG;
    if (k_in <= 0 || n_out <= 0) return EXL3_ERR_INVALID_ARG;
    if (!bits_ok(bits) || k_in % 128 || n_out % 128 || n_out / 128 > exl3::kMaxBlocks) return EXL3_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scale) || !aligned16(su) || !aligned16(sv) ||
        !aligned16(y))
        return EXL3_ERR_MISALIGNED;
    const size_t need = exl3_workspace_bytes(1, k_in, n_out, bits);
    if (need == 0 || need > kNoAllocScratchBytes) return EXL3_ERR_WORKSPACE;   // beyond the fixed scratch
    int st = check_arch();
    if (st != EXL3_OK) return st;
    void* ws = nullptr;
    st = noalloc_scratch(&ws);
    if (st != EXL3_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the array keeps the last call's contents: the status word and the
    // arrival counters must start at zero
    cudaError_t e = cudaMemsetAsync(ws, 0, exl3::ws_data_off(), s);
    if (e != cudaSuccess) return cuda_fail(e);
    exl3::GemmArgs a = single_args(1, x, packed, scale, su, sv, y, y_fp32, k_in, n_out, bits, ws, kNoAllocScratchBytes);
    a.pdl = 0;                       // follows a memset: ordinary stream order
    e = exl3::launch_gemv_m1(a, s);
    return e == cudaSuccess ? EXL3_OK : cuda_fail(e);
}
