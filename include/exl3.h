/*
 * exl3.h -- C ABI of libexl3: matrix-vector and skinny-matrix products
 * against EXL3-style trellis-quantised weights on NVIDIA B200 (sm_100a).
 *
 * What is computed.  The pages this library follows name the EXL3 trellis
 * format (a 27B-class model at a little over 3 bits per weight; orcasaq2-rocm
 * README, opening paragraph) and its decode-time product, which that page's
 * port moved onto the GPU's vector ALUs (same page, second paragraph), and a
 * tensor-core GEMV that verifies a handful of drafted tokens, with verify
 * batches of up to 32 rows (exl3-rdna4-recipe, section "What we added on top
 * of upstream"), but they never define the format.  The format fixed here:
 *   - W is K_in x N_out, stored as 16x16 tiles; tile (tk, tn) is tile number
 *     tk*(N_out/16) + tn and holds 8*K uint32 words (K = bits per weight) that
 *     form one tail-biting bitstream of 256*K bits.  Stream bit j is bit
 *     31-(j%32) of word j/32 (most significant bit first).
 *   - weight i of a tile (row i/16, column i%16 of the tile) is decoded from
 *     the 16 stream bits ending at bit (i+1)*K (positions modulo 256*K; the
 *     earliest bit is the most significant) with the 3INST map
 *         x = state*89226354 + 64248484  (mod 2^32)
 *         m = (x & 0x8FFF8FFF) ^ 0x3B603B60
 *         w = fp16(m[15:0]) + fp16(m[31:16])   (one rounding to fp16, RNE)
 *   - y = sv .* H( scale .* ( H(su .* x) W ) ), where H is the normalised
 *     128-point Hadamard transform (Sylvester order, entries
 *     (-1)^popcount(i&j)/sqrt(128)) applied to each contiguous 128-element
 *     block, su (K_in) and sv (N_out) are +-1 sign vectors and scale (N_out)
 *     is a per-output-channel fp16 scale.
 *
 * Conventions shared by every entry point.
 *   - All array arguments are DEVICE pointers (cudaMalloc / PyTorch CUDA
 *     memory) owned by the caller; the library allocates nothing, frees
 *     nothing and never synchronises the stream.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it and the call returns.
 *   - fp16 arrays are passed as uint16_t bit patterns (IEEE binary16).
 *   - Every pointer must be 16-byte aligned (EXL3_ERR_MISALIGNED otherwise).
 *   - Arguments are validated on the host before anything is enqueued; an
 *     invalid call returns its status and enqueues nothing.  A CUDA launch
 *     failure returns EXL3_ERR_CUDA (exl3_last_cuda_error() gives the
 *     cudaError_t).  Faults inside a kernel surface, CUDA-style, at the
 *     caller's next synchronisation.
 *   - The device current on the calling thread must be a B200 (compute
 *     capability 10.0); otherwise EXL3_ERR_ARCH.
 */
#ifndef EXL3_H
#define EXL3_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EXL3_API __attribute__((visibility("default")))
#else
#define EXL3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    EXL3_OK = 0,
    EXL3_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad mode     */
    EXL3_ERR_UNSUPPORTED = 2,  /* bits not in {2,3,4}; shape not a multiple of
                                  128 (16 for decode); m outside [1, 32]; more
                                  than 1,048,576 output channels in one call    */
    EXL3_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned               */
    EXL3_ERR_WORKSPACE = 4,    /* workspace null or smaller than required        */
    EXL3_ERR_ARCH = 5,         /* current device is not compute capability 10.0 */
    EXL3_ERR_CUDA = 6,         /* a CUDA runtime call failed                     */
    EXL3_ERR_TIMEOUT = 7,      /* a kernel's bounded wait expired (see
                                  exl3_workspace_status)                         */
    EXL3_ERR_BOUNDS = 8        /* debug builds only: an index check inside a
                                  kernel failed (see exl3_workspace_status)      */
};

/* Human-readable name of a status code (static string, never NULL). */
EXL3_API const char *exl3_status_string(int status);

/* cudaError_t of the last CUDA failure seen by this thread (0 if none). */
EXL3_API int exl3_last_cuda_error(void);

/* Library version, major*10000 + minor*100 + patch. */
EXL3_API int exl3_version(void);

/*
 * exl3_workspace_bytes -- size of the caller-allocated workspace that
 * exl3_gemv / exl3_gemm_small_m need for this problem: a status word, a fixed
 * 32 KB region of arrival counters (one per 128-channel output block; at most
 * 8192 blocks, i.e. 1,048,576 output channels, per call), then the call's own
 * split-K partial sums (fp32, L2-resident in practice) and rotated input.
 * The workspace must be zero-filled once before its first use; every call
 * leaves the counters at zero again and writes its own data only past the
 * counter region, so one workspace (sized for the largest call) serves any
 * sequence of calls of any shapes on the SAME stream without clearing.  Calls
 * that may run concurrently need separate workspaces.  Returns 0 for an
 * unsupported problem.  Host-only, no CUDA call.
 */
EXL3_API size_t exl3_workspace_bytes(int m, int k_in, int n_out, int bits);

/*
 * exl3_kernel_launches -- number of kernel launches one exl3_gemv /
 * exl3_gemm_small_m call with these arguments enqueues (0 if unsupported).
 * Host-only, no CUDA call.
 */
EXL3_API int exl3_kernel_launches(int m, int k_in, int n_out, int bits);

/*
 * exl3_workspace_status -- synchronises `stream`, then reads and clears the
 * workspace status word.  Returns EXL3_OK, or EXL3_ERR_TIMEOUT if a kernel
 * that used this workspace gave up a bounded wait (its output is then not
 * valid).  Every wait in the multi-row kernels gives up after 2 s.
 * Debug builds (the library compiled with -DEXL3_DEBUG_BOUNDS, built as
 * libexl3_debug.so next to libexl3.so) check the index of every access of the
 * product kernels to the packed words, the workspace and the outputs; a
 * failed check skips the access (no trap) and this call then returns
 * EXL3_ERR_BOUNDS.
 * Testing that path: while the uint32 at byte offset 4 of the workspace is
 * nonzero, exl3_gemm_small_m (m >= 2) and exl3_gemm_siblings (m >= 2) let
 * only the first v - 1 rotated-input copies of each CTA through (v = the
 * word's value; v = 1 withholds them all), and exl3_gemm_large_m withholds
 * every operand copy; the waits for the withheld copies run out and the call
 * finishes with EXL3_ERR_TIMEOUT here.  Keep that word zero in normal use.
 */
EXL3_API int exl3_workspace_status(void *workspace, void *stream);

/*
 * exl3_decode_tiles -- decode a whole trellis-packed matrix to fp16.
 *   packed : (k_in/16)*(n_out/16)*8*bits uint32 words, tile layout above.
 *   w_out  : k_in x n_out fp16, row-major (w_out[k*n_out + n] = W[k][n]).
 *   k_in, n_out : positive multiples of 16.   bits : 2, 3 or 4.
 * Bit-exact: every output equals the RNE-rounded 3INST weight.
 */
EXL3_API int exl3_decode_tiles(const uint32_t *packed, int k_in, int n_out, int bits,
                      uint16_t *w_out, void *stream);

/*
 * exl3_hadamard128 -- blockwise normalised Hadamard-128 with a sign vector.
 *   in, out : rows x n fp16, row-major; out may alias in.
 *   signs   : n fp16 values, each +1 or -1 (the same vector for every row).
 *   n       : positive multiple of 128.   rows : >= 1.
 *   mode 0  : out = H(signs .* in)   (the input-side rotation)
 *   mode 1  : out = signs .* H(in)   (the output-side rotation)
 * Computed in fp32, rounded once to fp16 (RNE).
 */
EXL3_API int exl3_hadamard128(const uint16_t *in, uint16_t *out, const uint16_t *signs,
                     int rows, int n, int mode, void *stream);

/*
 * exl3_gemv -- y = sv .* H(scale .* (H(su .* x) W)) for one input row (M = 1).
 *   x      : k_in fp16.              packed : trellis words of W (k_in x n_out).
 *   scale  : n_out fp16.             su : k_in fp16 +-1.   sv : n_out fp16 +-1.
 *   y      : n_out outputs, fp16 (y_fp32 == 0) or fp32 (y_fp32 != 0).
 *   k_in, n_out : positive multiples of 128.   bits : 2, 3 or 4.
 *   workspace, ws_bytes : at least exl3_workspace_bytes(1, k_in, n_out, bits)
 *                         bytes, zero-filled before first use (see above).
 * Accumulation is fp32; the reduction order is fixed, so repeated calls give
 * bitwise-identical y.
 */
EXL3_API int exl3_gemv(const uint16_t *x, const uint32_t *packed, const uint16_t *scale,
              const uint16_t *su, const uint16_t *sv, void *y, int y_fp32,
              int k_in, int n_out, int bits, void *workspace, size_t ws_bytes,
              void *stream);

/*
 * exl3_gemm_small_m -- the same product for m input rows (1 <= m <= 32): the
 * speculative-draft verification batch.
 *   x : m x k_in fp16, row-major.   y : m x n_out (fp16 or fp32), row-major.
 *   Other arguments as exl3_gemv; workspace at least
 *   exl3_workspace_bytes(m, k_in, n_out, bits).
 * Deterministic as exl3_gemv.  Different m may use different kernels, which
 * agree within rounding, not bitwise.
 * Timeouts (m >= 2): every wait inside the kernel is bounded (2 s).  If one
 * runs out the call has ALREADY returned EXL3_OK and y is not valid; nothing
 * reports it until exl3_workspace_status(workspace, stream), which
 * synchronises.  Callers that cannot rule out a stalled GPU poll it.  The
 * same holds for exl3_gemm_siblings and exl3_gemm_grouped at m >= 2 and for
 * exl3_gemm_large_m.  The single-row kernel (m = 1) never waits on anything.
 */
EXL3_API int exl3_gemm_small_m(int m, const uint16_t *x, const uint32_t *packed,
                      const uint16_t *scale, const uint16_t *su, const uint16_t *sv,
                      void *y, int y_fp32, int k_in, int n_out, int bits,
                      void *workspace, size_t ws_bytes, void *stream);

/*
 * exl3_gemm_large_m -- the same product for many input rows (prompt prefill;
 * the orcasaq2-rocm README reports prefill speeds next to its decode table):
 * the matrix is decoded once per call into the tensor-core operand layout in
 * the workspace, then multiplied on the tensor cores (tcgen05).
 *   m : 1 .. 2^20 rows (efficient from about a hundred; below 32 prefer
 *       exl3_gemm_small_m, which never materialises the decoded matrix).
 *   x : m x k_in fp16, row-major.   y : m x n_out (fp16 or fp32), row-major.
 *   Other arguments as exl3_gemm_small_m, except the workspace:
 *   workspace, ws_bytes : at least exl3_large_m_workspace_bytes(m, k_in,
 *     n_out, bits) bytes (2 bytes per weight plus 2 bytes per rotated input
 *     element, rounded up to the row tile), 256-byte aligned; its first word
 *     is the status word exl3_workspace_status reads.  No zero-fill needed.
 * Each output is one accumulator's fixed-order sum: repeated calls are
 * bitwise identical.  A bounded wait that runs out is reported only by
 * exl3_workspace_status (the call itself has returned EXL3_OK).
 */
EXL3_API size_t exl3_large_m_workspace_bytes(int m, int k_in, int n_out, int bits);
EXL3_API int exl3_gemm_large_m(int m, const uint16_t *x, const uint32_t *packed, const uint16_t *scale,
                               const uint16_t *su, const uint16_t *sv, void *y, int y_fp32, int k_in, int n_out,
                               int bits, void *workspace, size_t ws_bytes, void *stream);

/*
 * exl3_gemm_siblings -- the product for a group of matrices that take the
 * same input: y_i = sv_i .* H(scale_i .* (H(su .* x) W_i)) for i < n_mats,
 * in one pass that rotates x once and spreads all the groups' output blocks
 * over the GPU together.  The exl3-rdna4-recipe page fuses the MLP's
 * matrices into one native-code path for its verify batches (section "What
 * we added on top of upstream"); this is that fusion here: gate and up of an
 * MLP, or q, k and v of an attention block, whose inputs are the same
 * activation rows.
 *   x, su  : as exl3_gemm_small_m, shared by every matrix of the group.
 *   mats   : HOST array of n_mats (1..8) exl3_matrix_t; each gives its packed
 *            words, scale, sv and output y (m x n_out, row-major) and n_out
 *            (a positive multiple of 128).  All matrices have k_in rows and
 *            `bits` bits per weight.
 *   workspace, ws_bytes : at least exl3_workspace_bytes(m, k_in, sum of n_out,
 *            bits) bytes, zero-filled before first use.
 * Results equal the separate products within rounding (the reduction split
 * follows the group's total width); repeated calls are bitwise identical.
 */
typedef struct exl3_matrix {
    const uint32_t *packed;
    const uint16_t *scale;
    const uint16_t *sv;
    void *y;
    int n_out;
} exl3_matrix_t;

EXL3_API int exl3_gemm_siblings(int m, const uint16_t *x, const uint16_t *su, const exl3_matrix_t *mats,
                                int n_mats, int y_fp32, int k_in, int bits, void *workspace, size_t ws_bytes,
                                void *stream);

/*
 * exl3_gemm_grouped -- the products of up to 8 INDEPENDENT problems in one
 * pass: y_i = sv_i .* H(scale_i .* (H(su_i .* x_i) W_i)), each with its own
 * input rows, sign vectors, weights and shape, e.g. the seven matrices of one
 * transformer layer (q, k, v, o, gate, up, down) in a verify sweep where each
 * has its own activation rows.  The orcasaq2-rocm README (opening
 * paragraph) cuts the launches of a decode step by fusing steps; here the
 * same idea is applied to a layer's products: the whole group's work is split
 * over the GPU as one problem, so the small matrices leave no SMs idle, and
 * one launch (m = 1) or two (m >= 2: one rotation pre-pass for every member,
 * then one product launch) serve the group.
 *   m      : 1..32 rows, the same for every member.
 *   probs  : HOST array of n_probs (1..8) exl3_problem_t, each with device
 *            pointers x (m x k_in fp16), su (k_in), packed, scale (n_out), sv
 *            (n_out) and y (m x n_out, fp16 or fp32 as y_fp32), and its k_in
 *            and n_out (positive multiples of 128).  All members have `bits`
 *            bits per weight.
 *   workspace, ws_bytes : at least exl3_grouped_workspace_bytes(m, probs,
 *            n_probs, bits) bytes, 256-byte aligned, zero-filled before first
 *            use; reusable by later calls on the same stream.
 * Each y_i equals the separate product's within rounding (the work split
 * differs); repeated calls are bitwise identical.  The size query reads
 * only k_in and n_out of each problem (the pointers may be NULL there) and
 * returns 0 for an invalid group.
 */
typedef struct exl3_problem {
    const uint16_t *x;
    const uint16_t *su;
    const uint32_t *packed;
    const uint16_t *scale;
    const uint16_t *sv;
    void *y;
    int k_in;
    int n_out;
} exl3_problem_t;

EXL3_API size_t exl3_grouped_workspace_bytes(int m, const exl3_problem_t *probs, int n_probs, int bits);
EXL3_API int exl3_gemm_grouped(int m, const exl3_problem_t *probs, int n_probs, int y_fp32, int bits,
                               void *workspace, size_t ws_bytes, void *stream);

/*
 * exl3_gemv_noalloc -- exl3_gemv without a workspace argument.  The source
 * pages describe no counterpart of this entry point; it exists for callers that cannot
 * allocate device memory on the call path -- for example an inference engine
 * that reserves all of HBM for its own pool at start-up and forbids further
 * cudaMalloc, or a plugin whose host application owns the CUDA allocator --
 * and therefore cannot hand in the split-K workspace exl3_gemv needs.
 *   Arguments: as exl3_gemv, minus workspace and ws_bytes.
 *   Scratch: a fixed device array of 4 MiB inside the library, which every
 *     GPU that loads the library holds until the process exits.  Problems whose
 *     workspace (exl3_workspace_bytes(1, k_in, n_out, bits)) exceeds it are
 *     rejected with EXL3_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   Allocation: none -- no cudaMalloc, cudaFree or allocating library call.
 *     Each call clears the array's counters with cudaMemsetAsync on `stream`.
 *   Concurrency: all calls on a device share the one array, so calls that
 *     may overlap on the GPU (different streams without ordering) race and
 *     give wrong results; serialise them, or use exl3_gemv with separate
 *     workspaces.
 * Results are the same as exl3_gemv's.
 */
EXL3_API int exl3_gemv_noalloc(const uint16_t *x, const uint32_t *packed, const uint16_t *scale,
                               const uint16_t *su, const uint16_t *sv, void *y, int y_fp32,
                               int k_in, int n_out, int bits, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EXL3_H */
