/*
 * exl3_oracle.c -- plain, slow fp64 CPU reference for the EXL3 trellis GEMV.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: it is used by tests/, by the smoke check and by the
 * cpu_baseline / reference leg of bench.py, and by nothing else.  It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it computes, and where each step comes from:
 *
 *   The pages name the format (27B-class models at about 3 bits per weight:
 *   orcasaq2-rocm README and exl3-rdna4-recipe, opening paragraphs) but never
 *   define it.  The definition
 *   written out below is the format specification this library follows:
 *   16x16 tiles, each a
 *   tail-biting bitstream of 256*K bits; weight i of a tile is decoded from the
 *   16-bit window ending at bit (i+1)*K with the 3INST map
 *       x = state*89226354 + 64248484 (mod 2^32),
 *       m = (x & 0x8FFF8FFF) ^ 0x3B603B60, read as two fp16 halves and summed;
 *   each output channel takes an fp16 scale; activations and outputs pass
 *   through a normalised 128-point Hadamard with a seeded +-1 sign vector.
 *
 *   Readings taken where the definition is silent (each one is listed with
 *   its reason in the design notes):
 *     R1  stream bit j is bit 31-(j mod 32) of 32-bit word j/32 (MSB first);
 *         the earliest bit of a window is the state's most significant bit.
 *     R2  window bit positions wrap modulo 256*K (tail-biting).
 *     R3  weight i of tile (tk, tn) sits at row k = 16*tk + i/16 and column
 *         n = 16*tn + i%16 of W (K_in x N_out, y = x W).
 *     R4  tile (tk, tn) is tile number tk*(N_out/16) + tn; 8*K words per tile.
 *     R6  "summed": exact sum of the two halves, rounded once to fp16,
 *         round-to-nearest-even.
 *     R8  scale multiplies output channel n before the output rotation.
 *     R9  H[i][j] = (-1)^popcount(i & j) / sqrt(128) (Sylvester order) on
 *         contiguous 128-element blocks; input side: signs then H; output
 *         side: H then signs.
 *     R10 two sign vectors: su (K_in) on the input, sv (N_out) on the output.
 *
 * Everything here is fp64 (or exact integer) arithmetic; fp16 values are read
 * and rounded by the two converters in this file, written from the IEEE-754
 * binary16 definition.  Loops follow the definitions directly; the only
 * structure is the tile loop that the format itself imposes.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_HBLOCK 128

/* ---------------------------------------------------------------- fp16 --- */

/* binary16 bit pattern -> exact double value (IEEE-754 binary16 definition:
 * 1 sign bit, 5 exponent bits with bias 15, 10 fraction bits). */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round q >= 0 to the nearest integer, ties to the even integer. */
static double round_half_even(double q)
{
    double r = floor(q);
    double frac = q - r;                           /* exact for |q| < 2^52 */
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    return r;
}

/* double -> binary16 bit pattern, round to nearest, ties to even. */
uint16_t oracle_double_to_half_rne(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (isnan(v))
        return 0x7E00u;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: representable values are multiples of 2^-24 */
        double r = round_half_even(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)r);     /* r == 1024 is the smallest normal */
    }
    int e2;
    frexp(a, &e2);                                 /* a = mant * 2^e2, mant in [0.5, 1) */
    int E = e2 - 1;                                /* a in [2^E, 2^(E+1)) */
    double r = round_half_even(ldexp(a, 10 - E)); /* 11 significant bits */
    if (r == 2048.0) {
        r = 1024.0;
        E += 1;
    }
    if (E > 15)
        return (uint16_t)(sign | 0x7C00u);         /* overflow to infinity */
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)r - 1024));
}

/* -------------------------------------------------------------- 3INST --- */

/* Decode one 16-bit trellis state to the fp16 weight (bit pattern). */
uint16_t oracle_3inst(uint16_t state)
{
    uint32_t x = (uint32_t)state * 89226354u + 64248484u;   /* mod 2^32 */
    uint32_t m = (x & 0x8FFF8FFFu) ^ 0x3B603B60u;
    double lo = oracle_half_to_double((uint16_t)(m & 0xFFFFu));
    double hi = oracle_half_to_double((uint16_t)(m >> 16));
    return oracle_double_to_half_rne(lo + hi);               /* exact sum, one rounding (R6) */
}

/* ------------------------------------------------------------ stream --- */

/* Bit j of a tile's stream (R1, R2). */
static int stream_bit(const uint32_t *tile, long nbits, long j)
{
    j %= nbits;
    if (j < 0)
        j += nbits;
    return (int)((tile[j >> 5] >> (31 - (j & 31))) & 1u);
}

/* State of weight i: the 16 bits ending at bit (i+1)*K, earliest bit first. */
uint16_t oracle_state(const uint32_t *tile, int bits, int i)
{
    long nbits = 256L * bits;
    long start = (long)(i + 1) * bits - 16;
    uint32_t s = 0;
    for (int j = 0; j < 16; j++)
        s = (s << 1) | (uint32_t)stream_bit(tile, nbits, start + j);
    return (uint16_t)s;
}

/* Decode every tile of a K_in x N_out matrix into fp16 bits, row-major. */
void oracle_decode_tiles(const uint32_t *packed, long k_in, long n_out, int bits,
                         uint16_t *w_out)
{
    long tiles_n = n_out / 16;
    long tiles_k = k_in / 16;
#pragma omp parallel for schedule(static)
    for (long tk = 0; tk < tiles_k; tk++) {
        for (long tn = 0; tn < tiles_n; tn++) {
            const uint32_t *tile = packed + (tk * tiles_n + tn) * 8L * bits;   /* R4 */
            for (int i = 0; i < 256; i++) {
                long k = 16 * tk + i / 16;                                      /* R3 */
                long n = 16 * tn + i % 16;
                w_out[k * n_out + n] = oracle_3inst(oracle_state(tile, bits, i));
            }
        }
    }
}

/* ----------------------------------------------------------- Hadamard --- */

static int popcount7(unsigned v)
{
    int c = 0;
    for (; v; v >>= 1)
        c += (int)(v & 1u);
    return c;
}

/* mode 0: out = H (s .* in);   mode 1: out = s .* (H in);   per 128-block (R9).
 * Written as the matrix-vector product by the definition of H (no fast
 * transform).  in and out may not alias.  signs may be NULL (all +1). */
void oracle_hadamard128(const double *in, double *out, const double *signs,
                        long rows, long n, int mode)
{
    const double inv = 1.0 / sqrt((double)ORACLE_HBLOCK);
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        const double *v = in + r * n;
        double *o = out + r * n;
        for (long b = 0; b < n; b += ORACLE_HBLOCK) {
            for (int j = 0; j < ORACLE_HBLOCK; j++) {
                double acc = 0.0;
                for (int i = 0; i < ORACLE_HBLOCK; i++) {
                    double vi = v[b + i];
                    if (mode == 0 && signs)
                        vi *= signs[b + i];
                    acc += (popcount7((unsigned)(i & j)) & 1) ? -vi : vi;
                }
                acc *= inv;
                if (mode == 1 && signs)
                    acc *= signs[b + j];
                o[b + j] = acc;
            }
        }
    }
}

/* --------------------------------------------------------------- GEMM --- */

/* z[m][n] = scale[n] * sum_k xt[m][k] * W[k][n] for the channels of the
 * listed 128-channel output blocks, then y = sv .* H z on those blocks.
 * xt is the rotated input (M x K_in).  y_blocks is M x (nblocks*128).    */
static void gemm_blocks(const double *xt, const uint32_t *packed, const double *scale,
                        const double *sv, long M, long k_in, long n_out, int bits,
                        const long *blocks, long nblocks, double *y_blocks)
{
    long tiles_n = n_out / 16;
    long tiles_k = k_in / 16;
    long ncols = nblocks * ORACLE_HBLOCK;
    double *z = (double *)calloc((size_t)(M * ncols), sizeof(double));
    /* each column tile is owned by one thread: no shared accumulators */
#pragma omp parallel for schedule(dynamic, 1)
    for (long ct = 0; ct < nblocks * 8; ct++) {
        long tn = blocks[ct / 8] * 8 + ct % 8;
        double w[256];
        for (long tk = 0; tk < tiles_k; tk++) {
            const uint32_t *tile = packed + (tk * tiles_n + tn) * 8L * bits;
            for (int i = 0; i < 256; i++)
                w[i] = oracle_half_to_double(oracle_3inst(oracle_state(tile, bits, i)));
            for (long m = 0; m < M; m++) {
                const double *xr = xt + m * k_in + 16 * tk;
                double *zr = z + m * ncols + 16 * ct;
                for (int i = 0; i < 256; i++)
                    zr[i % 16] += xr[i / 16] * w[i];
            }
        }
    }
    for (long m = 0; m < M; m++)
        for (long c = 0; c < ncols; c++) {
            long n = blocks[c / ORACLE_HBLOCK] * ORACLE_HBLOCK + c % ORACLE_HBLOCK;
            z[m * ncols + c] *= scale[n];                                       /* R8 */
        }
    /* output rotation, block by block, with the signs of the block's channels */
    double *svb = (double *)malloc((size_t)ncols * sizeof(double));
    for (long c = 0; c < ncols; c++)
        svb[c] = sv[blocks[c / ORACLE_HBLOCK] * ORACLE_HBLOCK + c % ORACLE_HBLOCK];
    oracle_hadamard128(z, y_blocks, svb, M, ncols, 1);
    free(svb);
    free(z);
    (void)tiles_n;
}

/* Full product: y (M x N_out) = sv .* H( scale .* ( (H (su .* x)) W ) ). */
void oracle_gemm(const double *x, const uint32_t *packed, const double *scale,
                 const double *su, const double *sv, long M, long k_in, long n_out,
                 int bits, double *y)
{
    double *xt = (double *)malloc((size_t)(M * k_in) * sizeof(double));
    oracle_hadamard128(x, xt, su, M, k_in, 0);
    long nblocks = n_out / ORACLE_HBLOCK;
    long *blocks = (long *)malloc((size_t)nblocks * sizeof(long));
    for (long b = 0; b < nblocks; b++)
        blocks[b] = b;
    gemm_blocks(xt, packed, scale, sv, M, k_in, n_out, bits, blocks, nblocks, y);
    free(blocks);
    free(xt);
}

/* Same result restricted to some 128-channel output blocks (for sampled
 * checks of full-size problems).  y_blocks is M x (nblocks*128), the blocks'
 * columns in the order listed. */
void oracle_gemm_sampled(const double *x, const uint32_t *packed, const double *scale,
                         const double *su, const double *sv, long M, long k_in,
                         long n_out, int bits, const long *blocks, long nblocks,
                         double *y_blocks)
{
    double *xt = (double *)malloc((size_t)(M * k_in) * sizeof(double));
    oracle_hadamard128(x, xt, su, M, k_in, 0);
    gemm_blocks(xt, packed, scale, sv, M, k_in, n_out, bits, blocks, nblocks, y_blocks);
    free(xt);
}
