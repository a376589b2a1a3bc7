/*
 * oracle.h -- plain, slow CPU restatement of the weight-only quantized linear
 * layer y = x . dequant(Wq)^T for the three weight formats.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this code: only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header or table with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *  [NSS]  ExecuTorch PR "[cuda] Nestest Superscale Quantization for CUDA
 *         Weights (int4 / int6)", section "Quant schema update" (formats,
 *         w = (q - zero) * scale, group sizes, super-block 256, the z_pack
 *         word) and section "Why this design" (int6 symmetric, int8 code).
 *  [MTL]  Hugging Face Transformers docs, "Metal" quantization page: weights
 *         packed into uint32 tensors with per-group scales and biases,
 *         bit widths 2/4/8, group size configurable (default 64).
 *
 * Layout conventions (the readings of what the pages leave open are listed
 * in the repository's design notes; each is restated at its function):
 *  - W is N rows x K columns; row n holds its K codes contiguously.
 *  - Every array below is row-major with rows contiguous.
 *  - fp16 / bf16 values travel as their raw 16-bit patterns (uint16_t).
 *
 * Arithmetic: every float operation is one IEEE binary32 operation rounded to
 * nearest-even, in the order written; the file is compiled with
 * -ffp-contract=off and without fast-math so no FMA contraction happens.
 * The matmul accumulates in binary64, sequentially over k.
 */
#ifndef QL_ORACLE_H
#define QL_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- scalar conversions, written from the IEEE 754 format definitions ---- */
float    or_f32_from_f16(uint16_t h);     /* binary16 -> binary32 (exact)      */
float    or_f32_from_bf16(uint16_t b);    /* bfloat16 -> binary32 (exact)      */
uint16_t or_bf16_from_f32(float f);       /* binary32 -> bfloat16, nearest-even */

/* ---- int4 nested superscale ([NSS] "Quant schema update", int4 bullet) ----
 * q  : u8 [N][K]      codes 0..15 (only the low 4 bits are stored)
 * sc : u8 [N][K/32]   per-group scale code
 * zc : u8 [N][K/32]   per-group zero code
 * ss : fp16 [N][K/256] per-super-block scale step
 * zs : fp16 [N][K/256] per-super-block zero step
 * packed:
 * codes : u8  [N][K/2]   byte i = q[2i] | q[2i+1] << 4   (low nibble first)
 * gmeta : u16 [N][K/32]  sc | zc << 8
 * steps : u32 [N][K/256] ss | zs << 16   (the one 32-bit "z_pack" word)
 */
void or_int4_pack(int64_t N, int64_t K, const uint8_t *q, const uint8_t *sc,
                  const uint8_t *zc, const uint16_t *ss, const uint16_t *zs,
                  uint8_t *codes, uint16_t *gmeta, uint32_t *steps);
void or_int4_unpack(int64_t N, int64_t K, const uint8_t *codes,
                    const uint16_t *gmeta, const uint32_t *steps, uint8_t *q,
                    uint8_t *sc, uint8_t *zc, uint16_t *ss, uint16_t *zs);
/* w[n][k] = (q - Z) * S with S = sc*ss and Z = zc*zs, all binary32 */
void or_int4_dequant(int64_t N, int64_t K, const uint8_t *codes,
                     const uint16_t *gmeta, const uint32_t *steps, float *w);

/* ---- int6 symmetric nested superscale ([NSS], int6 bullet) ----
 * q  : i8 [N][K]       codes -32..31 (low 6 bits, two's complement, stored)
 * sc : i8 [N][K/16]    per-group scale code
 * st : fp16 [N][K/256] per-super-block step
 * packed:
 * codes : u8 [N][3K/4]  each run of 4 codes -> 24-bit little-endian unit
 *                       u24 = sum_i (q[4j+i] & 63) << 6i
 * gmeta : i8 [N][K/16]  sc
 * steps : u16 [N][K/256] st
 */
void or_int6_pack(int64_t N, int64_t K, const int8_t *q, const int8_t *sc,
                  const uint16_t *st, uint8_t *codes, int8_t *gmeta,
                  uint16_t *steps);
void or_int6_unpack(int64_t N, int64_t K, const uint8_t *codes,
                    const int8_t *gmeta, const uint16_t *steps, int8_t *q,
                    int8_t *sc, uint16_t *st);
/* w[n][k] = q * S with S = sc*st, binary32 */
void or_int6_dequant(int64_t N, int64_t K, const uint8_t *codes,
                     const int8_t *gmeta, const uint16_t *steps, float *w);

/* ---- uint32-packed affine ([MTL]) ----
 * bits in {2,4,8}; G = group size along K.
 * q     : u8 [N][K]      codes 0..2^bits-1
 * s     : bf16 [N][K/G]  per-group scale
 * b     : bf16 [N][K/G]  per-group bias
 * packed:
 * codes : u32 [N][K*bits/32]  word t = sum_i (q[tP+i] & (2^bits-1)) << bits*i,
 *                             P = 32/bits (first code in the lowest bits)
 * gmeta : u32 [N][K/G]        s | b << 16
 */
void or_affine_pack(int64_t N, int64_t K, int bits, int G, const uint8_t *q,
                    const uint16_t *s, const uint16_t *b, uint32_t *codes,
                    uint32_t *gmeta);
void or_affine_unpack(int64_t N, int64_t K, int bits, int G,
                      const uint32_t *codes, const uint32_t *gmeta, uint8_t *q,
                      uint16_t *s, uint16_t *b);
/* w[n][k] = q*s + b, binary32 (product first, then the add) */
void or_affine_dequant(int64_t N, int64_t K, int bits, int G,
                       const uint32_t *codes, const uint32_t *gmeta, float *w);

/* ---- the linear layer ----
 * y[m][n] = sum_k f64(x[m][k]) * f64(w[n][k]), summed over k = 0..K-1 in
 * order, in binary64.  x is bf16 [M][K]; w is binary32 [N][K].
 */
void or_matmul_f64(int64_t M, int64_t N, int64_t K, const uint16_t *x_bf16,
                   const float *w, double *y);

/* Round every element of a binary64 array to bfloat16 (via binary32 first
 * only when that is exact is NOT assumed: rounding is done from the double
 * value directly, nearest-even). */
void or_bf16_from_f64_array(int64_t n, const double *y, uint16_t *out);

/* int6, planar storage: the codes of each 256-weight super-block of a row as
 * 128 bytes of low nibbles (weight i at byte i/2, even i low) followed by 64
 * bytes of bits 4-5 (weight i at byte 128 + i/4, bits 2*(i%4)); codes
 * [N][3K/4] bytes.  Same q, sc, st, gmeta, steps and dequantisation as the
 * dense int6 functions. */
void or_int6p_pack(int64_t N, int64_t K, const int8_t *q, const int8_t *sc,
                   const uint16_t *st, uint8_t *codes, int8_t *gmeta,
                   uint16_t *steps);
void or_int6p_unpack(int64_t N, int64_t K, const uint8_t *codes,
                     const int8_t *gmeta, const uint16_t *steps, int8_t *q,
                     int8_t *sc, uint16_t *st);
void or_int6p_dequant(int64_t N, int64_t K, const uint8_t *codes,
                      const int8_t *gmeta, const uint16_t *steps, float *w);

/* number of OpenMP threads the oracle's loops use (1 without OpenMP) */
int or_num_threads(void);

/* set the number of OpenMP threads of the following calls (timing only; the
 * results do not depend on it) */
void or_set_num_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
