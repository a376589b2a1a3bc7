/*
 * oracle.c -- plain CPU restatement of the weight-only quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): used by the tests, the smoke check
 * and the benchmark's CPU baseline; never by the product path.
 *
 * Build: cc -O2 -std=c99 -ffp-contract=off -fno-fast-math -fopenmp
 *        -shared -fPIC oracle.c -lm
 * Every binary32 operation below is a single correctly rounded operation in
 * the order written (x86-64 SSE arithmetic, no contraction).
 */
#include "oracle.h"

#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE 754 conversions written from the format definitions                 */
/* ------------------------------------------------------------------------ */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * normal:    (-1)^s * (1 + f/1024) * 2^(e-15)
 * subnormal: (-1)^s * (f/1024) * 2^-14                                   */
float or_f32_from_f16(uint16_t h) {
  int s = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0x1f) {
    v = f ? NAN : INFINITY;
  } else if (e == 0) {
    v = ldexp((double)f, -24);
  } else {
    v = ldexp((double)(1024 + f), e - 25);
  }
  return (float)(s ? -v : v); /* exact: every binary16 value is a binary32 */
}

/* bfloat16 is the top half of a binary32 pattern. */
float or_f32_from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static uint16_t bf16_bits_of_f32_trunc(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* Nearest-even rounding of a real value v (given exactly as a double) to
 * bfloat16, by comparing the two bfloat16 neighbours of v. */
static uint16_t bf16_round_from_double(double v) {
  if (isnan(v)) return 0x7fc0;
  int neg = signbit(v) != 0;
  double a = fabs(v);
  uint16_t sign = neg ? 0x8000 : 0;
  /* largest finite bfloat16 and the rounding threshold halfway to 2^128 */
  const double maxbf = ldexp(255.0, 120);        /* (2 - 2^-7) * 2^127 */
  const double halfway = ldexp(511.0, 119);      /* (2 - 2^-8) * 2^127 */
  if (a >= halfway) return sign | 0x7f80;        /* rounds to infinity */
  if (a >= maxbf) return sign | 0x7f7f;
  if (a == 0.0) return sign;
  /* spacing of bfloat16 values around a: 2^(e-7) for a in [2^e, 2^(e+1)),
   * with e clamped to -126 in the subnormal range */
  int e;
  frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) -> a in [2^(e-1), 2^e) */
  e -= 1;
  if (e < -126) e = -126;
  double ulp = ldexp(1.0, e - 7);
  double lo = floor(a / ulp) * ulp; /* exact: a/ulp is a scaling by 2^k */
  double hi = lo + ulp;
  double dlo = a - lo, dhi = hi - a;
  double r;
  if (dlo < dhi) {
    r = lo;
  } else if (dhi < dlo) {
    r = hi;
  } else {
    /* tie: pick the neighbour whose last significand bit is zero */
    double k = lo / ulp;
    r = (fmod(k, 2.0) == 0.0) ? lo : hi;
  }
  /* r is exactly a bfloat16 value, so its binary32 form truncates cleanly */
  return sign | bf16_bits_of_f32_trunc((float)r);
}

uint16_t or_bf16_from_f32(float f) { return bf16_round_from_double((double)f); }

void or_bf16_from_f64_array(int64_t n, const double *y, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_round_from_double(y[i]);
}

int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void or_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* int4 nested superscale: group 32, super-block 256 (8 groups).            */
/* [NSS] "Quant schema update": scale = uint8 code x per-256 fp16 step,     */
/* zero = uint8 code x per-256 fp16 step, both steps in one 32-bit word,    */
/* w = (q - zero) * scale.                                                  */
/* ------------------------------------------------------------------------ */

void or_int4_pack(int64_t N, int64_t K, const uint8_t *q, const uint8_t *sc,
                  const uint8_t *zc, const uint16_t *ss, const uint16_t *zs,
                  uint8_t *codes, uint16_t *gmeta, uint32_t *steps) {
  const int64_t ng = K / 32, nsb = K / 256;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t i = 0; i < K / 2; ++i) {
      uint8_t lo = q[n * K + 2 * i] & 0xf;
      uint8_t hi = q[n * K + 2 * i + 1] & 0xf;
      codes[n * (K / 2) + i] = (uint8_t)(lo | (hi << 4));
    }
    for (int64_t g = 0; g < ng; ++g)
      gmeta[n * ng + g] =
          (uint16_t)(sc[n * ng + g] | ((uint16_t)zc[n * ng + g] << 8));
    for (int64_t j = 0; j < nsb; ++j)
      steps[n * nsb + j] =
          (uint32_t)ss[n * nsb + j] | ((uint32_t)zs[n * nsb + j] << 16);
  }
}

void or_int4_unpack(int64_t N, int64_t K, const uint8_t *codes,
                    const uint16_t *gmeta, const uint32_t *steps, uint8_t *q,
                    uint8_t *sc, uint8_t *zc, uint16_t *ss, uint16_t *zs) {
  const int64_t ng = K / 32, nsb = K / 256;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = codes[n * (K / 2) + k / 2];
      q[n * K + k] = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
    }
    for (int64_t g = 0; g < ng; ++g) {
      sc[n * ng + g] = (uint8_t)(gmeta[n * ng + g] & 0xff);
      zc[n * ng + g] = (uint8_t)(gmeta[n * ng + g] >> 8);
    }
    for (int64_t j = 0; j < nsb; ++j) {
      ss[n * nsb + j] = (uint16_t)(steps[n * nsb + j] & 0xffff);
      zs[n * nsb + j] = (uint16_t)(steps[n * nsb + j] >> 16);
    }
  }
}

void or_int4_dequant(int64_t N, int64_t K, const uint8_t *codes,
                     const uint16_t *gmeta, const uint32_t *steps, float *w) {
  const int64_t ng = K / 32, nsb = K / 256;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / 32, j = k / 256;
      uint8_t byte = codes[n * (K / 2) + k / 2];
      int q = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
      uint16_t gm = gmeta[n * ng + g];
      uint32_t st = steps[n * nsb + j];
      float scale_step = or_f32_from_f16((uint16_t)(st & 0xffff));
      float zero_step = or_f32_from_f16((uint16_t)(st >> 16));
      float S = (float)(gm & 0xff) * scale_step; /* scale = code x step */
      float Z = (float)(gm >> 8) * zero_step;    /* zero  = code x step */
      float t = (float)q - Z;                    /* q - zero            */
      w[n * K + k] = t * S;                      /* (q - zero) * scale  */
    }
  }
}

/* ------------------------------------------------------------------------ */
/* int6 symmetric: group 16, super-block 256 (16 groups), no zero.          */
/* [NSS] "Quant schema update": scale = int8 code x per-256 fp16 step.      */
/* Dense 6-bit storage, 4 codes per 3 bytes (LSB-first 24-bit units).       */
/* ------------------------------------------------------------------------ */

void or_int6_pack(int64_t N, int64_t K, const int8_t *q, const int8_t *sc,
                  const uint16_t *st, uint8_t *codes, int8_t *gmeta,
                  uint16_t *steps) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < K / 4; ++j) {
      uint32_t u = 0;
      for (int i = 0; i < 4; ++i)
        u |= ((uint32_t)(uint8_t)q[n * K + 4 * j + i] & 0x3f) << (6 * i);
      codes[n * rb + 3 * j + 0] = (uint8_t)(u & 0xff);
      codes[n * rb + 3 * j + 1] = (uint8_t)((u >> 8) & 0xff);
      codes[n * rb + 3 * j + 2] = (uint8_t)((u >> 16) & 0xff);
    }
    for (int64_t g = 0; g < ng; ++g) gmeta[n * ng + g] = sc[n * ng + g];
    for (int64_t j = 0; j < nsb; ++j) steps[n * nsb + j] = st[n * nsb + j];
  }
}

static int int6_code_at(const uint8_t *row, int64_t k) {
  int64_t j = k / 4;
  int i = (int)(k % 4);
  uint32_t u = (uint32_t)row[3 * j] | ((uint32_t)row[3 * j + 1] << 8) |
               ((uint32_t)row[3 * j + 2] << 16);
  int field = (int)((u >> (6 * i)) & 0x3f);
  return field >= 32 ? field - 64 : field; /* two's complement, 6 bits */
}

void or_int6_unpack(int64_t N, int64_t K, const uint8_t *codes,
                    const int8_t *gmeta, const uint16_t *steps, int8_t *q,
                    int8_t *sc, uint16_t *st) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k)
      q[n * K + k] = (int8_t)int6_code_at(codes + n * rb, k);
    for (int64_t g = 0; g < ng; ++g) sc[n * ng + g] = gmeta[n * ng + g];
    for (int64_t j = 0; j < nsb; ++j) st[n * nsb + j] = steps[n * nsb + j];
  }
}

void or_int6_dequant(int64_t N, int64_t K, const uint8_t *codes,
                     const int8_t *gmeta, const uint16_t *steps, float *w) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int q = int6_code_at(codes + n * rb, k);
      float step = or_f32_from_f16(steps[n * nsb + k / 256]);
      float S = (float)gmeta[n * ng + k / 16] * step; /* scale = code x step */
      w[n * K + k] = (float)q * S;                     /* q * scale          */
    }
  }
}

/* ------------------------------------------------------------------------ */
/* int6, planar storage.  [REV] "Correctness" note 2 describes the reference */
/* int6 decode kernel's 16-byte load as spanning one 32-weight group at 4    */
/* bits, i.e. the 6-bit codes are held as a 4-bit plane plus a 2-bit plane.  */
/* Reading: per 256-weight super-block of a row, 128 bytes of low nibbles    */
/* (weight i of the super-block at byte i/2, even i in the low nibble), then */
/* 64 bytes of the codes' bits 4-5 (weight i at byte 128 + i/4, bits         */
/* 2*(i%4)); the codes are the same two's-complement 6-bit values as the     */
/* dense layout, and so are the metadata and the dequantisation.             */
/* ------------------------------------------------------------------------ */

void or_int6p_pack(int64_t N, int64_t K, const int8_t *q, const int8_t *sc,
                   const uint16_t *st, uint8_t *codes, int8_t *gmeta,
                   uint16_t *steps) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < nsb; ++j) {
      uint8_t *blk = codes + n * rb + 192 * j;
      for (int b = 0; b < 192; ++b) blk[b] = 0;
      for (int i = 0; i < 256; ++i) {
        uint32_t f = (uint32_t)(uint8_t)q[n * K + 256 * j + i] & 0x3f; /* 6-bit field */
        blk[i / 2] |= (uint8_t)((f & 0xf) << (4 * (i % 2)));          /* low plane   */
        blk[128 + i / 4] |= (uint8_t)((f >> 4) << (2 * (i % 4)));     /* high plane  */
      }
    }
    for (int64_t g = 0; g < ng; ++g) gmeta[n * ng + g] = sc[n * ng + g];
    for (int64_t j = 0; j < nsb; ++j) steps[n * nsb + j] = st[n * nsb + j];
  }
}

static int int6p_code_at(const uint8_t *row, int64_t k) {
  const uint8_t *blk = row + 192 * (k / 256);
  int i = (int)(k % 256);
  int lo = (blk[i / 2] >> (4 * (i % 2))) & 0xf;
  int hi = (blk[128 + i / 4] >> (2 * (i % 4))) & 0x3;
  int field = lo | (hi << 4);
  return field >= 32 ? field - 64 : field; /* two's complement, 6 bits */
}

void or_int6p_unpack(int64_t N, int64_t K, const uint8_t *codes,
                     const int8_t *gmeta, const uint16_t *steps, int8_t *q,
                     int8_t *sc, uint16_t *st) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k)
      q[n * K + k] = (int8_t)int6p_code_at(codes + n * rb, k);
    for (int64_t g = 0; g < ng; ++g) sc[n * ng + g] = gmeta[n * ng + g];
    for (int64_t j = 0; j < nsb; ++j) st[n * nsb + j] = steps[n * nsb + j];
  }
}

void or_int6p_dequant(int64_t N, int64_t K, const uint8_t *codes,
                      const int8_t *gmeta, const uint16_t *steps, float *w) {
  const int64_t ng = K / 16, nsb = K / 256, rb = 3 * K / 4;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int q = int6p_code_at(codes + n * rb, k);
      float step = or_f32_from_f16(steps[n * nsb + k / 256]);
      float S = (float)gmeta[n * ng + k / 16] * step; /* scale = code x step */
      w[n * K + k] = (float)q * S;                     /* q * scale          */
    }
  }
}

/* ------------------------------------------------------------------------ */
/* uint32-packed affine ([MTL]): codes of `bits` bits packed into uint32    */
/* words along K, per-group scale and bias, w = q * scale + bias.           */
/* ------------------------------------------------------------------------ */

void or_affine_pack(int64_t N, int64_t K, int bits, int G, const uint8_t *q,
                    const uint16_t *s, const uint16_t *b, uint32_t *codes,
                    uint32_t *gmeta) {
  const int P = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t nw = K / P, ng = K / G;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t t = 0; t < nw; ++t) {
      uint32_t word = 0;
      for (int i = 0; i < P; ++i)
        word |= ((uint32_t)q[n * K + t * P + i] & mask) << (bits * i);
      codes[n * nw + t] = word;
    }
    for (int64_t g = 0; g < ng; ++g)
      gmeta[n * ng + g] = (uint32_t)s[n * ng + g] | ((uint32_t)b[n * ng + g] << 16);
  }
}

void or_affine_unpack(int64_t N, int64_t K, int bits, int G,
                      const uint32_t *codes, const uint32_t *gmeta, uint8_t *q,
                      uint16_t *s, uint16_t *b) {
  const int P = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t nw = K / P, ng = K / G;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k)
      q[n * K + k] = (uint8_t)((codes[n * nw + k / P] >> (bits * (k % P))) & mask);
    for (int64_t g = 0; g < ng; ++g) {
      s[n * ng + g] = (uint16_t)(gmeta[n * ng + g] & 0xffff);
      b[n * ng + g] = (uint16_t)(gmeta[n * ng + g] >> 16);
    }
  }
}

void or_affine_dequant(int64_t N, int64_t K, int bits, int G,
                       const uint32_t *codes, const uint32_t *gmeta, float *w) {
  const int P = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t nw = K / P, ng = K / G;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      uint32_t q = (codes[n * nw + k / P] >> (bits * (k % P))) & mask;
      uint32_t gm = gmeta[n * ng + k / G];
      float scale = or_f32_from_bf16((uint16_t)(gm & 0xffff));
      float bias = or_f32_from_bf16((uint16_t)(gm >> 16));
      float p = (float)q * scale; /* q * scale */
      w[n * K + k] = p + bias;    /* + bias    */
    }
  }
}

/* ------------------------------------------------------------------------ */
/* y = x . W^T in binary64                                                  */
/* ------------------------------------------------------------------------ */

void or_matmul_f64(int64_t M, int64_t N, int64_t K, const uint16_t *x_bf16,
                   const float *w, double *y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += (double)or_f32_from_bf16(x_bf16[m * K + k]) * (double)w[n * K + k];
      y[m * N + n] = acc;
    }
  }
}
