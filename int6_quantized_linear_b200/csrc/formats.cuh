// formats.cuh -- exact binary32 dequantisation of 32 consecutive weights of a
// row, for each weight format.  Each routine performs the definition's
// operations one by one with explicit round-to-nearest intrinsics (never
// contracted into FMA), so the result is bit-identical to the definition:
//
//  int4 (ExecuTorch PR "[cuda] Nestest Superscale Quantization for CUDA
//       Weights (int4 / int6)", "Quant schema update", int4 bullet):
//       S = sc*ss, Z = zc*zs, w = (q - Z) * S
//  int6 (same section, int6 bullet):  S = sc*st, w = q * S
//  affine (Transformers "Metal" quantization page): w = q*scale + bias
//
// A "chunk" is 32 consecutive weights of one row starting at a multiple of
// 32: one int4 group, two int6 groups, and a part of one affine group (the
// affine group size is a multiple of 32).
#pragma once
#include "common.cuh"

namespace ql {

enum : int { FMT_INT4 = 1, FMT_INT6 = 2, FMT_AFFINE = 3, FMT_INT6P = 4 };

// ---- int4 -----------------------------------------------------------------
// c: the chunk's 16 code bytes as 4 little-endian words (low nibble = even k)
// gm: the group's 16-bit metadata word (scale code | zero code << 8)
// st: the super-block's step word (fp16 scale step | fp16 zero step << 16)
QL_DEVI void int4_decode32(const uint32_t (&c)[4], uint32_t gm, uint32_t st, float (&w)[32]) {
  const float S = __fmul_rn((float)(gm & 0xffu), f16_bits_to_f32(st));
  const float Z = __fmul_rn((float)((gm >> 8) & 0xffu), f16_bits_to_f32(st >> 16));
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t q = (c[i >> 3] >> (4 * (i & 7))) & 0xfu;
    w[i] = __fmul_rn(__fsub_rn((float)q, Z), S);
  }
}

// ---- int6 -----------------------------------------------------------------
// c: the chunk's 24 code bytes as 6 little-endian words; every 3 bytes hold
//    4 six-bit two's-complement codes, first code in the lowest bits.
// sc2: the two groups' int8 scale codes (group 2j in the low byte)
// st: the super-block's fp16 step (low 16 bits)
QL_DEVI void int6_decode32(const uint32_t (&c)[6], uint32_t sc2, uint32_t st, float (&w)[32]) {
  const float step = f16_bits_to_f32(st);
  const float S0 = __fmul_rn((float)(int8_t)(sc2 & 0xffu), step);
  const float S1 = __fmul_rn((float)(int8_t)((sc2 >> 8) & 0xffu), step);
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // 8 units of 3 bytes
    const int bit = 24 * j;
    const int wi = bit >> 5, sh = bit & 31;
    uint32_t u;
    if (sh <= 8) {
      u = c[wi] >> sh;
    } else {
      u = __funnelshift_r(c[wi], c[wi + 1], sh);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int f = (int)((u >> (6 * i)) & 0x3fu);
      const int q = (f ^ 32) - 32;  // sign-extend 6 bits
      w[4 * j + i] = __fmul_rn((float)q, (4 * j + i) < 16 ? S0 : S1);
    }
  }
}

// ---- int6, planar storage -------------------------------------------------
// The review of the ExecuTorch PR ("Correctness" note 2) describes the
// reference int6 decode kernel's 16-byte load as one 32-weight group at 4
// bits: the codes sit in a 4-bit plane and a 2-bit plane.  Per 256-weight
// super-block: 128 bytes of low nibbles (even weight low), then 64 bytes of
// bits 4-5 (weight i at bits 2*(i%4) of byte 128 + i/4).
// lo: the chunk's 16 low-plane bytes as 4 words; hi: its 8 high-plane bytes
// as 2 words; sc2, st as int6_decode32.
QL_DEVI void int6p_decode32(const uint32_t (&lo)[4], const uint32_t (&hi)[2], uint32_t sc2, uint32_t st,
                            float (&w)[32]) {
  const float step = f16_bits_to_f32(st);
  const float S0 = __fmul_rn((float)(int8_t)(sc2 & 0xffu), step);
  const float S1 = __fmul_rn((float)(int8_t)((sc2 >> 8) & 0xffu), step);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int f = (int)(((lo[i >> 3] >> (4 * (i & 7))) & 0xfu) | (((hi[i >> 4] >> (2 * (i & 15))) & 0x3u) << 4));
    const int q = (f ^ 32) - 32;  // sign-extend 6 bits
    w[i] = __fmul_rn((float)q, i < 16 ? S0 : S1);
  }
}

// ---- affine ---------------------------------------------------------------
// c: the chunk's 32*bits/8 code bytes as BITS words (first code lowest)
// gm: the group's word (bf16 scale | bf16 bias << 16)
template <int BITS>
QL_DEVI void affine_decode32(const uint32_t (&c)[BITS], uint32_t gm, float (&w)[32]) {
  constexpr int P = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const float s = bf16_bits_to_f32(gm);
  const float b = bf16_bits_to_f32(gm >> 16);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t q = (c[i / P] >> (BITS * (i % P))) & MASK;
    w[i] = __fadd_rn(__fmul_rn((float)q, s), b);
  }
}

}  // namespace ql
