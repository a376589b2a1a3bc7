// pack_dequant.cuh -- packing, unpacking and standalone dequantisation.
//
// All three are HBM-bound elementwise passes over flat index spaces: because
// K is a multiple of 256 (int4, int6) or a whole number of 16-byte code words
// (affine), row boundaries never split a unit, so each thread handles whole
// 16-byte output units with vector loads and stores.
#pragma once
#include "formats.cuh"

namespace ql {

struct PackArgs {
  int64_t N, K;
  int bits, G;
  const uint8_t *q;
  const uint8_t *meta0, *meta1;
  const uint16_t *step0, *step1;
  uint8_t *codes;
  uint8_t *gmeta;
  uint8_t *steps;
};

// ---- pack ------------------------------------------------------------------
// Index space = [codes units | gmeta units | steps units], grid-stride.
__global__ void __launch_bounds__(256) pack_int4_kernel(PackArgs a) {
  const int64_t nA = a.N * a.K / 32, nB = a.N * a.K / 256, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {  // 32 codes -> 16 bytes, byte i = q[2i] | q[2i+1] << 4
      const uint4 *src = reinterpret_cast<const uint4 *>(a.q + 32 * u);
      uint4 in[2] = {src[0], src[1]};
      const uint32_t *iw = reinterpret_cast<const uint32_t *>(in);
      uint32_t o[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {  // output word t <- input words 2t, 2t+1 (8 codes)
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t code = (iw[2 * t + (i >> 2)] >> (8 * (i & 3))) & 0xfu;
          r |= code << (4 * i);
        }
        o[t] = r;
      }
      reinterpret_cast<uint4 *>(a.codes)[u] = make_uint4(o[0], o[1], o[2], o[3]);
    } else if (u < nA + nB) {  // 8 groups: sc | zc << 8
      const int64_t v = u - nA;
      const uint2 s = reinterpret_cast<const uint2 *>(a.meta0)[v];
      const uint2 z = reinterpret_cast<const uint2 *>(a.meta1)[v];
      const uint8_t *sb = reinterpret_cast<const uint8_t *>(&s);
      const uint8_t *zb = reinterpret_cast<const uint8_t *>(&z);
      uint32_t o[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        o[t] = (uint32_t)sb[2 * t] | ((uint32_t)zb[2 * t] << 8) | ((uint32_t)sb[2 * t + 1] << 16) |
               ((uint32_t)zb[2 * t + 1] << 24);
      reinterpret_cast<uint4 *>(a.gmeta)[v] = make_uint4(o[0], o[1], o[2], o[3]);
    } else {  // one super-block: ss | zs << 16
      const int64_t v = u - nA - nB;
      reinterpret_cast<uint32_t *>(a.steps)[v] = (uint32_t)a.step0[v] | ((uint32_t)a.step1[v] << 16);
    }
  }
}

__global__ void __launch_bounds__(256) pack_int6_kernel(PackArgs a) {
  const int64_t nA = a.N * a.K / 64, nB = a.N * a.K / 256, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {  // 64 codes -> 48 bytes: 16 units of (c0 | c1<<6 | c2<<12 | c3<<18)
      const uint4 *src = reinterpret_cast<const uint4 *>(a.q + 64 * u);
      uint4 in[4] = {src[0], src[1], src[2], src[3]};
      const uint32_t *iw = reinterpret_cast<const uint32_t *>(in);
      uint32_t o[12];
#pragma unroll
      for (int t = 0; t < 12; ++t) o[t] = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint32_t w4 = iw[j];  // 4 codes, one per byte
        const uint32_t u24 = (w4 & 0x3fu) | (((w4 >> 8) & 0x3fu) << 6) | (((w4 >> 16) & 0x3fu) << 12) |
                             (((w4 >> 24) & 0x3fu) << 18);
        const int bit = 24 * j, wi = bit >> 5, sh = bit & 31;
        o[wi] |= u24 << sh;
        if (sh > 8) o[wi + 1] |= u24 >> (32 - sh);
      }
      uint4 *dst = reinterpret_cast<uint4 *>(a.codes + 48 * u);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
    } else if (u < nA + nB) {  // scale codes: 16-byte copy
      const int64_t v = u - nA;
      reinterpret_cast<uint4 *>(a.gmeta)[v] = reinterpret_cast<const uint4 *>(a.meta0)[v];
    } else {
      const int64_t v = u - nA - nB;
      reinterpret_cast<uint16_t *>(a.steps)[v] = a.step0[v];
    }
  }
}

// int6 planar: unit = 32 codes -> 16 low-plane bytes (at 192 j + 16 t of the row's super-block j,
// chunk t) and 8 high-plane bytes (at 192 j + 128 + 8 t); metadata as dense int6.
__global__ void __launch_bounds__(256) pack_int6p_kernel(PackArgs a) {
  const int64_t nA = a.N * a.K / 32, nB = a.N * a.K / 256, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {
      const uint4 *src = reinterpret_cast<const uint4 *>(a.q + 32 * u);
      uint4 in[2] = {src[0], src[1]};
      const uint32_t *iw = reinterpret_cast<const uint32_t *>(in);  // code i in byte i % 4 of word i / 4
      uint32_t lo[4] = {0u, 0u, 0u, 0u}, hi[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t f = (iw[i >> 2] >> (8 * (i & 3))) & 0x3fu;
        lo[i >> 3] |= (f & 0xfu) << (4 * (i & 7));
        hi[i >> 4] |= (f >> 4) << (2 * (i & 15));
      }
      const int64_t sb = u >> 3, t = u & 7;  // super-block (over all rows: K is a multiple of 256) and chunk
      uint8_t *blk = a.codes + 192 * sb;
      *reinterpret_cast<uint4 *>(blk + 16 * t) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint2 *>(blk + 128 + 8 * t) = make_uint2(hi[0], hi[1]);
    } else if (u < nA + nB) {  // scale codes: 16-byte copy
      const int64_t v = u - nA;
      reinterpret_cast<uint4 *>(a.gmeta)[v] = reinterpret_cast<const uint4 *>(a.meta0)[v];
    } else {
      const int64_t v = u - nA - nB;
      reinterpret_cast<uint16_t *>(a.steps)[v] = a.step0[v];
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(256) pack_affine_kernel(PackArgs a) {
  constexpr int P = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t nA = a.N * a.K * BITS / 128, nB = a.N * a.K / a.G;
  const int64_t total = nA + nB;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {  // 4 output words <- 4P codes
      const uint8_t *src = a.q + (int64_t)4 * P * u;
      uint32_t o[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < P; i += 4) {
          const uint32_t w4 = *reinterpret_cast<const uint32_t *>(src + t * P + i);
#pragma unroll
          for (int b = 0; b < 4; ++b) r |= ((w4 >> (8 * b)) & MASK) << (BITS * (i + b));
        }
        o[t] = r;
      }
      reinterpret_cast<uint4 *>(a.codes)[u] = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      const int64_t v = u - nA;
      const uint16_t *s = reinterpret_cast<const uint16_t *>(a.meta0);
      const uint16_t *b = reinterpret_cast<const uint16_t *>(a.meta1);
      reinterpret_cast<uint32_t *>(a.gmeta)[v] = (uint32_t)s[v] | ((uint32_t)b[v] << 16);
    }
  }
}

// ---- unpack (inverse) --------------------------------------------------------
struct UnpackArgs {
  int64_t N, K;
  int bits, G;
  const uint8_t *codes, *gmeta, *steps;
  uint8_t *q, *meta0, *meta1;
  uint16_t *step0, *step1;
};

__global__ void __launch_bounds__(256) unpack_int4_kernel(UnpackArgs a) {
  const int64_t nA = a.N * a.K / 32, nB = a.N * a.K / 32, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {
      const uint4 in = reinterpret_cast<const uint4 *>(a.codes)[u];
      const uint32_t iw[4] = {in.x, in.y, in.z, in.w};
      uint32_t o[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {  // output word t = codes 4t..4t+3
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = 4 * t + i;
          r |= ((iw[k >> 3] >> (4 * (k & 7))) & 0xfu) << (8 * i);
        }
        o[t] = r;
      }
      uint4 *dst = reinterpret_cast<uint4 *>(a.q + 32 * u);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else if (u < nA + nB) {
      const int64_t v = u - nA;
      const uint16_t gm = reinterpret_cast<const uint16_t *>(a.gmeta)[v];
      if (a.meta0) a.meta0[v] = (uint8_t)(gm & 0xff);
      if (a.meta1) a.meta1[v] = (uint8_t)(gm >> 8);
    } else {
      const int64_t v = u - nA - nB;
      const uint32_t st = reinterpret_cast<const uint32_t *>(a.steps)[v];
      if (a.step0) a.step0[v] = (uint16_t)(st & 0xffff);
      if (a.step1) a.step1[v] = (uint16_t)(st >> 16);
    }
  }
}

__global__ void __launch_bounds__(256) unpack_int6_kernel(UnpackArgs a) {
  const int64_t nA = a.N * a.K / 64, nB = a.N * a.K / 16, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {
      const uint4 *src = reinterpret_cast<const uint4 *>(a.codes + 48 * u);
      uint4 in[3] = {src[0], src[1], src[2]};
      const uint32_t *iw = reinterpret_cast<const uint32_t *>(in);
      uint32_t o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int bit = 24 * j, wi = bit >> 5, sh = bit & 31;
        const uint32_t u24 = (sh <= 8) ? (iw[wi] >> sh) : __funnelshift_r(iw[wi], iw[wi + 1], sh);
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t f = (u24 >> (6 * i)) & 0x3fu;
          const uint32_t byte = (f & 0x20u) ? (f | 0xc0u) : f;  // sign-extend into the byte
          r |= byte << (8 * i);
        }
        o[j] = r;
      }
      uint4 *dst = reinterpret_cast<uint4 *>(a.q + 64 * u);
#pragma unroll
      for (int t = 0; t < 4; ++t) dst[t] = make_uint4(o[4 * t], o[4 * t + 1], o[4 * t + 2], o[4 * t + 3]);
    } else if (u < nA + nB) {
      const int64_t v = u - nA;
      if (a.meta0) a.meta0[v] = a.gmeta[v];
    } else {
      const int64_t v = u - nA - nB;
      if (a.step0) a.step0[v] = reinterpret_cast<const uint16_t *>(a.steps)[v];
    }
  }
}

__global__ void __launch_bounds__(256) unpack_int6p_kernel(UnpackArgs a) {
  const int64_t nA = a.N * a.K / 32, nB = a.N * a.K / 16, nC = a.N * a.K / 256;
  const int64_t total = nA + nB + nC;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {
      const int64_t sb = u >> 3, t = u & 7;
      const uint8_t *blk = a.codes + 192 * sb;
      const uint4 l = *reinterpret_cast<const uint4 *>(blk + 16 * t);
      const uint2 h = *reinterpret_cast<const uint2 *>(blk + 128 + 8 * t);
      const uint32_t lo[4] = {l.x, l.y, l.z, l.w}, hi[2] = {h.x, h.y};
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t r = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int i = 4 * j + b;
          const uint32_t f = ((lo[i >> 3] >> (4 * (i & 7))) & 0xfu) | (((hi[i >> 4] >> (2 * (i & 15))) & 0x3u) << 4);
          r |= ((f & 0x20u) ? (f | 0xc0u) : f) << (8 * b);  // sign-extend into the byte
        }
        o[j] = r;
      }
      uint4 *dst = reinterpret_cast<uint4 *>(a.q + 32 * u);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else if (u < nA + nB) {
      const int64_t v = u - nA;
      if (a.meta0) a.meta0[v] = a.gmeta[v];
    } else {
      const int64_t v = u - nA - nB;
      if (a.step0) a.step0[v] = reinterpret_cast<const uint16_t *>(a.steps)[v];
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(256) unpack_affine_kernel(UnpackArgs a) {
  constexpr int P = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int64_t nA = a.N * a.K / P, nB = a.N * a.K / a.G;
  const int64_t total = nA + nB;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    if (u < nA) {  // one word -> P bytes (P is 4, 8 or 16: whole 32-bit stores)
      const uint32_t wd = reinterpret_cast<const uint32_t *>(a.codes)[u];
      uint32_t *dst = reinterpret_cast<uint32_t *>(a.q + (int64_t)P * u);
#pragma unroll
      for (int t = 0; t < P / 4; ++t) {
        uint32_t r = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) r |= ((wd >> (BITS * (4 * t + i))) & MASK) << (8 * i);
        dst[t] = r;
      }
    } else {
      const int64_t v = u - nA;
      const uint32_t gm = reinterpret_cast<const uint32_t *>(a.gmeta)[v];
      if (a.meta0) reinterpret_cast<uint16_t *>(a.meta0)[v] = (uint16_t)(gm & 0xffff);
      if (a.meta1) reinterpret_cast<uint16_t *>(a.meta1)[v] = (uint16_t)(gm >> 16);
    }
  }
}

// ---- chunk loaders (global memory) -------------------------------------------
struct WeightPtrs {
  const uint8_t *codes;
  const uint8_t *gmeta;
  const uint8_t *steps;
  int64_t K;
  int G;
};

// Decode chunk c (weights 32c .. 32c+31) of row n, exactly.
template <int FMT, int BITS>
QL_DEVI void load_decode32(const WeightPtrs &p, int64_t n, int64_t c, float (&w)[32]) {
  if constexpr (FMT == FMT_INT4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.codes + n * (p.K / 2)) + c);
    const uint32_t cw[4] = {v.x, v.y, v.z, v.w};
    const uint32_t gm = __ldg(reinterpret_cast<const uint16_t *>(p.gmeta) + n * (p.K / 32) + c);
    const uint32_t st = __ldg(reinterpret_cast<const uint32_t *>(p.steps) + n * (p.K / 256) + (c >> 3));
    int4_decode32(cw, gm, st, w);
  } else if constexpr (FMT == FMT_INT6) {
    const uint2 *src = reinterpret_cast<const uint2 *>(p.codes + n * (3 * p.K / 4) + 24 * c);
    const uint2 v0 = __ldg(src), v1 = __ldg(src + 1), v2 = __ldg(src + 2);
    const uint32_t cw[6] = {v0.x, v0.y, v1.x, v1.y, v2.x, v2.y};
    const uint32_t sc2 = __ldg(reinterpret_cast<const uint16_t *>(p.gmeta + n * (p.K / 16)) + c);
    const uint32_t st = __ldg(reinterpret_cast<const uint16_t *>(p.steps) + n * (p.K / 256) + (c >> 3));
    int6_decode32(cw, sc2, st, w);
  } else if constexpr (FMT == FMT_INT6P) {
    const uint8_t *blk = p.codes + n * (3 * p.K / 4) + 192 * (c >> 3);
    const uint4 l = __ldg(reinterpret_cast<const uint4 *>(blk + 16 * (c & 7)));
    const uint2 h = __ldg(reinterpret_cast<const uint2 *>(blk + 128 + 8 * (c & 7)));
    const uint32_t lo[4] = {l.x, l.y, l.z, l.w}, hi[2] = {h.x, h.y};
    const uint32_t sc2 = __ldg(reinterpret_cast<const uint16_t *>(p.gmeta + n * (p.K / 16)) + c);
    const uint32_t st = __ldg(reinterpret_cast<const uint16_t *>(p.steps) + n * (p.K / 256) + (c >> 3));
    int6p_decode32(lo, hi, sc2, st, w);
  } else {
    const uint32_t *src = reinterpret_cast<const uint32_t *>(p.codes + n * (p.K * BITS / 8)) + BITS * c;
    uint32_t cw[BITS];
    if constexpr (BITS == 2) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src));
      cw[0] = v.x; cw[1] = v.y;
    } else {
#pragma unroll
      for (int t = 0; t < BITS / 4; ++t) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src) + t);
        cw[4 * t] = v.x; cw[4 * t + 1] = v.y; cw[4 * t + 2] = v.z; cw[4 * t + 3] = v.w;
      }
    }
    const uint32_t gm = __ldg(reinterpret_cast<const uint32_t *>(p.gmeta) + n * (p.K / p.G) + (32 * c) / p.G);
    affine_decode32<BITS>(cw, gm, w);
  }
}

// ---- standalone dequantisation -----------------------------------------------
template <int FMT, int BITS, bool OUT_BF16>
__global__ void __launch_bounds__(256) dequant_kernel(WeightPtrs p, int64_t N, void *out) {
  const int64_t cpr = p.K / 32, total = N * cpr;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = u / cpr, c = u - n * cpr;
    float w[32];
    load_decode32<FMT, BITS>(p, n, c, w);
    if constexpr (OUT_BF16) {
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + 32 * u);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        dst[t] = make_uint4(pack_bf16x2(w[8 * t], w[8 * t + 1]), pack_bf16x2(w[8 * t + 2], w[8 * t + 3]),
                            pack_bf16x2(w[8 * t + 4], w[8 * t + 5]), pack_bf16x2(w[8 * t + 6], w[8 * t + 7]));
    } else {
      float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + 32 * u);
#pragma unroll
      for (int t = 0; t < 8; ++t) dst[t] = make_float4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
    }
  }
}


// Metadata encoder (the int4 / int6 metadata of the ExecuTorch PR "[cuda] Nestest Superscale
// Quantization for CUDA Weights", "Quant schema update"; its review, "Correctness" note 1 and
// "Things done well"): one thread per (row, super-block) of one per-group float field.
// int4 (SIGNED false): step = fp16(max / 255), code = clamp(rint(v / step_f), 0, 255);
// int6 (SIGNED true):  step = fp16(max|v| / 127), code = clamp(rint(v / step_f), -127, 127);
// step_f is the fp16-rounded step, so encoder and decoder reconstruct with the same value; the
// divisions are IEEE binary32, rint rounds half to even, a zero max gives step 0 and codes 0.
// A non-finite value (or a negative one for int4) sets QL_DEV_RANGE.
template <bool SIGNED, int PER>
__global__ void __launch_bounds__(256) quantize_meta_kernel(const float *v0, const float *v1, int64_t rows, int64_t G,
                                                            uint8_t *codes0, uint8_t *codes1, uint16_t *steps0,
                                                            uint16_t *steps1) {
  // blockIdx.y picks the array (int4: scale, zero); thread t = (row, super-block) owns elements
  // t * PER .. t * PER + PER - 1, read as 16-byte vectors, and writes its PER codes in one store
  const float *v = blockIdx.y ? v1 : v0;
  uint8_t *codes = blockIdx.y ? codes1 : codes0;
  uint16_t *steps = blockIdx.y ? steps1 : steps0;
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= rows * (G / PER)) return;
  const float4 *src = reinterpret_cast<const float4 *>(v) + t * (PER / 4);
  float x[PER];
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) {
    const float4 f = __ldg(src + i);
    x[4 * i] = f.x; x[4 * i + 1] = f.y; x[4 * i + 2] = f.z; x[4 * i + 3] = f.w;
  }
  float m = 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    bad |= !isfinite(x[i]) || (!SIGNED && x[i] < 0.f);
    m = fmaxf(m, SIGNED ? fabsf(x[i]) : x[i]);
  }
  if (bad) atomicOr(&g_ql_status, QL_DEV_RANGE);
  const __half st = __float2half_rn(__fdiv_rn(m, SIGNED ? 127.f : 255.f));
  const float sf = __half2float(st);
  const float lo = SIGNED ? -127.f : 0.f, hi = SIGNED ? 127.f : 255.f;
  uint32_t w[PER / 4];
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) w[i] = 0u;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float q = sf > 0.f ? fminf(hi, fmaxf(lo, rintf(__fdiv_rn(x[i], sf)))) : 0.f;
    const uint32_t b = SIGNED ? (uint32_t)(uint8_t)(int8_t)(int)q : (uint32_t)(uint8_t)(int)q;
    w[i / 4] |= b << (8 * (i % 4));
  }
  if constexpr (PER == 8) {
    reinterpret_cast<uint2 *>(codes)[t] = make_uint2(w[0], w[1]);
  } else {
    reinterpret_cast<uint4 *>(codes)[t] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  steps[t] = __half_as_ushort(st);
}
}  // namespace ql
