// gemv.cuh -- decode-shaped layer y[M][N] = x[M][K] . W^T for small M.
//
// Simple form (affine weights whose group size has no tensor-core kernel):
// one warp per output row; lane l takes chunks l, l+32, ... of the row (32
// weights each, coalesced loads), decodes the exact binary32 weights and
// accumulates x*w in fp32; a warp-shuffle reduction finishes the row.  The
// trip count over chunks is the same for every lane of a warp, so full-mask
// shuffles are always reached.
#pragma once
#include "gemm_prep.cuh"
#include "pack_dequant.cuh"

namespace ql {

// Optional per-output-row bias (bf16 [N], may be NULL), added in fp32 before the one rounding.
QL_DEVI float bias_at(const __nv_bfloat16 *bias, int64_t n) { return bias ? __bfloat162float(bias[n]) : 0.f; }

template <int FMT, int BITS, int MT>
__global__ void __launch_bounds__(256) gemv_simple_kernel(WeightPtrs p, int64_t N, const __nv_bfloat16 *x,
                                                          int M, const __nv_bfloat16 *bias, __nv_bfloat16 *y) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t cpr = p.K / 32;
  for (int64_t n = warp; n < N; n += nwarps) {
    for (int m0 = 0; m0 < M; m0 += MT) {
      float acc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.f;
      for (int64_t c0 = 0; c0 < cpr; c0 += 32) {  // uniform trip count across the warp
        const int64_t c = c0 + lane;
        if (c < cpr) {
          float w[32];
          load_decode32<FMT, BITS>(p, n, c, w);
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m0 + m < M) {
              const uint4 *xr = reinterpret_cast<const uint4 *>(x + (int64_t)(m0 + m) * p.K + 32 * c);
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const uint4 v = __ldg(xr + t);
                const uint32_t xv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  acc[m] = fmaf(w[8 * t + 2 * i], __uint_as_float(xv[i] << 16), acc[m]);
                  acc[m] = fmaf(w[8 * t + 2 * i + 1], __uint_as_float(xv[i] & 0xffff0000u), acc[m]);
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m0 + m < M) y[(int64_t)(m0 + m) * N + n] = __float2bfloat16_rn(acc[m] + bias_at(bias, n));
      }
    }
  }
}


// ===========================================================================
// Tensor-core decode GEMV for int4 at M = 1 (integer MMA).
//
// Each warp owns a tile of 16 weight rows and a range of super-blocks.  The
// codes of one super-block of the tile (16 rows x 128 bytes) arrive by TMA
// into a per-warp ring in shared memory.  Lane (g = lane/4, c = lane%4) reads
// whole 16-byte groups -- groups c and c+4 of two tile rows -- and turns each
// 32-bit word of 8 nibbles into two u8x4 registers with one bit operation
// each: w & 0xF0F0F0F0 holds the odd-k codes times 16, (w << 4) & 0xF0F0F0F0
// the even-k codes times 16.
//
// mma.sync.m16n8k32 (u8 x s8 / u8 x u8, s32 accumulate) multiplies these
// 16x32 fragments by a "diagonal" x operand: column n of B holds x only in
// the k-slots that carry group n's codes and zeros elsewhere, so D[row][n]
// collects group n's partial dot product.  x enters as fixed point per
// 32-element group, x_int = rint(x * 2^a_g), as up to three bytes x_int =
// 65536 * hi + 256 * mid + lo (a signed high byte, unsigned middle and low
// bytes), one MMA each:
//   - 16-bit (the group's max |x| scaled into [2^14, 2^15), lo = 0: no third
//     MMA), exact for every bf16 element within 2^7 of the group's largest
//     magnitude, the rest rounded to 2^-15 of it;
//   - 24-bit (max |x| in [2^22, 2^23)), exact within 2^15, for every group of
//     a super-block in which some group's 16-bit rounding error exceeds 2^-12
//     of that group's mass outside its largest element (a dominant outlier,
//     where the 16-bit form would lose the other elements).
// Per (row, group) of a super-block the integer sums are exact and below 2^22
// in magnitude, so the accumulators start at 1.5 * 2^23 (as bits) and read
// back as floats with one subtraction.  The streaming loop runs the high and
// middle bytes only and applies the scale and zero once per (row, group):
//     T = 256 * D_hi + D_mid,   y += S * G_x * (T + Z * G_y)
// with S = sc * ss, Z = zc * zs, X_g = sum_k x_int_k and (G_x, G_y) =
// (2^-a_g / 16, -16 X_g), which for 16-bit x is the whole product.  For 24-bit
// x, T is 2^-8 of 16 sum_k q_k x_int_k less the low bytes' share, so (G_x, G_y)
// = (2^8 * 2^-a_g / 16, -16 X_g / 2^8), G_x carries the 24-bit marker
// (mark_24bit), and after the loop an out-of-line pass adds S G_x 2^-8 D_lo for
// the marked super-blocks, reading their weights again (gemv_m1_low_bytes).
// Each CTA (four tiles over one part of K) converts its part of x itself into
// shared memory -- the x bytes in the order the fragments read them, (G_x, G_y)
// per group and a 24-bit flag per super-block -- after its weight copies have
// started and griddepcontrol.wait has let the previous kernel on the stream
// finish.  Lanes that hold no x for an MMA read a zero block, so no per-MMA
// selects are needed.
// ===========================================================================

constexpr int GEMV_MT_MAX_CTAS = 4096;  // bound on the CTAs of one multi-token launch (sizes its partial sums)

// The split of K over the CTAs of the multi-token and int6 GEMVs: units -- 64-row groups -- 0 .. extra - 1
// take P + 1 parts and the rest P, so that units x parts can match
// the resident slots exactly and no SM idles while the others stream.  Part w of the grid belongs to
// unit `unit`, is its part `part` of `pu`, and the unit's parts start at grid index `first`.
struct SplitK {
  int P, extra;
  __host__ __device__ int64_t total(int64_t units) const { return units * P + extra; }
  // 32-bit arithmetic: a grid has fewer than 2^31 parts
  __host__ __device__ void locate(int w, int64_t &unit, int &part, int &pu, int64_t &first) const {
    const int big = extra * (P + 1);
    int u, f;
    if (w < big) {
      u = w / (P + 1);
      pu = P + 1;
      f = u * pu;
    } else {
      const int q = (w - big) / P;
      u = extra + q;
      pu = P;
      f = big + q * P;
    }
    part = w - f;
    unit = u;
    first = f;
  }
};

// P = slots / units parts per unit (at least 1, at most NS, the super-blocks of K).  With fill, when
// the units alone nearly fill the slots (P = 1), the leftover slots take the second halves of as many
// units (measured: the int4 multi-token and int6 kernels at 432 row groups of 444 slots gain 3-4 %);
// when K is already split, or without fill, the parts stay even (uneven parts measured slower there:
// the unsplit CTAs remain the critical path and the split adds its partial sums).
inline SplitK split_k(int64_t units, int64_t slots, int64_t NS, bool fill) {
  SplitK s;
  const int64_t P = std::max<int64_t>(1, std::min<int64_t>(NS, slots / units));
  s.P = (int)P;
  s.extra = fill && P == 1 && NS > 1 ? (int)std::max<int64_t>(0, std::min<int64_t>(units, slots - units)) : 0;
  return s;
}

// M = 1 x block per super-block (in the CTA's shared memory): 8 x (G_x, G_y) (64 B) and the (hi, mid)
// x words (1 KB), then the lo x words (512 B), written and read only for a 24-bit super-block
constexpr int GEMV_XBLOB = 1600, GEMV_XCOPY = 1088, GEMV_XB_Q = 64, GEMV_XB_L = 1088;

struct GemvWorkspace {
  uint4 *xq;        // int4 M > 1 / affine: [K/32 groups][M tokens][4][16 B] (hi, mid) B-operand words, then
                    //   [K/32][M][4][8 B] lo words (gemv_xprep_mt_kernel); int6: see gemv_xprep_int6_kernel
  float2 *gsum;     // M > 1: [K/32][M]: (G_x, G_y); int6: per 16-element group scales
  float *partial;   // [CTA][M][64 rows]: sums of one K range
  int *counters;    // parts finished so far, per 64-row group
  uint8_t *flags;   // [K/256][16]: byte m non-zero when token m's x of that super-block is 24-bit
};

// floats of partial sums: the multi-token and int6 kernels' bound, or the M = 1 kernel's when a wide
// layer splits K only so that each part's x fits a CTA (64 sums a CTA, parts of at least 20 super-blocks)
inline size_t gemv_partial_floats(int64_t M, int64_t N, int64_t K) {
  const size_t mt = (size_t)GEMV_MT_MAX_CTAS * 64 * M;
  const size_t m1 = (size_t)64 * ((N + 63) / 64) * ((K / 256 + 19) / 20);
  return mt > m1 ? mt : m1;
}

inline size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return align256((size_t)M * K * 7) + align256((size_t)M * (K / 32) * 8) +
         align256(gemv_partial_floats(M, N, K) * 4) + align256((size_t)((N + 15) / 16) * 4) +
         align256((size_t)(K / 256) * 16);
}

inline GemvWorkspace gemv_workspace_carve(void *base, int64_t M, int64_t N, int64_t K) {
  uint8_t *p = static_cast<uint8_t *>(base);
  GemvWorkspace w;
  w.xq = reinterpret_cast<uint4 *>(p);
  p += align256((size_t)M * K * 7);
  w.gsum = reinterpret_cast<float2 *>(p);
  p += align256((size_t)M * (K / 32) * 8);
  w.partial = reinterpret_cast<float *>(p);
  p += align256(gemv_partial_floats(M, N, K) * 4);
  w.counters = reinterpret_cast<int *>(p);
  p += align256((size_t)((N + 15) / 16) * 4);
  w.flags = p;
  return w;
}

// Counter bump with acquire-release semantics at GPU scope; returns the old value.
QL_DEVI int atomic_add_acq_rel_gpu(int *addr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}


// The 24-bit marker: the lowest mantissa bit of a group's x scale G_x.  For 16-bit x, G_x is a power of
// two (that bit is 0); for 24-bit x it is a normal power of two with the bit set, which changes it by
// 2^-23 relative -- below the fp32 rounding of the sums it scales -- so the streaming loops use G_x as
// stored, OR its bits together once per super-block and add the low bytes' share after the loop only
// when the bit turned up.
QL_DEVI float mark_24bit(float gx) { return __uint_as_float(__float_as_uint(gx) | 1u); }
QL_DEVI float unmark(float gx) { return __uint_as_float(__float_as_uint(gx) & ~1u); }

// Whether a group's 16-bit fixed point loses too much: the summed rounding error of its elements,
// x * 2^a - rint(x * 2^a) with a the 16-bit exponent, above 2^-12 of the group's mass outside its
// largest element (all in units of 2^-a).  err and mass are a lane's partial sums; the four lanes
// of a group combine them.
QL_DEVI bool group_needs_24bit(float err, float mass, float amax_scaled) {
  err += __shfl_xor_sync(0xffffffffu, err, 1);
  err += __shfl_xor_sync(0xffffffffu, err, 2);
  mass += __shfl_xor_sync(0xffffffffu, mass, 1);
  mass += __shfl_xor_sync(0xffffffffu, mass, 2);
  return err > (mass - amax_scaled) * (1.f / 4096.f);
}

// x conversion for the int4 M = 1 kernel, NP lanes per 32-element group (1, 2 or 4; lane part p holds
// k = p 32/NP .. (p + 1) 32/NP - 1), 8 NP lanes per super-block: fixed point with the group's max and sum
// (combined over its lanes by shuffles), 16-bit unless some group of the super-block needs 24 bits (then
// the whole super-block is 24-bit), byte split in fragment order into the super-block's block blk
// (shared memory, GEMV_XBLOB bytes): the eight groups' (G_x, G_y), then chunk (j, kind) of group grp at
// [j][kind][grp] of the (hi, mid) region -- the high-byte and middle-byte words of k = 8j + kind +
// {0, 2, 4, 6}, each paired with a zero word so that one 16-byte load gives the B pairs of two MMAs:
// (x, 0) for groups 0-3 (their lanes feed b0), (0, x) for groups 4-7 (b1) -- and, for 24-bit x only,
// the low-byte word paired the same way (8 bytes) in the lo region.  v: the lane's 32/NP bf16; live: the
// lane holds a group (every lane takes part in the shuffles and the vote).  Returns whether the
// super-block is 24-bit.
template <int NP>
QL_DEVI bool gemv_m1_convert_group(const uint4 (&v)[4], bool live, int grp, int part, uint8_t *blk) {
  constexpr int EL = 32 / NP;  // elements a lane
  const int lane = threadIdx.x & 31;
  float xs[EL];
  float amax = 0.f;
#pragma unroll
  for (int q = 0; q < EL / 8; ++q) {
    const uint32_t u[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[8 * q + 2 * i] = bf16_bits_to_f32(u[i]);
      xs[8 * q + 2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
    }
  }
#pragma unroll
  for (int k = 0; k < EL; ++k) amax = fmaxf(amax, fabsf(xs[k]));
#pragma unroll
  for (int o = 1; o < NP; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const int a16 = scale_exponent(amax, 14);  // max |x_int| < 2^15
  const float s16 = exp2i(a16);
  float err = 0.f, mass = 0.f;
#pragma unroll
  for (int k = 0; k < EL; ++k) {
    const float sv = xs[k] * s16;
    err += fabsf(sv - rintf(sv));
    mass += fabsf(sv);
  }
#pragma unroll
  for (int o = 1; o < NP; o <<= 1) {
    err += __shfl_xor_sync(0xffffffffu, err, o);
    mass += __shfl_xor_sync(0xffffffffu, mass, o);
  }
  // 16-bit fixed point loses too much when the summed rounding error is above 2^-12 of the group's mass
  // outside its largest element (all in units of 2^-a16)
  const bool wide = live && err > (mass - amax * s16) * (1.f / 4096.f);
  constexpr uint32_t SEG = 8 * NP == 32 ? 0xffffffffu : (1u << (8 * NP)) - 1u;  // the super-block's lanes
  const bool sb24 = ((__ballot_sync(0xffffffffu, wide) >> (lane & ~(8 * NP - 1))) & SEG) != 0u;
  const int a = sb24 ? scale_exponent(amax, 22) : a16;  // 24-bit: max |x_int| < 2^23
  const float sc = exp2i(a);
  int xi[EL];
  int sum = 0;  // |sum| < 32 * 2^23
#pragma unroll
  for (int k = 0; k < EL; ++k) {
    xi[k] = __float2int_rn(xs[k] * sc);
    sum += xi[k];
  }
#pragma unroll
  for (int o = 1; o < NP; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (!live) return sb24;
  // byte b of a word = the chosen byte of value b: the value's top byte is byte 2 (24-bit) or byte 1
  // (16-bit, no low byte), its middle byte the one below; gathered by byte permutes
  const uint32_t th = sb24 ? 2u : 1u, sel_hi = th | ((4u + th) << 4), sel_mid = (th - 1u) | ((3u + th) << 4);
  auto gather = [](int v0, int v1, int v2, int v3, uint32_t sel) {
    return __byte_perm(__byte_perm((uint32_t)v0, (uint32_t)v1, sel), __byte_perm((uint32_t)v2, (uint32_t)v3, sel),
                       0x5410u);
  };
#pragma unroll
  for (int jj = 0; jj < EL / 8; ++jj)
#pragma unroll
    for (int kind = 0; kind < 2; ++kind) {
      const int j = part * (EL / 8) + jj;
      const int *vv = xi + 8 * jj + kind;  // values k = 8j + kind + {0, 2, 4, 6}
      const uint32_t hi = gather(vv[0], vv[2], vv[4], vv[6], sel_hi), mid = gather(vv[0], vv[2], vv[4], vv[6], sel_mid);
      const uint32_t lo = sb24 ? gather(vv[0], vv[2], vv[4], vv[6], 0x40u) : 0u;
      const int ch = 8 * (2 * j + kind) + grp;  // chunk (j, kind) of group grp
      reinterpret_cast<uint4 *>(blk + GEMV_XB_Q)[ch] = grp < 4 ? make_uint4(hi, 0u, mid, 0u) : make_uint4(0u, hi, 0u, mid);
      if (sb24) reinterpret_cast<uint2 *>(blk + GEMV_XB_L)[ch] = grp < 4 ? make_uint2(lo, 0u) : make_uint2(0u, lo);
    }
  if (part == 0) {  // (G_x, G_y) = (2^-a / 16, -16 X) scaled by (2^v, 2^-v), v = 8 (24-bit) or 0 (16-bit)
    const float vs = sb24 ? 256.f : 1.f, vi = sb24 ? 1.f / 256.f : 1.f, gx = exp2i(-a) * 0.0625f * vs;
    reinterpret_cast<float2 *>(blk)[grp] = make_float2(sb24 ? mark_24bit(gx) : gx, -16.f * (float)sum * vi);
  }
  return sb24;
}

// A byte of a metadata word as a float: 2^23 + b, to be fused into an FMA with -2^23 * step.
QL_DEVI float byte_magic(uint32_t w, int i) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650 | i));
}

QL_DEVI uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
QL_DEVI float4 lds128f(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
QL_DEVI float2 lds64f(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
  return v;
}
QL_DEVI uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
QL_DEVI uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

// Wait for an mbarrier phase, letting the hardware suspend the thread (up to a hint, in ns) instead
// of spinning; bounded like mbar_wait_bounded.
QL_DEVI bool mbar_wait_suspend(uint32_t bar, uint32_t parity, volatile int *abort) {
  const long long t0 = clock64();
  const uint32_t hint = 1000000u;
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (clock64() - t0 > QL_WAIT_LIMIT_CYCLES) {
      atomicOr(&g_ql_status, QL_DEV_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// ACC = C + A * B (first MMA of a chain) and ACC += A * B, with A = u8 codes x 16 and B = the
// high (signed) or low (unsigned) x bytes
#define QL_IMMA0(TB, ACC, C, A0, A1, A2, A3, B0, B1)                                                  \
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8." TB ".s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "  \
      "{%10,%11,%12,%13};"                                                                              \
      : "=r"(ACC[0]), "=r"(ACC[1]), "=r"(ACC[2]), "=r"(ACC[3])                                        \
      : "r"(A0), "r"(A1), "r"(A2), "r"(A3), "r"(B0), "r"(B1), "r"(C[0]), "r"(C[1]), "r"(C[2]), "r"(C[3]))
#define QL_IMMA(TB, ACC, A0, A1, A2, A3, B0, B1)                                                      \
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8." TB ".s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "  \
      "{%0,%1,%2,%3};"                                                                                  \
      : "+r"(ACC[0]), "+r"(ACC[1]), "+r"(ACC[2]), "+r"(ACC[3])                                        \
      : "r"(A0), "r"(A1), "r"(A2), "r"(A3), "r"(B0), "r"(B1))

constexpr int32_t GEMV_ACC0 = 0x4B400000;    // 1.5 * 2^23 as float bits: integer sums below 2^22 read back exactly
constexpr float GEMV_ACC0_F = 12582912.f;

constexpr int GEMV_RING = 4;   // super-blocks in flight per warp
constexpr int GEMV_CTAS_PER_SM = 3;
constexpr int GEMV_WARPS = 4;     // warps per CTA: four 16-row tiles over the same part of K
// a stage of a warp's ring = one super-block of a 16-row tile: its codes (16 rows x 128 B, 128-byte
// swizzle) in the codes ring, its group words in the group-word ring: int4 16 B a row (u16 sc | zc per
// group; the step words come through L1), 4-bit affine 4 (256 / G) B a row ((s, b) bf16 per group)
static_assert(GEMV_XB_Q + 1024 == GEMV_XCOPY && GEMV_XB_L + 512 == GEMV_XBLOB && GEMV_XBLOB % 16 == 0, "x block");
constexpr int GEMV_ZERO_BYTES = 1024;  // zero x chunks at a 128-byte stride, for lanes that feed no x

template <int FMT, int G>
struct M1Layout {
  static constexpr int GM_ROW = FMT == FMT_INT4 ? 16 : 4 * (256 / G);
  static constexpr int GM_STAGE = 16 * GM_ROW;
  static constexpr int XSB_MAX = GM_ROW > 16 ? 20 : 22;  // super-blocks of x a CTA converts and keeps
  static constexpr int CODES_BYTES = GEMV_WARPS * GEMV_RING * 2048;  // 1024-aligned stages
  static constexpr int GMETA_BYTES = GEMV_WARPS * GEMV_RING * GM_STAGE;
  static constexpr uint32_t STAGE_TX = 2048 + GM_STAGE;
  // dynamic shared memory: codes rings, group-word rings, the CTA's x blocks and their 24-bit flags,
  // zero block, mbarriers
  static constexpr int USED = CODES_BYTES + GMETA_BYTES + XSB_MAX * GEMV_XBLOB + 32 + GEMV_ZERO_BYTES +
                              GEMV_WARPS * GEMV_RING * 8 + 1024;
  static_assert(GEMV_CTAS_PER_SM * (USED + 1024) <= 233472, "three CTAs an SM");
  // affine: a request that keeps a third CTA off an SM, so a layer with half as many tile groups as
  // slots spreads over two thirds of the SMs instead of being packed onto half of them
  static constexpr int FLOOR = 233472 / 3;
  static constexpr int SMEM = FMT == FMT_AFFINE && USED < FLOOR ? FLOOR : USED;
};

struct GemvTcParams {
  const uint8_t *codes, *gmeta;  // [N][K/2], group words [N][K/16] (int4) or [N][4K/G]: read directly only
                                 // by the 24-bit tail
  const uint8_t *steps;          // int4: [N][K/256] step words
  const __nv_bfloat16 *bias;     // [N] or NULL
  const __nv_bfloat16 *x;        // [K]
  int64_t N, K;
  int P;           // parts of K: CTA b takes part b % P of tiles 4 (b / P) .. + 3
  float *partial;  // P > 1: [tile][part][16 rows], added by gemv_m1_sum_parts
  __nv_bfloat16 *y;
};

// The low bytes of 24-bit x for one warp of the M = 1 kernel: S G_x 2^-8 D_lo per (row, 32-k slice) of
// every flagged super-block of its range (S = sc ss for int4, the group's s for affine), the weights read
// again from global memory (q0, q1: the code rows of rows r0, r1 at the range's first super-block;
// m0, m1: their group words; st0, st1: int4 step words) and x from the CTA's blocks in shared memory
// (xs: the first block; fl: the blocks' 24-bit flags).  Flagged super-blocks are rare, so this runs out
// of line and leaves the streaming loop's registers alone.  Returns the sums to add for rows r0 and r1
// (the lane's slices 2c, 2c + 1).
template <int FMT, int G>
__device__ __noinline__ float2 gemv_m1_low_bytes(const uint8_t *q0, const uint8_t *q1, const uint8_t *m0,
                                                 const uint8_t *m1, const uint32_t *st0, const uint32_t *st1,
                                                 const uint8_t *xs, const uint8_t *fl, int nsb) {
  constexpr int GM_ROW = M1Layout<FMT, G>::GM_ROW;
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const bool on0 = (g == c), feed = on0 || (g == c + 4);
  const uint2 *xlg = reinterpret_cast<const uint2 *>(xs + GEMV_XB_L) + (on0 ? c : c + 4);
  const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
  float a0 = 0.f, a1 = 0.f;
  for (int i = 0; i < nsb; ++i) {
    if (fl[i] == 0) continue;  // the same for the whole warp
    const uint4 *c0 = reinterpret_cast<const uint4 *>(q0 + (int64_t)i * 128);
    const uint4 *c1 = reinterpret_cast<const uint4 *>(q1 + (int64_t)i * 128);
    const uint4 v00 = __ldg(c0 + c), v01 = __ldg(c0 + c + 4), v10 = __ldg(c1 + c), v11 = __ldg(c1 + c + 4);
    const uint32_t u00[4] = {v00.x, v00.y, v00.z, v00.w}, u01[4] = {v01.x, v01.y, v01.z, v01.w};
    const uint32_t u10[4] = {v10.x, v10.y, v10.z, v10.w}, u11[4] = {v11.x, v11.y, v11.z, v11.w};
    const uint2 *lg = xlg + (int64_t)i * (GEMV_XBLOB / 8);
    int32_t dl[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint2 le = feed ? lg[16 * j] : make_uint2(0u, 0u);      // even k
      const uint2 lo = feed ? lg[16 * j + 8] : make_uint2(0u, 0u);  // odd k
      const uint32_t h00 = u00[j] & 0xF0F0F0F0u, h10 = u10[j] & 0xF0F0F0F0u;
      const uint32_t h01 = u01[j] & 0xF0F0F0F0u, h11 = u11[j] & 0xF0F0F0F0u;
      const uint32_t e00 = (u00[j] << 4) & 0xF0F0F0F0u, e10 = (u10[j] << 4) & 0xF0F0F0F0u;
      const uint32_t e01 = (u01[j] << 4) & 0xF0F0F0F0u, e11 = (u11[j] << 4) & 0xF0F0F0F0u;
      if (j == 0) QL_IMMA0("u8", dl, acc_init, h00, h10, h01, h11, lo.x, lo.y);
      else QL_IMMA("u8", dl, h00, h10, h01, h11, lo.x, lo.y);
      QL_IMMA("u8", dl, e00, e10, e01, e11, le.x, le.y);
    }
    // (G_x, G_y) of groups 2c, 2c + 1; S = sc * ss per row and group
    const float4 Gx = reinterpret_cast<const float4 *>(xs + (int64_t)i * GEMV_XBLOB)[c];
    const float gx0 = unmark(Gx.x) * (1.f / 256.f), gx1 = unmark(Gx.z) * (1.f / 256.f);
    float s0a, s0b, s1a, s1b;  // the scales of slices 2c, 2c + 1 for rows r0, r1
    if constexpr (FMT == FMT_INT4) {
      const uint32_t cm0 = __ldg(reinterpret_cast<const uint32_t *>(m0 + (int64_t)i * GM_ROW) + c);
      const uint32_t cm1 = __ldg(reinterpret_cast<const uint32_t *>(m1 + (int64_t)i * GM_ROW) + c);
      const float ss0 = f16_bits_to_f32(__ldg(st0 + i)), ss1 = f16_bits_to_f32(__ldg(st1 + i));
      s0a = fmaf(byte_magic(cm0, 0), ss0, -8388608.f * ss0);
      s0b = fmaf(byte_magic(cm0, 2), ss0, -8388608.f * ss0);
      s1a = fmaf(byte_magic(cm1, 0), ss1, -8388608.f * ss1);
      s1b = fmaf(byte_magic(cm1, 2), ss1, -8388608.f * ss1);
    } else {  // slice 2c + h lies in group (2c + h) * 32 / G
      const uint32_t *w0 = reinterpret_cast<const uint32_t *>(m0 + (int64_t)i * GM_ROW);
      const uint32_t *w1 = reinterpret_cast<const uint32_t *>(m1 + (int64_t)i * GM_ROW);
      s0a = bf16_bits_to_f32(__ldg(w0 + 2 * c * 32 / G));
      s0b = bf16_bits_to_f32(__ldg(w0 + (2 * c + 1) * 32 / G));
      s1a = bf16_bits_to_f32(__ldg(w1 + 2 * c * 32 / G));
      s1b = bf16_bits_to_f32(__ldg(w1 + (2 * c + 1) * 32 / G));
    }
    a0 = fmaf(s0a * gx0, __int_as_float(dl[0]) - GEMV_ACC0_F, a0);
    a0 = fmaf(s0b * gx1, __int_as_float(dl[1]) - GEMV_ACC0_F, a0);
    a1 = fmaf(s1a * gx0, __int_as_float(dl[2]) - GEMV_ACC0_F, a1);
    a1 = fmaf(s1b * gx1, __int_as_float(dl[3]) - GEMV_ACC0_F, a1);
  }
  return make_float2(a0, a1);
}

// One CTA = four 16-row tiles over the same part of K.  After the grid it depends on has finished,
// its warps convert the part's x (GEMV_XSB_MAX super-blocks at most) into shared memory once for all
// four tiles -- no separate pass, no hand-over between kernels -- while the first stages of the weights,
// started before that wait, are in flight.  The weights of a super-block arrive by one stage of a
// per-warp ring: the codes box (TMA, 128-byte swizzle: 16-byte chunk j of row r at chunk j ^ (r & 7))
// and the group words box (TMA), both completing on the stage's mbarrier.  MMA row g (and g + 8) reads
// tile row pg = (g >> 1) | ((g & 1) << 2), so the two rows of one 8-lane shared-load phase differ in
// bit 2 and their chunks never share banks.  The loop runs RING super-blocks per turn so every
// shared-memory offset inside a stage is a constant; step words come through the L1 cache RING - 1
// super-blocks ahead.  With K split (P > 1), each part's row sums go to the workspace and a small
// dependent kernel adds them in part order, so the result does not depend on timing.
template <int FMT, int G>
__device__ __forceinline__ void gemv_m1_body(const CUtensorMap &map_codes, const CUtensorMap &map_gmeta,
                                             const GemvTcParams &p) {
  using L = M1Layout<FMT, G>;
  constexpr int GM_ROW = L::GM_ROW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *gm_ring = smem + L::CODES_BYTES;
  uint8_t *xblk = gm_ring + L::GMETA_BYTES;                 // [XSB_MAX][GEMV_XBLOB]
  uint8_t *xflag = xblk + L::XSB_MAX * GEMV_XBLOB;          // [XSB_MAX]
  uint8_t *zero_blk = xflag + 32;
  uint64_t *bars = reinterpret_cast<uint64_t *>(zero_blk + GEMV_ZERO_BYTES);
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles = (p.N + 15) / 16;
  const int P = p.P;
  const int part = (int)(blockIdx.x % (unsigned)P);
  const int64_t tile = (int64_t)(blockIdx.x / (unsigned)P) * GEMV_WARPS + warp;
  const int g = lane >> 2, c = lane & 3;
  const bool active = tile < n_tiles;  // warps past the last tile stream nothing
  const int NS = (int)(p.K / 256);
  const int sb0 = part * NS / P, nsb = (part + 1) * NS / P - sb0;  // the CTA's part of K
  const int nsw = active ? nsb : 0;                                // super-blocks this warp streams
  const uint32_t cring = smem_u32(smem + warp * GEMV_RING * 2048);
  const uint32_t gring = smem_u32(gm_ring + warp * GEMV_RING * L::GM_STAGE);
  const uint32_t bar0 = smem_u32(bars + warp * GEMV_RING);
  if (threadIdx.x == 0) abort_flag = 0;
  for (int t = threadIdx.x; t < GEMV_ZERO_BYTES / 16; t += blockDim.x)
    reinterpret_cast<uint4 *>(zero_blk)[t] = make_uint4(0u, 0u, 0u, 0u);
  if (lane == 0) {
    for (int s = 0; s < GEMV_RING; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the next call's kernel may be scheduled as this grid's CTAs retire; it waits for this grid to
  // finish before it reads x
  pdl_launch_dependents();
  // stage s of super-block i: weights only (codes, group words), independent of x
  auto issue_w = [&](int i, int s) {
    const uint32_t bar = bar0 + 8 * s;
    mbar_arrive_expect_tx(bar, L::STAGE_TX);
    tma_load_2d(cring + s * 2048, &map_codes, bar, (sb0 + i) * 128, (int32_t)(tile * 16));
    tma_load_2d(gring + s * L::GM_STAGE, &map_gmeta, bar, (sb0 + i) * GM_ROW, (int32_t)(tile * 16));
  };
  const int nis = copies_withheld() ? 0 : nsw;  // super-blocks whose copies this warp starts
  const int pre = nis < GEMV_RING - 1 ? nis : GEMV_RING - 1;
  int issued = pre;  // super-blocks whose stage copies were started (lane 0's count is the one used)
  if (lane == 0) {
    tma_prefetch_desc(&map_codes);
    tma_prefetch_desc(&map_gmeta);
    for (int i = 0; i < pre; ++i) issue_w(i, i);
  }
  const int pg = (g >> 1) | ((g & 1) << 2);
  int64_t r0 = tile * 16 + pg, r1 = r0 + 8;
  if (r0 >= p.N) r0 = p.N - 1;  // rows past the end are computed on a valid row and discarded
  if (r1 >= p.N) r1 = p.N - 1;
  const uint32_t *st0 = reinterpret_cast<const uint32_t *>(p.steps) + r0 * NS + sb0;
  const uint32_t *st1 = reinterpret_cast<const uint32_t *>(p.steps) + r1 * NS + sb0;
  uint32_t sr0[GEMV_RING], sr1[GEMV_RING];  // int4 step words of the next RING - 1 super-blocks, by stage
#pragma unroll
  for (int s = 0; s < GEMV_RING; ++s) {
    sr0[s] = 0u;
    sr1[s] = 0u;
    if (FMT == FMT_INT4 && s < pre) {
      sr0[s] = __ldg(st0 + s);
      sr1[s] = __ldg(st1 + s);
    }
  }
  // x of the part: its first 128 groups one a thread, the rest (at most 8 * XSB_MAX - 128) two or four
  // lanes a group, so that the second pass is as short as the first allows
  static_assert(8 * L::XSB_MAX <= 2 * 32 * GEMV_WARPS, "two passes");
  const int ng = 8 * nsb, rest = ng - 32 * GEMV_WARPS;
  const int np = rest <= 0 ? 0 : rest <= 8 * GEMV_WARPS ? 4 : rest <= 16 * GEMV_WARPS ? 2 : 1;  // lanes a group
  const uint4 *xg = reinterpret_cast<const uint4 *>(p.x + (int64_t)sb0 * 256);
  const int q1 = (int)threadIdx.x;                                          // pass 1: group q1
  const int q2 = 32 * GEMV_WARPS + (np ? (int)threadIdx.x / np : 0);        // pass 2: group q2,
  const int part2 = np ? (int)threadIdx.x % np : 0, per2 = np ? 4 / np : 0;  // part part2 of it
  if (q1 < ng) prefetch_l2(xg + 4 * q1);
  if (np && q2 < ng) prefetch_l2(xg + 4 * q2);
  pdl_wait();  // x may be the output of the kernel launched before this one
  {
    uint4 v1[4], v2[4];  // both passes' loads in flight before either converts
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v1[e] = q1 < ng ? __ldg(xg + 4 * q1 + e) : make_uint4(0u, 0u, 0u, 0u);
      v2[e] = np && q2 < ng && e < per2 ? __ldg(xg + 4 * q2 + part2 * per2 + e) : make_uint4(0u, 0u, 0u, 0u);
    }
    {
      const bool live = q1 < ng;
      const bool sb24 = gemv_m1_convert_group<1>(v1, live, q1 & 7, 0, xblk + (live ? q1 >> 3 : 0) * GEMV_XBLOB);
      if (live && (q1 & 7) == 0) xflag[q1 >> 3] = sb24 ? 1 : 0;
    }
    if (np) {  // the same for the whole CTA
      const bool live = q2 < ng;
      uint8_t *blk = xblk + (live ? q2 >> 3 : 0) * GEMV_XBLOB;
      const bool sb24 = np == 4   ? gemv_m1_convert_group<4>(v2, live, q2 & 7, part2, blk)
                        : np == 2 ? gemv_m1_convert_group<2>(v2, live, q2 & 7, part2, blk)
                                  : gemv_m1_convert_group<1>(v2, live, q2 & 7, part2, blk);
      if (live && (q2 & 7) == 0 && part2 == 0) xflag[q2 >> 3] = sb24 ? 1 : 0;
    }
  }
  __syncthreads();  // the part's x blocks are complete

  // per-lane shared-memory addresses (offsets inside a stage are added as constants)
  const bool on0 = (g == c), on1 = (g == c + 4);
  const uint32_t xs0 = smem_u32(xblk);
  const uint32_t xa0 = on0 ? xs0 + GEMV_XB_Q + 16 * c : on1 ? xs0 + GEMV_XB_Q + 16 * (c + 4) : smem_u32(zero_blk);
  const uint32_t xstep = (on0 || on1) ? GEMV_XBLOB : 0u;  // lanes that feed no x read the zero block
  const uint32_t a00 = cring + pg * 128 + ((c ^ pg) << 4), a01 = cring + pg * 128 + (((c + 4) ^ pg) << 4);
  const uint32_t a10 = a00 + 1024, a11 = a01 + 1024;  // row pg + 8: same swizzle phase, next atom
  // group words of the lane's slices 2c, 2c + 1: int4 the u16 pair at 4c; affine group (2c) * 32 / G
  const uint32_t am = gring + pg * GM_ROW + (FMT == FMT_INT4 ? 4 * c : 4 * (2 * c * 32 / G));
  const uint32_t ag = xs0 + 16 * c;

  const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
  float acc0 = 0.f, acc1 = 0.f;
  uint32_t x24s = 0u;  // bit 0: some super-block's G_x carries the 24-bit marker
  bool ok = true;
  for (int base = 0; base < nsw && ok; base += GEMV_RING) {
    const uint32_t par = (uint32_t)((base / GEMV_RING) & 1);
    const uint32_t xt = xa0 + (uint32_t)base * xstep, gt = ag + (uint32_t)base * GEMV_XBLOB;
#pragma unroll
    for (int s = 0; s < GEMV_RING; ++s) {
      const int i = base + s;
      if (i >= nsw) break;
      // refill the stage released by the previous super-block with super-block i + RING - 1
      const int nx = i + GEMV_RING - 1;
      const int sn = (s + GEMV_RING - 1) % GEMV_RING;
      __syncwarp();  // every lane has read that stage in the previous turn
      if (nx < nis) {
        if (lane == 0) {
          issue_w(nx, sn);
          issued = nx + 1;
        }
        if constexpr (FMT == FMT_INT4) {
          sr0[sn] = __ldg(st0 + nx);
          sr1[sn] = __ldg(st1 + nx);
        }
      }
      if (!mbar_wait_suspend(bar0 + 8 * s, par, &abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t so = s * 2048, sg = s * L::GM_STAGE;
      const uint4 w00 = lds128(a00 + so), w10 = lds128(a10 + so);  // (r0 | r1, group c)
      const uint4 w01 = lds128(a01 + so), w11 = lds128(a11 + so);  // (r0 | r1, group c+4)
      const float4 Gx = lds128f(gt + s * GEMV_XBLOB);              // (G_x, G_y) of groups 2c, 2c+1
      // group words of rows r0, r1 (row r1 = pg + 8): int4 one word; affine group 64 one, group 32 two
      uint32_t cm0, cm1, cn0 = 0u, cn1 = 0u;
      if constexpr (FMT == FMT_INT4 || G == 64) {
        cm0 = lds32(am + sg);
        cm1 = lds32(am + sg + 8 * GM_ROW);
      } else {
        const uint2 u0 = lds64(am + sg), u1 = lds64(am + sg + 8 * GM_ROW);
        cm0 = u0.x, cn0 = u0.y, cm1 = u1.x, cn1 = u1.y;
      }
      const uint32_t xi = xt + (uint32_t)s * xstep;
      const uint32_t ww00[4] = {w00.x, w00.y, w00.z, w00.w}, ww01[4] = {w01.x, w01.y, w01.z, w01.w};
      const uint32_t ww10[4] = {w10.x, w10.y, w10.z, w10.w}, ww11[4] = {w11.x, w11.y, w11.z, w11.w};
      // D[q]: q = 0 (r0, group 2c), 1 (r0, 2c+1), 2 (r1, 2c), 3 (r1, 2c+1); T = 256 D_hi + D_mid
      int32_t dh[4], dm[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 xe = lds128(xi + 256 * j), xo = lds128(xi + 256 * j + 128);  // even k, odd k
        const uint32_t h00 = ww00[j] & 0xF0F0F0F0u, h10 = ww10[j] & 0xF0F0F0F0u;  // odd k, x16
        const uint32_t h01 = ww01[j] & 0xF0F0F0F0u, h11 = ww11[j] & 0xF0F0F0F0u;
        if (j == 0) {
          QL_IMMA0("s8", dh, acc_init, h00, h10, h01, h11, xo.x, xo.y);
          QL_IMMA0("u8", dm, acc_init, h00, h10, h01, h11, xo.z, xo.w);
        } else {
          QL_IMMA("s8", dh, h00, h10, h01, h11, xo.x, xo.y);
          QL_IMMA("u8", dm, h00, h10, h01, h11, xo.z, xo.w);
        }
        const uint32_t e00 = (ww00[j] << 4) & 0xF0F0F0F0u, e10 = (ww10[j] << 4) & 0xF0F0F0F0u;  // even k, x16
        const uint32_t e01 = (ww01[j] << 4) & 0xF0F0F0F0u, e11 = (ww11[j] << 4) & 0xF0F0F0F0u;
        QL_IMMA("s8", dh, e00, e10, e01, e11, xe.x, xe.y);
        QL_IMMA("u8", dm, e00, e10, e01, e11, xe.z, xe.w);
      }
      float t[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        t[q] = fmaf(__int_as_float(dh[q]) - GEMV_ACC0_F, 256.f, __int_as_float(dm[q]) - GEMV_ACC0_F);
      x24s |= __float_as_uint(Gx.x);
      if constexpr (FMT == FMT_INT4) {
        // S = sc * ss and Z = zc * zs, each one FMA from the byte placed in the mantissa of 2^23
        const uint32_t cs0 = sr0[s], cs1 = sr1[s];
        const float ss0 = f16_bits_to_f32(cs0), zs0 = f16_bits_to_f32(cs0 >> 16);
        const float ss1 = f16_bits_to_f32(cs1), zs1 = f16_bits_to_f32(cs1 >> 16);
        const float nss0 = -8388608.f * ss0, nzs0 = -8388608.f * zs0;
        const float nss1 = -8388608.f * ss1, nzs1 = -8388608.f * zs1;
        const float S00 = fmaf(byte_magic(cm0, 0), ss0, nss0) * Gx.x, Z00 = fmaf(byte_magic(cm0, 1), zs0, nzs0);
        const float S01 = fmaf(byte_magic(cm0, 2), ss0, nss0) * Gx.z, Z01 = fmaf(byte_magic(cm0, 3), zs0, nzs0);
        const float S10 = fmaf(byte_magic(cm1, 0), ss1, nss1) * Gx.x, Z10 = fmaf(byte_magic(cm1, 1), zs1, nzs1);
        const float S11 = fmaf(byte_magic(cm1, 2), ss1, nss1) * Gx.z, Z11 = fmaf(byte_magic(cm1, 3), zs1, nzs1);
        acc0 = fmaf(S00, fmaf(Z00, Gx.y, t[0]), acc0);
        acc0 = fmaf(S01, fmaf(Z01, Gx.w, t[1]), acc0);
        acc1 = fmaf(S10, fmaf(Z10, Gx.y, t[2]), acc1);
        acc1 = fmaf(S11, fmaf(Z11, Gx.w, t[3]), acc1);
      } else {  // w = q s + b: s G_x T + b 2^-a X, with b 2^-a X = -b G_x G_y
        const uint32_t wa0 = cm0, wb0 = G == 64 ? cm0 : cn0, wa1 = cm1, wb1 = G == 64 ? cm1 : cn1;
        const float ga0 = bf16_bits_to_f32(wa0) * Gx.x, gb0 = bf16_bits_to_f32(wb0) * Gx.z;
        const float ga1 = bf16_bits_to_f32(wa1) * Gx.x, gb1 = bf16_bits_to_f32(wb1) * Gx.z;
        acc0 = fmaf(ga0, t[0], fmaf(-bf16_bits_to_f32(wa0 >> 16) * Gx.x, Gx.y, acc0));
        acc0 = fmaf(gb0, t[1], fmaf(-bf16_bits_to_f32(wb0 >> 16) * Gx.z, Gx.w, acc0));
        acc1 = fmaf(ga1, t[2], fmaf(-bf16_bits_to_f32(wa1 >> 16) * Gx.x, Gx.y, acc1));
        acc1 = fmaf(gb1, t[3], fmaf(-bf16_bits_to_f32(wb1 >> 16) * Gx.z, Gx.w, acc1));
      }
    }
  }
  if (!ok && lane == 0) {  // a wait gave up: let this warp's copies in flight land first
    for (int i = issued - GEMV_RING; i < issued; ++i) {
      if (i < 0) continue;
      const long long t0 = clock64();
      while (!mbar_try_wait(bar0 + 8 * (i % GEMV_RING), (uint32_t)((i / GEMV_RING) & 1)) &&
             clock64() - t0 < QL_WAIT_LIMIT_CYCLES) {
      }
    }
  }
  if (__any_sync(0xffffffffu, (x24s & 1u) != 0u) && ok) {  // rare
    const int64_t gm_stride = p.K / 256 * GM_ROW;  // group-word bytes a row
    const float2 lb = gemv_m1_low_bytes<FMT, G>(p.codes + r0 * (p.K / 2) + (int64_t)sb0 * 128,
                                                p.codes + r1 * (p.K / 2) + (int64_t)sb0 * 128,
                                                p.gmeta + r0 * gm_stride + (int64_t)sb0 * GM_ROW,
                                                p.gmeta + r1 * gm_stride + (int64_t)sb0 * GM_ROW, st0, st1, xblk,
                                                xflag, nsw);
    acc0 += lb.x;
    acc1 += lb.y;
  }
  // the four lanes of a row hold its groups 2c, 2c+1: sum them
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
  if (P == 1) {
    if (active && ok && c == 0) {
      const int64_t ra = tile * 16 + pg, rb = ra + 8;
      if (ra < p.N) p.y[ra] = __float2bfloat16_rn(acc0 + bias_at(p.bias, ra));
      if (rb < p.N) p.y[rb] = __float2bfloat16_rn(acc1 + bias_at(p.bias, rb));
    }
    return;
  }
  // K split: this part's sums of the tile's rows go to the workspace; gemv_m1_sum_parts, the dependent
  // launch after this grid, adds the P parts in part order
  if (!active) return;
  {  // lane r < 16 stores the sum of tile row r (held by lane 4g with pg(g) = r mod 8)
    const int rr = lane & 15, prow = rr & 7;
    const int src = 4 * (((prow & 3) << 1) | (prow >> 2));
    const float v0 = __shfl_sync(0xffffffffu, acc0, src), v1 = __shfl_sync(0xffffffffu, acc1, src);
    if (lane < 16) p.partial[(tile * P + part) * 16 + rr] = rr < 8 ? v0 : v1;
  }
}

// The parts of a K split of the M = 1 kernel, added in part order: one thread per output row.  Launched
// as a programmatic dependent of that kernel (it lets the next kernel start, then waits for the parts).
__global__ void __launch_bounds__(256) gemv_m1_sum_parts(const float *partial, int P, int64_t N,
                                                         const __nv_bfloat16 *bias, __nv_bfloat16 *y) {
  pdl_launch_dependents();
  const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  pdl_wait();
  if (r >= N) return;
  const float *src = partial + (r >> 4) * P * 16 + (r & 15);
  float sum = 0.f;
  for (int q = 0; q < P; ++q) sum += src[q * 16];
  y[r] = __float2bfloat16_rn(sum + bias_at(bias, r));
}

// int4 (nested superscale) at M = 1
__global__ void __launch_bounds__(32 * GEMV_WARPS, GEMV_CTAS_PER_SM)
    gemv_int4_m1_tc_kernel(const __grid_constant__ CUtensorMap map_codes,
                           const __grid_constant__ CUtensorMap map_gmeta, GemvTcParams p) {
  gemv_m1_body<FMT_INT4, 32>(map_codes, map_gmeta, p);
}

// 4-bit affine (group G = 32 or 64) at M = 1: the same nibble layout, (s, b) per group
template <int G>
__global__ void __launch_bounds__(32 * GEMV_WARPS, GEMV_CTAS_PER_SM)
    gemv_affine4_m1_tc_kernel(const __grid_constant__ CUtensorMap map_codes,
                              const __grid_constant__ CUtensorMap map_gmeta, GemvTcParams p) {
  gemv_m1_body<FMT_AFFINE, G>(map_codes, map_gmeta, p);
}


// ===========================================================================
// Tensor-core decode GEMV with the tokens as MMA columns: int4 at 2 <= M <= 8, and 2-, 4- and 8-bit
// affine (group 32 or 64) at 1 <= M <= 8.
//
// The same integer MMA (m16n8k32, u8 codes x16 against the high / low bytes of
// 16-bit fixed-point x) with the 8 MMA columns as the tokens (a dense B):
// one MMA pair per (16 rows, 32-weight group) covers every token, so D is the
// group partial of 16 rows x 8 tokens and the scale and zero are applied per
// (row, token, group).  Lane (g, c) supplies code word c of the group for tile
// rows g and g + 8 (even-k codes to slots 4c.., odd-k codes to slots 4c+16..)
// and, as column g, token g's x bytes of those slots; it ends with the sums of
// rows g, g + 8 for tokens 2c, 2c + 1.
//
// x is 16- or 24-bit fixed point per (token, group) as in the M = 1 kernel
// (high, middle and, for 24-bit super-blocks, low byte: one MMA each).  A CTA is one producer warp and four consumer warps on 64 weight rows (four
// 16-row tiles) and a range of super-blocks: each stage (codes box, group-word
// box, every token's x words and group sums) is fetched once and read by all
// four.  When the row groups alone do not fill one wave of GEMV_MT_CTAS_PER_SM
// CTAs per SM, K is split over P CTAs per row group; each writes its sums to the
// workspace and the CTA that finds the others done (a counter per row group,
// cleared by the preparation pass) adds the P parts in part order and writes y.
// ===========================================================================

// x preparation for M > 1: 4 lanes per (token, 32-element group), so one warp holds one token's
// eight groups of a super-block; 16-bit fixed point unless some group of them needs 24 bits (then
// all eight are 24-bit and the token's flag byte of the super-block is set).  Lane c owns
// k = 8c .. 8c + 7 and writes its MMA word quad (even-k high bytes, odd-k high bytes, even-k middle
// bytes, odd-k middle bytes) and word pair (even-k low bytes, odd-k low bytes; zero for 16-bit).
__global__ void __launch_bounds__(256) gemv_xprep_mt_kernel(const __nv_bfloat16 *x, int64_t M, int64_t K,
                                                            int64_t n_counters, GemvWorkspace ws) {
  pdl_launch_dependents();  // the streaming kernel may start fetching weights now
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t ng = K / 32;
  const int64_t gq = t >> 2;  // (token, group), token-major
  const int c = (int)(t & 3);
  const bool live = gq < M * ng;  // every lane takes part in the shuffles
  const int64_t m = live ? gq / ng : 0, g = live ? gq - m * ng : 0;
  if (live) prefetch_l2(x + m * K + 32 * g + 8 * c);
  pdl_wait();               // x (and this workspace) may belong to the kernel launched before this one
  if (t < n_counters) ws.counters[t] = 0;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (live) v = __ldg(reinterpret_cast<const uint4 *>(x + m * K + 32 * g + 8 * c));
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  float xs[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xs[2 * i] = bf16_bits_to_f32(u[i]);
    xs[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
    amax = fmaxf(amax, fmaxf(fabsf(xs[2 * i]), fabsf(xs[2 * i + 1])));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  const int a16 = scale_exponent(amax, 14);  // max |x_int| < 2^15
  const float s16 = exp2i(a16);
  float err = 0.f, mass = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float sv = xs[k] * s16;
    err += fabsf(sv - rintf(sv));
    mass += fabsf(sv);
  }
  const bool wide = group_needs_24bit(err, mass, amax * s16);
  const bool sb24 = __any_sync(0xffffffffu, wide && live);  // the warp holds one (token, super-block)
  const int a = sb24 ? scale_exponent(amax, 22) : a16;     // 24-bit: max |x_int| < 2^23
  const float sc = exp2i(a);
  const int hs = sb24 ? 16 : 8;  // the value's top byte: bits 16.. (24-bit) or 8.. (16-bit, lo = 0)
  uint32_t eh = 0, oh = 0, em = 0, om = 0, el = 0, ol = 0;
  int sum = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int xe = __float2int_rn(xs[2 * b] * sc), xo = __float2int_rn(xs[2 * b + 1] * sc);
    sum += xe + xo;
    eh |= ((uint32_t)(xe >> hs) & 0xffu) << (8 * b);
    em |= ((uint32_t)(xe >> (hs - 8)) & 0xffu) << (8 * b);
    el |= ((uint32_t)xe & 0xffu) << (8 * b);
    oh |= ((uint32_t)(xo >> hs) & 0xffu) << (8 * b);
    om |= ((uint32_t)(xo >> (hs - 8)) & 0xffu) << (8 * b);
    ol |= ((uint32_t)xo & 0xffu) << (8 * b);
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  if (!live) return;
  ws.xq[(g * M + m) * 4 + c] = make_uint4(eh, oh, em, om);
  if (sb24) reinterpret_cast<uint2 *>(ws.xq + M * K / 8)[(g * M + m) * 4 + c] = make_uint2(el, ol);
  if (c == 0) {  // (G_x, G_y) = (2^-a / 16, -16 X) scaled by (2^v, 2^-v), v = 8 (24-bit) or 0 (16-bit)
    const float v = sb24 ? 256.f : 1.f, vi = sb24 ? 1.f / 256.f : 1.f, gx = exp2i(-a) * 0.0625f * v;
    ws.gsum[g * M + m] = make_float2(sb24 ? mark_24bit(gx) : gx, -16.f * (float)sum * vi);
  }
  if ((threadIdx.x & 31) == 0) ws.flags[(g >> 3) * 16 + m] = sb24 ? 1 : 0;
}

constexpr int GEMV_MT_WARPS = 4;  // consumer warps per CTA; warp 4 produces
constexpr int GEMV_MT_THREADS = 32 * (GEMV_MT_WARPS + 1);
// int4: three CTAs an SM, so at most 128 registers a thread (an SM partition's 16K registers hold four
// of their warps).  Affine: two CTAs an SM with up to GEMV_MT_AFFINE_NREG registers a thread (three
// warps a partition) -- at the row counts it serves its per-CTA rate, not the CTA count, bounds it,
// and the extra registers raise that rate.
constexpr int GEMV_MT_CTAS_PER_SM = 3;
constexpr int GEMV_MT_AFFINE_CTAS_PER_SM = 2;
#define GEMV_MT_AFFINE_NREG 168
// the warps of the resident CTAs spread over an SM's four partitions of 16K registers each
static_assert(((GEMV_MT_AFFINE_CTAS_PER_SM * GEMV_MT_THREADS / 32 + 3) / 4) * 32 * GEMV_MT_AFFINE_NREG <= 16384 &&
                  ((GEMV_MT_CTAS_PER_SM * GEMV_MT_THREADS / 32 + 3) / 4) * 32 * 128 <= 16384,
              "register budgets of the multi-token kernels");
template <int FMT>
constexpr int gemv_mt_ctas_per_sm() { return FMT == FMT_INT4 ? GEMV_MT_CTAS_PER_SM : GEMV_MT_AFFINE_CTAS_PER_SM; }

// Stage layout of the multi-token kernel per format, for one 256-weight super-block of 64 rows:
// codes [64 rows][CODE_ROW B] as swizzled boxes of CODE_BOX B (128-byte swizzle; 64-byte swizzle for
// the 64-byte rows of 2-bit codes), group words [64][META_ROW B], group sums [8][M][8 B], (hi, mid) x
// words [8 groups][M][4][16 B].  A 24-bit super-block's lo x words are read from global memory.  int4 and 4-bit affine codes share one layout (a nibble per weight, low
// nibble first); 8-bit affine codes are bytes; 2-bit codes are 16 per word, lowest bits first.
template <int FMT, int BITS, int G>
struct MtLayout {
  static constexpr int CODE_ROW = FMT == FMT_INT4 ? 128 : 256 * BITS / 8;
  static constexpr int CODE_BOX = CODE_ROW < 128 ? CODE_ROW : 128;
  static constexpr int CODE_BOXES = CODE_ROW / CODE_BOX;
  static constexpr int META_ROW = FMT == FMT_INT4 ? 16 : 4 * (256 / G);  // int4: 8 x u16; affine: 256/G x u32
  static constexpr int ST_GMETA = CODE_BOXES * 64 * CODE_BOX;
  static constexpr int ST_GSUM = ST_GMETA + 64 * META_ROW;
  static constexpr int ST_X = ST_GSUM + 512;
  static constexpr int STAGE = (ST_X + 4096 + 1023) / 1024 * 1024;
  // CTAs an SM holds (gemv_mt_ctas_per_sm) and the deepest ring (up to 4 stages for int4, 6 for affine)
  // with which they share its 228 KB of shared memory (1 KB of it reserved per CTA)
  static constexpr int CTAS = FMT == FMT_INT4 ? GEMV_MT_CTAS_PER_SM : GEMV_MT_AFFINE_CTAS_PER_SM;
  static constexpr int PER_CTA = 233472 / CTAS - 1024 - (1024 + 6 * 16 + 16);
  static constexpr int RING = (FMT == FMT_INT4 ? 4 : 6) < PER_CTA / STAGE ? (FMT == FMT_INT4 ? 4 : 6) : PER_CTA / STAGE;
  static constexpr int USED = RING * STAGE + RING * 16 + 16 + 1024;  // stages, barriers, flags, alignment
  // affine: the request also keeps a CTAS + 1-th CTA off the SM, so the row groups spread over more SMs
  static constexpr int FLOOR = FMT == FMT_INT4 ? 0 : 233472 / (CTAS + 1);
  static constexpr int SMEM = USED > FLOOR ? USED : FLOOR;
  static_assert(RING >= 3 && CTAS * (SMEM + 1024) <= 233472 && (CTAS + 1) * (SMEM + 1024) > 233472 || FMT == FMT_INT4,
                "affine ring and occupancy");
};

struct GemvMtParams {
  const uint8_t *codes, *gmeta;  // read directly only by the 24-bit tail
  const uint8_t *steps;       // int4 step words; unused for affine
  const __nv_bfloat16 *bias;  // [N] or NULL
  int64_t N, K;
  int M;  // 1 .. 8 tokens (int4: 2 .. 8)
  SplitK split;  // of K over the CTAs of the grid, per 64-row group
  GemvWorkspace ws;
  __nv_bfloat16 *y;
};

template <int FMT, int BITS, int G>
inline constexpr int gemv_mt_smem_bytes() { return MtLayout<FMT, BITS, G>::SMEM; }

// The low bytes of 24-bit x for one consumer warp of the multi-token kernel: S G_x 2^-8 D_lo per (row,
// token, 32-weight group) of every super-block of the range [sb0, sb0 + nsb) in which some token's x
// is 24-bit, the weights read again from global memory (rows c0, c1; rows past N read row N - 1 and
// their sums are never stored).  Flagged super-blocks are rare, so this runs out of line and leaves
// the streaming loop's registers alone.  Returns the sums to add for (row g | g + 8) x (token 2c |
// 2c + 1).
template <int FMT, int BITS, int G>
__device__ __noinline__ float4 gemv_mt_low_bytes(const uint8_t *codes, const uint8_t *gmeta, int64_t c0, int64_t c1,
                                                 const uint32_t *st0, const uint32_t *st1, const uint8_t *flags,
                                                 const float2 *gsum, const uint2 *xlg, int64_t K, int M, int sb0,
                                                 int nsb) {
  using L = MtLayout<FMT, BITS, G>;
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int tk0 = 2 * c, tk1 = 2 * c + 1;
  const uint64_t fmask = M >= 8 ? ~0ull : ((1ull << (8 * M)) - 1);  // the flag bytes of tokens < M
  const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
  constexpr int64_t CB = FMT == FMT_INT4 ? 128 : 32 * BITS;  // code bytes per row and super-block
  constexpr int64_t MB = L::META_ROW;                         // group-word bytes per row and super-block
  constexpr float SF = (FMT == FMT_INT4 || BITS == 4) ? 1.f : 16.f;
  const uint8_t *q0 = codes + c0 * (K / 256) * CB, *q1 = codes + c1 * (K / 256) * CB;
  const uint8_t *g0 = gmeta + c0 * (K / 256) * MB, *g1 = gmeta + c1 * (K / 256) * MB;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < nsb; ++i) {
    const int64_t sb = sb0 + i;
    const uint2 fw = __ldg(reinterpret_cast<const uint2 *>(flags + sb * 16));
    const uint64_t f24 = ((uint64_t)fw.y << 32 | fw.x) & fmask;
    if (f24 == 0) continue;  // the same for the whole warp
    const bool mine24 = g < M && ((f24 >> (8 * g)) & 0xffu) != 0;  // token g: this lane's column
    float ss0 = 0.f, ss1 = 0.f;
    if constexpr (FMT == FMT_INT4) {
      ss0 = f16_bits_to_f32(__ldg(st0 + i));
      ss1 = f16_bits_to_f32(__ldg(st1 + i));
    }
#pragma unroll 1
    for (int gg = 0; gg < 8; ++gg) {
      uint32_t e0, e1, o0, o1;  // as in the streaming loop, from the unswizzled rows
      if constexpr (FMT == FMT_INT4 || BITS == 4) {
        const uint32_t w0 = __ldg(reinterpret_cast<const uint32_t *>(q0 + sb * CB + 16 * gg + 4 * c));
        const uint32_t w1 = __ldg(reinterpret_cast<const uint32_t *>(q1 + sb * CB + 16 * gg + 4 * c));
        e0 = (w0 << 4) & 0xF0F0F0F0u; e1 = (w1 << 4) & 0xF0F0F0F0u;
        o0 = w0 & 0xF0F0F0F0u; o1 = w1 & 0xF0F0F0F0u;
      } else if constexpr (BITS == 2) {
        const uint32_t sel = (c & 1) ? 0x4342u : 0x4140u;
        const uint32_t t0 = __byte_perm(__ldg(reinterpret_cast<const uint32_t *>(q0 + sb * CB + 8 * gg + 4 * (c >> 1))), 0u, sel);
        const uint32_t t1 = __byte_perm(__ldg(reinterpret_cast<const uint32_t *>(q1 + sb * CB + 8 * gg + 4 * (c >> 1))), 0u, sel);
        const uint32_t u0 = (t0 | (t0 << 4)) & 0x0F0F0F0Fu, u1 = (t1 | (t1 << 4)) & 0x0F0F0F0Fu;
        e0 = u0 & 0x03030303u; e1 = u1 & 0x03030303u;
        o0 = (u0 >> 2) & 0x03030303u; o1 = (u1 >> 2) & 0x03030303u;
      } else {
        const uint2 w0 = __ldg(reinterpret_cast<const uint2 *>(q0 + sb * CB + 32 * gg + 8 * c));
        const uint2 w1 = __ldg(reinterpret_cast<const uint2 *>(q1 + sb * CB + 32 * gg + 8 * c));
        e0 = __byte_perm(w0.x, w0.y, 0x6420); e1 = __byte_perm(w1.x, w1.y, 0x6420);
        o0 = __byte_perm(w0.x, w0.y, 0x7531); o1 = __byte_perm(w1.x, w1.y, 0x7531);
      }
      const int64_t grp = sb * 8 + gg;
      const uint2 xl = mine24 ? __ldg(xlg + (grp * M + g) * 4 + c) : make_uint2(0u, 0u);
      int32_t dl[4];
      QL_IMMA0("u8", dl, acc_init, e0, e1, o0, o1, xl.x, xl.y);
      const float ga = tk0 < M ? unmark(__ldg(&gsum[grp * M + tk0].x)) * (1.f / 256.f) : 0.f;
      const float gb = tk1 < M ? unmark(__ldg(&gsum[grp * M + tk1].x)) * (1.f / 256.f) : 0.f;
      float S0, S1;
      if constexpr (FMT == FMT_INT4) {
        const int bsc = 2 * (gg & 1);
        S0 = fmaf(byte_magic(__ldg(reinterpret_cast<const uint32_t *>(g0 + sb * MB) + (gg >> 1)), bsc), ss0, -8388608.f * ss0);
        S1 = fmaf(byte_magic(__ldg(reinterpret_cast<const uint32_t *>(g1 + sb * MB) + (gg >> 1)), bsc), ss1, -8388608.f * ss1);
      } else {
        S0 = bf16_bits_to_f32(__ldg(reinterpret_cast<const uint32_t *>(g0 + sb * MB) + gg * 32 / G)) * SF;
        S1 = bf16_bits_to_f32(__ldg(reinterpret_cast<const uint32_t *>(g1 + sb * MB) + gg * 32 / G)) * SF;
      }
      acc.x = fmaf(S0 * ga, __int_as_float(dl[0]) - GEMV_ACC0_F, acc.x);
      acc.y = fmaf(S0 * gb, __int_as_float(dl[1]) - GEMV_ACC0_F, acc.y);
      acc.z = fmaf(S1 * ga, __int_as_float(dl[2]) - GEMV_ACC0_F, acc.z);
      acc.w = fmaf(S1 * gb, __int_as_float(dl[3]) - GEMV_ACC0_F, acc.w);
    }
  }
  return acc;
}

// int4: w = (q - zc zs)(sc ss) with the step word per super-block; affine (2 / 4 / 8 bits, group 32
// or 64): w = q s + b with (s, b) bf16 per group.  Per (row, token, 32-weight slice) the integer MMA
// gives T = sum_k A_k x_int_k with A = 16 q (nibbles) or q (2-bit fields, bytes); then
//   int4:   y += S (2^-a / 16) (T - 16 Z X)
//   affine: y += s' (2^-a / 16) T + b 2^-a X      (s' = s for nibbles, 16 s otherwise)
template <int FMT, int BITS, int G>
__device__ __forceinline__ void gemv_mt_body(const CUtensorMap &map_codes, const CUtensorMap &map_gmeta,
                                             const GemvMtParams &p) {
  using L = MtLayout<FMT, BITS, G>;
  constexpr int RING = L::RING;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + RING * L::STAGE);  // full[R], empty[R]
  int *flags = reinterpret_cast<int *>(bars + 2 * RING);                   // abort, last-part
  volatile int *abort_flag = flags;
  const uint32_t sbase = smem_u32(smem);
  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + RING + s); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = p.M;
  const int NS = (int)(p.K / 256);
  int64_t rg, first;  // 64-row group, index of its first part
  int part, P;        // this CTA is part `part` of the P splitting the group's K
  p.split.locate((int)blockIdx.x, rg, part, P, first);
  const int sb0 = part * NS / P, nsb = (part + 1) * NS / P - sb0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), GEMV_MT_WARPS);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  // the (G_x, G_y) slots of tokens M..7 in every stage: never written by the copies, read (and their
  // sums dropped) by lanes whose tokens are past M; zero, so they carry no 24-bit marker
  if (threadIdx.x < (8 - M) * 16) {
#pragma unroll
    for (int s = 0; s < RING; ++s) reinterpret_cast<uint32_t *>(smem + s * L::STAGE + L::ST_GSUM + M * 64)[threadIdx.x] = 0u;
  }
  __syncthreads();
  pdl_launch_dependents();  // the next call's preparation pass waits for this grid before touching anything

  if (warp == GEMV_MT_WARPS) {  // producer
    if (lane == 0) {
      tma_prefetch_desc(&map_codes);
      tma_prefetch_desc(&map_gmeta);
      const uint32_t tx = L::ST_GSUM + (uint32_t)M * (64 + 512);  // codes, group words, sums, x
      auto issue_w = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
        mbar_arrive_expect_tx(bar_full(s), tx);
#pragma unroll
        for (int bx = 0; bx < L::CODE_BOXES; ++bx)
          tma_load_2d(st + bx * 64 * L::CODE_BOX, &map_codes, bar_full(s), (sb0 + i) * L::CODE_ROW + bx * L::CODE_BOX,
                      (int32_t)(rg * 64));
        tma_load_2d(st + L::ST_GMETA, &map_gmeta, bar_full(s), (sb0 + i) * L::META_ROW, (int32_t)(rg * 64));
      };
      auto issue_x = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
        const int64_t g0 = (int64_t)(sb0 + i) * 8;  // first 32-element group of the super-block
        bulk_load(st + L::ST_GSUM, p.ws.gsum + g0 * M, (uint32_t)M * 64, bar_full(s));
        bulk_load(st + L::ST_X, p.ws.xq + g0 * M * 4, (uint32_t)M * 512, bar_full(s));
      };
      const int nis = copies_withheld() ? 0 : nsb;  // super-blocks whose copies are started
      const int pre = nis < RING ? nis : RING;
      for (int i = 0; i < pre; ++i) issue_w(i, i);  // weights need no x
      pdl_wait();
      for (int i = 0; i < pre; ++i) issue_x(i, i);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int i = pre;
      for (; i < nis; ++i) {  // unit i reuses the stage of unit i - RING
        if (!mbar_wait_bounded(bar_empty(s), ph, abort_flag)) {
          ok = false;
          break;
        }
        issue_w(i, s);
        issue_x(i, s);
        if (++s == RING) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {  // let the copies in flight land before the CTA can exit
        for (int j = i - 1; j >= 0 && j >= i - RING; --j) {
          const long long t0 = clock64();
          while (!mbar_try_wait(bar_full(j % RING), (uint32_t)((j / RING) & 1)) &&
                 clock64() - t0 < QL_WAIT_LIMIT_CYCLES) {
          }
        }
      }
    }
  } else {  // consumers: warp w owns box rows 16w + g and 16w + g + 8
    const int g = lane >> 2, c = lane & 3;
    const int r0 = 16 * warp + g, r1 = r0 + 8;
    int64_t n0 = rg * 64 + r0, n1 = n0 + 8;
    const int64_t c0 = n0 < p.N ? n0 : p.N - 1, c1 = n1 < p.N ? n1 : p.N - 1;
    const uint32_t *st0 = reinterpret_cast<const uint32_t *>(p.steps) + c0 * NS + sb0;
    const uint32_t *st1 = reinterpret_cast<const uint32_t *>(p.steps) + c1 * NS + sb0;
    uint32_t sr0[RING], sr1[RING];  // int4 step words by stage, RING - 1 super-blocks ahead
#pragma unroll
    for (int s = 0; s < RING; ++s) {
      sr0[s] = 0u;
      sr1[s] = 0u;
      if constexpr (FMT == FMT_INT4) {
        if (s < RING - 1 && s < nsb) {
          sr0[s] = __ldg(st0 + s);
          sr1[s] = __ldg(st1 + s);
        }
      }
    }
    const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
    const uint2 *xlg = reinterpret_cast<const uint2 *>(p.ws.xq + (int64_t)M * p.K / 8);  // lo x words
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // (row g | g + 8) x (token 2c | 2c + 1)
    const uint32_t sw = (uint32_t)(r0 & 7);
    uint32_t x24s = 0u;  // bit 0: some super-block's G_x of token 2c or 2c + 1 carries the 24-bit marker
    bool ok = true;
    for (int base = 0; base < nsb && ok; base += RING) {
      const uint32_t par = (uint32_t)((base / RING) & 1);
#pragma unroll
      for (int s = 0; s < RING; ++s) {
        const int i = base + s;
        if (i >= nsb) break;
        if constexpr (FMT == FMT_INT4) {
          const int nx = i + RING - 1, sn = (s + RING - 1) % RING;
          if (nx < nsb) {
            sr0[sn] = __ldg(st0 + nx);
            sr1[sn] = __ldg(st1 + nx);
          }
        }
        if (!mbar_wait_bounded(bar_full(s), par, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t stg = sbase + s * L::STAGE;
        // group words of rows r0, r1 (int4: 8 x u16 sc|zc; affine: 256/G x u32 s|b)
        uint32_t gw0[L::META_ROW / 4], gw1[L::META_ROW / 4];
#pragma unroll
        for (int q = 0; q < L::META_ROW / 16; ++q) {
          const uint4 a = lds128(stg + L::ST_GMETA + r0 * L::META_ROW + 16 * q);
          const uint4 b = lds128(stg + L::ST_GMETA + r1 * L::META_ROW + 16 * q);
          gw0[4 * q] = a.x; gw0[4 * q + 1] = a.y; gw0[4 * q + 2] = a.z; gw0[4 * q + 3] = a.w;
          gw1[4 * q] = b.x; gw1[4 * q + 1] = b.y; gw1[4 * q + 2] = b.z; gw1[4 * q + 3] = b.w;
        }
        float ss0 = 0.f, zs0 = 0.f, ss1 = 0.f, zs1 = 0.f, nss0 = 0.f, nzs0 = 0.f, nss1 = 0.f, nzs1 = 0.f;
        if constexpr (FMT == FMT_INT4) {
          const uint32_t cs0 = sr0[s], cs1 = sr1[s];
          ss0 = f16_bits_to_f32(cs0); zs0 = f16_bits_to_f32(cs0 >> 16);
          ss1 = f16_bits_to_f32(cs1); zs1 = f16_bits_to_f32(cs1 >> 16);
          nss0 = -8388608.f * ss0; nzs0 = -8388608.f * zs0;
          nss1 = -8388608.f * ss1; nzs1 = -8388608.f * zs1;
        }
        // A operand of group gg: even-k and odd-k codes of rows r0, r1 (x16 for nibbles)
        auto codes = [&](int gg, uint32_t &e0, uint32_t &e1, uint32_t &o0, uint32_t &o1) {
          if constexpr (FMT == FMT_INT4 || BITS == 4) {
            const uint32_t coff = (((uint32_t)gg ^ sw) << 4) + 4 * c;
            const uint32_t w0 = lds32(stg + r0 * 128 + coff), w1 = lds32(stg + r1 * 128 + coff);
            e0 = (w0 << 4) & 0xF0F0F0F0u; e1 = (w1 << 4) & 0xF0F0F0F0u;
            o0 = w0 & 0xF0F0F0F0u; o1 = w1 & 0xF0F0F0F0u;
          } else if constexpr (BITS == 2) {
            // 2-bit: slice gg is 8 B of the 64-byte row (64-byte swizzle: 16-byte chunk ^ (row / 2) % 4);
            // lane c takes the half-word of k = 8c .. 8c + 7, spreads its nibbles to bytes (one byte
            // permute, one shift-or) and splits even and odd k with two masks
            const uint32_t off = ((((uint32_t)gg >> 1) ^ (((uint32_t)r0 >> 1) & 3u)) << 4) + 8 * (gg & 1) + 4 * (c >> 1);
            const uint32_t sel = (c & 1) ? 0x4342u : 0x4140u;
            const uint32_t t0 = __byte_perm(lds32(stg + r0 * 64 + off), 0u, sel);
            const uint32_t t1 = __byte_perm(lds32(stg + r1 * 64 + off), 0u, sel);
            const uint32_t u0 = (t0 | (t0 << 4)) & 0x0F0F0F0Fu, u1 = (t1 | (t1 << 4)) & 0x0F0F0F0Fu;
            e0 = u0 & 0x03030303u; e1 = u1 & 0x03030303u;
            o0 = (u0 >> 2) & 0x03030303u; o1 = (u1 >> 2) & 0x03030303u;
          } else {  // bytes: slice gg is 32 B of box gg / 4; lane c takes bytes 8c .. 8c + 7
            const uint32_t ch = (uint32_t)(2 * (gg & 3) + (c >> 1));
            const uint32_t off = (uint32_t)(gg >> 2) * 8192 + ((ch ^ sw) << 4) + 8 * (c & 1);
            const uint2 w0 = lds64(stg + r0 * 128 + off), w1 = lds64(stg + r1 * 128 + off);
            e0 = __byte_perm(w0.x, w0.y, 0x6420); e1 = __byte_perm(w1.x, w1.y, 0x6420);
            o0 = __byte_perm(w0.x, w0.y, 0x7531); o1 = __byte_perm(w1.x, w1.y, 0x7531);
          }
        };
        // the weight scale of group gg for rows r0, r1 (int4: S = sc * ss; affine: s, times 16 when the
        // codes enter the MMA as q rather than 16 q)
        constexpr float SF = (FMT == FMT_INT4 || BITS == 4) ? 1.f : 16.f;
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) {
          uint32_t e0, e1, o0, o1;
          codes(gg, e0, e1, o0, o1);
          const uint4 xv = lds128(stg + L::ST_X + ((gg * M + g) * 4 + c) * 16);
          // (G_x, G_y) of tokens 2c and 2c + 1: 8-byte records, so two 8-byte loads (odd M)
          const float2 Ga = lds64f(stg + L::ST_GSUM + (gg * M + 2 * c) * 8);
          const float2 Gb = lds64f(stg + L::ST_GSUM + (gg * M + 2 * c + 1) * 8);
          if (gg == 0) x24s |= __float_as_uint(Ga.x) | __float_as_uint(Gb.x);  // zero for tokens past M
          const float gax = Ga.x, gbx = Gb.x;
          int32_t dh[4], dm[4];
          QL_IMMA0("s8", dh, acc_init, e0, e1, o0, o1, xv.x, xv.y);
          QL_IMMA0("u8", dm, acc_init, e0, e1, o0, o1, xv.z, xv.w);
          float t[4];  // T = 256 D_hi + D_mid
#pragma unroll
          for (int q = 0; q < 4; ++q)
            t[q] = fmaf(__int_as_float(dh[q]) - GEMV_ACC0_F, 256.f, __int_as_float(dm[q]) - GEMV_ACC0_F);
          if constexpr (FMT == FMT_INT4) {
            const uint32_t gw0g = gw0[gg >> 1], gw1g = gw1[gg >> 1];
            const int bsc = 2 * (gg & 1);
            const float S0 = fmaf(byte_magic(gw0g, bsc), ss0, nss0), Z0 = fmaf(byte_magic(gw0g, bsc + 1), zs0, nzs0);
            const float S1 = fmaf(byte_magic(gw1g, bsc), ss1, nss1), Z1 = fmaf(byte_magic(gw1g, bsc + 1), zs1, nzs1);
            acc[0] = fmaf(S0 * gax, fmaf(Z0, Ga.y, t[0]), acc[0]);
            acc[1] = fmaf(S0 * gbx, fmaf(Z0, Gb.y, t[1]), acc[1]);
            acc[2] = fmaf(S1 * gax, fmaf(Z1, Ga.y, t[2]), acc[2]);
            acc[3] = fmaf(S1 * gbx, fmaf(Z1, Gb.y, t[3]), acc[3]);
          } else {
            // slice gg lies in affine group gg * 32 / G of the super-block; its word holds (s, b) bf16
            const uint32_t gw0g = gw0[gg * 32 / G], gw1g = gw1[gg * 32 / G];
            const float s0 = bf16_bits_to_f32(gw0g) * SF, b0 = bf16_bits_to_f32(gw0g >> 16);
            const float s1 = bf16_bits_to_f32(gw1g) * SF, b1 = bf16_bits_to_f32(gw1g >> 16);
            // b 2^-a X = -b G_x G_y
            acc[0] = fmaf(s0 * gax, t[0], fmaf(-b0 * gax, Ga.y, acc[0]));
            acc[1] = fmaf(s0 * gbx, t[1], fmaf(-b0 * gbx, Gb.y, acc[1]));
            acc[2] = fmaf(s1 * gax, t[2], fmaf(-b1 * gax, Ga.y, acc[2]));
            acc[3] = fmaf(s1 * gbx, t[3], fmaf(-b1 * gbx, Gb.y, acc[3]));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
      }
    }
    // publish: rows n0, n1 x tokens 2c, 2c + 1
    const int tk0 = 2 * c, tk1 = 2 * c + 1;
    if (__any_sync(0xffffffffu, (x24s & 1u) != 0u) && ok) {  // rare
      const float4 lb = gemv_mt_low_bytes<FMT, BITS, G>(p.codes, p.gmeta, c0, c1, st0, st1, p.ws.flags, p.ws.gsum,
                                                        xlg, p.K, M, sb0, nsb);
      acc[0] += lb.x;
      acc[1] += lb.y;
      acc[2] += lb.z;
      acc[3] += lb.w;
    }
    if (ok) {
      if (P == 1) {
        if (n0 < p.N) {
          const float b0 = bias_at(p.bias, n0);
          if (tk0 < M) p.y[(int64_t)tk0 * p.N + n0] = __float2bfloat16_rn(acc[0] + b0);
          if (tk1 < M) p.y[(int64_t)tk1 * p.N + n0] = __float2bfloat16_rn(acc[1] + b0);
        }
        if (n1 < p.N) {
          const float b1 = bias_at(p.bias, n1);
          if (tk0 < M) p.y[(int64_t)tk0 * p.N + n1] = __float2bfloat16_rn(acc[2] + b1);
          if (tk1 < M) p.y[(int64_t)tk1 * p.N + n1] = __float2bfloat16_rn(acc[3] + b1);
        }
      } else {
        float *mine = p.ws.partial + (int64_t)blockIdx.x * M * 64;
        if (tk0 < M) {
          mine[tk0 * 64 + r0] = acc[0];
          mine[tk0 * 64 + r1] = acc[2];
        }
        if (tk1 < M) {
          mine[tk1 * 64 + r0] = acc[1];
          mine[tk1 * 64 + r1] = acc[3];
        }
      }
    }
  }
  if (P > 1) {  // the CTA that completes a row group adds its P parts in part order
    __syncthreads();  // every partial store precedes thread 0's release
    if (threadIdx.x == 0 && !*abort_flag) flags[1] = atomic_add_acq_rel_gpu(p.ws.counters + rg, 1) == P - 1;
    __syncthreads();  // thread 0's acquire precedes the reads of the other parts
    if (flags[1] && warp < GEMV_MT_WARPS) {
      const float *base = p.ws.partial + first * M * 64;
      for (int e = threadIdx.x; e < M * 64; e += GEMV_MT_WARPS * 32) {
        const int tk = e >> 6, r = e & 63;
        float sum = 0.f;
        for (int q = 0; q < P; ++q) sum += __ldcg(base + (int64_t)q * M * 64 + e);
        const int64_t n = rg * 64 + r;
        if (n < p.N) p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(sum + bias_at(p.bias, n));
      }
    }
  }
}

// The kernels: the same body under the register budget of each format (see gemv_mt_ctas_per_sm).
__global__ void __launch_bounds__(GEMV_MT_THREADS, GEMV_MT_CTAS_PER_SM)
    gemv_mt_int4_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_gmeta,
                        GemvMtParams p) {
  gemv_mt_body<FMT_INT4, 4, 32>(map_codes, map_gmeta, p);
}

template <int BITS, int G>
__global__ void __maxnreg__(GEMV_MT_AFFINE_NREG)
    gemv_mt_affine_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_gmeta,
                          GemvMtParams p) {
  gemv_mt_body<FMT_AFFINE, BITS, G>(map_codes, map_gmeta, p);
}

}  // namespace ql
