// Tensor-core decode GEMV for the symmetric int6 format at 1 <= M <= 8 tokens, for both storages
// of its codes (dense, and planar: see int6p_a_words).
//
// Format (ExecuTorch PR "[cuda] Nestest Superscale Quantization for CUDA Weights
// (int4 / int6)", "Quant schema update", int6 bullet): 6-bit two's-complement
// codes, four per three bytes along K (code i of a 16-weight group at bits
// 6i .. 6i+5 of its 12 little-endian bytes), one int8 scale code per 16 weights
// and one fp16 step per 256: w = q * (code * step), no zero point.
//
// The integer MMA (mma.sync m16n8k32, s8 x s8 / s8 x u8, s32 accumulate) runs
// with a "diagonal" B operand, as in the int4 M = 1 kernel: within a set of 8
// groups of a super-block, k-slots 4c .. 4c+3 of a k-step carry four codes of
// group c and slots 16+4c .. of group c+4, and column n of B holds x only in
// the slots of group n, so D[row][n] is group n's partial dot product and the
// scale is applied once per (row, group).  Each group's 16 codes become four
// A registers (4 q as s8, the codes in the top six bits of each byte) with two
// byte permutes, at most two shifts and one or two masks each; the k-step j
// register holds codes int6_kperm(j, 0..3), and the x bytes are written in the
// same order by the preparation pass.  x enters as fixed point per 16-element
// group, x_int = rint(x * 2^a): 16-bit (max |x_int| in [2^14, 2^15)) or, for a
// super-block whose 16-bit form would lose too much (as in the int4 kernels),
// 24-bit (max |x_int| in [2^22, 2^23): exact for every bf16 element within 2^15
// of the group's largest magnitude), split into a signed high and unsigned
// middle and low bytes, one MMA each; per (row, group) the sums are exact below
// 2^19, so the accumulators start at the bits of 1.5 * 2^23 and read back with
// one subtraction.  The streaming loop runs the high and middle bytes:
//     T = 256 D_hi + D_mid,   y += S G T
// with S = code * step (exact in fp32) and G = 2^-a / 4 for 16-bit x (the whole
// product).  For 24-bit x, G = 2^8 * 2^-a / 4 carries the 24-bit marker
// (mark_24bit) and an out-of-line pass after the loop adds S G 2^-8 D_lo for
// the marked super-blocks (gemv_int6_low_bytes).
//
// A CTA is a producer warp and four consumer warps on 64 weight rows and a
// range of super-blocks.  A stage holds the codes box (64 rows x 208 bytes: the
// super-block's 192 bytes plus the first 16 of the next, so rows sit 52 words
// apart and the loads of one k-step hit 32 distinct banks), the scale codes
// (64 x 16 B), and every token's x words and group scales; all arrive on one
// mbarrier.  When the row groups alone leave a wave of 3 CTAs per SM unfilled,
// K is split over P CTAs per row group and the CTA that completes a group adds
// the parts in part order.
#pragma once

#include "gemv.cuh"

namespace ql {

// Byte b of the k-step j A register holds code int6_kperm(j, b) of the group (times 4).  Dense
// storage: the order two byte permutes per register give; planar storage: code 4b + j.
template <bool PLANAR>
__host__ __device__ constexpr int int6_kperm(int j, int b) {
  return PLANAR ? 4 * b + j
       : j == 0 ? 4 * b
       : j == 1 ? (b == 0 ? 9 : b == 1 ? 1 : b == 2 ? 13 : 5)
       : j == 2 ? (b == 0 ? 2 : b == 1 ? 10 : b == 2 ? 6 : 14)
                : 4 * b + 3;
}

// The four A registers of one group from its code words w0 w1 w2.  Codes 4i + 3 already sit in the
// top six bits of a byte; codes 4i in the low six bits of one; codes 4i + 1 and 4i + 2 straddle two
// bytes, gathered in byte pairs and shifted so the code lands in the top six bits.
QL_DEVI void int6_a_words(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t (&a)[4]) {
  const uint32_t t0 = __byte_perm(__byte_perm(w0, w1, 0x0630), w2, 0x5210);  // codes 0 4 8 12, low bits
  a[0] = (t0 << 2) & 0xFCFCFCFCu;
  const uint32_t p1 = __byte_perm(w0, w1, 0x4310), q1 = __byte_perm(w1, w2, 0x6532);  // 1 5 | 9 13
  a[1] = ((p1 << 4) & 0xFC00FC00u) | ((q1 >> 4) & 0x00FC00FCu);
  const uint32_t p2 = __byte_perm(w0, w1, 0x5421), q2 = __byte_perm(w1, w2, 0x7643);  // 2 6 | 10 14
  a[2] = ((p2 >> 2) & 0x00FC00FCu) | ((q2 << 6) & 0xFC00FC00u);
  const uint32_t t3 = __byte_perm(__byte_perm(w0, w1, 0x0052), w2, 0x7410);  // codes 3 7 11 15, top bits
  a[3] = t3 & 0xFCFCFCFCu;
}

// Planar storage (a 4-bit and a 2-bit plane per super-block, as the review of the ExecuTorch PR
// describes the reference int6 kernel's loads): the four A registers of one group from its two
// low-plane words l0, l1 (nibble i = code i, i < 8 in l0) and its high-plane word h (bits 2i, 2i+1 =
// bits 4-5 of code i).  Register j takes codes j, 4 + j, 8 + j, 12 + j: their nibbles are the low (j
// even) or high (j odd) halves of bytes j/2 and 2 + j/2 of l0 and of l1 (one byte permute per pair of
// registers), and their high fields sit at bits 2j of each byte of h.
QL_DEVI void int6p_a_words(uint32_t l0, uint32_t l1, uint32_t h, uint32_t (&a)[4]) {
  const uint32_t t01 = __byte_perm(l0, l1, 0x6420), t23 = __byte_perm(l0, l1, 0x7531);
  a[0] = ((t01 << 2) & 0x3C3C3C3Cu) | ((h << 6) & 0xC0C0C0C0u);
  a[1] = ((t01 >> 2) & 0x3C3C3C3Cu) | ((h << 4) & 0xC0C0C0C0u);
  a[2] = ((t23 << 2) & 0x3C3C3C3Cu) | ((h << 2) & 0xC0C0C0C0u);
  a[3] = ((t23 >> 2) & 0x3C3C3C3Cu) | (h & 0xC0C0C0C0u);
}

// x preparation: one thread per (token, 16-element group), so a half-warp holds one token's 16 groups
// of a super-block (16- or 24-bit as in the int4 kernels; flag byte [sb][m] and the scale's marker say which).  Entry
// (sb, m, set, j, gi) of the x words
// is the B pairs of k-step j for group 8 set + gi: (hi, 0, mid, 0) for gi < 4 (its lane feeds b0),
// (0, hi, 0, mid) for gi >= 4 (b1), and (lo, 0) or (0, lo) in the low-byte region that follows the
// K/256 * M * 1024 bytes of the first (24-bit x only); the group scale goes to gscale[sb][m][16].
// Also zeroes the first n_counters row-group counters.
template <bool PLANAR>
__global__ void __launch_bounds__(256) gemv_xprep_int6_kernel(const __nv_bfloat16 *x, int64_t M, int64_t K,
                                                              int64_t n_counters, GemvWorkspace ws) {
  pdl_launch_dependents();  // the streaming kernel may start fetching weights now
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t ng = K / 16;
  const bool live = t < M * ng;  // every lane takes part in the ballot below
  const int64_t m = live ? t / ng : 0, gg = live ? t - m * ng : 0;
  const uint4 *src = reinterpret_cast<const uint4 *>(x + m * K + 16 * gg);
  if (live) prefetch_l2(src);
  pdl_wait();               // x (and this workspace) may belong to the kernel launched before this one
  if (t < n_counters) ws.counters[t] = 0;
  uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
  if (live) {
    v0 = __ldg(src);
    v1 = __ldg(src + 1);
  }
  const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  float xs[16];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    xs[2 * i] = bf16_bits_to_f32(u[i]);
    xs[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
    amax = fmaxf(amax, fmaxf(fabsf(xs[2 * i]), fabsf(xs[2 * i + 1])));
  }
  // 16-bit fixed point unless some group of this (token, super-block) -- the 16 threads of a
  // half-warp -- would lose too much (see group_needs_24bit): then all 16 groups are 24-bit
  const int a16 = scale_exponent(amax, 14);
  const float s16 = exp2i(a16);
  float err = 0.f, mass = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float sv = xs[k] * s16;
    err += fabsf(sv - rintf(sv));
    mass += fabsf(sv);
  }
  const bool wide = live && err > (mass - amax * s16) * (1.f / 4096.f);
  const uint32_t ballot = __ballot_sync(0xffffffffu, wide);
  const bool sb24 = ((ballot >> (threadIdx.x & 16)) & 0xffffu) != 0u;
  const int a = sb24 ? scale_exponent(amax, 22) : a16;  // bf16 inputs: max |x_int| < 2^23 (2^15 for 16-bit)
  const float sc = exp2i(a);
  const int hs = sb24 ? 16 : 8;  // the value's top byte: bits 16.. (24-bit) or 8.. (16-bit, lo = 0)
  int xi[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) xi[k] = __float2int_rn(xs[k] * sc);
  if (!live) return;
  const int64_t sb = gg >> 4;
  const int gl = (int)(gg & 15), set = gl >> 3, gi = gl & 7;
  const int64_t ent = (((sb * M + m) * 2 + set) * 4) * 8 + gi;
  uint4 *dst = ws.xq + ent;
  uint2 *dst8 = reinterpret_cast<uint2 *>(ws.xq + (K / 256) * M * 64) + ent;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t hi = 0, mid = 0, lo = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int v = xi[int6_kperm<PLANAR>(j, b)];
      hi |= ((uint32_t)(v >> hs) & 0xffu) << (8 * b);
      mid |= ((uint32_t)(v >> (hs - 8)) & 0xffu) << (8 * b);
      lo |= ((uint32_t)v & 0xffu) << (8 * b);
    }
    dst[8 * j] = gi < 4 ? make_uint4(hi, 0u, mid, 0u) : make_uint4(0u, hi, 0u, mid);
    if (sb24) dst8[8 * j] = gi < 4 ? make_uint2(lo, 0u) : make_uint2(0u, lo);
  }
  // the group scale 2^-a / 4, times 2^8 for 24-bit x (whose T = 256 D_hi + D_mid is then 2^-8 of
  // 4 sum q x_int, less the low byte's 2^-8 D_lo) and then carrying the 24-bit marker (mark_24bit)
  const float gsc = exp2i(-a) * (sb24 ? 64.f : 0.25f);
  reinterpret_cast<float *>(ws.gsum)[(sb * M + m) * 16 + gl] = sb24 ? mark_24bit(gsc) : gsc;
  if (gl == 0) ws.flags[sb * 16 + m] = sb24 ? 1 : 0;
}

#define QL_IMMA6_0(TB, ACC, C, A0, A1, A2, A3, B0, B1)                                                \
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8." TB ".s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "  \
      "{%10,%11,%12,%13};"                                                                              \
      : "=r"(ACC[0]), "=r"(ACC[1]), "=r"(ACC[2]), "=r"(ACC[3])                                        \
      : "r"(A0), "r"(A1), "r"(A2), "r"(A3), "r"(B0), "r"(B1), "r"(C[0]), "r"(C[1]), "r"(C[2]), "r"(C[3]))
#define QL_IMMA6(TB, ACC, A0, A1, A2, A3, B0, B1)                                                     \
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8." TB ".s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "  \
      "{%0,%1,%2,%3};"                                                                                  \
      : "+r"(ACC[0]), "+r"(ACC[1]), "+r"(ACC[2]), "+r"(ACC[3])                                        \
      : "r"(A0), "r"(A1), "r"(A2), "r"(A3), "r"(B0), "r"(B1))

constexpr int GEMV6_WARPS = 4;  // consumer warps per CTA (64 rows); warp 4 produces
constexpr int GEMV6_THREADS = 32 * (GEMV6_WARPS + 1);
constexpr int GEMV6_CTAS_PER_SM = 3;
constexpr int GEMV6_CODE_ROW = 208;  // bytes per row in a stage: 192 of the super-block + 16 of the next

// Stage layout for up to TM tokens: codes [64][208], scale codes [64][16], group scales [TM][16] f32,
// (hi, mid) x words [TM][2 sets][4 k-steps][8 groups][16 B] (a 24-bit super-block's lo x words are
// read from global memory).  The ring is as deep (4, 3 or 2 stages) as three CTAs per SM allow.
template <int TM>
struct Int6Layout {
  static constexpr int ST_SC = 64 * GEMV6_CODE_ROW;
  static constexpr int ST_G = ST_SC + 64 * 16;
  static constexpr int ST_X = ST_G + TM * 64;
  static constexpr int STAGE = (ST_X + TM * 1024 + 127) / 128 * 128;
  static constexpr int EXTRA = 16 + 2 * 4 * 8 + 16 + 128;  // zero slot, barriers, flags, alignment
  static constexpr int RING = GEMV6_CTAS_PER_SM * (4 * STAGE + EXTRA + 1024) <= 233472   ? 4
                            : GEMV6_CTAS_PER_SM * (3 * STAGE + EXTRA + 1024) <= 233472 ? 3
                                                                                        : 2;
  static constexpr int SMEM = RING * STAGE + EXTRA;
};

struct Gemv6Params {
  const uint8_t *codes, *sc;  // [N][3K/4], [N][K/16]: read directly only by the 24-bit tail
  const uint16_t *steps;      // fp16 [N][K/256]
  const __nv_bfloat16 *bias;  // [N] or NULL
  int64_t N, K;
  int M;  // 1 .. TM tokens
  SplitK split;  // of K over the CTAs of the grid, per 64-row group
  GemvWorkspace ws;
  __nv_bfloat16 *y;
};

// The low bytes of 24-bit x for one consumer warp of the int6 kernel: S G 2^-8 D_lo per (row, token,
// 16-weight group) of every super-block of the range [sb0, sb0 + nsb) in which some token's x is
// 24-bit, the weights read again from global memory (rows c0, c1; rows past N read row N - 1 and their
// sums are never stored).  Flagged super-blocks are rare, so this runs out of line and leaves the
// streaming loop's registers alone.  Returns the sums to add per (token, row r0 | r1).
template <int TM>
struct Int6LowBytes {
  float v[TM][2];
};

template <int TM, bool PLANAR>
__device__ __noinline__ Int6LowBytes<TM> gemv_int6_low_bytes(const uint8_t *codes, const uint8_t *sc, int64_t c0,
                                                             int64_t c1, const uint16_t *st0, const uint16_t *st1,
                                                             const uint8_t *flags, const float *gscale,
                                                             const uint2 *xlg, int64_t K, int M, int sb0, int nsb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const bool on = (g & 3) == c;  // lane (g, c) feeds x for group g of a set
  const uint64_t fmask = M >= 8 ? ~0ull : ((1ull << (8 * M)) - 1);  // the flag bytes of tokens < M
  const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
  const uint8_t *q0 = codes + c0 * (K / 256) * 192, *q1 = codes + c1 * (K / 256) * 192;
  const uint8_t *s0p = sc + c0 * (K / 16), *s1p = sc + c1 * (K / 16);
  const int bo = 8 * ((2 * c) & 3);
  Int6LowBytes<TM> out;
#pragma unroll
  for (int m = 0; m < TM; ++m) out.v[m][0] = out.v[m][1] = 0.f;
  for (int i = 0; i < nsb; ++i) {
    const int64_t sb = sb0 + i;
    const uint2 fw = __ldg(reinterpret_cast<const uint2 *>(flags + sb * 16));
    const uint64_t f24 = ((uint64_t)fw.y << 32 | fw.x) & fmask;
    if (f24 == 0) continue;  // the same for the whole warp
    const float p0 = f16_bits_to_f32(__ldg(st0 + i)), p1 = f16_bits_to_f32(__ldg(st1 + i));
    const uint8_t *b0 = q0 + sb * 192, *b1 = q1 + sb * 192;
    const float *gsc = gscale + sb * M * 16;
    const uint2 *xls = xlg + sb * M * 64;
#pragma unroll 1
    for (int set = 0; set < 2; ++set) {
      uint32_t A00[4], A01[4], A10[4], A11[4];  // as in the streaming loop, from the rows in global memory
      const int gl = 8 * set + c;
      if constexpr (PLANAR) {
        const uint2 l00 = __ldg(reinterpret_cast<const uint2 *>(b0 + 8 * gl)), l01 = __ldg(reinterpret_cast<const uint2 *>(b0 + 8 * gl + 32));
        const uint2 l10 = __ldg(reinterpret_cast<const uint2 *>(b1 + 8 * gl)), l11 = __ldg(reinterpret_cast<const uint2 *>(b1 + 8 * gl + 32));
        int6p_a_words(l00.x, l00.y, __ldg(reinterpret_cast<const uint32_t *>(b0 + 128 + 4 * gl)), A00);
        int6p_a_words(l01.x, l01.y, __ldg(reinterpret_cast<const uint32_t *>(b0 + 144 + 4 * gl)), A01);
        int6p_a_words(l10.x, l10.y, __ldg(reinterpret_cast<const uint32_t *>(b1 + 128 + 4 * gl)), A10);
        int6p_a_words(l11.x, l11.y, __ldg(reinterpret_cast<const uint32_t *>(b1 + 144 + 4 * gl)), A11);
      } else {
        const uint32_t *w0 = reinterpret_cast<const uint32_t *>(b0 + 12 * gl);
        const uint32_t *w1 = reinterpret_cast<const uint32_t *>(b1 + 12 * gl);
        int6_a_words(__ldg(w0), __ldg(w0 + 1), __ldg(w0 + 2), A00);
        int6_a_words(__ldg(w0 + 12), __ldg(w0 + 13), __ldg(w0 + 14), A01);
        int6_a_words(__ldg(w1), __ldg(w1 + 1), __ldg(w1 + 2), A10);
        int6_a_words(__ldg(w1 + 12), __ldg(w1 + 13), __ldg(w1 + 14), A11);
      }
      const uint32_t sw0 = __ldg(reinterpret_cast<const uint32_t *>(s0p + sb * 16 + 8 * set + 4 * (c >> 1)));
      const uint32_t sw1 = __ldg(reinterpret_cast<const uint32_t *>(s1p + sb * 16 + 8 * set + 4 * (c >> 1)));
      const float S00 = __fmul_rn((float)(int8_t)(sw0 >> bo), p0), S01 = __fmul_rn((float)(int8_t)(sw0 >> (bo + 8)), p0);
      const float S10 = __fmul_rn((float)(int8_t)(sw1 >> bo), p1), S11 = __fmul_rn((float)(int8_t)(sw1 >> (bo + 8)), p1);
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        if (m < M && ((f24 >> (8 * m)) & 0xffu) != 0) {  // the same for the warp
          int32_t dl[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint2 xl = on ? __ldg(xls + ((m * 2 + set) * 4 + j) * 8 + g) : make_uint2(0u, 0u);
            if (j == 0) QL_IMMA6_0("u8", dl, acc_init, A00[0], A10[0], A01[0], A11[0], xl.x, xl.y);
            else QL_IMMA6("u8", dl, A00[j], A10[j], A01[j], A11[j], xl.x, xl.y);
          }
          const float2 G = __ldg(reinterpret_cast<const float2 *>(gsc + m * 16 + 8 * set + 2 * c));
          const float gx = unmark(G.x) * (1.f / 256.f), gy = unmark(G.y) * (1.f / 256.f);
          out.v[m][0] = fmaf(S00 * gx, __int_as_float(dl[0]) - GEMV_ACC0_F, out.v[m][0]);
          out.v[m][0] = fmaf(S01 * gy, __int_as_float(dl[1]) - GEMV_ACC0_F, out.v[m][0]);
          out.v[m][1] = fmaf(S10 * gx, __int_as_float(dl[2]) - GEMV_ACC0_F, out.v[m][1]);
          out.v[m][1] = fmaf(S11 * gy, __int_as_float(dl[3]) - GEMV_ACC0_F, out.v[m][1]);
        }
      }
    }
  }
  return out;
}

template <int TM, bool PLANAR>
__global__ void __launch_bounds__(GEMV6_THREADS, GEMV6_CTAS_PER_SM)
    gemv_int6_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_sc,
                     Gemv6Params p) {
  using L = Int6Layout<TM>;
  constexpr int RING = L::RING;
  constexpr int MP = TM < 4 ? TM : 4;  // tokens per MMA group
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t *zero16 = smem + RING * L::STAGE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(zero16 + 16);  // full[R], empty[R]
  int *flags = reinterpret_cast<int *>(bars + 2 * RING);        // abort, last-part
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
  if (threadIdx.x < 4) reinterpret_cast<uint32_t *>(zero16)[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), GEMV6_WARPS);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  // the group scales of tokens M..TM-1 in every stage: never written by the copies, read (and their
  // sums dropped) for odd M; zero, so they carry no 24-bit marker
  if (threadIdx.x < (TM - M) * 16) {
#pragma unroll
    for (int s = 0; s < RING; ++s) reinterpret_cast<uint32_t *>(smem + s * L::STAGE + L::ST_G + M * 64)[threadIdx.x] = 0u;
  }
  __syncthreads();
  pdl_launch_dependents();  // the next call's preparation pass waits for this grid before touching anything

  if (warp == GEMV6_WARPS) {  // producer
    if (lane == 0) {
      tma_prefetch_desc(&map_codes);
      tma_prefetch_desc(&map_sc);
      const uint32_t tx = (uint32_t)L::ST_G + (uint32_t)M * (64 + 1024);
      const float *gscale = reinterpret_cast<const float *>(p.ws.gsum);
      auto issue_w = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
        mbar_arrive_expect_tx(bar_full(s), tx);
        tma_load_2d(st, &map_codes, bar_full(s), (sb0 + i) * 192, (int32_t)(rg * 64));
        tma_load_2d(st + L::ST_SC, &map_sc, bar_full(s), (sb0 + i) * 16, (int32_t)(rg * 64));
      };
      auto issue_x = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
        const int64_t sb = sb0 + i;
        bulk_load(st + L::ST_G, gscale + sb * M * 16, (uint32_t)M * 64, bar_full(s));
        bulk_load(st + L::ST_X, p.ws.xq + sb * M * 64, (uint32_t)M * 1024, bar_full(s));
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
    const int64_t n0 = rg * 64 + r0, n1 = n0 + 8;
    const int64_t c0 = n0 < p.N ? n0 : p.N - 1, c1 = n1 < p.N ? n1 : p.N - 1;
    const uint16_t *st0 = p.steps + c0 * NS + sb0, *st1 = p.steps + c1 * NS + sb0;
    uint32_t sr0[RING], sr1[RING];  // step bits by stage, RING - 1 super-blocks ahead
#pragma unroll
    for (int s = 0; s < RING; ++s) {
      sr0[s] = 0u;
      sr1[s] = 0u;
      if (s < RING - 1 && s < nsb) {
        sr0[s] = __ldg(st0 + s);
        sr1[s] = __ldg(st1 + s);
      }
    }
    // lane (g, c) feeds x for group g of a set when g = c (b0) or g = c + 4 (b1); otherwise zeros
    const bool on = (g & 3) == c;
    const uint32_t zero_a = smem_u32(zero16);
    const int32_t acc_init[4] = {GEMV_ACC0, GEMV_ACC0, GEMV_ACC0, GEMV_ACC0};
    const uint2 *xlg = reinterpret_cast<const uint2 *>(p.ws.xq + (p.K / 256) * M * 64);  // lo x words
    float acc[TM][2];  // (token) x (row r0 | r1)
#pragma unroll
    for (int m = 0; m < TM; ++m) acc[m][0] = acc[m][1] = 0.f;
    uint32_t x24s = 0u;  // bit 0: some super-block's group scale carries the 24-bit marker
    bool ok = true;
    for (int base = 0; base < nsb && ok; base += RING) {
      const uint32_t par = (uint32_t)((base / RING) & 1);
#pragma unroll
      for (int s = 0; s < RING; ++s) {
        const int i = base + s;
        if (i >= nsb) break;
        const int nx = i + RING - 1, sn = (s + RING - 1) % RING;
        if (nx < nsb) {
          sr0[sn] = __ldg(st0 + nx);
          sr1[sn] = __ldg(st1 + nx);
        }
        if (!mbar_wait_bounded(bar_full(s), par, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t stg = sbase + s * L::STAGE;
        const float stp0 = f16_bits_to_f32(sr0[s]), stp1 = f16_bits_to_f32(sr1[s]);
        // scale codes of the D columns: groups 8 set + 2c, 8 set + 2c + 1 of rows r0, r1
        const uint32_t scw00 = lds32(stg + L::ST_SC + r0 * 16 + 4 * (c >> 1));
        const uint32_t scw01 = lds32(stg + L::ST_SC + r0 * 16 + 8 + 4 * (c >> 1));
        const uint32_t scw10 = lds32(stg + L::ST_SC + r1 * 16 + 4 * (c >> 1));
        const uint32_t scw11 = lds32(stg + L::ST_SC + r1 * 16 + 8 + 4 * (c >> 1));
        const int bo = 8 * ((2 * c) & 3);
        float S[2][2][2];  // [set][row][column half]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          S[0][0][h] = __fmul_rn((float)(int8_t)(scw00 >> (bo + 8 * h)), stp0);
          S[1][0][h] = __fmul_rn((float)(int8_t)(scw01 >> (bo + 8 * h)), stp0);
          S[0][1][h] = __fmul_rn((float)(int8_t)(scw10 >> (bo + 8 * h)), stp1);
          S[1][1][h] = __fmul_rn((float)(int8_t)(scw11 >> (bo + 8 * h)), stp1);
        }
        // A operand of set `set`: groups 8 set + c (slots 4c ..) and 8 set + c + 4 (slots 16 + 4c ..) of
        // rows r0, r1, as [row][group half]
        auto a_words = [&](int set, uint32_t (&A00)[4], uint32_t (&A01)[4], uint32_t (&A10)[4], uint32_t (&A11)[4]) {
          if constexpr (PLANAR) {  // group gg: low plane bytes 8 gg .., high plane bytes 128 + 4 gg ..
            const uint32_t gl = 8 * set + c;
            const uint32_t a0 = stg + r0 * GEMV6_CODE_ROW, a1 = stg + r1 * GEMV6_CODE_ROW;
            const uint2 l00 = lds64(a0 + 8 * gl), l01 = lds64(a0 + 8 * gl + 32);
            const uint2 l10 = lds64(a1 + 8 * gl), l11 = lds64(a1 + 8 * gl + 32);
            int6p_a_words(l00.x, l00.y, lds32(a0 + 128 + 4 * gl), A00);
            int6p_a_words(l01.x, l01.y, lds32(a0 + 144 + 4 * gl), A01);
            int6p_a_words(l10.x, l10.y, lds32(a1 + 128 + 4 * gl), A10);
            int6p_a_words(l11.x, l11.y, lds32(a1 + 144 + 4 * gl), A11);
          } else {
            const uint32_t o = stg + 12 * (8 * set + c);
            const uint32_t a0 = o + r0 * GEMV6_CODE_ROW, a1 = o + r1 * GEMV6_CODE_ROW;
            int6_a_words(lds32(a0), lds32(a0 + 4), lds32(a0 + 8), A00);
            int6_a_words(lds32(a0 + 48), lds32(a0 + 52), lds32(a0 + 56), A01);
            int6_a_words(lds32(a1), lds32(a1 + 4), lds32(a1 + 8), A10);
            int6_a_words(lds32(a1 + 48), lds32(a1 + 52), lds32(a1 + 56), A11);
          }
        };
#pragma unroll
        for (int set = 0; set < 2; ++set) {
          uint32_t A00[4], A01[4], A10[4], A11[4];
          a_words(set, A00, A01, A10, A11);
          // up to four tokens at a time: eight independent accumulator chains (hi / mid) per k-step
#pragma unroll
          for (int m0 = 0; m0 < TM; m0 += MP) {
            if (m0 < M) {
              int32_t dh[MP][4], dm[MP][4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int mm = 0; mm < MP; ++mm) {
                  const int m = m0 + mm;  // a token past M (odd M) reads stale stage words; its sums are never stored
                  const uint32_t xrow = stg + L::ST_X + ((m * 2 + set) * 4 + j) * 128 + 16 * g;
                  const uint4 xv = lds128(on ? xrow : zero_a);
                  if (j == 0) {
                    QL_IMMA6_0("s8", dh[mm], acc_init, A00[0], A10[0], A01[0], A11[0], xv.x, xv.y);
                    QL_IMMA6_0("u8", dm[mm], acc_init, A00[0], A10[0], A01[0], A11[0], xv.z, xv.w);
                  } else {
                    QL_IMMA6("s8", dh[mm], A00[j], A10[j], A01[j], A11[j], xv.x, xv.y);
                    QL_IMMA6("u8", dm[mm], A00[j], A10[j], A01[j], A11[j], xv.z, xv.w);
                  }
                }
              }
#pragma unroll
              for (int mm = 0; mm < MP; ++mm) {
                const int m = m0 + mm;
                // D[q]: q = 0 (r0, group 8 set + 2c), 1 (r0, + 1), 2 (r1, 2c), 3 (r1, + 1)
                const float2 G = lds64f(stg + L::ST_G + (m * 16 + 8 * set + 2 * c) * 4);
                if (set == 0) x24s |= __float_as_uint(G.x);  // zero for tokens past M
                float t[4];  // T = 256 D_hi + D_mid
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  t[q] = fmaf(__int_as_float(dh[mm][q]) - GEMV_ACC0_F, 256.f, __int_as_float(dm[mm][q]) - GEMV_ACC0_F);
                acc[m][0] = fmaf(S[set][0][0] * G.x, t[0], acc[m][0]);
                acc[m][0] = fmaf(S[set][0][1] * G.y, t[1], acc[m][0]);
                acc[m][1] = fmaf(S[set][1][0] * G.x, t[2], acc[m][1]);
                acc[m][1] = fmaf(S[set][1][1] * G.y, t[3], acc[m][1]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
      }
    }
    if (__any_sync(0xffffffffu, (x24s & 1u) != 0u) && ok) {  // rare
      const Int6LowBytes<TM> lb = gemv_int6_low_bytes<TM, PLANAR>(p.codes, p.sc, c0, c1, st0, st1, p.ws.flags,
                                                                 reinterpret_cast<const float *>(p.ws.gsum), xlg,
                                                                 p.K, M, sb0, nsb);
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        acc[m][0] += lb.v[m][0];
        acc[m][1] += lb.v[m][1];
      }
    }
    // the four lanes of a row hold its groups 2c, 2c + 1 of each set: sum them
#pragma unroll
    for (int m = 0; m < TM; ++m) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        acc[m][r] += __shfl_xor_sync(0xffffffffu, acc[m][r], 1);
        acc[m][r] += __shfl_xor_sync(0xffffffffu, acc[m][r], 2);
      }
    }
    if (ok) {
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        if (m < M && (m & 3) == c) {  // lane c publishes tokens c, c + 4
          if (P == 1) {
            if (n0 < p.N) p.y[(int64_t)m * p.N + n0] = __float2bfloat16_rn(acc[m][0] + bias_at(p.bias, n0));
            if (n1 < p.N) p.y[(int64_t)m * p.N + n1] = __float2bfloat16_rn(acc[m][1] + bias_at(p.bias, n1));
          } else {
            float *mine = p.ws.partial + ((int64_t)blockIdx.x * M + m) * 64;
            mine[r0] = acc[m][0];
            mine[r1] = acc[m][1];
          }
        }
      }
    }
  }
  if (P > 1) {  // the CTA that completes a row group adds its P parts in part order
    __syncthreads();  // every partial store precedes thread 0's release
    if (threadIdx.x == 0 && !*abort_flag) flags[1] = atomic_add_acq_rel_gpu(p.ws.counters + rg, 1) == P - 1;
    __syncthreads();  // thread 0's acquire precedes the reads of the other parts
    if (flags[1] && warp < GEMV6_WARPS) {
      const float *base = p.ws.partial + first * M * 64;
      for (int e = threadIdx.x; e < M * 64; e += GEMV6_WARPS * 32) {
        const int tk = e >> 6, r = e & 63;
        float sum = 0.f;
        for (int q = 0; q < P; ++q) sum += __ldcg(base + (int64_t)q * M * 64 + e);
        const int64_t n = rg * 64 + r;
        if (n < p.N) p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(sum + bias_at(p.bias, n));
      }
    }
  }
}

}  // namespace ql
