// gemm_sm100.cuh -- prefill-shaped layer on the 5th-generation tensor core.
//
//   y[M][N] = x[M][K] . W^T,  x bf16, W quantized, y bf16, fp32 accumulation
//
// Persistent kernel, one CTA per SM, tiles of BN=128 weight rows x TT tokens,
// K streamed in BK=64 steps through a shared-memory ring of x and code tiles.
// The dequantised weight tile never touches shared memory: the dequantisers
// write it into tensor memory (TMEM), where the MMAs of M = 128 (weight rows,
// A read from TMEM) x N = TT (tokens, B = the x tile in shared memory) consume
// it.  Shared memory then carries only the x tile (written once by TMA, read
// once by the tensor core) and the packed codes: a shared-memory weight tile
// would add its store, and a second token half would read it again, roughly
// doubling the bytes shared memory moves per MMA.  Within a tile the pace is
// set by the one thread that issues the MMAs (its per-stage waits, commits and
// bookkeeping).  Two token tiles:
//   TT = 256 (prefill): one M = 128, N = 256 MMA per 16-k slice.  The
//     accumulator (128 lanes x 256 columns) and a ring of A stages (32 columns
//     each) share the 512 TMEM columns, so there is one accumulator and the
//     epilogue of a tile runs between two tiles' MMAs.
//   TT = 32 (up to 32 tokens): one M = 128, N = 32 MMA per slice, two 32-column
//     accumulators (an epilogue overlaps the next tile), the A ring beside them.
// Warp roles:
//   warp 0      TMA producer: scaled fp16 x tile (TT x 64, 128-byte
//               swizzle) and the packed code tile (128 rows x BK codes)
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (f16 x f16 -> f32)
//   warps 2-3   (int4) copy each super-block's group and step words into a
//               metadata ring, MSLOTS super-blocks ahead
//   warps 4-7   epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32*(w%4).., one weight row per lane), undo the two
//               power-of-two scales (exponents added first), round to bf16,
//               store y
//   warps 8..    dequantisers: packed codes + metadata -> weight times 2^b_n
//               -> fp16, one whole 64-weight tile row per thread, into the
//               TMEM lanes of the warp's quarter.  Groups of four warps take
//               the stages in turn: two groups (warps 8-15) at TT = 256, four
//               (warps 8-23) at TT = 32.
// The operands are fp16 rather than bf16 because rounding every weight to
// bf16 costs ~1% of rms(y); fp16 costs ~0.1% (see gemm_prep.cuh for the
// scaling that keeps fp32 range).  Loop state advances by counters: no
// division runs per stage.
// Every mbarrier wait is bounded; a wait that gives up sets the device status
// word and makes every role leave its loop.
#pragma once
#include "gemm_prep.cuh"
#include "pack_dequant.cuh"

namespace ql {
namespace gemm {

constexpr int BM = 256;  // tokens per tile of the prefill form (the MMA's N)
constexpr int BN = 128;  // weight rows per tile
constexpr int BK = 64;
constexpr int WARP_TMA = 0;
constexpr int WARP_MMA = 1;
constexpr int WARP_META0 = 2;    // int4: two warps copy each super-block's group and step words ahead
constexpr int NUM_META_WARPS = 2;
constexpr int WARP_EPI0 = 4;
constexpr int WARP_DEQ0 = 8;
// dequantising warps: groups of four (one per TMEM lane quarter) take turns on the stages.  CPS is the
// CTAs resident per SM.  The 32-token form, whose MMAs are short and whose pace is its stage chain, has
// four groups at one CTA an SM, or two at two CTAs an SM (a layer with more 128-row tiles than SMs
// then runs every tile at once); the 256-token form has two (its register budget).
__host__ __device__ constexpr int deq_warps(int tt, int cps = 1) { return tt == BM || cps == 2 ? 8 : 16; }
__host__ __device__ constexpr int num_threads(int tt, int cps = 1) { return (WARP_DEQ0 + deq_warps(tt, cps)) * 32; }
constexpr int TT_SMALL = 32;          // token tile for up to 32 tokens
// int4 metadata ring: one slot per 256-weight super-block (four k-stages): [BN rows][16 bytes] of group
// words (the u32 of stage kb holds its two 32-weight groups), then [BN rows][4 bytes] of step words.
// Whole super-blocks make a row's copy one 16-byte and one 4-byte cp.async, against two 4-byte copies a
// stage, each from another row's line (int4 K is a multiple of 256, so no super-block straddles tiles).
constexpr int MSLOTS = 3;
constexpr int META_SLOT_BYTES = BN * 16 + BN * 4;
constexpr int SMEM_LIMIT = 232448;        // dynamic shared memory a CTA may use

__host__ __device__ constexpr int code_bits(int fmt, int bits) {
  return fmt == FMT_INT4 ? 4 : ((fmt == FMT_INT6 || fmt == FMT_INT6P) ? 6 : bits);
}
__host__ __device__ constexpr int p_row_bytes(int fmt, int bits) { return BK * code_bits(fmt, bits) / 8; }
__host__ __device__ constexpr int p_bytes(int fmt, int bits) { return BN * p_row_bytes(fmt, bits); }

// TT is the token tile: BM = 256 (one accumulator of 256 columns) or TT_SMALL = 32 (two of 32); the
// A ring of the dequantised weight tiles follows the accumulators in TMEM.
__host__ __device__ constexpr int a_bytes(int tt) { return tt * BK * 2; }  // the fp16 x tile
__host__ __device__ constexpr uint32_t tmem_cols(int tt) { return tt == BM ? 512u : 256u; }
__host__ __device__ constexpr int num_acc(int tt) { return tt == BM ? 1 : 2; }
__host__ __device__ constexpr uint32_t ta_acol0(int tt) { return (uint32_t)(num_acc(tt) * tt); }
constexpr uint32_t TA_ACOLS = BK / 2;   // an A stage: 64 fp16 per row = 32 columns

// Stages of the ring: as many as fit, up to six (TT = 256: six A stages of 32 columns fit beside the
// 256-column accumulator).  int4 adds the metadata ring [MSLOTS][META_SLOT_BYTES] and its barriers.
constexpr int NUM_BARS_PER_STAGE = 3;  // tma_full, b_full, empty
constexpr int NUM_BARS_FIXED = 5;      // acc_full[2], acc_empty[2], final
__host__ __device__ constexpr int stage_bytes(int fmt, int bits, int tt) {
  return a_bytes(tt) + p_bytes(fmt, bits);
}
__host__ __device__ constexpr int meta_bytes(int fmt) { return fmt == FMT_INT4 ? MSLOTS * META_SLOT_BYTES : 0; }
__host__ __device__ constexpr int meta_bars(int fmt) { return fmt == FMT_INT4 ? 2 * MSLOTS : 0; }
// each epilogue warp's copy of the tile's token scale exponents, one signed byte per token
__host__ __device__ constexpr int xe_bytes(int tt) { return 4 * tt; }
__host__ __device__ constexpr int smem_need(int fmt, int bits, int tt, int st) {
  return st * stage_bytes(fmt, bits, tt) + meta_bytes(fmt) + xe_bytes(tt) +
         (NUM_BARS_PER_STAGE * st + NUM_BARS_FIXED + meta_bars(fmt)) * 8 + 16 + 1024;
}
__host__ __device__ constexpr int stages(int fmt, int bits, int tt) {
  return smem_need(fmt, bits, tt, 6) <= SMEM_LIMIT ? 6
       : smem_need(fmt, bits, tt, 5) <= SMEM_LIMIT ? 5
       : smem_need(fmt, bits, tt, 4) <= SMEM_LIMIT ? 4 : 3;
}

// byte offsets inside the dynamic shared memory (base aligned to 1024)
__host__ __device__ constexpr int off_a(int tt, int s) { return s * a_bytes(tt); }
__host__ __device__ constexpr int off_p(int fmt, int bits, int tt, int s) {
  return stages(fmt, bits, tt) * a_bytes(tt) + s * p_bytes(fmt, bits);
}
__host__ __device__ constexpr int off_meta(int fmt, int bits, int tt, int s) {
  return stages(fmt, bits, tt) * stage_bytes(fmt, bits, tt) + s * META_SLOT_BYTES;
}
__host__ __device__ constexpr int off_xe(int fmt, int bits, int tt) {
  return stages(fmt, bits, tt) * stage_bytes(fmt, bits, tt) + meta_bytes(fmt);
}
__host__ __device__ constexpr int off_bar(int fmt, int bits, int tt) { return off_xe(fmt, bits, tt) + xe_bytes(tt); }
// barriers: tma_full[S], b_full[S], empty[S], acc_full[2], acc_empty[2], final, (int4) meta_full[MS],
// meta_empty[MS]; then the tmem base and the abort flag
__host__ __device__ constexpr int smem_bytes(int fmt, int bits, int tt) {
  return smem_need(fmt, bits, tt, stages(fmt, bits, tt));
}

struct Params {
  int64_t M, N, K;
  int G;
  const __nv_bfloat16 *bias;  // [N] or NULL: added in fp32 before the rounding to bf16
  const uint8_t *gmeta;
  const uint8_t *steps;
  __nv_bfloat16 *y;
  GemmWorkspace ws;
};

// Metadata of one 32-weight chunk (see formats.cuh): int4 (gm, st); int6
// (two scale codes, st); affine (gm, unused).
template <int FMT>
QL_DEVI void load_meta(const Params &p, int64_t n, int64_t c, uint32_t &gm, uint32_t &st) {
  if (n >= p.N) {
    gm = 0;
    st = 0;
    return;
  }
  if constexpr (FMT == FMT_INT4) {
    gm = __ldg(reinterpret_cast<const uint16_t *>(p.gmeta) + n * (p.K / 32) + c);
    st = __ldg(reinterpret_cast<const uint32_t *>(p.steps) + n * (p.K / 256) + (c >> 3));
  } else if constexpr (FMT == FMT_INT6 || FMT == FMT_INT6P) {
    gm = __ldg(reinterpret_cast<const uint16_t *>(p.gmeta + n * (p.K / 16)) + c);
    st = __ldg(reinterpret_cast<const uint16_t *>(p.steps) + n * (p.K / 256) + (c >> 3));
  } else {
    gm = __ldg(reinterpret_cast<const uint32_t *>(p.gmeta) + n * (p.K / p.G) + (32 * c) / p.G);
    st = 0;
  }
}

// Decode one chunk whose codes sit in shared memory at `src` (int6 planar: the chunk's 16 low-plane
// bytes at `src`, its 8 high-plane bytes at `src_hi`).
template <int FMT, int BITS>
QL_DEVI void smem_decode32(const uint8_t *src, const uint8_t *src_hi, uint32_t gm, uint32_t st, float (&w)[32]) {
  if constexpr (FMT == FMT_INT6P) {
    const uint4 l = *reinterpret_cast<const uint4 *>(src);
    const uint2 h = *reinterpret_cast<const uint2 *>(src_hi);
    const uint32_t lo[4] = {l.x, l.y, l.z, l.w}, hi[2] = {h.x, h.y};
    int6p_decode32(lo, hi, gm, st, w);
  } else if constexpr (FMT == FMT_INT4) {
    const uint4 v = *reinterpret_cast<const uint4 *>(src);
    const uint32_t c[4] = {v.x, v.y, v.z, v.w};
    int4_decode32(c, gm, st, w);
  } else if constexpr (FMT == FMT_INT6) {
    const uint2 *s2 = reinterpret_cast<const uint2 *>(src);
    const uint2 a = s2[0], b = s2[1], d = s2[2];
    const uint32_t c[6] = {a.x, a.y, b.x, b.y, d.x, d.y};
    int6_decode32(c, gm, st, w);
  } else {
    uint32_t c[BITS];
    if constexpr (BITS == 2) {
      const uint2 v = *reinterpret_cast<const uint2 *>(src);
      c[0] = v.x;
      c[1] = v.y;
    } else {
#pragma unroll
      for (int t = 0; t < BITS / 4; ++t) {
        const uint4 v = reinterpret_cast<const uint4 *>(src)[t];
        c[4 * t] = v.x; c[4 * t + 1] = v.y; c[4 * t + 2] = v.z; c[4 * t + 3] = v.w;
      }
    }
    affine_decode32<BITS>(c, gm, w);
  }
}

// Words of one 32-weight chunk's codes, read from shared memory (int4, affine): code_bits words.
template <int FMT, int BITS>
QL_DEVI void load_code_words(const uint8_t *src, uint32_t (&cw)[code_bits(FMT, BITS)]) {
  if constexpr (code_bits(FMT, BITS) == 2) {
    const uint2 v = *reinterpret_cast<const uint2 *>(src);
    cw[0] = v.x;
    cw[1] = v.y;
  } else {
#pragma unroll
    for (int t = 0; t < code_bits(FMT, BITS) / 4; ++t) {
      const uint4 v = reinterpret_cast<const uint4 *>(src)[t];
      cw[4 * t] = v.x; cw[4 * t + 1] = v.y; cw[4 * t + 2] = v.z; cw[4 * t + 3] = v.w;
    }
  }
}

// One 32-weight chunk of a tile row -> 16 words of fp16 pairs, each weight times 2^b_n (sc is the
// row's 2^b_n).  Word 4 q + e holds weights (8 q + e, 8 q + e + 4): the k order of the x tile, whose
// 16-byte chunks hold k = 0,4,1,5,2,6,3,7 of their 8 values.  int4 and affine take the chunk's code
// words `cw`; int6 (and int6 planar, with its high-plane bytes at `src_hi`) decode from `src`.
template <int FMT, int BITS>
QL_DEVI void chunk_to_f16(const uint32_t (&cw)[code_bits(FMT, BITS)], const uint8_t *src, const uint8_t *src_hi,
                          uint32_t gm, uint32_t st, float sc, uint32_t (&o)[16]) {
  if constexpr (FMT == FMT_INT4) {
    // packed-half arithmetic: q as 1024+q / 64+q from one bit operation, then
    // w * 2^b_n = q * S' - Z * S' in fp16 with S' = S * 2^b_n; the codes sc, zc become floats
    // by placing the byte in the mantissa of 2^23 and subtracting 2^23 (exact)
    const float scf = __uint_as_float(0x4B000000u | (gm & 0xffu)) - 8388608.f;
    const float zcf = __uint_as_float(0x4B000000u | ((gm >> 8) & 0xffu)) - 8388608.f;
    const float S = __fmul_rn(scf, f16_bits_to_f32(st)) * sc;
    const float ZS = __fmul_rn(zcf, f16_bits_to_f32(st >> 16)) * S;
    const __half2 s2 = __float2half2_rn(S), nz2 = __float2half2_rn(-ZS);
    const __half2 m1024 = __float2half2_rn(1024.f), m64 = __float2half2_rn(64.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t wd = cw[q], w8 = wd >> 8;
      uint32_t pr[4];
      pr[0] = (wd & 0x000F000Fu) | 0x64006400u;  // (1024 + n0, 1024 + n4)
      pr[1] = (wd & 0x00F000F0u) | 0x54005400u;  // (64 + n1, 64 + n5)
      pr[2] = (w8 & 0x000F000Fu) | 0x64006400u;  // (1024 + n2, 1024 + n6)
      pr[3] = (w8 & 0x00F000F0u) | 0x54005400u;  // (64 + n3, 64 + n7)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 qv = __hsub2(*reinterpret_cast<const __half2 *>(&pr[e]), (e & 1) ? m64 : m1024);
        const __half2 wv = __hfma2(qv, s2, nz2);
        o[4 * q + e] = *reinterpret_cast<const uint32_t *>(&wv);
      }
    }
  } else if constexpr (FMT == FMT_AFFINE) {
    // packed-half arithmetic: the codes become 1024 + q halves by bit operations (q exact after
    // one subtraction), then w * 2^b_n = q * s' + b' in one fused multiply-add with s' = s * 2^b_n
    // and b' = b * 2^b_n, which are exact in fp16 (bf16 values scaled into fp16's range), so each
    // weight is rounded once
    const __half2 s2 = __float2half2_rn(bf16_bits_to_f32(gm) * sc);
    const __half2 b2 = __float2half2_rn(bf16_bits_to_f32(gm >> 16) * sc);
    const __half2 m1024 = __float2half2_rn(1024.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // output words 4q..: weights 8q .. 8q+7 of the chunk, as (k, k+4) pairs
      uint32_t pr[4];
      if constexpr (BITS == 4) {
        const uint32_t wd = cw[q], w8 = wd >> 8;
        pr[0] = (wd & 0x000F000Fu) | 0x64006400u;  // (1024 + n0, 1024 + n4)
        pr[1] = ((wd >> 4) & 0x000F000Fu) | 0x64006400u;
        pr[2] = (w8 & 0x000F000Fu) | 0x64006400u;
        pr[3] = ((w8 >> 4) & 0x000F000Fu) | 0x64006400u;
      } else if constexpr (BITS == 8) {
        const uint32_t w0 = cw[2 * q], w1 = cw[2 * q + 1];  // k 0..3, k 4..7
        const uint32_t t0 = __byte_perm(w0, w1, 0x5140), t1 = __byte_perm(w0, w1, 0x7362);  // (0 4 1 5) (2 6 3 7)
        pr[0] = __byte_perm(t0, 0x64646464u, 0x4140);
        pr[1] = __byte_perm(t0, 0x64646464u, 0x4342);
        pr[2] = __byte_perm(t1, 0x64646464u, 0x4140);
        pr[3] = __byte_perm(t1, 0x64646464u, 0x4342);
      } else {  // 2-bit: codes 8q .. 8q+7 are bits 16 (q & 1) .. of word q / 2
        const uint32_t wd = cw[q >> 1] >> (16 * (q & 1));
        const uint32_t u = __byte_perm(wd, 0u, 0x4140);  // codes 0-3 in byte 0, codes 4-7 in byte 2
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = ((u >> (2 * e)) & 0x00030003u) | 0x64006400u;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 qv = __hsub2(*reinterpret_cast<const __half2 *>(&pr[e]), m1024);
        const __half2 wv = __hfma2(qv, s2, b2);
        o[4 * q + e] = *reinterpret_cast<const uint32_t *>(&wv);
      }
    }
  } else {
    float w[32];
    smem_decode32<FMT, BITS>(src, src_hi, gm, st, w);
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[4 * q + e] = pack_f16x2(w[8 * q + e] * sc, w[8 * q + e + 4] * sc);
  }
}

template <int FMT, int BITS, int TT, int CPS = 1>
__global__ void __launch_bounds__(num_threads(TT, CPS), CPS)
    gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
                Params p) {
  constexpr int NACC = num_acc(TT);  // accumulators in TMEM
  constexpr uint32_t A_COL0 = ta_acol0(TT);
  // dequantising warps per stage: TT = 256 alternates stages between two groups of four
  static_assert(CPS == 1 || (CPS == 2 && TT != BM), "two CTAs an SM: the 32-token form only");
  constexpr int DEQ_WARPS = deq_warps(TT, CPS), NG = DEQ_WARPS / 4;  // dequantiser groups
  constexpr int DEQ_PER_STAGE = 4;                                   // one group fills a stage
  static_assert(NG >= 1 && 4 % NG == 0, "groups take whole turns within a super-block");

  constexpr int PROW = p_row_bytes(FMT, BITS);
  constexpr int STAGES = stages(FMT, BITS, TT);
  constexpr uint32_t STAGE_TX = a_bytes(TT) + p_bytes(FMT, BITS);
  constexpr uint32_t TMEM_COLS = tmem_cols(TT);
  static_assert(NG < STAGES, "a group's step through the ring crosses its end at most once");
  static_assert(A_COL0 + STAGES * TA_ACOLS <= TMEM_COLS, "A ring beside the accumulators");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + off_bar(FMT, BITS, TT));
  uint32_t *tmem_holder =
      reinterpret_cast<uint32_t *>(bars + NUM_BARS_PER_STAGE * STAGES + NUM_BARS_FIXED + meta_bars(FMT));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
  auto bar_tma_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_b_full = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + 2 * STAGES + s); };
  auto bar_acc_full = [&](int a) { return smem_u32(bars + 3 * STAGES + a); };
  auto bar_acc_empty = [&](int a) { return smem_u32(bars + 3 * STAGES + 2 + a); };
  const uint32_t bar_final = smem_u32(bars + 3 * STAGES + 4);
  auto bar_meta_full = [&](int s) { return smem_u32(bars + 3 * STAGES + 5 + s); };
  auto bar_meta_empty = [&](int s) { return smem_u32(bars + 3 * STAGES + 5 + MSLOTS + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m_tiles = (p.M + TT - 1) / TT, n_tiles = (p.N + BN - 1) / BN;
  const int64_t num_tiles = m_tiles * n_tiles;
  const int num_kb = (int)(p.K / BK);
  const int64_t my_tiles = (num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const int64_t total_it = my_tiles * num_kb;  // k-stages this CTA runs, in order

  // (k-step, tile) of a stage, advanced one stage at a time
  struct Cursor {
    int kb;
    int64_t tile, n_tile, m_tile;
  };
  auto cursor0 = [&]() {
    Cursor c;
    c.kb = 0;
    c.tile = blockIdx.x;
    c.n_tile = c.tile / m_tiles;
    c.m_tile = c.tile - c.n_tile * m_tiles;
    return c;
  };
  auto advance = [&](Cursor &c) {
    if (++c.kb == num_kb) {
      c.kb = 0;
      c.tile += gridDim.x;
      c.n_tile = c.tile / m_tiles;
      c.m_tile = c.tile - c.n_tile * m_tiles;
    }
  };
  // slot and phase of a ring position, advanced one use at a time
  auto step_ring = [](int &slot, uint32_t &phase, int depth) {
    if (++slot == depth) {
      slot = 0;
      phase ^= 1u;
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_tma_full(s), 1);
      mbar_init(bar_b_full(s), DEQ_PER_STAGE);
      mbar_init(bar_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_acc_full(a), 1);
      mbar_init(bar_acc_empty(a), 4);
    }
    mbar_init(bar_final, 1);
    if constexpr (FMT == FMT_INT4) {
      for (int s = 0; s < MSLOTS; ++s) {
        mbar_init(bar_meta_full(s), NUM_META_WARPS * 32);  // one cp.async arrival per copying thread
        mbar_init(bar_meta_empty(s), DEQ_WARPS);            // every dequantising warp, once a super-block
      }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // launched as a programmatic dependent of the weight-scale pass (which waits for the x pass): the
  // set-up above overlapped them; the workspace they write is read only from here on
  pdl_wait();

  if (warp == WARP_TMA) {
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_codes);
      int64_t it = 0;
      int s = 0;
      uint32_t ph = 0;
      Cursor cur = cursor0();
      bool ok = true;
      const int64_t n_it = copies_withheld() ? 0 : total_it;  // steps whose copies are started
      for (; it < n_it; ++it) {
        if (!mbar_wait_bounded(bar_empty(s), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar_tma_full(s), STAGE_TX);
        tma_load_2d(sbase + off_a(TT, s), &map_x, bar_tma_full(s), cur.kb * BK, (int32_t)(cur.m_tile * TT));
        if constexpr (FMT == FMT_INT6P) {  // k-step kb: low-plane bytes 32 (kb % 4) .. and high-plane
                                           // bytes 128 + 16 (kb % 4) .. of super-block kb / 4, by 16-byte boxes
          const int32_t x0 = 192 * (cur.kb >> 2) + 32 * (cur.kb & 3), xh = 192 * (cur.kb >> 2) + 128 + 16 * (cur.kb & 3);
          tma_load_2d(sbase + off_p(FMT, BITS, TT, s), &map_codes, bar_tma_full(s), x0, (int32_t)(cur.n_tile * BN));
          tma_load_2d(sbase + off_p(FMT, BITS, TT, s) + 16 * BN, &map_codes, bar_tma_full(s), x0 + 16,
                      (int32_t)(cur.n_tile * BN));
          tma_load_2d(sbase + off_p(FMT, BITS, TT, s) + 32 * BN, &map_codes, bar_tma_full(s), xh,
                      (int32_t)(cur.n_tile * BN));
        } else {
          tma_load_2d(sbase + off_p(FMT, BITS, TT, s), &map_codes, bar_tma_full(s), cur.kb * PROW,
                      (int32_t)(cur.n_tile * BN));
        }
        step_ring(s, ph, STAGES);
        advance(cur);
      }
      if (!ok) {  // let copies already issued land before the CTA can exit
        for (int64_t j = it - 1; j >= 0 && j >= it - STAGES; --j) {
          const long long t0 = clock64();
          while (!mbar_try_wait(bar_tma_full((int)(j % STAGES)), (uint32_t)((j / STAGES) & 1)) &&
                 clock64() - t0 < QL_WAIT_LIMIT_CYCLES) {
          }
        }
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      // D[weight row][token] += W tile (A, M = 128) x x tile (B, N = TT).  This one thread sets the
      // kernel's pace, so its loop is unrolled over the ring's slots: slot j's x-tile descriptor
      // and A columns are compile-time offsets from slot 0's, and the phase flips once a ring cycle.
      constexpr uint32_t idesc = umma_idesc_f16_f32(BN, TT);
      constexpr uint32_t XDESC_STEP = (uint32_t)(a_bytes(TT) >> 4);  // descriptor address units
      const uint64_t xdesc0 = umma_desc_k_sw128(sbase + off_a(TT, 0));
      const uint32_t a_tmem0 = tmem_base + A_COL0;
      int64_t tcount = 0, tile = blockIdx.x;
      int kb = 0;  // stage within the current tile
      uint32_t ph = 0, d_tmem = tmem_base;
      bool ok = true, issued = false;
      // start a tile: its accumulator must have been drained (bounded wait)
      auto begin_tile = [&]() {
        const int a = (int)(tcount % NACC);
        const uint32_t ause = (uint32_t)(tcount / NACC);
        if (!mbar_wait_bounded(bar_acc_empty(a), (ause & 1) ^ 1, abort_flag)) return false;
        tc_fence_after();
        d_tmem = tmem_base + (uint32_t)(a * TT);  // accumulator a: columns a * TT ..
        return true;
      };
      if (tile < num_tiles) ok = begin_tile();
      while (ok && tile < num_tiles) {
#pragma unroll
        for (int j = 0; j < STAGES; ++j) {
          if (!ok || tile >= num_tiles) break;
          // b_full alone: its arrivals come from dequantisers that waited for this stage's tma_full,
          // so the x tile has landed before the MMAs read it (and a copy that never lands ends their
          // wait, and so this one, by the abort flag)
          if (!mbar_wait_bounded(bar_b_full(j), ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t xdesc = xdesc0 + (uint64_t)(j * XDESC_STEP);
          const uint32_t a_tmem = a_tmem0 + (uint32_t)(j * TA_ACOLS);  // lanes 0..127
          // 16 fp16 = 8 TMEM columns; 32 bytes = 2 descriptor units
          umma_f16_tmem_a(d_tmem, a_tmem, xdesc, idesc, kb != 0);
#pragma unroll
          for (int kk = 1; kk < BK / 16; ++kk) umma_f16_tmem_a(d_tmem, a_tmem + 8 * kk, xdesc + 2 * kk, idesc, 1u);
          umma_commit(bar_empty(j));
          issued = true;
          if (++kb == num_kb) {  // the tile's last stage
            kb = 0;
            umma_commit(bar_acc_full((int)(tcount % NACC)));
            tile += gridDim.x;
            ++tcount;
            if (tile < num_tiles) ok = begin_tile();
          }
        }
        ph ^= 1u;
      }
      if (issued) {  // all MMAs retired before teardown
        umma_commit(bar_final);
        const long long t0 = clock64();
        while (!mbar_try_wait(bar_final, 0) && clock64() - t0 < QL_WAIT_LIMIT_CYCLES) {
        }
      }
    }
  } else if (warp >= WARP_META0 && warp < WARP_META0 + NUM_META_WARPS) {
    if constexpr (FMT == FMT_INT4) {
      // for every super-block, each tile row's 16 bytes of group words and its step word, up to
      // MSLOTS super-blocks ahead of the dequantisers
      const int t = threadIdx.x - WARP_META0 * 32;  // 0..63: rows t and t + 64
      int ms = 0;
      uint32_t phm = 0;
      Cursor cur = cursor0();
      for (int64_t it = 0; it < total_it; it += 4) {
        if (!mbar_wait_bounded(bar_meta_empty(ms), phm ^ 1u, abort_flag)) break;
        const uint32_t dst = sbase + off_meta(FMT, BITS, TT, ms);
#pragma unroll
        for (int i = 0; i < BN / 64; ++i) {
          const int r = t + 64 * i;
          const int64_t n = cur.n_tile * BN + r;
          const bool valid = n < p.N;
          const int64_t nn = valid ? n : p.N - 1;
          cp_async16(dst + r * 16, p.gmeta + nn * (p.K / 16) + 16 * (cur.kb >> 2), valid);
          cp_async4(dst + BN * 16 + r * 4, p.steps + 4 * (nn * (p.K / 256) + (cur.kb >> 2)), valid);
        }
        cp_async_arrive_noinc(bar_meta_full(ms));
        step_ring(ms, phm, MSLOTS);
        for (int j = 0; j < 4; ++j) advance(cur);
      }
      cp_async_wait_all();  // no copy may land after the CTA is gone
    }
  } else if (warp >= WARP_EPI0 && warp < WARP_EPI0 + 4) {
    // lane = weight row n of the tile (TMEM lane 32 e + lane); its TT columns = the tile's tokens
    const int e = warp - WARP_EPI0;  // TMEM lane quarter
    int64_t tcount = 0;
    for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const int64_t n_tile = tile / m_tiles, m_tile = tile - n_tile * m_tiles;
      const int a = (int)(tcount % NACC);
      const uint32_t ause = (uint32_t)(tcount / NACC);
      // the tile's scale exponents and bias, loaded while its MMAs run: lane l holds the exponents of
      // tokens l, l + 32, .. (a load per column chunk would put an L2 round trip between the chunks)
      const int64_t n = n_tile * BN + 32 * e + lane;
      const int we = n < p.N ? p.ws.wexp[n] : 0;
      const float bn = (p.bias && n < p.N) ? __bfloat162float(p.bias[n]) : 0.f;
      // (each exponent lies in [-126, 126], so one signed byte holds it: a chunk's 16 are one broadcast
      // 16-byte load from this warp's own copy, which no other warp touches)
      int8_t *xe_s = reinterpret_cast<int8_t *>(smem + off_xe(FMT, BITS, TT)) + TT * e;
      int xe_lo = 1 << 20, xe_hi = -(1 << 20);
      __syncwarp();  // every lane is done with the previous tile's copy
#pragma unroll
      for (int j = 0; j < TT / 32; ++j) {
        const int64_t m = m_tile * TT + 32 * j + lane;
        const int xe = m < p.M ? p.ws.xexp[m] : 0;
        xe_s[32 * j + lane] = (int8_t)xe;
        xe_lo = min(xe_lo, xe);
        xe_hi = max(xe_hi, xe);
      }
      __syncwarp();
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        xe_lo = min(xe_lo, __shfl_xor_sync(0xffffffffu, xe_lo, o));
        xe_hi = max(xe_hi, __shfl_xor_sync(0xffffffffu, xe_hi, o));
      }
      // every exponent sum of the warp's rows and the tile's tokens is that of a normal float: then
      // D * 2^e is one multiplication by 2^e built from its bits, the same single rounding as mul_pow2
      const bool one_mul = __all_sync(0xffffffffu, xe_lo + we >= -126 && xe_hi + we <= 127);
      const int w_bits = we * (1 << 23) + 0x3F800000;  // bits of 2^(xe + we) = xe * 2^23 + w_bits
      if (!mbar_wait_bounded(bar_acc_full(a), ause & 1, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < TT / 16; ++c) {  // 16 tokens at a time
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(32 * e) << 16) + (uint32_t)(a * TT + 16 * c), r);
        tmem_ld_wait();
        if (c == TT / 16 - 1) {  // the accumulator is in registers: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_acc_empty(a));
        }
        const int64_t m0 = m_tile * TT + 16 * c;
        const uint4 xv = *reinterpret_cast<const uint4 *>(xe_s + 16 * c);  // tokens 16c .. 16c + 15
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        // y = D * 2^-(a_m + b_n) (exponents added first), + bias, one rounding
        if (one_mul) {
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int xe = (int)(int8_t)(xw[t >> 2] >> (8 * (t & 3)));
            r[t] = __float_as_uint(__fmul_rn(__uint_as_float(r[t]), __int_as_float(xe * (1 << 23) + w_bits)) + bn);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int xe = (int)(int8_t)(xw[t >> 2] >> (8 * (t & 3)));
            r[t] = __float_as_uint(mul_pow2(__uint_as_float(r[t]), xe + we) + bn);
          }
        }
        if (n < p.N) {  // token t of row n: the warp's 32 rows are 64 contiguous bytes of y's row m0 + t
          __nv_bfloat16 *dst = p.y + m0 * p.N + n;
          const int64_t rows_left = p.M - m0;
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            if (t < rows_left) *dst = __float2bfloat16_rn(__uint_as_float(r[t]));
            dst += p.N;
          }
        }
      }
    }
  } else if (warp >= WARP_DEQ0) {
    auto row_scale = [&](int64_t n) { return n < p.N ? p.ws.wsc[n] : 0.f; };
    // Stages go round the NG groups of four warps (warps 8-11 take stages 0, NG, 2 NG, ..., warps
    // 12-15 stages 1, NG + 1, ...).  A thread fills one whole tile row (64 weights, both 32-weight
    // chunks) of its stage into TMEM lane r = its warp's lane quarter + lane, columns A_COL0 + 32 s ..:
    // the A operand of that stage's MMAs.
    const int wd = warp - WARP_DEQ0;     // 0 .. DEQ_WARPS - 1
    const int g = wd >> 2;               // stages it = g, g + NG, ...
    const int r = 32 * (wd & 3) + lane;  // tile row
    const uint32_t t_row = tmem_base + ((uint32_t)(32 * (wd & 3)) << 16) + A_COL0;
    auto step_ng = [](int &slot, uint32_t &phase, int depth) {
      slot += NG;
      if (slot >= depth) {
        slot -= depth;
        phase ^= 1u;
      }
    };
    Cursor cur = cursor0();
    for (int j = 0; j < g; ++j) advance(cur);
    int s = g, ms = 0;  // every group visits every super-block's slot
    uint32_t ph = 0, phm = 0;
    uint32_t gm[2] = {0, 0}, st[2] = {0, 0};
    float sc = 0.f;
    if (g < total_it) {
      if constexpr (FMT != FMT_INT4) {
        load_meta<FMT>(p, cur.n_tile * BN + r, (int64_t)cur.kb * 2, gm[0], st[0]);
        load_meta<FMT>(p, cur.n_tile * BN + r, (int64_t)cur.kb * 2 + 1, gm[1], st[1]);
      }
      sc = row_scale(cur.n_tile * BN + r);
    }
    for (int64_t it = g; it < total_it; it += NG) {
      Cursor nx = cur;  // this group's next stage
      for (int j = 0; j < NG; ++j) advance(nx);
      uint32_t ngm[2] = {0, 0}, nst[2] = {0, 0};
      float nsc = sc;
      if (it + NG < total_it) {  // its metadata (int6, affine) and row scale, loaded ahead
        const int64_t n = nx.n_tile * BN + r;
        if constexpr (FMT != FMT_INT4) {
          load_meta<FMT>(p, n, (int64_t)nx.kb * 2, ngm[0], nst[0]);
          load_meta<FMT>(p, n, (int64_t)nx.kb * 2 + 1, ngm[1], nst[1]);
        }
        if (nx.n_tile != cur.n_tile) nsc = row_scale(n);
      }
      if constexpr (FMT == FMT_INT4) {  // this stage's group and step words, from the metadata ring
        const int q = (int)(it & 3);  // stage of the super-block: this group sees q = g, g + NG, ..
        if (q == g && !__all_sync(0xffffffffu, mbar_wait_bounded(bar_meta_full(ms), phm, abort_flag))) break;
        const uint8_t *slot = smem + off_meta(FMT, BITS, TT, ms);
        const uint32_t w = *reinterpret_cast<const uint32_t *>(slot + r * 16 + 4 * q);
        gm[0] = w & 0xffffu;
        gm[1] = w >> 16;
        st[0] = st[1] = *reinterpret_cast<const uint32_t *>(slot + BN * 16 + r * 4);
        if (q == g + 4 - NG) {  // this group's last stage of the super-block: release the slot
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_meta_empty(ms));
          step_ring(ms, phm, MSLOTS);
        }
      }
      // the codes have landed, and the MMAs that last read this A stage have completed (they
      // released the stage before TMA refilled it)
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_tma_full(s), ph, abort_flag))) break;
      tc_fence_after();
      const uint8_t *prow = smem + off_p(FMT, BITS, TT, s) + r * PROW;
      uint32_t o[32];
      if constexpr (PROW == 32 && (FMT == FMT_INT4 || FMT == FMT_AFFINE)) {
        // the row's two 16-byte chunks, read in the order (h ^ bit 2 of r) so that the 32 lanes'
        // first reads cover all 32 banks in four wavefronts (rows are 32 bytes apart)
        const int sw = (r >> 2) & 1;
        const uint4 va = reinterpret_cast<const uint4 *>(prow)[sw];
        const uint4 vb = reinterpret_cast<const uint4 *>(prow)[sw ^ 1];
        const uint4 c0 = sw ? vb : va, c1 = sw ? va : vb;
        const uint32_t cw0[4] = {c0.x, c0.y, c0.z, c0.w}, cw1[4] = {c1.x, c1.y, c1.z, c1.w};
        uint32_t o0[16], o1[16];
        chunk_to_f16<FMT, BITS>(cw0, nullptr, nullptr, gm[0], st[0], sc, o0);
        chunk_to_f16<FMT, BITS>(cw1, nullptr, nullptr, gm[1], st[1], sc, o1);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          o[i] = o0[i];
          o[16 + i] = o1[i];
        }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint8_t *src = prow + h * (PROW / 2);
          const uint8_t *src_hi = nullptr;
          if constexpr (FMT == FMT_INT6P) {
            src = smem + off_p(FMT, BITS, TT, s) + h * 16 * BN + r * 16;
            src_hi = smem + off_p(FMT, BITS, TT, s) + 32 * BN + r * 16 + 8 * h;
          }
          uint32_t cw[code_bits(FMT, BITS)];
          if constexpr (FMT == FMT_INT4 || FMT == FMT_AFFINE) load_code_words<FMT, BITS>(src, cw);
          uint32_t oh[16];
          chunk_to_f16<FMT, BITS>(cw, src, src_hi, gm[h], st[h], sc, oh);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[16 * h + i] = oh[i];
        }
      }
      tmem_st_32x32b_x32(t_row + (uint32_t)s * TA_ACOLS, o);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_b_full(s));
      step_ng(s, ph, STAGES);
      cur = nx;
      sc = nsc;
      gm[0] = ngm[0];
      gm[1] = ngm[1];
      st[0] = nst[0];
      st[1] = nst[1];
    }
  }

  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace ql
