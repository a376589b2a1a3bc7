// Tensor-core GEMV for uint32-packed affine weights (2, 4 or 8 bits, group 32 or 64) at 9 <= M <= 32
// tokens, on fp16 operands.
//
// Format (Hugging Face Transformers "Metal" quantization page, introduction and the loading of
// pre-quantized checkpoints): w = q * scale + bias, (scale, bias) bf16 per group of G weights along K.
//
// Past eight tokens the integer GEMVs' per-(row, token, group) scale-and-bias combine grows with the
// token count, while dequantising each weight once and sharing it across the tokens does not.  So here
// every weight is dequantised once into fp16 (packed halves: q = (1024 + q) - 1024 exactly, then
// q * s' + b' with one rounding) and fed as the A operand of mma.sync m16n8k16 (f16 x f16 -> f32)
// against NT = 2 or 4 column tiles of 8 tokens each, whose B fragments are the tokens' fp16 x.
//
// Scaling (all exact powers of two, undone at the end):
//  - x: the GEMM's fp16 copy of x (x_to_f16_kernel), one exponent per token row, stored within every
//    8 elements in the order k = 0,4,1,5,2,6,3,7 -- which is the m16n8k16 B fragment order for the
//    nibble pairs below, so one 16-byte load gives a lane all four B registers of a 32-k slice;
//  - w: per row, 2^e with a bound on the row's |w| scaled into [2^14, 2^15), from its group words alone
//    (max over the groups of (2^bits - 1)|s| + |b|), found by each consumer warp when it starts, while
//    the first stages are in flight (the GEMM's weight scaling: nothing within 2^29 of the row's
//    largest weight loses bits).
// The MMAs accumulate the whole K range in fp32, in two sets per token tile (even and odd slices, so
// the dependency chain between MMAs is half as long); the epilogue adds the sets, multiplies by
// 2^-e 2^-a and adds the bias before the one rounding to bf16.
//
// Operands per lane (g = lane / 4, c = lane % 4) and 32-k slice: the 8 codes k = 8c .. 8c + 7 of rows
// r0 = 16 w + g and r1 = r0 + 8 (one code word for 4 bits), paired (k, k + 4) for k = 0..3 by one
// shift-and-mask each into (1024 + q) halves; pair (0,4) and (1,5) are the first MMA's a0/a1 and
// a2/a3, pairs (2,6) and (3,7) the second's.  Token n*8 + g's x words (x0,x4) (x1,x5) (x2,x6) (x3,x7)
// are the two MMAs' b0/b1 in the same pairing.
//
// A CTA is a producer warp and four consumer warps on 64 rows; each stage holds a super-block's codes
// (TMA box, swizzled), its group words, and the tokens' x slices (eight TMA boxes of 32 k, one per
// slice, 64-byte swizzle -- 16-byte chunk c of token row t at c ^ ((t >> 1) & 3) -- so the eight lanes
// of a quarter-warp, tokens 2q and 2q + 1 x chunks 0..3, hit eight distinct bank groups; rows past M
// zero-filled).  Two CTAs share an SM (the shared-memory request keeps a third
// off, as for the multi-token affine kernel).
#pragma once

#include "gemv.cuh"

namespace ql {

template <int BITS, int G, int NT>
struct F16Layout {
  static constexpr int CODE_ROW = 32 * BITS;  // bytes per row and super-block
  static constexpr int CODE_BOX = CODE_ROW < 128 ? CODE_ROW : 128;
  static constexpr int CODE_BOXES = CODE_ROW / CODE_BOX;
  static constexpr int META_ROW = 4 * (256 / G);  // (s, b) bf16 pairs of the super-block's groups
  static constexpr int XROWS = 8 * NT;
  static constexpr int XBOX = XROWS * 64;          // one 32-k box (a slice) of every token row
  static constexpr int ST_X = CODE_BOXES * 64 * CODE_BOX;
  static constexpr int ST_META = ST_X + 8 * XBOX;
  static constexpr int STAGE = (ST_META + 64 * META_ROW + 1023) / 1024 * 1024;
  static constexpr uint32_t TX = ST_X + 8 * XBOX + 64 * META_ROW;
  static constexpr int CTAS = 2;
  static constexpr int PER_CTA = 233472 / CTAS - 1024 - (1024 + 6 * 16 + 16);
  static constexpr int RING = 6 < PER_CTA / STAGE ? 6 : PER_CTA / STAGE;
  static constexpr int USED = RING * STAGE + RING * 16 + 16 + 1024;  // stages, barriers, flags, alignment
  static constexpr int FLOOR = 233472 / (CTAS + 1);                  // keeps a third CTA off the SM
  static constexpr int SMEM = USED > FLOOR ? USED : FLOOR;
  static_assert(RING >= 3 && CTAS * (SMEM + 1024) <= 233472, "fp16 GEMV ring");
};

struct GemvF16Params {
  const uint8_t *gmeta;       // [N][K/G] (s, b) words, read directly for the rows' weight exponents
  const __nv_bfloat16 *bias;  // [N] or NULL
  const int *xexp;            // [M]: -a, the tokens' x exponents
  int64_t N, K;
  int M;
  SplitK split;  // of K over the CTAs of the grid, per 64-row group
  GemvWorkspace ws;  // partial sums and counters of a K split
  __nv_bfloat16 *y;
};

#define QL_HMMA(D, A0, A1, A2, A3, B0, B1)                                                                \
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, " \
               "{%0,%1,%2,%3};"                                                                          \
               : "+f"(D[0]), "+f"(D[1]), "+f"(D[2]), "+f"(D[3])                                          \
               : "r"(A0), "r"(A1), "r"(A2), "r"(A3), "r"(B0), "r"(B1))

QL_DEVI uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
QL_DEVI __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// (1024 + q) halves -> q * s + b (q exact, one rounding)
QL_DEVI uint32_t dq_pair(uint32_t magic, __half2 s, __half2 b) {
  const __half2 q = __hsub2(bits_h2(magic), __half2half2(__ushort_as_half((unsigned short)0x6400u)));
  return h2_bits(__hfma2(q, s, b));
}

// The four (1024 + q) pairs (k, k + 4), k = 0..3, of one lane's 8 codes of a 32-k slice of row r.
template <int BITS>
QL_DEVI void slice_pairs(uint32_t stg, int r, int sl, int c, uint32_t (&m)[4]) {
  if constexpr (BITS == 4) {  // 16 B per slice; 128-byte swizzle: chunk sl of row r at sl ^ (r % 8)
    const uint32_t w = lds32(stg + r * 128 + (((uint32_t)sl ^ (uint32_t)(r & 7)) << 4) + 4 * c);
#pragma unroll
    for (int s = 0; s < 4; ++s) m[s] = ((w >> (4 * s)) & 0x000F000Fu) | 0x64006400u;
  } else if constexpr (BITS == 2) {  // 8 B per slice of a 64-byte row (64-byte swizzle); a half-word a lane
    const uint32_t off = ((((uint32_t)sl >> 1) ^ (((uint32_t)r >> 1) & 3u)) << 4) + 8 * (sl & 1) + 4 * (c >> 1);
    const uint32_t t = __byte_perm(lds32(stg + r * 64 + off), 0u, (c & 1) ? 0x4342u : 0x4140u);  // bytes 0, 2
#pragma unroll
    for (int s = 0; s < 4; ++s) m[s] = ((t >> (2 * s)) & 0x00030003u) | 0x64006400u;
  } else {  // bytes: 32 B per slice in the 128-byte boxes of the 256-byte row
    const uint32_t ch = (uint32_t)(2 * (sl & 3) + (c >> 1));
    const uint2 w = lds64(stg + (uint32_t)(sl >> 2) * 8192 + r * 128 + ((ch ^ (uint32_t)(r & 7)) << 4) + 8 * (c & 1));
#pragma unroll
    for (int s = 0; s < 4; ++s)
      m[s] = (__byte_perm(w.x, w.y, (uint32_t)(s | (s << 4) | ((4 + s) << 8) | ((4 + s) << 12))) & 0x00FF00FFu) |
             0x64006400u;
  }
}

template <int BITS, int G, int NT>
__global__ void __launch_bounds__(GEMV_MT_THREADS, 2)
    gemv_f16_kernel(const __grid_constant__ CUtensorMap map_codes, const __grid_constant__ CUtensorMap map_meta,
                    const __grid_constant__ CUtensorMap map_x, GemvF16Params p) {
  using L = F16Layout<BITS, G, NT>;
  constexpr int RING = L::RING;
  constexpr float QMAX = (float)((1 << BITS) - 1);
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
  __syncthreads();
  pdl_launch_dependents();  // the next call's preparation pass waits for this grid before touching anything

  if (warp == GEMV_MT_WARPS) {  // producer
    if (lane == 0) {
      tma_prefetch_desc(&map_codes);
      tma_prefetch_desc(&map_meta);
      tma_prefetch_desc(&map_x);
      auto issue_w = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
        mbar_arrive_expect_tx(bar_full(s), L::TX);
#pragma unroll
        for (int bx = 0; bx < L::CODE_BOXES; ++bx)
          tma_load_2d(st + bx * 64 * L::CODE_BOX, &map_codes, bar_full(s), (sb0 + i) * L::CODE_ROW + bx * L::CODE_BOX,
                      (int32_t)(rg * 64));
        tma_load_2d(st + L::ST_META, &map_meta, bar_full(s), (sb0 + i) * L::META_ROW, (int32_t)(rg * 64));
      };
      auto issue_x = [&](int i, int s) {
        const uint32_t st = sbase + s * L::STAGE;
#pragma unroll
        for (int bx = 0; bx < 8; ++bx)
          tma_load_2d(st + L::ST_X + bx * L::XBOX, &map_x, bar_full(s), (sb0 + i) * 256 + 32 * bx, 0);
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
    // the rows' weight exponents: lane c takes groups c, c + 4, .. of rows n0, n1 (rows past N read
    // row N - 1; their sums are never stored), the four lanes of a row combine by shuffles
    constexpr int NG = 256 / G;
    int e0, e1;
    {
      const int64_t ng = p.K / G;
      const uint32_t *w0 = reinterpret_cast<const uint32_t *>(p.gmeta) + (n0 < p.N ? n0 : p.N - 1) * ng;
      const uint32_t *w1 = reinterpret_cast<const uint32_t *>(p.gmeta) + (n1 < p.N ? n1 : p.N - 1) * ng;
      float bound0 = 0.f, bound1 = 0.f;
      for (int64_t q = c; q < ng; q += 4) {
        const uint32_t u0 = __ldg(w0 + q), u1 = __ldg(w1 + q);
        bound0 = fmaxf(bound0, fmaf(QMAX, fabsf(bf16_bits_to_f32(u0)), fabsf(bf16_bits_to_f32(u0 >> 16))));
        bound1 = fmaxf(bound1, fmaf(QMAX, fabsf(bf16_bits_to_f32(u1)), fabsf(bf16_bits_to_f32(u1 >> 16))));
      }
      bound0 = fmaxf(bound0, __shfl_xor_sync(0xffffffffu, bound0, 1));
      bound0 = fmaxf(bound0, __shfl_xor_sync(0xffffffffu, bound0, 2));
      bound1 = fmaxf(bound1, __shfl_xor_sync(0xffffffffu, bound1, 1));
      bound1 = fmaxf(bound1, __shfl_xor_sync(0xffffffffu, bound1, 2));
      e0 = scale_exponent(bound0, 14);
      e1 = scale_exponent(bound1, 14);
    }
    const float f0 = exp2i(e0), f1 = exp2i(e1);
    float D[2][NT][4];  // [slice parity][token tile] x (row r0 | r1) x (token 2c | 2c + 1)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int n = 0; n < NT; ++n) D[h][n][0] = D[h][n][1] = D[h][n][2] = D[h][n][3] = 0.f;
    bool ok = true;
    for (int base = 0; base < nsb && ok; base += RING) {
      const uint32_t par = (uint32_t)((base / RING) & 1);
#pragma unroll 1
      for (int s = 0; s < RING; ++s) {
        const int i = base + s;
        if (i >= nsb) break;
        if (!mbar_wait_bounded(bar_full(s), par, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t stg = sbase + s * L::STAGE;
        // the super-block's (s, b) of rows r0, r1 as fp16 pairs (s', s'), (b', b'), times 2^e
        __half2 sc0[NG], bi0[NG], sc1[NG], bi1[NG];
#pragma unroll
        for (int q4 = 0; q4 < NG / 4; ++q4) {
          const uint4 a = lds128(stg + L::ST_META + r0 * L::META_ROW + 16 * q4);
          const uint4 b = lds128(stg + L::ST_META + r1 * L::META_ROW + 16 * q4);
          const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            sc0[4 * q4 + j] = __float2half2_rn(bf16_bits_to_f32(wa[j]) * f0);
            bi0[4 * q4 + j] = __float2half2_rn(bf16_bits_to_f32(wa[j] >> 16) * f0);
            sc1[4 * q4 + j] = __float2half2_rn(bf16_bits_to_f32(wb[j]) * f1);
            bi1[4 * q4 + j] = __float2half2_rn(bf16_bits_to_f32(wb[j] >> 16) * f1);
          }
        }
#pragma unroll
        for (int sl = 0; sl < 8; ++sl) {
          const int q = sl * 32 / G;  // the slice's group
          uint32_t m0[4], m1[4];
          slice_pairs<BITS>(stg, r0, sl, c, m0);
          slice_pairs<BITS>(stg, r1, sl, c, m1);
          uint32_t a0[4], a1[4];  // pair k of rows r0, r1
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            a0[k] = dq_pair(m0[k], sc0[q], bi0[q]);
            a1[k] = dq_pair(m1[k], sc1[q], bi1[q]);
          }
          const uint32_t xb = stg + L::ST_X + (uint32_t)sl * L::XBOX;
          const uint32_t chunk = (uint32_t)c ^ (uint32_t)((g >> 1) & 3);  // 64-byte swizzle of token row n*8 + g
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint4 xv = lds128(xb + (uint32_t)(n * 8 + g) * 64 + (chunk << 4));  // token n*8 + g
            QL_HMMA(D[sl & 1][n], a0[0], a1[0], a0[1], a1[1], xv.x, xv.y);
            QL_HMMA(D[sl & 1][n], a0[2], a1[2], a0[3], a1[3], xv.z, xv.w);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty(s));
      }
    }
    if (ok) {  // rows n0, n1 x tokens n*8 + 2c, n*8 + 2c + 1
      const float p0 = exp2i(-e0), p1 = exp2i(-e1);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = n * 8 + 2 * c + h;
          if (t >= M) continue;
          const float v0 = (D[0][n][h] + D[1][n][h]) * p0, v1 = (D[0][n][2 + h] + D[1][n][2 + h]) * p1;
          if (P == 1) {
            const float xs = exp2i(__ldg(p.xexp + t));
            if (n0 < p.N) p.y[(int64_t)t * p.N + n0] = __float2bfloat16_rn(fmaf(v0, xs, bias_at(p.bias, n0)));
            if (n1 < p.N) p.y[(int64_t)t * p.N + n1] = __float2bfloat16_rn(fmaf(v1, xs, bias_at(p.bias, n1)));
          } else {
            float *mine = p.ws.partial + (int64_t)blockIdx.x * M * 64;
            mine[t * 64 + r0] = v0;
            mine[t * 64 + r1] = v1;
          }
        }
      }
    }
  }
  if (P > 1) {  // the CTA that completes a row group adds its P parts in part order
    __syncthreads();  // every partial store precedes thread 0's release
    if (threadIdx.x == 0 && !*abort_flag) flags[1] = atomic_add_acq_rel_gpu(p.ws.counters + rg, 1) == P - 1;
    __syncthreads();  // thread 0's acquire precedes the reads of the other parts
    if (flags[1] && warp < GEMV_MT_WARPS) {
      const float *pbase = p.ws.partial + first * M * 64;
      for (int e = threadIdx.x; e < M * 64; e += GEMV_MT_WARPS * 32) {
        const int tk = e >> 6, r = e & 63;
        float sum = 0.f;
        for (int q = 0; q < P; ++q) sum += __ldcg(pbase + (int64_t)q * M * 64 + e);
        const int64_t n = rg * 64 + r;
        if (n < p.N)
          p.y[(int64_t)tk * p.N + n] = __float2bfloat16_rn(fmaf(sum, exp2i(__ldg(p.xexp + tk)), bias_at(p.bias, n)));
      }
    }
  }
}

}  // namespace ql
