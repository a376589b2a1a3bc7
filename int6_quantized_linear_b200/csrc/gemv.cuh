// gemv.cuh -- decode-shaped layer y[M][N] = x[M][K] . W^T for small M.
//
// Simple form: one warp per output row; lane l takes chunks l, l+32, ... of
// the row (32 weights each: one int4 group, 16-byte coalesced loads), decodes
// the exact binary32 weights and accumulates x*w in fp32; a warp-shuffle
// reduction finishes the row.  The trip count over chunks is the same for
// every lane of a warp, so full-mask shuffles are always reached.
#pragma once
#include "gemm_prep.cuh"
#include "pack_dequant.cuh"

namespace ql {

template <int FMT, int BITS, int MT>
__global__ void __launch_bounds__(256) gemv_simple_kernel(WeightPtrs p, int64_t N, const __nv_bfloat16 *x,
                                                          int M, __nv_bfloat16 *y) {
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
          if (m0 + m < M) y[(int64_t)(m0 + m) * N + n] = __float2bfloat16_rn(acc[m]);
      }
    }
  }
}


// ===========================================================================
// Tensor-core decode GEMV for int4 at M = 1.
//
// Each warp owns a tile of 16 weight rows and a range of super-blocks.  The
// codes of one super-block of the tile (16 rows x 128 bytes) arrive by TMA
// into a per-warp ring in shared memory.  Lane (g = lane/4, c = lane%4) reads
// whole 16-byte groups -- groups c and c+4 of two tile rows -- and turns every
// 32-bit word of 8 nibbles into four f16x2 registers with one bit operation
// each (after one shift per word): the nibble is OR-ed into the mantissa of
// 1024.0 (even k) or of 64.0 (odd k), giving 1024+q or 64+q exactly.
//
// mma.sync.m16n8k16 then multiplies these 16x16 weight fragments by a
// "diagonal" x operand: column n of B holds x only in the two k-slots that
// carry group n's weights and zeros elsewhere, so after the 16 MMAs of a
// super-block D[row][n] is group n's partial dot product
//     D = sum_k (bias_k + q_k) * x'_k,     bias_k = 1024 (k even) / 64 (k odd)
// with x' = x * 2^a_g, x scaled per 32-element group by a power of two that
// puts the group's max |x| in [2^15, 2^16) (exact in fp16).  The scale and
// zero are applied once per (row, group):
//     y += S * 2^-a_g * (D - B'_g - Z * X'_g),  B'_g = sum bias_k x'_k, X'_g = sum x'_k.
// A short preparation pass writes x' in the order the fragments read it and
// (B'_g, X'_g, 2^-a_g); lanes that hold no x for an MMA read a zero block,
// so no per-MMA selects are needed.  The streaming kernel is launched as a
// programmatic dependent of that pass and starts fetching weights before the
// pass has finished (griddepcontrol.wait guards the first read of x).
// ===========================================================================

struct GemvWorkspace {
  uint32_t *xperm;  // [M][K/32 groups][16] f16x2 pairs: pair t = (x'[8(t/4)+t%4], x'[8(t/4)+t%4+4])
  float4 *gsum;     // [M][K/32] (B'_g, X'_g, 2^-a_g, 0)
  uint32_t *zero;   // 64 zero bytes
};

inline size_t gemv_workspace_bytes(int64_t M, int64_t K) {
  return align256((size_t)M * K * 2) + align256((size_t)M * (K / 32) * 16) + 256;
}

inline GemvWorkspace gemv_workspace_carve(void *base, int64_t M, int64_t K) {
  uint8_t *p = static_cast<uint8_t *>(base);
  GemvWorkspace w;
  w.xperm = reinterpret_cast<uint32_t *>(p);
  p += align256((size_t)M * K * 2);
  w.gsum = reinterpret_cast<float4 *>(p);
  p += align256((size_t)M * (K / 32) * 16);
  w.zero = reinterpret_cast<uint32_t *>(p);
  return w;
}

QL_DEVI void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
QL_DEVI void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One thread per 32-element group of x: scale into fp16 range, reorder into
// fragment pairs, sum.
__global__ void __launch_bounds__(256) gemv_xprep_kernel(const __nv_bfloat16 *x, int64_t M, int64_t K,
                                                         GemvWorkspace ws) {
  pdl_launch_dependents();
  const int64_t ng = K / 32;
  const int64_t gi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // over M * ng
  if (gi == 0) {
#pragma unroll
    for (int t = 0; t < 16; ++t) ws.zero[t] = 0u;
  }
  if (gi >= M * ng) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(x) + 4 * gi;  // 32 bf16 = 64 bytes
  float xs[32];
  float amax = 0.f;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint4 v = __ldg(src + t);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xs[8 * t + 2 * j] = bf16_bits_to_f32(u[j]);
      xs[8 * t + 2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
      amax = fmaxf(amax, fmaxf(fabsf(xs[8 * t + 2 * j]), fabsf(xs[8 * t + 2 * j + 1])));
    }
  }
  const int a = scale_exponent(amax, 15);
  const float sc = exp2i(a);
  uint32_t pr[16];
  float be = 0.f, bo = 0.f;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const int k0 = 8 * (t >> 2) + (t & 3);
    const __half2 h = __floats2half2_rn(xs[k0] * sc, xs[k0 + 4] * sc);
    pr[t] = *reinterpret_cast<const uint32_t *>(&h);
    const float2 f = __half22float2(h);  // the values the MMA will see
    if (t & 1) bo += f.x + f.y; else be += f.x + f.y;
  }
  uint4 *dst = reinterpret_cast<uint4 *>(ws.xperm + 16 * gi);
#pragma unroll
  for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pr[4 * t], pr[4 * t + 1], pr[4 * t + 2], pr[4 * t + 3]);
  ws.gsum[gi] = make_float4(1024.f * be + 64.f * bo, be + bo, exp2i(-a), 0.f);
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

// Wait for an mbarrier phase, letting the hardware suspend the thread (up to the hint, in ns)
// instead of spinning; bounded like mbar_wait_bounded.
QL_DEVI bool mbar_wait_suspend(uint32_t bar, uint32_t parity, volatile int *abort) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
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

// One MMA of the GEMV: builds the four f16x2 A registers from the code words in place
// ((w & mask) | magic: 1024+q for a nibble in bits 0-3 of a half, 64+q for bits 4-7) and
// multiplies them into acc.
#define QL_GEMV_MMA(MASK, MAGIC, W0, W1, W2, W3, B0, B1)                                              \
  asm volatile(                                                                                         \
      "{\n\t.reg .b32 a0, a1, a2, a3;\n\t"                                                            \
      "lop3.b32 a0, %4, " MASK ", " MAGIC ", 0xEA;\n\t"                                               \
      "lop3.b32 a1, %5, " MASK ", " MAGIC ", 0xEA;\n\t"                                               \
      "lop3.b32 a2, %6, " MASK ", " MAGIC ", 0xEA;\n\t"                                               \
      "lop3.b32 a3, %7, " MASK ", " MAGIC ", 0xEA;\n\t"                                               \
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {a0,a1,a2,a3}, {%8,%9}, "     \
      "{%0,%1,%2,%3};\n\t}"                                                                             \
      : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3])                                        \
      : "r"(W0), "r"(W1), "r"(W2), "r"(W3), "r"(B0), "r"(B1))

constexpr int GEMV_RING = 4;   // super-blocks in flight per warp (RING - 1 copies ahead)
constexpr int GEMV_WARPS = 4;  // warps per CTA: GEMV_WARPS / parts tiles, each split over `parts` warps
constexpr int GEMV_STAGE_BYTES = 16 * 128;  // one super-block of a 16-row tile: 16 rows x 128 code bytes

struct GemvTcParams {
  const uint8_t *gmeta, *steps;
  int64_t N, K;
  int parts;  // warps splitting K for one tile (1, 2 or 4)
  GemvWorkspace ws;
  __nv_bfloat16 *y;
};

// dynamic shared memory: [warp][stage] code tiles (1024-aligned), mbarriers, reduction buffer
inline constexpr int gemv_smem_bytes() {
  return GEMV_WARPS * GEMV_RING * GEMV_STAGE_BYTES + GEMV_WARPS * GEMV_RING * 8 + GEMV_WARPS * 16 * 4 + 1024;
}

// Codes arrive by TMA: each warp runs its own GEMV_RING-deep ring of 16-row x 128-byte boxes (one
// super-block of its tile) with one mbarrier per stage.  The box is stored with the 128-byte
// swizzle (16-byte chunk j of row r at chunk j ^ (r & 7)); MMA row g (and g + 8) reads tile row
// pg = (g >> 1) | ((g & 1) << 2), so the two rows of one 8-lane shared-load phase differ in bit 2
// and their chunks never share banks.  Group words, step words, x and the group sums are small
// and come through the L1 cache, one super-block ahead.
__global__ void __launch_bounds__(32 * GEMV_WARPS, 4)
    gemv_int4_m1_tc_kernel(const __grid_constant__ CUtensorMap map_codes, GemvTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + GEMV_WARPS * GEMV_RING * GEMV_STAGE_BYTES);
  float *red = reinterpret_cast<float *>(bars + GEMV_WARPS * GEMV_RING);  // [GEMV_WARPS][16]
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = p.parts, T = GEMV_WARPS / P;
  const int tl = warp / P, part = warp - tl * P;
  const int64_t n_tiles = (p.N + 15) / 16;
  const int64_t tile = (int64_t)blockIdx.x * T + tl;
  const int g = lane >> 2, c = lane & 3;
  const bool active = tile < n_tiles;
  const int NS = (int)(p.K / 256);
  const int sb0 = active ? part * NS / P : 0, nsb = active ? (part + 1) * NS / P - sb0 : 0;
  const uint32_t ring = smem_u32(smem + warp * GEMV_RING * GEMV_STAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars + warp * GEMV_RING);
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0) {
    for (int s = 0; s < GEMV_RING; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // i-th super-block of this warp's range goes to stage i % RING; its wait parity is (i / RING) & 1
  auto issue = [&](int i) {
    const int s = i % GEMV_RING;
    mbar_arrive_expect_tx(bar0 + 8 * s, GEMV_STAGE_BYTES);
    tma_load_2d(ring + s * GEMV_STAGE_BYTES, &map_codes, bar0 + 8 * s, (sb0 + i) * 128, (int32_t)(tile * 16));
  };
  int issued = 0;
  if (lane == 0) {
    tma_prefetch_desc(&map_codes);
    for (; issued < GEMV_RING - 1 && issued < nsb; ++issued) issue(issued);  // weights need no x
  }
  const int pg = (g >> 1) | ((g & 1) << 2);
  int64_t r0 = tile * 16 + pg, r1 = r0 + 8;
  if (r0 >= p.N) r0 = p.N - 1;  // rows past the end are computed on a valid row and discarded
  if (r1 >= p.N) r1 = p.N - 1;
  const uint32_t *gm0 = reinterpret_cast<const uint32_t *>(p.gmeta + r0 * (p.K / 16)) + 4 * sb0 + c;
  const uint32_t *gm1 = reinterpret_cast<const uint32_t *>(p.gmeta + r1 * (p.K / 16)) + 4 * sb0 + c;
  const uint32_t *st0 = reinterpret_cast<const uint32_t *>(p.steps) + r0 * NS + sb0;
  const uint32_t *st1 = reinterpret_cast<const uint32_t *>(p.steps) + r1 * NS + sb0;
  uint32_t m0 = 0, m1 = 0, s0 = 0, s1 = 0;
  if (nsb > 0) {
    m0 = __ldg(gm0); m1 = __ldg(gm1);
    s0 = __ldg(st0); s1 = __ldg(st1);
  }
  pdl_wait();  // x in fragment order and its group sums are ready from here on

  // x operand: lane (g, c) feeds column g from its b0 slots when g == c, from b1 when g == c + 4;
  // other lanes read the zero block
  const bool on0 = (g == c), on1 = (g == c + 4);
  const uint4 *xb0 = reinterpret_cast<const uint4 *>(on0 ? p.ws.xperm + 16 * c + 128 * sb0 : p.ws.zero);
  const uint4 *xb1 = reinterpret_cast<const uint4 *>(on1 ? p.ws.xperm + 16 * (c + 4) + 128 * sb0 : p.ws.zero);
  const int xinc0 = on0 ? 32 : 0, xinc1 = on1 ? 32 : 0;  // uint4 per super-block (8 groups x 64 B)
  const float4 *gs = p.ws.gsum + 8 * sb0 + 2 * c;        // (B', X', 2^-a) of groups 2c, 2c+1; + 8 per sb
  // shared-memory offsets of this lane's four 16-byte chunks inside a stage
  const uint32_t o00 = pg * 128 + ((c ^ pg) << 4), o01 = pg * 128 + (((c + 4) ^ pg) << 4);
  const uint32_t o10 = (pg + 8) * 128 + ((c ^ pg) << 4), o11 = (pg + 8) * 128 + (((c + 4) ^ pg) << 4);

  float acc0 = 0.f, acc1 = 0.f;
  for (int i = 0; i < nsb; ++i) {
    // refill the stage released at the end of the previous turn (RING - 1 stages stay in flight)
    if (lane == 0 && issued < nsb) issue(issued++);
    const uint32_t cm0 = m0, cm1 = m1, cs0 = s0, cs1 = s1;
    if (i + 1 < nsb) {
      m0 = __ldg(gm0 + 4 * (i + 1)); m1 = __ldg(gm1 + 4 * (i + 1));
      s0 = __ldg(st0 + i + 1); s1 = __ldg(st1 + i + 1);
    }
    const float4 G0 = __ldg(gs), G1 = __ldg(gs + 1);
    gs += 8;
    const int s = i % GEMV_RING;
    if (!mbar_wait_suspend(bar0 + 8 * s, (uint32_t)((i / GEMV_RING) & 1), &abort_flag)) break;
    const uint32_t stg = ring + s * GEMV_STAGE_BYTES;
    const uint4 a00 = lds128(stg + o00), a10 = lds128(stg + o10);  // (r0 | r1, group c)
    const uint4 a01 = lds128(stg + o01), a11 = lds128(stg + o11);  // (r0 | r1, group c+4)
    __syncwarp();  // every lane has read the stage: the next turn may refill it
    // two independent accumulator chains (even / odd words) halve the MMA dependency latency
    float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t w00[4] = {a00.x, a00.y, a00.z, a00.w}, w01[4] = {a01.x, a01.y, a01.z, a01.w};
    const uint32_t w10[4] = {a10.x, a10.y, a10.z, a10.w}, w11[4] = {a11.x, a11.y, a11.z, a11.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 xv0 = __ldg(xb0 + j), xv1 = __ldg(xb1 + j);
      const uint32_t v00 = w00[j] >> 8, v10 = w10[j] >> 8, v01 = w01[j] >> 8, v11 = w11[j] >> 8;
      float(&acc)[4] = (j & 1) ? e : d;
      QL_GEMV_MMA("0x000F000F", "0x64006400", w00[j], w10[j], w01[j], w11[j], xv0.x, xv1.x);  // (n0, n4)
      QL_GEMV_MMA("0x00F000F0", "0x54005400", w00[j], w10[j], w01[j], w11[j], xv0.y, xv1.y);  // (n1, n5)
      QL_GEMV_MMA("0x000F000F", "0x64006400", v00, v10, v01, v11, xv0.z, xv1.z);              // (n2, n6)
      QL_GEMV_MMA("0x00F000F0", "0x54005400", v00, v10, v01, v11, xv0.w, xv1.w);              // (n3, n7)
    }
    xb0 += xinc0;
    xb1 += xinc1;
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] += e[q];
    // d0: (r0, group 2c)  d1: (r0, 2c+1)  d2: (r1, 2c)  d3: (r1, 2c+1)
    // S = sc * ss and Z = zc * zs, each one FMA from the byte placed in the mantissa of 2^23
    const float ss0 = f16_bits_to_f32(cs0), zs0 = f16_bits_to_f32(cs0 >> 16);
    const float ss1 = f16_bits_to_f32(cs1), zs1 = f16_bits_to_f32(cs1 >> 16);
    const float nss0 = -8388608.f * ss0, nzs0 = -8388608.f * zs0;
    const float nss1 = -8388608.f * ss1, nzs1 = -8388608.f * zs1;
    const float S00 = fmaf(byte_magic(cm0, 0), ss0, nss0) * G0.z, Z00 = fmaf(byte_magic(cm0, 1), zs0, nzs0);
    const float S01 = fmaf(byte_magic(cm0, 2), ss0, nss0) * G1.z, Z01 = fmaf(byte_magic(cm0, 3), zs0, nzs0);
    const float S10 = fmaf(byte_magic(cm1, 0), ss1, nss1) * G0.z, Z10 = fmaf(byte_magic(cm1, 1), zs1, nzs1);
    const float S11 = fmaf(byte_magic(cm1, 2), ss1, nss1) * G1.z, Z11 = fmaf(byte_magic(cm1, 3), zs1, nzs1);
    acc0 = fmaf(S00, fmaf(-Z00, G0.y, d[0] - G0.x), acc0);
    acc0 = fmaf(S01, fmaf(-Z01, G1.y, d[1] - G1.x), acc0);
    acc1 = fmaf(S10, fmaf(-Z10, G0.y, d[2] - G0.x), acc1);
    acc1 = fmaf(S11, fmaf(-Z11, G1.y, d[3] - G1.x), acc1);
  }
  if (abort_flag && lane == 0) {  // a wait gave up: let this warp's copies in flight land first
    for (int i = issued - GEMV_RING; i < issued; ++i) {
      if (i < 0) continue;
      const long long t0 = clock64();
      while (!mbar_try_wait(bar0 + 8 * (i % GEMV_RING), (uint32_t)((i / GEMV_RING) & 1)) &&
             clock64() - t0 < QL_WAIT_LIMIT_CYCLES) {
      }
    }
  }
  // the four lanes of a row hold its groups 2c, 2c+1: sum them
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
  acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
  acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
  if (c == 0) {
    red[warp * 16 + pg] = acc0;
    red[warp * 16 + pg + 8] = acc1;
  }
  __syncthreads();
  if (part == 0 && lane < 16 && active) {
    float sum = 0.f;
    for (int q = 0; q < P; ++q) sum += red[(warp + q) * 16 + lane];
    const int64_t r = tile * 16 + lane;
    if (r < p.N) p.y[r] = __float2bfloat16_rn(sum);
  }
}

}  // namespace ql
