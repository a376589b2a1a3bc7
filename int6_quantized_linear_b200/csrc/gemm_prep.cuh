// gemm_prep.cuh -- the two short passes that let the tensor-core GEMM run on
// fp16 operands without giving up fp32 range.
//
// fp16 keeps 11 significant bits (bf16 keeps 8); rounding each weight to bf16
// alone puts the layer's error near 1% of rms(y), fp16 brings it to ~0.1%.
// fp16's range is what needs care, so both operands are scaled by exact
// powers of two that the epilogue undoes:
//
//  x:  a_m per token row, chosen so max_k |x[m][k]| * 2^a_m lies in
//      [2^15, 2^16).  A bf16 value scaled into that range is exactly an fp16
//      value unless it is more than 2^29 below the row's maximum.
//  W:  b_n per weight row, chosen so a bound on max_k |w[n][k]| times 2^b_n
//      lies in [2^14, 2^15) (headroom for the rounding to fp16).  The bound
//      comes from the metadata alone:  int4 |S|*max(|Z|, |15-Z|),
//      int6 (either storage) 32*|S|,  affine max(|bias|, |(2^bits-1)*scale + bias|).
//
// The epilogue undoes both scales with the combined exponent -(a_m + b_n), so
// no intermediate product can overflow or underflow where the result does not.
//
// Workspace layout (caller-provided, 256-byte aligned sections):
//   x16   fp16 [M][K]   scaled activations
//   xexp  s32  [M]      -a_m
//   wsc   f32  [N']     2^b_n   (N' = N rounded up to 256; rows N.. hold 0)
//   wexp  s32  [N']     -b_n    (rows N.. hold 0)
#pragma once
#include "formats.cuh"

namespace ql {

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct GemmWorkspace {
  __half *x16;
  int *xexp;
  float *wsc;
  int *wexp;
};

// the per-row weight scales are padded to whole 256-row tiles
__host__ __device__ inline size_t padded_rows(int64_t N) { return (size_t)((N + 255) / 256 * 256); }

inline size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return align256((size_t)M * K * 2) + align256((size_t)M * 4) + 2 * align256(padded_rows(N) * 4);
}

inline GemmWorkspace gemm_workspace_carve(void *base, int64_t M, int64_t N, int64_t K) {
  uint8_t *p = static_cast<uint8_t *>(base);
  GemmWorkspace w;
  w.x16 = reinterpret_cast<__half *>(p);
  p += align256((size_t)M * K * 2);
  w.xexp = reinterpret_cast<int *>(p);
  p += align256((size_t)M * 4);
  w.wsc = reinterpret_cast<float *>(p);
  p += align256(padded_rows(N) * 4);
  w.wexp = reinterpret_cast<int *>(p);
  return w;
}

// 2^e as a binary32 for e in [-126, 127]
QL_DEVI float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// d * 2^e for any e in [-252, 253] as two exact power-of-two multiplications: the result is the
// nearest binary32 of the exact product whenever that product is a normal float.
QL_DEVI float mul_pow2(float d, int e) {
  const int e1 = max(-126, min(127, e));
  return (d * exp2i(e1)) * exp2i(max(-126, min(127, e - e1)));
}

// Exponent that puts amax * 2^s into [2^top, 2^(top+1)); 0 for zero or non-finite.
QL_DEVI int scale_exponent(float amax, int top) {
  if (!(amax > 0.f) || !isfinite(amax)) return 0;
  int e = ((__float_as_int(amax) >> 23) & 0xff) - 127;  // floor(log2(amax)) for normal amax
  if (e == -127) e = -118 - __clz(__float_as_int(amax) & 0x7fffff);  // subnormal: m * 2^-149
  int s = top - e;
  return s < -126 ? -126 : (s > 126 ? 126 : s);
}

// One CTA of 256 threads per token row: find max|x|, then write the scaled fp16 row.  Within every
// 8-element chunk the elements are stored in the order k = 0,4,1,5,2,6,3,7 (pairs (0,4) (1,5) (2,6)
// (3,7)): the weight operand is written in the same order, which is the order a single bit operation
// pulls nibble pairs out of a code word (the MMA's sum over k does not depend on it).  Rows of up to
// X2F16_REGS * 256 16-byte vectors are read once and kept in registers; longer rows are read again for
// the conversion.
// DEP: launched as a programmatic dependent (of whatever precedes it on the stream) by the fp16 GEMV,
// whose streaming kernel is in turn its dependent: the pass lets that kernel start, waits for its own
// predecessor before reading x, and clears the first n_counters K-split counters (the grid has at
// least n_counters threads).
constexpr int X2F16_THREADS = 256, X2F16_REGS = 4;

QL_DEVI uint4 x_chunk_to_f16(uint4 v, float sc) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // pair j = (x[j], x[j + 4]): u[j / 2] holds x[j & ~1], x[j | 1]
    const uint32_t a = u[j >> 1], b = u[2 + (j >> 1)];
    const float lo = (j & 1) ? __uint_as_float(a & 0xffff0000u) : __uint_as_float(a << 16);
    const float hi = (j & 1) ? __uint_as_float(b & 0xffff0000u) : __uint_as_float(b << 16);
    const __half2 h = __floats2half2_rn(lo * sc, hi * sc);
    o[j] = *reinterpret_cast<const uint32_t *>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

QL_DEVI float chunk_amax(uint4 v, float amax) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(u[j] << 16)), fabsf(__uint_as_float(u[j] & 0xffff0000u))));
  return amax;
}

template <bool DEP = false>
__global__ void __launch_bounds__(X2F16_THREADS) x_to_f16_kernel(const __nv_bfloat16 *x, int64_t M, int64_t K,
                                                                 GemmWorkspace ws, int *counters = nullptr,
                                                                 int64_t n_counters = 0) {
  __shared__ float red[X2F16_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t m = blockIdx.x;
  const int64_t nv = K / 8;  // 16-byte vectors of the row
  const uint4 *row = reinterpret_cast<const uint4 *>(x + m * K);
  if constexpr (!DEP) pdl_launch_dependents();  // the GEMM's weight-scale pass needs nothing from here
  if constexpr (DEP) {
    pdl_launch_dependents();
    if (m < M && tid < nv) prefetch_l2(row + tid);
    pdl_wait();
    const int64_t t = m * X2F16_THREADS + tid;
    if (t < n_counters) counters[t] = 0;
  }
  if (m >= M) return;  // whole CTAs leave together
  const bool in_regs = nv <= (int64_t)X2F16_REGS * X2F16_THREADS;
  uint4 v[X2F16_REGS];
  float amax = 0.f;
  if (in_regs) {
#pragma unroll
    for (int r = 0; r < X2F16_REGS; ++r) {
      const int64_t i = tid + (int64_t)r * X2F16_THREADS;
      v[r] = i < nv ? __ldg(row + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int r = 0; r < X2F16_REGS; ++r) amax = chunk_amax(v[r], amax);
  } else {
    for (int64_t i = tid; i < nv; i += X2F16_THREADS) amax = chunk_amax(__ldg(row + i), amax);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < X2F16_THREADS / 32; ++w) amax = fmaxf(amax, red[w]);
  const int a = scale_exponent(amax, 15);
  const float sc = exp2i(a);
  uint4 *out = reinterpret_cast<uint4 *>(ws.x16 + m * K);
  if (in_regs) {
#pragma unroll
    for (int r = 0; r < X2F16_REGS; ++r) {
      const int64_t i = tid + (int64_t)r * X2F16_THREADS;
      if (i < nv) out[i] = x_chunk_to_f16(v[r], sc);
    }
  } else {
    for (int64_t i = tid; i < nv; i += X2F16_THREADS) out[i] = x_chunk_to_f16(__ldg(row + i), sc);
  }
  if (tid == 0) ws.xexp[m] = -a;
}

// One warp per weight row: bound max|w| from the metadata (lanes stride over the groups, then a
// max-reduction), pick b_n.  The grid covers the rows up to N rounded to 256: rows past N get
// scale 0 and exponent 0, so the padded columns of a tile are defined (and never stored).
template <int FMT, int BITS>
__device__ __forceinline__ void w_scale_row(const uint8_t *gmeta, const uint8_t *steps, int64_t N, int64_t K,
                                            int G, GemmWorkspace ws, int64_t n, int lane) {
  if (n >= N) {
    if (lane == 0) {
      ws.wsc[n] = 0.f;
      ws.wexp[n] = 0;
    }
    return;
  }
  float bound = 0.f;
  if constexpr (FMT == FMT_INT4) {
    const uint16_t *gm = reinterpret_cast<const uint16_t *>(gmeta) + n * (K / 32);
    const uint32_t *st = reinterpret_cast<const uint32_t *>(steps) + n * (K / 256);
    for (int64_t g = lane; g < K / 32; g += 32) {
      const uint32_t s = __ldg(st + (g >> 3));
      const float ss = f16_bits_to_f32(s), zs = f16_bits_to_f32(s >> 16);
      const uint32_t c = __ldg(gm + g);
      const float S = __fmul_rn((float)(c & 0xffu), ss);
      const float Z = __fmul_rn((float)(c >> 8), zs);
      bound = fmaxf(bound, __fmul_rn(fabsf(S), fmaxf(fabsf(Z), fabsf(__fsub_rn(15.f, Z)))));
    }
  } else if constexpr (FMT == FMT_INT6 || FMT == FMT_INT6P) {
    const int8_t *gm = reinterpret_cast<const int8_t *>(gmeta) + n * (K / 16);
    const uint16_t *st = reinterpret_cast<const uint16_t *>(steps) + n * (K / 256);
    for (int64_t g = lane; g < K / 16; g += 32) {
      const float step = f16_bits_to_f32(__ldg(st + (g >> 4)));
      bound = fmaxf(bound, __fmul_rn(32.f, fabsf(__fmul_rn((float)__ldg(gm + g), step))));
    }
  } else {
    const uint32_t *gm = reinterpret_cast<const uint32_t *>(gmeta) + n * (K / G);
    const float qmax = (float)((1 << BITS) - 1);
    for (int64_t g = lane; g < K / G; g += 32) {
      const uint32_t c = __ldg(gm + g);
      const float s = bf16_bits_to_f32(c), b = bf16_bits_to_f32(c >> 16);
      bound = fmaxf(bound, fmaxf(fabsf(b), fabsf(__fadd_rn(__fmul_rn(qmax, s), b))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bound = fmaxf(bound, __shfl_xor_sync(0xffffffffu, bound, o));
  if (lane == 0) {
    const int e = scale_exponent(bound, 14);
    ws.wsc[n] = exp2i(e);
    ws.wexp[n] = -e;
  }
}

// Launched as a programmatic dependent of the GEMM's x pass: it reads only the weights' metadata, so it
// runs alongside that pass, and waits for it before exiting -- the GEMM, a programmatic dependent of
// this kernel, then finds both passes' results complete.
template <int FMT, int BITS>
__global__ void __launch_bounds__(256) w_scale_kernel(const uint8_t *gmeta, const uint8_t *steps, int64_t N,
                                                       int64_t K, int G, GemmWorkspace ws) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t n = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  if (n < (int64_t)padded_rows(N)) w_scale_row<FMT, BITS>(gmeta, steps, N, K, G, ws, n, lane);
  pdl_wait();
}

}  // namespace ql
