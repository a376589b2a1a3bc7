// gemv.cuh -- decode-shaped layer y[M][N] = x[M][K] . W^T for small M.
//
// Simple form: one warp per output row; lane l takes chunks l, l+32, ... of
// the row (32 weights each: one int4 group, 16-byte coalesced loads), decodes
// the exact binary32 weights and accumulates x*w in fp32; a warp-shuffle
// reduction finishes the row.  The trip count over chunks is the same for
// every lane of a warp, so full-mask shuffles are always reached.
#pragma once
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

}  // namespace ql
