// qlinear.cu -- the C ABI (include/qlinear.h): host-side validation, launch
// configuration and TMA descriptor encoding.  Single translation unit: the
// kernels live in the included .cuh files and share one device status word.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/qlinear.h"
#include "gemm_sm100.cuh"
#include "gemv.cuh"
#include "gemv_int6.cuh"
#include "gemv_f16.cuh"
#include "pack_dequant.cuh"

using namespace ql;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  int sms = 0;
  int major = 0, minor = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A CUDA call on the host failed: clear the runtime's last-error slot (a non-sticky error would
// otherwise make the next call's launch check report this failure as its own) and say so.
inline ql_status cuda_failed() {
  (void)cudaGetLastError();
  return QL_ERR_CUDA;
}

ql_status device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_failed();
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return cuda_failed();
    d.init = true;
  }
  *out = &d;
  return QL_OK;
}

ql_status check_desc(const ql_desc *d) {
  if (!d) return QL_ERR_NULL;
  if (d->N < 1 || d->K < 1) return QL_ERR_SHAPE;
  switch (d->fmt) {
    case QL_INT4_NSS:
    case QL_INT6_SYM:
    case QL_INT6_PLANAR:
      if (d->K % 256 != 0) return QL_ERR_SHAPE;
      return QL_OK;
    case QL_AFFINE_U32:
      if (d->bits != 2 && d->bits != 4 && d->bits != 8) return QL_ERR_SHAPE;
      if (d->group != 32 && d->group != 64 && d->group != 128) return QL_ERR_SHAPE;
      if (d->K % d->group != 0 || (d->K * d->bits) % 128 != 0) return QL_ERR_SHAPE;
      return QL_OK;
    default:
      return QL_ERR_UNSUPPORTED;
  }
}

void sizes(const ql_desc *d, size_t *c, size_t *g, size_t *s) {
  const size_t N = (size_t)d->N, K = (size_t)d->K;
  switch (d->fmt) {
    case QL_INT4_NSS: *c = N * K / 2; *g = N * (K / 32) * 2; *s = N * (K / 256) * 4; break;
    case QL_INT6_SYM:
    case QL_INT6_PLANAR: *c = N * 3 * K / 4; *g = N * (K / 16); *s = N * (K / 256) * 2; break;
    default: *c = N * K * d->bits / 8; *g = N * (K / d->group) * 4; *s = 0; break;
  }
}

ql_status check_packed(const ql_desc *d, const void *codes, const void *gmeta, const void *steps) {
  if (!codes || !gmeta || (d->fmt != QL_AFFINE_U32 && !steps)) return QL_ERR_NULL;
  if (!aligned16(codes) || !aligned16(gmeta) || (d->fmt != QL_AFFINE_U32 && !aligned16(steps)))
    return QL_ERR_ALIGN;
  return QL_OK;
}

inline int grid_for(int64_t units, int sms, int per_sm = 8) {
  int64_t g = (units + 255) / 256;
  const int64_t cap = (int64_t)sms * per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

inline ql_status launched() {
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

WeightPtrs make_ptrs(const ql_desc *d, const ql_packed_const *w) {
  WeightPtrs p;
  p.codes = static_cast<const uint8_t *>(w->codes);
  p.gmeta = static_cast<const uint8_t *>(w->gmeta);
  p.steps = static_cast<const uint8_t *>(w->steps);
  p.K = d->K;
  p.G = d->group;
  return p;
}

// ---- TMA descriptors ---------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A tensor map is a pure function of these arguments, so the last few encodings are kept per host
// thread and reused: a decode loop calls the same layers with the same buffers over and over, and the
// encoding is host time on every call's critical path.
struct TmapKey {
  const void *base;
  uint64_t inner, outer, row_bytes;
  uint32_t box_inner, box_outer;
  int dt, sw;
  bool operator==(const TmapKey &o) const {
    return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
           box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && sw == o.sw;
  }
};

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  constexpr int kEntries = 32;
  struct Entry {
    TmapKey key;
    CUtensorMap map;
    bool valid;
  };
  static thread_local Entry cache[kEntries] = {};
  static thread_local int next = 0;
  const TmapKey key{base, inner, outer, row_bytes, box_inner, box_outer, (int)dt, (int)sw};
  for (int i = 0; i < kEntries; ++i)
    if (cache[i].valid && cache[i].key == key) {
      *map = cache[i].map;
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  if (fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cache[next] = Entry{key, *map, true};
  next = (next + 1) % kEntries;
  return true;
}

template <int FMT, int BITS, int TT, int CPS = 1>
ql_status launch_gemm_tt(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                         void *y, void *workspace, cudaStream_t st, int sms) {
  using namespace ql::gemm;
  const int64_t N = d->N, K = d->K;
  const uint64_t row_bytes = (uint64_t)K * code_bits(FMT, BITS) / 8;
  const GemmWorkspace ws = gemm_workspace_carve(workspace, M, N, K);
  // pass 1: scaled fp16 activations; pass 2: per-row weight scales
  // the weight-scale pass and the GEMM are programmatic dependents: each starts while the kernel before
  // it drains (the scale pass needs nothing from the x pass and waits for it only before exiting; the
  // GEMM waits after its set-up)
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  x_to_f16_kernel<false><<<(unsigned)M, X2F16_THREADS, 0, st>>>(static_cast<const __nv_bfloat16 *>(x), M, K, ws);
  {
    cudaLaunchConfig_t wc = {};
    wc.gridDim = dim3((unsigned)(((int64_t)padded_rows(N) * 32 + 255) / 256));
    wc.blockDim = dim3(256);
    wc.stream = st;
    wc.attrs = pdl;
    wc.numAttrs = 1;
    if (cudaLaunchKernelEx(&wc, w_scale_kernel<FMT, BITS>, static_cast<const uint8_t *>(w->gmeta),
                           static_cast<const uint8_t *>(w->steps), N, K, d->group, ws) != cudaSuccess)
      return cuda_failed();
  }
  CUtensorMap mx, mc;
  if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.x16, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, BK, TT,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cuda_failed();
  // int6 planar: a k-step's codes are three 16-byte pieces of its super-block (two of the low plane,
  // one of the high plane), loaded as three boxes of 16 bytes x BN rows
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, row_bytes, (uint64_t)N, row_bytes,
                 FMT == FMT_INT6P ? 16u : (uint32_t)p_row_bytes(FMT, BITS), BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cuda_failed();
  Params p;
  p.M = M; p.N = N; p.K = K; p.G = d->group;
  p.bias = static_cast<const __nv_bfloat16 *>(bias);
  p.gmeta = static_cast<const uint8_t *>(w->gmeta);
  p.steps = static_cast<const uint8_t *>(w->steps);
  p.y = static_cast<__nv_bfloat16 *>(y);
  p.ws = ws;
  const int smem = smem_bytes(FMT, BITS, TT);
  auto kern = gemm_kernel<FMT, BITS, TT, CPS>;
  static thread_local int configured_dev = -1;  // per (kernel instantiation, thread)
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return cuda_failed();
    configured_dev = dev;
  }
  const int64_t tiles = ((M + TT - 1) / TT) * ((N + BN - 1) / BN);
  const int slots = CPS * sms;
  const int grid = (int)(tiles < slots ? tiles : slots);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(num_threads(TT, CPS));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mx, mc, p) != cudaSuccess) return cuda_failed();
  return launched();
}

// Up to 32 tokens: tiles of 32 tokens (MMA N = 32), so no MMA runs on padding tokens -- two CTAs an SM
// when the layer has more 128-row tiles than SMs (every tile then runs at once instead of some SMs
// taking two in turn); from 33 tokens: tiles of 256 tokens.  Both take 128 weight rows as the MMA's
// M = 128 operand.
template <int FMT, int BITS>
ql_status launch_gemm(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                      void *y, void *workspace, cudaStream_t st, int sms) {
  if (M <= gemm::TT_SMALL) {
    if ((d->N + gemm::BN - 1) / gemm::BN > sms)
      return launch_gemm_tt<FMT, BITS, gemm::TT_SMALL, 2>(d, w, x, M, bias, y, workspace, st, sms);
    return launch_gemm_tt<FMT, BITS, gemm::TT_SMALL>(d, w, x, M, bias, y, workspace, st, sms);
  }
  return launch_gemm_tt<FMT, BITS, gemm::BM>(d, w, x, M, bias, y, workspace, st, sms);
}

// Affine layers the tensor-core GEMVs serve: group 32 or 64, K a multiple of 256 (the integer
// multi-token kernel up to 8 tokens, the fp16 kernel from 9 to 32).
inline bool affine_tc(const ql_desc *d) { return (d->group == 32 || d->group == 64) && d->K % 256 == 0; }

// Which GEMV calls run on the tensor-core GEMM: affine with other groups from M = 8 (measured faster
// there than on the CUDA-core kernel: M=32 70-74 us vs 537-551 us).  int4 and int6 have tensor-core
// GEMVs over their whole GEMV range (M <= 8).
inline bool gemv_runs_on_gemm(const ql_desc *d, int64_t M) {
  return d->fmt == QL_AFFINE_U32 && !affine_tc(d) && M >= 8;
}

inline size_t gemv_call_workspace_bytes(const ql_desc *d, int64_t M) {
  const size_t own = gemv_workspace_bytes(M, d->N, d->K);
  if (!gemv_runs_on_gemm(d, M)) return own;
  const size_t gemm = gemm_workspace_bytes(M, d->N, d->K);
  return own > gemm ? own : gemm;
}

template <int FMT, int BITS>
ql_status launch_gemm(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                      void *y, void *workspace, cudaStream_t st, int sms);

// Multi-token tensor-core GEMV (int4 at 2..8 tokens; 2-, 4- and 8-bit affine with group 32 or 64 at
// 1..8 tokens): x preparation, then the streaming kernel as its programmatic dependent.
template <int FMT, int BITS, int G>
ql_status launch_gemv_mt(const ql_desc *d, const ql_packed_const *w, const __nv_bfloat16 *xb, int64_t M,
                         const __nv_bfloat16 *bb, __nv_bfloat16 *yb, void *workspace, cudaStream_t st, int sms) {
  using L = MtLayout<FMT, BITS, G>;
  const int64_t N = d->N, K = d->K, NS = K / 256, TG = (N + 63) / 64;
  const GemvWorkspace ws = gemv_workspace_carve(workspace, M, N, K);
  cudaLaunchAttribute pa[1];
  pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pa[0].val.programmaticStreamSerializationAllowed = 1;
  {
    const int64_t threads = std::max<int64_t>(4 * M * (K / 32), TG);
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3((unsigned)((threads + 255) / 256));
    pc.blockDim = dim3(256);
    pc.stream = st;
    pc.attrs = pa;
    pc.numAttrs = 1;
    if (cudaLaunchKernelEx(&pc, gemv_xprep_mt_kernel, xb, M, K, TG, ws) != cudaSuccess) return cuda_failed();
  }
  GemvMtParams p;
  p.codes = static_cast<const uint8_t *>(w->codes);
  p.gmeta = static_cast<const uint8_t *>(w->gmeta);
  p.steps = static_cast<const uint8_t *>(w->steps);
  p.bias = bb;
  p.N = N;
  p.K = K;
  p.M = (int)M;
  // split K over the CTAs of a 64-row group so that the groups fill one wave of resident CTAs
  p.split = split_k(TG, (int64_t)sms * gemv_mt_ctas_per_sm<FMT>(), NS, FMT == FMT_INT4);
  const int64_t ctas = p.split.total(TG);
  if (p.split.P + (p.split.extra > 0) > 1 && ctas > GEMV_MT_MAX_CTAS) return QL_ERR_RANGE;  // partial sums' room
  p.ws = ws;
  p.y = yb;
  const uint64_t code_row = FMT == FMT_INT4 ? (uint64_t)K / 2 : (uint64_t)K * BITS / 8;
  const uint64_t meta_row = FMT == FMT_INT4 ? (uint64_t)K / 16 : (uint64_t)K / G * 4;
  CUtensorMap mc, mg;  // codes: boxes of 64 rows x CODE_BOX bytes, swizzled; group words: 64 rows x META_ROW
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, code_row, (uint64_t)N, code_row, L::CODE_BOX, 64,
                 L::CODE_BOX == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_2d(&mg, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->gmeta, meta_row, (uint64_t)N, meta_row, L::META_ROW, 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cuda_failed();
  auto kern = [] {
    if constexpr (FMT == FMT_INT4) return gemv_mt_int4_kernel;
    else return gemv_mt_affine_kernel<BITS, G>;
  }();
  static thread_local int configured_dev = -1;  // per instantiation and thread
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
      return cuda_failed();
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(GEMV_MT_THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cfg.attrs = pa;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mc, mg, p) != cudaSuccess) return cuda_failed();
  return launched();
}

// Tensor-core int6 GEMV at 1..TM tokens: x preparation, then the streaming kernel as its dependent.
template <int TM, bool PLANAR>
ql_status launch_gemv_int6(const ql_desc *d, const ql_packed_const *w, const __nv_bfloat16 *xb, int64_t M,
                           const __nv_bfloat16 *bb, __nv_bfloat16 *yb, void *workspace, cudaStream_t st, int sms) {
  using L = Int6Layout<TM>;
  const int64_t N = d->N, K = d->K, NS = K / 256, TG = (N + 63) / 64;
  const GemvWorkspace ws = gemv_workspace_carve(workspace, M, N, K);
  // split K over the CTAs of a 64-row group so that the groups fill one wave of resident CTAs
  const SplitK split = split_k(TG, (int64_t)sms * GEMV6_CTAS_PER_SM, NS, true);
  const int64_t ctas = split.total(TG);
  const bool splits = split.P + (split.extra > 0) > 1;  // some group's K is split
  if (splits && ctas > GEMV_MT_MAX_CTAS) return QL_ERR_RANGE;  // partial sums' room
  cudaLaunchAttribute pa[1];
  pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pa[0].val.programmaticStreamSerializationAllowed = 1;
  {
    const int64_t threads = std::max<int64_t>(M * (K / 16), splits ? TG : 0);
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3((unsigned)((threads + 255) / 256));
    pc.blockDim = dim3(256);
    pc.stream = st;
    pc.attrs = pa;
    pc.numAttrs = 1;
    if (cudaLaunchKernelEx(&pc, gemv_xprep_int6_kernel<PLANAR>, xb, M, K, splits ? TG : (int64_t)0, ws) !=
        cudaSuccess)
      return cuda_failed();
  }
  Gemv6Params p;
  p.codes = static_cast<const uint8_t *>(w->codes);
  p.sc = static_cast<const uint8_t *>(w->gmeta);
  p.steps = static_cast<const uint16_t *>(w->steps);
  p.bias = bb;
  p.N = N;
  p.K = K;
  p.M = (int)M;
  p.split = split;
  p.ws = ws;
  p.y = yb;
  const uint64_t code_row = (uint64_t)K * 3 / 4, sc_row = (uint64_t)K / 16;
  CUtensorMap mc, ms;  // codes: 64 rows x 208 bytes (a super-block and 16 bytes more); scale codes: 64 x 16 B
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, code_row, (uint64_t)N, code_row, GEMV6_CODE_ROW, 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&ms, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->gmeta, sc_row, (uint64_t)N, sc_row, 16, 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cuda_failed();
  auto kern = gemv_int6_kernel<TM, PLANAR>;
  static thread_local int configured_dev = -1;  // per instantiation and thread
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
      return cuda_failed();
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(GEMV6_THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cfg.attrs = pa;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mc, ms, p) != cudaSuccess) return cuda_failed();
  return launched();
}

// fp16 tensor-core GEMV for affine at 9..32 tokens (NT column tiles of 8): the x pass (fp16, one
// exponent per token, programmatic dependent of what precedes it), then the streaming kernel as its
// dependent.  x16 and the token exponents sit at the start of the workspace (the GEMM's layout), the
// partial sums and counters of a K split where the GEMV layout has them (past 7 M K bytes).
template <int BITS, int G, int NT>
ql_status launch_gemv_f16(const ql_desc *d, const ql_packed_const *w, const __nv_bfloat16 *xb, int64_t M,
                          const __nv_bfloat16 *bb, __nv_bfloat16 *yb, void *workspace, cudaStream_t st, int sms) {
  using L = F16Layout<BITS, G, NT>;
  const int64_t N = d->N, K = d->K, NS = K / 256, TG = (N + 63) / 64;
  const GemmWorkspace gw = gemm_workspace_carve(workspace, M, N, K);
  const GemvWorkspace vw = gemv_workspace_carve(workspace, M, N, K);
  const SplitK split = split_k(TG, (int64_t)sms * L::CTAS, NS, false);
  const int64_t ctas = split.total(TG);
  const bool splits = split.P > 1;
  if (splits && ctas > GEMV_MT_MAX_CTAS) return QL_ERR_RANGE;  // partial sums' room
  cudaLaunchAttribute pa[1];
  pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pa[0].val.programmaticStreamSerializationAllowed = 1;
  {
    const int64_t n_counters = splits ? TG : 0;
    const int64_t blocks = std::max<int64_t>(M, (n_counters + X2F16_THREADS - 1) / X2F16_THREADS);  // a CTA per token row
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3((unsigned)blocks);
    pc.blockDim = dim3(X2F16_THREADS);
    pc.stream = st;
    pc.attrs = pa;
    pc.numAttrs = 1;
    if (cudaLaunchKernelEx(&pc, x_to_f16_kernel<true>, xb, M, K, gw, vw.counters, n_counters) != cudaSuccess)
      return cuda_failed();
  }
  GemvF16Params p;
  p.gmeta = static_cast<const uint8_t *>(w->gmeta);
  p.bias = bb;
  p.xexp = gw.xexp;
  p.N = N;
  p.K = K;
  p.M = (int)M;
  p.split = split;
  p.ws = vw;
  p.y = yb;
  const uint64_t code_row = (uint64_t)K * BITS / 8, meta_row = (uint64_t)K / G * 4;
  CUtensorMap mc, mg, mx;  // codes: 64 rows x CODE_BOX bytes, swizzled; group words: 64 x META_ROW; x: 8 NT x 32 halves
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, code_row, (uint64_t)N, code_row, L::CODE_BOX, 64,
                 L::CODE_BOX == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode_2d(&mg, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->gmeta, meta_row, (uint64_t)N, meta_row, L::META_ROW, 64,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, gw.x16, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 32,
                 (uint32_t)L::XROWS, CU_TENSOR_MAP_SWIZZLE_64B))
    return cuda_failed();
  auto kern = gemv_f16_kernel<BITS, G, NT>;
  static thread_local int configured_dev = -1;  // per instantiation and thread
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
      return cuda_failed();
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(GEMV_MT_THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cfg.attrs = pa;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mc, mg, mx, p) != cudaSuccess) return cuda_failed();
  return launched();
}

// M = 1 on the diagonal-x kernel (int4, or 4-bit affine with group 32 / 64): each CTA converts its part
// of x, then streams four 16-row tiles over it (+ the kernel that adds the parts when K is split)
template <int FMT, int G>
ql_status launch_gemv_m1(const ql_desc *d, const ql_packed_const *w, const __nv_bfloat16 *xb,
                         const __nv_bfloat16 *bb, __nv_bfloat16 *yb, void *workspace, cudaStream_t st, int sms) {
  using L = M1Layout<FMT, G>;
  const int64_t M = 1;
  const int64_t NS = d->K / 256, n_tiles = (d->N + 15) / 16, groups = (n_tiles + GEMV_WARPS - 1) / GEMV_WARPS;
  // split K so that the tile groups fill the resident CTA slots, and so that each part's x fits the
  // CTA's blocks; the parts' sums go through the workspace (16 floats a tile and part)
  int64_t P = std::max<int64_t>(1, std::min<int64_t>(NS, (int64_t)sms * GEMV_CTAS_PER_SM / groups));
  P = std::max<int64_t>(P, (NS + L::XSB_MAX - 1) / L::XSB_MAX);
  if (P > 1 && groups * GEMV_WARPS * P * 16 > (int64_t)gemv_partial_floats(M, d->N, d->K)) return QL_ERR_RANGE;
  const GemvWorkspace ws = gemv_workspace_carve(workspace, M, d->N, d->K);
  GemvTcParams p;
  p.codes = static_cast<const uint8_t *>(w->codes);
  p.gmeta = static_cast<const uint8_t *>(w->gmeta);
  p.steps = static_cast<const uint8_t *>(w->steps);
  p.bias = bb;
  p.x = xb;
  p.N = d->N;
  p.K = d->K;
  p.P = (int)P;
  p.partial = ws.partial;
  p.y = yb;
  const uint64_t gm_row = (uint64_t)NS * L::GM_ROW;  // group-word bytes a row
  CUtensorMap mc, mg;  // codes as [N][K/2] bytes, boxes of 16 rows x 128 bytes, 128-byte swizzle;
                       // group words as [N][gm_row] bytes, boxes of 16 rows x GM_ROW bytes
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)d->K / 2, (uint64_t)d->N,
                 (uint64_t)d->K / 2, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mg, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->gmeta, gm_row, (uint64_t)d->N, gm_row, L::GM_ROW, 16,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cuda_failed();
  auto kern = FMT == FMT_INT4 ? gemv_int4_m1_tc_kernel : gemv_affine4_m1_tc_kernel<G>;
  static thread_local int configured_dev = -1;  // per instantiation and thread
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
      return cuda_failed();
    configured_dev = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * P));
  cfg.blockDim = dim3(32 * GEMV_WARPS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // programmatic dependent of whatever precedes it
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mc, mg, p) != cudaSuccess) return cuda_failed();
  if (P > 1) {  // the parts' sums, added by the kernel that depends on this one
    cudaLaunchConfig_t rc = {};
    rc.gridDim = dim3((unsigned)((d->N + 255) / 256));
    rc.blockDim = dim3(256);
    rc.stream = st;
    rc.attrs = attr;
    rc.numAttrs = 1;
    if (cudaLaunchKernelEx(&rc, gemv_m1_sum_parts, (const float *)ws.partial, (int)P, (int64_t)d->N, bb, yb) !=
        cudaSuccess)
      return cuda_failed();
  }
  return launched();
}

template <int FMT, int BITS>
ql_status launch_gemv(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                      void *y, void *workspace, cudaStream_t st, int sms) {
  const auto *xb = static_cast<const __nv_bfloat16 *>(x);
  auto *yb = static_cast<__nv_bfloat16 *>(y);
  const auto *bb = static_cast<const __nv_bfloat16 *>(bias);
  if (gemv_runs_on_gemm(d, M)) return launch_gemm<FMT, BITS>(d, w, x, M, bias, y, workspace, st, sms);
  if constexpr (FMT == FMT_INT4) {
    if (M >= 2) return launch_gemv_mt<FMT_INT4, 4, 32>(d, w, xb, M, bb, yb, workspace, st, sms);
  }
  if constexpr (FMT == FMT_INT6 || FMT == FMT_INT6P) {  // M <= 8; dense or planar code storage
    constexpr bool PL = FMT == FMT_INT6P;
    if (M == 1) return launch_gemv_int6<1, PL>(d, w, xb, M, bb, yb, workspace, st, sms);
    if (M == 2) return launch_gemv_int6<2, PL>(d, w, xb, M, bb, yb, workspace, st, sms);
    if (M <= 4) return launch_gemv_int6<4, PL>(d, w, xb, M, bb, yb, workspace, st, sms);
    return launch_gemv_int6<8, PL>(d, w, xb, M, bb, yb, workspace, st, sms);
  }
  if constexpr (FMT == FMT_AFFINE) {  // bits 2, 4, 8
    if constexpr (BITS == 4) {  // one token: the diagonal-x kernel of int4 (the same nibble layout)
      if (affine_tc(d) && M == 1)
        return d->group == 64 ? launch_gemv_m1<FMT_AFFINE, 64>(d, w, xb, bb, yb, workspace, st, sms)
                              : launch_gemv_m1<FMT_AFFINE, 32>(d, w, xb, bb, yb, workspace, st, sms);
    }
    if (affine_tc(d) && M <= 8) {
      if (d->group == 64) return launch_gemv_mt<FMT_AFFINE, BITS, 64>(d, w, xb, M, bb, yb, workspace, st, sms);
      return launch_gemv_mt<FMT_AFFINE, BITS, 32>(d, w, xb, M, bb, yb, workspace, st, sms);
    }
    if (affine_tc(d)) {  // 9..32 tokens
      if (d->group == 64)
        return M <= 16 ? launch_gemv_f16<BITS, 64, 2>(d, w, xb, M, bb, yb, workspace, st, sms)
                       : launch_gemv_f16<BITS, 64, 4>(d, w, xb, M, bb, yb, workspace, st, sms);
      return M <= 16 ? launch_gemv_f16<BITS, 32, 2>(d, w, xb, M, bb, yb, workspace, st, sms)
                     : launch_gemv_f16<BITS, 32, 4>(d, w, xb, M, bb, yb, workspace, st, sms);
    }
  }
  if constexpr (FMT == FMT_INT4) {
    if (M == 1) return launch_gemv_m1<FMT_INT4, 32>(d, w, xb, bb, yb, workspace, st, sms);
  }
  if constexpr (FMT == FMT_AFFINE) {  // groups without the multi-token kernel, M < 8: CUDA cores
    const WeightPtrs p = make_ptrs(d, w);
    const int64_t rows_per_block = 8;
    int64_t g = (d->N + rows_per_block - 1) / rows_per_block;
    const int64_t cap = (int64_t)sms * 16;
    if (g > cap) g = cap;
    if (M == 1)
      gemv_simple_kernel<FMT, BITS, 1><<<(int)g, 256, 0, st>>>(p, d->N, xb, (int)M, bb, yb);
    else if (M == 2)
      gemv_simple_kernel<FMT, BITS, 2><<<(int)g, 256, 0, st>>>(p, d->N, xb, (int)M, bb, yb);
    else if (M <= 4)
      gemv_simple_kernel<FMT, BITS, 4><<<(int)g, 256, 0, st>>>(p, d->N, xb, (int)M, bb, yb);
    else
      gemv_simple_kernel<FMT, BITS, 8><<<(int)g, 256, 0, st>>>(p, d->N, xb, (int)M, bb, yb);
    return launched();
  } else {
    return QL_ERR_UNSUPPORTED;  // int4 and int6 returned above for every M in range
  }
}

}  // namespace

// ---- the GEMM for callers that cannot allocate -------------------------------
// Some callers of this library may not allocate device memory at all: plug-in
// and custom-op interfaces of inference runtimes hand an op its input and
// output pointers but no allocator, and serving processes that reserve all of
// HBM up front for their own pool would see cudaMalloc fail (or stall the
// device while it synchronises).  qlinear_gemm_noalloc serves them with the
// GEMM's workspace taken from this fixed device array instead.
#define QL_NOALLOC_SCRATCH_BYTES (32u << 20)  // 32 MiB on every GPU that loads the library
static __device__ __align__(256) unsigned char g_gemm_noalloc_scratch[QL_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_gemm_noalloc_scratch per device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
void *g_noalloc_addr[kMaxDevices] = {};

ql_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_failed();
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemm_noalloc_scratch) != cudaSuccess || p == nullptr) return cuda_failed();
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return QL_OK;
}
}  // namespace

extern "C" {

int32_t qlinear_version(void) { return 1; }

const char *qlinear_status_string(ql_status s) {
  switch (s) {
    case QL_OK: return "ok";
    case QL_ERR_NULL: return "a required pointer is NULL";
    case QL_ERR_SHAPE: return "shape, bit width or group size not allowed for this format";
    case QL_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case QL_ERR_RANGE:
      return "value out of range: M for this entry point, a problem larger than the fixed scratch array, "
             "or (from qlinear_sync_status) an encoder input outside its domain";
    case QL_ERR_UNSUPPORTED: return "unknown format or unsupported device";
    case QL_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case QL_ERR_TIMEOUT: return "a device-side bounded wait gave up";
  }
  return "unknown status";
}

ql_status qlinear_packed_bytes(const ql_desc *d, size_t *c, size_t *g, size_t *s) {
  if (!c || !g || !s) return QL_ERR_NULL;
  const ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  sizes(d, c, g, s);
  return QL_OK;
}

ql_status qlinear_pack(const ql_desc *d, const ql_unpacked *in, const ql_packed *out, ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!in || !out || !in->q || !in->meta0) return QL_ERR_NULL;
  if ((d->fmt == QL_INT4_NSS && (!in->meta1 || !in->step0 || !in->step1)) ||
      ((d->fmt == QL_INT6_SYM || d->fmt == QL_INT6_PLANAR) && !in->step0) ||
      (d->fmt == QL_AFFINE_U32 && !in->meta1))
    return QL_ERR_NULL;
  if ((st = check_packed(d, out->codes, out->gmeta, out->steps)) != QL_OK) return st;
  const void *ins[5] = {in->q, in->meta0, in->meta1, in->step0, in->step1};
  for (const void *p : ins)
    if (p && !aligned16(p)) return QL_ERR_ALIGN;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  PackArgs a;
  a.N = d->N; a.K = d->K; a.bits = d->bits; a.G = d->group;
  a.q = static_cast<const uint8_t *>(in->q);
  a.meta0 = static_cast<const uint8_t *>(in->meta0);
  a.meta1 = static_cast<const uint8_t *>(in->meta1);
  a.step0 = static_cast<const uint16_t *>(in->step0);
  a.step1 = static_cast<const uint16_t *>(in->step1);
  a.codes = static_cast<uint8_t *>(out->codes);
  a.gmeta = static_cast<uint8_t *>(out->gmeta);
  a.steps = static_cast<uint8_t *>(out->steps);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t NK = d->N * d->K;
  switch (d->fmt) {
    case QL_INT4_NSS: pack_int4_kernel<<<grid_for(NK / 32 + NK / 128, di->sms), 256, 0, s>>>(a); break;
    case QL_INT6_SYM: pack_int6_kernel<<<grid_for(NK / 64 + NK / 128, di->sms), 256, 0, s>>>(a); break;
    case QL_INT6_PLANAR: pack_int6p_kernel<<<grid_for(NK / 32 + NK / 128, di->sms), 256, 0, s>>>(a); break;
    default: {
      const int g = grid_for(NK * d->bits / 128 + NK / d->group, di->sms);
      if (d->bits == 2) pack_affine_kernel<2><<<g, 256, 0, s>>>(a);
      else if (d->bits == 4) pack_affine_kernel<4><<<g, 256, 0, s>>>(a);
      else pack_affine_kernel<8><<<g, 256, 0, s>>>(a);
    }
  }
  return launched();
}

ql_status qlinear_unpack(const ql_desc *d, const ql_packed_const *in, const ql_unpacked_out *out,
                         ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!in || !out || !out->q) return QL_ERR_NULL;
  if ((st = check_packed(d, in->codes, in->gmeta, in->steps)) != QL_OK) return st;
  const void *outs[5] = {out->q, out->meta0, out->meta1, out->step0, out->step1};
  for (const void *p : outs)
    if (p && !aligned16(p)) return QL_ERR_ALIGN;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  UnpackArgs a;
  a.N = d->N; a.K = d->K; a.bits = d->bits; a.G = d->group;
  a.codes = static_cast<const uint8_t *>(in->codes);
  a.gmeta = static_cast<const uint8_t *>(in->gmeta);
  a.steps = static_cast<const uint8_t *>(in->steps);
  a.q = static_cast<uint8_t *>(out->q);
  a.meta0 = static_cast<uint8_t *>(out->meta0);
  a.meta1 = static_cast<uint8_t *>(out->meta1);
  a.step0 = static_cast<uint16_t *>(out->step0);
  a.step1 = static_cast<uint16_t *>(out->step1);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t NK = d->N * d->K;
  switch (d->fmt) {
    case QL_INT4_NSS: unpack_int4_kernel<<<grid_for(NK / 32 * 2 + NK / 256, di->sms), 256, 0, s>>>(a); break;
    case QL_INT6_SYM: unpack_int6_kernel<<<grid_for(NK / 64 + NK / 16, di->sms), 256, 0, s>>>(a); break;
    case QL_INT6_PLANAR: unpack_int6p_kernel<<<grid_for(NK / 32 + NK / 16, di->sms), 256, 0, s>>>(a); break;
    default: {
      const int g = grid_for(NK * d->bits / 32 + NK / d->group, di->sms);
      if (d->bits == 2) unpack_affine_kernel<2><<<g, 256, 0, s>>>(a);
      else if (d->bits == 4) unpack_affine_kernel<4><<<g, 256, 0, s>>>(a);
      else unpack_affine_kernel<8><<<g, 256, 0, s>>>(a);
    }
  }
  return launched();
}

ql_status qlinear_dequant(const ql_desc *d, const ql_packed_const *w, void *out, int32_t out_dtype,
                          ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!w || !out) return QL_ERR_NULL;
  if ((st = check_packed(d, w->codes, w->gmeta, w->steps)) != QL_OK) return st;
  if (!aligned16(out)) return QL_ERR_ALIGN;
  if (out_dtype != QL_OUT_F32 && out_dtype != QL_OUT_BF16) return QL_ERR_SHAPE;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  const WeightPtrs p = make_ptrs(d, w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int g = grid_for(d->N * d->K / 32, di->sms);
  const bool bf = out_dtype == QL_OUT_BF16;
#define QL_DQ(F, B)                                                        \
  do {                                                                     \
    if (bf) dequant_kernel<F, B, true><<<g, 256, 0, s>>>(p, d->N, out);    \
    else dequant_kernel<F, B, false><<<g, 256, 0, s>>>(p, d->N, out);      \
  } while (0)
  switch (d->fmt) {
    case QL_INT4_NSS: QL_DQ(FMT_INT4, 4); break;
    case QL_INT6_SYM: QL_DQ(FMT_INT6, 6); break;
    case QL_INT6_PLANAR: QL_DQ(FMT_INT6P, 6); break;
    default:
      if (d->bits == 2) QL_DQ(FMT_AFFINE, 2);
      else if (d->bits == 4) QL_DQ(FMT_AFFINE, 4);
      else QL_DQ(FMT_AFFINE, 8);
  }
#undef QL_DQ
  return launched();
}

ql_status qlinear_gemv_workspace_bytes(const ql_desc *d, int64_t M, size_t *bytes) {
  const ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!bytes) return QL_ERR_NULL;
  const int64_t mmax = d->fmt == QL_AFFINE_U32 ? 32 : 8;
  if (M < 1 || M > mmax) return QL_ERR_RANGE;
  *bytes = gemv_call_workspace_bytes(d, M);
  return QL_OK;
}

static ql_status gemv_call(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                           void *y, void *workspace, size_t workspace_bytes, ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!w || !x || !y || !workspace) return QL_ERR_NULL;
  if ((st = check_packed(d, w->codes, w->gmeta, w->steps)) != QL_OK) return st;
  if (!aligned16(x) || !aligned16(y) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QL_ERR_ALIGN;
  if (bias && !aligned16(bias)) return QL_ERR_ALIGN;
  const int64_t mmax = d->fmt == QL_AFFINE_U32 ? 32 : 8;
  if (M < 1 || M > mmax) return QL_ERR_RANGE;
  if (workspace_bytes < gemv_call_workspace_bytes(d, M)) return QL_ERR_SHAPE;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d->fmt) {
    case QL_INT4_NSS: return launch_gemv<FMT_INT4, 4>(d, w, x, M, bias, y, workspace, s, di->sms);
    case QL_INT6_SYM: return launch_gemv<FMT_INT6, 6>(d, w, x, M, bias, y, workspace, s, di->sms);
    case QL_INT6_PLANAR: return launch_gemv<FMT_INT6P, 6>(d, w, x, M, bias, y, workspace, s, di->sms);
    default:
      if (d->bits == 2) return launch_gemv<FMT_AFFINE, 2>(d, w, x, M, bias, y, workspace, s, di->sms);
      if (d->bits == 4) return launch_gemv<FMT_AFFINE, 4>(d, w, x, M, bias, y, workspace, s, di->sms);
      return launch_gemv<FMT_AFFINE, 8>(d, w, x, M, bias, y, workspace, s, di->sms);
  }
}

ql_status qlinear_gemv(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, void *y,
                       void *workspace, size_t workspace_bytes, ql_stream_t stream) {
  return gemv_call(d, w, x, M, nullptr, y, workspace, workspace_bytes, stream);
}

ql_status qlinear_gemv_bias(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M,
                            const void *bias, void *y, void *workspace, size_t workspace_bytes,
                            ql_stream_t stream) {
  if (!bias) return QL_ERR_NULL;
  return gemv_call(d, w, x, M, bias, y, workspace, workspace_bytes, stream);
}

ql_status qlinear_gemm_workspace_bytes(const ql_desc *d, int64_t M, size_t *bytes) {
  const ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!bytes) return QL_ERR_NULL;
  if (M < 1 || M > (int64_t)INT32_MAX) return QL_ERR_RANGE;
  *bytes = gemm_workspace_bytes(M, d->N, d->K);
  return QL_OK;
}

static ql_status gemm_call(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, const void *bias,
                           void *y, void *workspace, size_t workspace_bytes, ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!w || !x || !y || !workspace) return QL_ERR_NULL;
  if ((st = check_packed(d, w->codes, w->gmeta, w->steps)) != QL_OK) return st;
  if (!aligned16(x) || !aligned16(y) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QL_ERR_ALIGN;
  if (bias && !aligned16(bias)) return QL_ERR_ALIGN;
  if (M < 1 || M > (int64_t)INT32_MAX) return QL_ERR_RANGE;
  if (d->K % gemm::BK != 0 || d->N > (int64_t)INT32_MAX) return QL_ERR_SHAPE;
  if (workspace_bytes < gemm_workspace_bytes(M, d->N, d->K)) return QL_ERR_SHAPE;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  if (di->major != 10) return QL_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d->fmt) {
    case QL_INT4_NSS: return launch_gemm<FMT_INT4, 4>(d, w, x, M, bias, y, workspace, s, di->sms);
    case QL_INT6_SYM: return launch_gemm<FMT_INT6, 6>(d, w, x, M, bias, y, workspace, s, di->sms);
    case QL_INT6_PLANAR: return launch_gemm<FMT_INT6P, 6>(d, w, x, M, bias, y, workspace, s, di->sms);
    default:
      if (d->bits == 2) return launch_gemm<FMT_AFFINE, 2>(d, w, x, M, bias, y, workspace, s, di->sms);
      if (d->bits == 4) return launch_gemm<FMT_AFFINE, 4>(d, w, x, M, bias, y, workspace, s, di->sms);
      return launch_gemm<FMT_AFFINE, 8>(d, w, x, M, bias, y, workspace, s, di->sms);
  }
}

ql_status qlinear_gemm(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, void *y,
                       void *workspace, size_t workspace_bytes, ql_stream_t stream) {
  return gemm_call(d, w, x, M, nullptr, y, workspace, workspace_bytes, stream);
}

ql_status qlinear_gemm_bias(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M,
                            const void *bias, void *y, void *workspace, size_t workspace_bytes,
                            ql_stream_t stream) {
  if (!bias) return QL_ERR_NULL;
  return gemm_call(d, w, x, M, bias, y, workspace, workspace_bytes, stream);
}

// Two packed layers with the same format and K side by side along N: every packed buffer is
// row-major per weight row with per-row metadata, so the result is each buffer of `a` followed by
// the same buffer of `b` (six device-to-device copies on the stream).
ql_status qlinear_concat_n(const ql_desc *da, const ql_packed_const *wa, const ql_desc *db,
                           const ql_packed_const *wb, const ql_packed *out, ql_stream_t stream) {
  ql_status st;
  if (!da || !db || !wa || !wb || !out) return QL_ERR_NULL;
  if ((st = check_desc(da)) != QL_OK || (st = check_desc(db)) != QL_OK) return st;
  if (da->fmt != db->fmt || da->bits != db->bits || da->group != db->group || da->K != db->K) return QL_ERR_SHAPE;
  if ((st = check_packed(da, wa->codes, wa->gmeta, wa->steps)) != QL_OK) return st;
  if ((st = check_packed(db, wb->codes, wb->gmeta, wb->steps)) != QL_OK) return st;
  ql_desc dc = *da;
  dc.N = da->N + db->N;
  if ((st = check_packed(&dc, out->codes, out->gmeta, out->steps)) != QL_OK) return st;
  size_t ca, ga, sa, cb, gb, sb;
  if ((st = qlinear_packed_bytes(da, &ca, &ga, &sa)) != QL_OK) return st;
  if ((st = qlinear_packed_bytes(db, &cb, &gb, &sb)) != QL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void *srcs[3][2] = {{wa->codes, wb->codes}, {wa->gmeta, wb->gmeta}, {wa->steps, wb->steps}};
  void *dsts[3] = {out->codes, out->gmeta, out->steps};
  const size_t na[3] = {ca, ga, sa}, nb[3] = {cb, gb, sb};
  for (int i = 0; i < 3; ++i) {
    if (na[i] + nb[i] == 0) continue;  // affine: no step buffer
    uint8_t *dst = static_cast<uint8_t *>(dsts[i]);
    if (cudaMemcpyAsync(dst, srcs[i][0], na[i], cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dst + na[i], srcs[i][1], nb[i], cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return cuda_failed();
  }
  return QL_OK;
}

ql_status qlinear_gemm_noalloc(const ql_desc *d, const ql_packed_const *w, const void *x, int64_t M, void *y,
                               ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (!w || !x || !y) return QL_ERR_NULL;
  if ((st = check_packed(d, w->codes, w->gmeta, w->steps)) != QL_OK) return st;
  if (!aligned16(x) || !aligned16(y)) return QL_ERR_ALIGN;
  if (M < 1 || M > (int64_t)INT32_MAX) return QL_ERR_RANGE;
  if (d->K % gemm::BK != 0 || d->N > (int64_t)INT32_MAX) return QL_ERR_SHAPE;
  if (gemm_workspace_bytes(M, d->N, d->K) > (size_t)QL_NOALLOC_SCRATCH_BYTES) return QL_ERR_RANGE;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  if (di->major != 10) return QL_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != QL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (d->fmt) {
    case QL_INT4_NSS: return launch_gemm<FMT_INT4, 4>(d, w, x, M, nullptr, y, scratch, s, di->sms);
    case QL_INT6_SYM: return launch_gemm<FMT_INT6, 6>(d, w, x, M, nullptr, y, scratch, s, di->sms);
    case QL_INT6_PLANAR: return launch_gemm<FMT_INT6P, 6>(d, w, x, M, nullptr, y, scratch, s, di->sms);
    default:
      if (d->bits == 2) return launch_gemm<FMT_AFFINE, 2>(d, w, x, M, nullptr, y, scratch, s, di->sms);
      if (d->bits == 4) return launch_gemm<FMT_AFFINE, 4>(d, w, x, M, nullptr, y, scratch, s, di->sms);
      return launch_gemm<FMT_AFFINE, 8>(d, w, x, M, nullptr, y, scratch, s, di->sms);
  }
}

ql_status qlinear_quantize_meta(const ql_desc *d, const float *scale, const float *zero, const ql_unpacked_out *out,
                                ql_stream_t stream) {
  ql_status st = check_desc(d);
  if (st != QL_OK) return st;
  if (d->fmt == QL_AFFINE_U32) return QL_ERR_UNSUPPORTED;
  const bool i4 = d->fmt == QL_INT4_NSS;
  if (!scale || !out || !out->meta0 || !out->step0) return QL_ERR_NULL;
  if (i4 && (!zero || !out->meta1 || !out->step1)) return QL_ERR_NULL;
  if (!aligned16(scale) || !aligned16(out->meta0) || !aligned16(out->step0)) return QL_ERR_ALIGN;
  if (i4 && (!aligned16(zero) || !aligned16(out->meta1) || !aligned16(out->step1))) return QL_ERR_ALIGN;
  DeviceInfo *di;
  if ((st = device_info(&di)) != QL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = d->N, K = d->K;
  const int per = i4 ? 8 : 16;                  // groups per 256-weight super-block
  const int64_t G = K / (i4 ? 32 : 16);         // groups per row
  const int64_t threads = N * (G / per);        // one per (row, super-block)
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  auto *c0 = static_cast<uint8_t *>(out->meta0);
  auto *s0 = static_cast<uint16_t *>(out->step0);
  if (i4)  // scale and zero fields in one launch (grid y)
    quantize_meta_kernel<false, 8><<<dim3(blocks, 2), 256, 0, s>>>(scale, zero, N, G, c0,
                                                                  static_cast<uint8_t *>(out->meta1), s0,
                                                                  static_cast<uint16_t *>(out->step1));
  else
    quantize_meta_kernel<true, 16><<<dim3(blocks, 1), 256, 0, s>>>(scale, scale, N, G, c0, c0, s0, s0);
  return launched();
}

ql_status qlinear_set_withhold_copies(int32_t on) {
  const int h = on ? 1 : 0;
  if (cudaMemcpyToSymbol(g_ql_withhold, &h, sizeof h) != cudaSuccess) return cuda_failed();
  return QL_OK;
}

ql_status qlinear_sync_status(ql_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return cuda_failed();
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_ql_status, sizeof v) != cudaSuccess) return cuda_failed();
  if (v != 0 && cudaMemcpyToSymbol(g_ql_status, &zero, sizeof zero) != cudaSuccess) return cuda_failed();
  return (v & QL_DEV_TIMEOUT) ? QL_ERR_TIMEOUT : (v & QL_DEV_RANGE) ? QL_ERR_RANGE : QL_OK;
}

}  // extern "C"
