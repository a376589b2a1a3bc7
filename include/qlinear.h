/*
 * qlinear.h -- C ABI of the B200 (sm_100a) weight-only quantized linear layer
 *
 *     y[M][N] = x[M][K] . dequant(Wq)[N][K]^T
 *
 * with group-wise dequantisation fused into the contraction.
 *
 * Formats (sources are web pages, cited by title and section):
 *
 *  QL_INT4_NSS   nested-superscale int4.  ExecuTorch PR "[cuda] Nestest
 *                Superscale Quantization for CUDA Weights (int4 / int6)",
 *                section "Quant schema update", int4 bullet: 4-bit codes,
 *                group 32, super-block 256; scale = uint8 code x per-256 fp16
 *                step, zero = uint8 code x per-256 fp16 step, both steps in
 *                one 32-bit word; w = (q - zero) * scale; 4.625 bits/weight.
 *  QL_INT6_SYM   symmetric int6, same page and section, int6 bullet: no zero,
 *                group 16, super-block 256, scale = int8 code x per-256 fp16
 *                step; 6.5625 bits/weight.  Section "Why this design" (b)
 *                gives the reason the int8 scale code is kept.
 *  QL_INT6_PLANAR the same int6 codes and metadata with the codes held as a
 *                4-bit plane and a 2-bit plane: the ExecuTorch PR's review,
 *                "Correctness" note 2, describes the reference int6 decode
 *                kernel's 16-byte load as one 32-weight group at 4 bits.
 *  QL_AFFINE_U32 uint32-packed affine.  Hugging Face Transformers docs,
 *                "Metal" quantization page, introduction: codes packed into
 *                uint32 words with per-group scales and biases; bit widths
 *                2, 4, 8; group size configurable, default 64;
 *                w = q * scale + bias.
 *
 * Layout of every weight buffer: W has N rows (output features) and K columns
 * (input features); each row's data is contiguous and rows follow each other
 * (row-major).  16-bit floats are raw IEEE binary16 / bfloat16 bit patterns.
 *
 *  QL_INT4_NSS  codes u8  [N][K/2]   byte i = q[2i] | q[2i+1] << 4
 *               gmeta u16 [N][K/32]  scale code | zero code << 8
 *               steps u32 [N][K/256] fp16 scale step | fp16 zero step << 16
 *  QL_INT6_SYM  codes u8  [N][3K/4]  every 4 codes form one little-endian
 *                                    24-bit unit: sum_i (q[4j+i] & 63) << 6i
 *               gmeta i8  [N][K/16]  scale code
 *               steps u16 [N][K/256] fp16 step
 *  QL_INT6_PLANAR codes u8 [N][3K/4]  per 256-weight super-block j of a row,
 *                                    192 bytes at 192j: bytes 0..127 hold
 *                                    the low 4 bits of code 256j+i at byte
 *                                    i/2 (even i in the low nibble), bytes
 *                                    128..191 its bits 4-5 at byte 128+i/4,
 *                                    bits 2*(i%4); gmeta, steps as QL_INT6_SYM
 *  QL_AFFINE_U32 codes u32 [N][K*bits/32]  word t = sum_i q[tP+i] << bits*i,
 *                                          P = 32/bits (first code lowest)
 *               gmeta u32 [N][K/group] bf16 scale | bf16 bias << 16
 *               steps (none)
 *
 * Dequantisation, exactly (each step one binary32 operation, nearest-even,
 * no fused multiply-add):
 *  int4:   S = f32(sc)*f32(ss); Z = f32(zc)*f32(zs); w = (f32(q) - Z) * S
 *  int6 (either storage):   S = f32(sc)*f32(st); w = f32(q) * S
 *  affine: w = f32(q)*f32(scale) + f32(bias)
 *
 * Conventions for every entry point:
 *  - Ownership: the caller allocates and frees every buffer (including the
 *    GEMM's workspace); pointers are device pointers unless stated
 *    otherwise.  The library allocates no device memory in any call.  It keeps one small static device status
 *    word per device and a host-side cache of kernel attributes.
 *  - Asynchrony: calls enqueue work on `stream` and return without
 *    synchronising (qlinear_sync_status excepted).
 *  - Errors: arguments are validated on the host before anything is
 *    launched; a non-QL_OK status means nothing was enqueued.  A launch
 *    failure returns QL_ERR_CUDA.  Kernels never trap: a device-side wait
 *    that gives up sets the device status word, which qlinear_sync_status
 *    reports as QL_ERR_TIMEOUT.
 *  - Alignment: every device pointer must be 16-byte aligned.
 *  - Values out of range in the data (e.g. an int8 scale code of -128) are
 *    not checked; they are defined by the formulas above.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ql_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  QL_OK = 0,
  QL_ERR_NULL = 1,        /* a required pointer is NULL                          */
  QL_ERR_SHAPE = 2,       /* N, K, M, bits or group not allowed for the format   */
  QL_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                    */
  QL_ERR_RANGE = 4,       /* a value out of range: M for the entry point, a      */
                          /* problem larger than qlinear_gemm_noalloc's fixed    */
                          /* scratch array, or (from qlinear_sync_status) an     */
                          /* encoder input outside its domain                    */
  QL_ERR_UNSUPPORTED = 5, /* unknown format, or the device is not sm_100         */
  QL_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed                */
  QL_ERR_TIMEOUT = 7      /* a device-side bounded wait gave up                  */
} ql_status;

typedef enum { QL_INT4_NSS = 1, QL_INT6_SYM = 2, QL_AFFINE_U32 = 3, QL_INT6_PLANAR = 4 } ql_format;

typedef enum { QL_OUT_F32 = 0, QL_OUT_BF16 = 1 } ql_out_dtype;

/* Describes one quantized weight matrix.
 *  fmt   : a ql_format value
 *  bits  : QL_AFFINE_U32: 2, 4 or 8.  Ignored (0) for int4 / int6.
 *  group : QL_AFFINE_U32: 32, 64 or 128.  Ignored (0) for int4 / int6, whose
 *          groups are fixed at 32 and 16 (int6 in either storage).
 *  N     : output features, N >= 1.
 *  K     : input features.  int4 / int6: K % 256 == 0.  affine:
 *          K % group == 0 and (K * bits) % 128 == 0 (whole 16-byte rows). */
typedef struct {
  int32_t fmt;
  int32_t bits;
  int32_t group;
  int32_t reserved;
  int64_t N;
  int64_t K;
} ql_desc;

/* The packed weight buffers (device pointers, caller-owned).  `steps` is
 * unused (may be NULL) for QL_AFFINE_U32. */
typedef struct {
  void *codes;
  void *gmeta;
  void *steps;
} ql_packed;

typedef struct {
  const void *codes;
  const void *gmeta;
  const void *steps;
} ql_packed_const;

/* The unpacked inputs of qlinear_pack (device pointers, caller-owned):
 *              q (one code per byte)   meta0          meta1        step0        step1
 *  int4:       u8 [N][K] 0..15         sc u8 [N][K/32] zc u8 [..]  ss f16 [N][K/256] zs f16 [..]
 *  int6 (both): i8 [N][K] -32..31      sc i8 [N][K/16] (unused)    st f16 [N][K/256] (unused)
 *  affine:     u8 [N][K] 0..2^bits-1   scale bf16 [N][K/group] bias bf16 [..] (unused) (unused)
 * Codes are reduced to their low `bits` bits (int6: two's complement low
 * 6 bits) when packed. */
typedef struct {
  const void *q;
  const void *meta0;
  const void *meta1;
  const void *step0;
  const void *step1;
} ql_unpacked;

/* Byte sizes of the three packed buffers for `desc` (host-only, no CUDA call).
 * Size closed forms: int4 K/2 + K/16 + K/64 bytes per row (4.625 bits per
 * weight); int6 (either storage) 3K/4 + K/16 + K/128 (6.5625); affine K*bits/8 + 4K/group
 * (bits + 32/group).  Errors: QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_UNSUPPORTED. */
ql_status qlinear_packed_bytes(const ql_desc *desc, size_t *codes_bytes,
                               size_t *gmeta_bytes, size_t *steps_bytes);

/* Pack unpacked codes and metadata into the layout above (one kernel).
 * Same page and section as each format; bit-exact by definition.
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_ALIGN, QL_ERR_UNSUPPORTED,
 * QL_ERR_CUDA. */
ql_status qlinear_pack(const ql_desc *desc, const ql_unpacked *in,
                       const ql_packed *out, ql_stream_t stream);

/* Where qlinear_unpack writes: same element types and shapes as ql_unpacked
 * (int6 codes come back sign-extended; unused members may be NULL). */
typedef struct {
  void *q;
  void *meta0;
  void *meta1;
  void *step0;
  void *step1;
} ql_unpacked_out;

/* Inverse of qlinear_pack (one kernel); bit-exact by definition.
 * Errors: as qlinear_pack. */
ql_status qlinear_unpack(const ql_desc *desc, const ql_packed_const *in,
                         const ql_unpacked_out *out, ql_stream_t stream);

/* Standalone dequantisation: out[N][K] = w as defined above, as binary32
 * (QL_OUT_F32, bit-exact) or as its nearest-even bfloat16 (QL_OUT_BF16).
 * The formulas are those of the ExecuTorch page's "Quant schema update"
 * (int4 / int6) and of the Transformers "Metal" page's introduction
 * (affine); that page's section on dequantisation describes the same
 * operation as turning a pre-quantized checkpoint back into float weights
 * where the fused kernels are not used.  `out`: device, [N][K] row-major,
 * 4 or 2 bytes per element, caller-owned, 16-byte aligned.
 * Errors: as qlinear_pack, plus QL_ERR_SHAPE for an unknown out_dtype. */
ql_status qlinear_dequant(const ql_desc *desc, const ql_packed_const *w,
                          void *out, int32_t out_dtype, ql_stream_t stream);

/* Metadata encoder: float per-group metadata -> the codes and per-256 fp16
 * steps that qlinear_pack takes (ExecuTorch PR above, "Quant schema update";
 * its review, "Correctness" note 1 and "Things done well").  One field at a
 * time, per 256-weight super-block of a row:
 *   int4: scale and zero, float32 [N][K/32] each, finite and >= 0 (zero in
 *         code units: w = (q - zero) * scale):
 *         step = RN_fp16(block max / 255)  (binary32 division, then fp16),
 *         code = clamp(round_half_even(v / f32(step)), 0, 255)  -> u8;
 *         out->meta0 = sc [N][K/32], out->meta1 = zc, out->step0 = ss
 *         [N][K/256] fp16 bits, out->step1 = zs.
 *   int6 (either storage): scale float32 [N][K/16], finite, either sign; `zero` unused:
 *         step = RN_fp16(block max|v| / 127),
 *         code = clamp(round_half_even(v / f32(step)), -127, 127) -> i8;
 *         out->meta0 = sc [N][K/16], out->step0 = st [N][K/256].
 * Codes are rounded against the fp16-rounded step, so qlinear_pack +
 * qlinear_dequant reconstruct code * step exactly as the encoder saw it.  A
 * super-block whose max is 0 gets step 0 and codes 0.  A negative (int4) or
 * non-finite input is not rejected on the host (it is device data): the
 * kernel records it and the next qlinear_sync_status returns QL_ERR_RANGE.
 * Device pointers, caller-owned, 16-byte aligned.  affine: QL_ERR_UNSUPPORTED.
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_ALIGN, QL_ERR_UNSUPPORTED,
 * QL_ERR_CUDA. */
ql_status qlinear_quantize_meta(const ql_desc *desc, const float *scale, const float *zero,
                                const ql_unpacked_out *out, ql_stream_t stream);

/* Bytes of caller-provided device workspace qlinear_gemv needs for `desc`
 * and M (host-only, no CUDA call): 7*M*K for x (24-bit fixed point, three
 * bytes per element plus the zero padding of the diagonal operands) in the
 * order the tensor-core fragments read it, 8*M*K/32 for the per-group x
 * scales and sums,
 * 4*max(4096*64*M, 64*ceil(N/64)*ceil(K/5120)) for the partial sums of a
 * K split, 4*ceil(N/16) for its
 * counters and 16*K/256 for the per-super-block precision flags, each part
 * rounded up to 256 bytes; for affine calls that run on
 * the GEMM (below) at least qlinear_gemm_workspace_bytes().
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_RANGE, QL_ERR_UNSUPPORTED. */
ql_status qlinear_gemv_workspace_bytes(const ql_desc *desc, int64_t M, size_t *bytes);

/* Decode-shaped layer, HBM-bound: y[M][N] (bf16) = x[M][K] (bf16) . W^T,
 * fp32 scales and accumulation, one nearest-even rounding to bf16 at the end.
 * 1 <= M <= 8 for int4 / int6; 1 <= M <= 32 for affine.
 *  - Tensor-core path (int4 and int6 at every M; affine with group 32 or 64
 *    and K % 256 == 0 at M <= 8): two launches (int4 and 4-bit affine at
 *    M = 1: one, plus a short kernel that adds the parts when K is split).
 *    Each x
 *    group (32 elements; 16 for int6) is turned into fixed point, x_int = rint(x *
 *    2^a): 16-bit (the group's max |x| scaled into [2^14, 2^15): exact for
 *    every bf16 element within 2^7 of the group's largest magnitude), or
 *    24-bit (max in [2^22, 2^23): exact within 2^15) for every group of a
 *    super-block (per token) in which some group's 16-bit rounding error
 *    exceeds 2^-12 of its mass outside its largest element; split into high,
 *    middle and (24-bit) low bytes in the order the tensor-core fragments
 *    read them, with the group's scale (and sum) -- by a short pass, or, for
 *    int4 and 4-bit affine (group 32 / 64) at M = 1, by each CTA of the
 *    streaming kernel for its part of K,
 *    into shared memory (K split into parts of at most 22 super-blocks, their
 *    partial sums in the workspace); then the streaming kernel
 *    multiplies the codes (as u8 or s8 bytes: 16q for nibbles, 4q for int6,
 *    q for 2- and 8-bit fields) by those bytes on the integer tensor core
 *    (mma.sync m16n8k32, exact s32 sums, one MMA per byte: high and middle
 *    in the streaming loop, the low bytes of 24-bit super-blocks in a pass
 *    after it that reads their weights again) and applies scale (and zero
 *    or bias) once per (row, group[, token]) in fp32.  int4 and 4-bit
 *    affine at M = 1 and int6 use a diagonal x operand (one MMA column per
 *    weight group); int4 at M >= 2 and the other affine calls use the tokens
 *    as MMA columns.  K may be split
 *    over warps or CTAs, the parts added in a fixed order through the
 *    workspace.
 *  - Affine with group 32 or 64 and K % 256 == 0 at 9 <= M <= 32: two
 *    launches, fp16 tensor cores.  A pass writes x as fp16 with one
 *    power-of-two scale per token (qlinear_gemm's first pass); the streaming
 *    kernel dequantises each weight once to fp16 (q * s' + b', one rounding,
 *    with (s, b) scaled per row by a power of two from the row's group
 *    words) and multiplies it with mma.sync m16n8k16 against two or four
 *    8-token column tiles, fp32 accumulation over K, both scales undone at
 *    the end.
 *  - Affine with other groups, or K % 256 != 0, at M < 8: one launch, exact
 *    binary32 weights, fp32 FMA; from M = 8: runs as qlinear_gemm.
 * ExecuTorch page above, "Quant schema update" (the int4 / int6 formats)
 * and the review's "Things done well" (the decode kernel's per-super-block
 * step word and full-warp trip counts).
 * `workspace`: at least qlinear_gemv_workspace_bytes(), 256-byte aligned,
 * caller-owned, overwritten; calls sharing one workspace must not overlap on
 * the GPU.  Consecutive tensor-core calls on one stream chain by
 * programmatic dependent launch: a call's weight stream may start while the
 * previous kernel on the stream drains, and its first kernel waits for that
 * kernel before it reads x or writes the workspace.
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE (also: workspace too small),
 * QL_ERR_ALIGN, QL_ERR_RANGE, QL_ERR_UNSUPPORTED, QL_ERR_CUDA. */
ql_status qlinear_gemv(const ql_desc *desc, const ql_packed_const *w,
                       const void *x, int64_t M, void *y, void *workspace,
                       size_t workspace_bytes, ql_stream_t stream);

/* qlinear_gemv plus a per-output-row bias: y[m][n] = RN_bf16(acc[m][n] +
 * f32(bias[n])), the bias added in fp32 before the one rounding.  `bias`:
 * bf16 [N] on the device, 16-byte aligned, not NULL.  Otherwise as
 * qlinear_gemv (Metal backend notes on the ExecuTorch page: "linear with
 * bias", "4-bit linear with bias").  Errors: as qlinear_gemv. */
ql_status qlinear_gemv_bias(const ql_desc *desc, const ql_packed_const *w,
                            const void *x, int64_t M, const void *bias, void *y,
                            void *workspace, size_t workspace_bytes, ql_stream_t stream);

/* Bytes of caller-provided device workspace qlinear_gemm needs for `desc`
 * and M (host-only, no CUDA call): 2*M*K for the fp16 copy of x, plus
 * 4*M + 8*ceil(N/256)*256 for the per-row scales, each part rounded up to
 * 256 bytes.  Errors: QL_ERR_NULL, QL_ERR_SHAPE, QL_ERR_RANGE,
 * QL_ERR_UNSUPPORTED. */
ql_status qlinear_gemm_workspace_bytes(const ql_desc *desc, int64_t M, size_t *bytes);

/* Prefill-shaped layer on the tcgen05 tensor cores: same result definition
 * as qlinear_gemv, any M >= 1 (meant for M >= 128).  The dequantisation is
 * fused into the contraction, as the Transformers "Metal" page's
 * introduction describes for its fused dequantize + matmul kernel; the
 * ExecuTorch page's "e2e results" measure this shape as prefill.  Three launches on
 * `stream`: (1) x is scaled per token row by a power of two 2^a_m that puts
 * the row's max |x| in [2^15, 2^16) and stored as fp16 in the workspace
 * (exact for every value within 2^29 of the row maximum); (2) each weight
 * row gets a power of two 2^b_n from a metadata bound on its max |w|;
 * (3) the persistent GEMM (tiles of 128 weight rows x 256 tokens, or x 32
 * tokens up to M = 32) dequantises each weight once per tile into fp16, into
 * tensor memory as the MMA's A operand -- int4 as q * S' - Z * S' in packed
 * halves with S' = S * 2^b_n, int6 / affine as the exact binary32 value times
 * 2^b_n rounded once -- contracts with fp32 accumulation in tensor memory,
 * and stores RN_bf16(acc * 2^-a_m * 2^-b_n).  fp16 operands rather than
 * bf16 keep the weight rounding at ~0.1% of rms(y) instead of ~1%.
 * `workspace`: device memory of at least qlinear_gemm_workspace_bytes(),
 * 256-byte aligned, owned by the caller, overwritten; calls sharing one
 * workspace must not overlap on the GPU.  K % 64 == 0.  Requires an sm_100
 * device.
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE (also: workspace too small),
 * QL_ERR_ALIGN, QL_ERR_RANGE, QL_ERR_UNSUPPORTED (format or device),
 * QL_ERR_CUDA. */
ql_status qlinear_gemm(const ql_desc *desc, const ql_packed_const *w,
                       const void *x, int64_t M, void *y, void *workspace,
                       size_t workspace_bytes, ql_stream_t stream);

/* qlinear_gemm plus a per-output-row bias (bf16 [N], added in fp32 before
 * the rounding to bf16), as qlinear_gemv_bias.  Errors: as qlinear_gemm. */
ql_status qlinear_gemm_bias(const ql_desc *desc, const ql_packed_const *w,
                            const void *x, int64_t M, const void *bias, void *y,
                            void *workspace, size_t workspace_bytes, ql_stream_t stream);

/* Two packed layers with the same format, bits, group and K, stacked along
 * N (fused projections such as QKV or gate/up; the ExecuTorch PR's
 * "_concat_coalesced_int4_along_n", review "Correctness" note 3): `out` is
 * the packed layer with N = a.N + b.N whose rows are a's rows then b's.
 * Every packed buffer is row-major per weight row with per-row metadata, so
 * each output buffer is a's buffer followed by b's (six device-to-device
 * copies on `stream`).  `out` buffers sized by qlinear_packed_bytes for the
 * stacked desc, caller-owned, 16-byte aligned.
 * Errors: QL_ERR_NULL, QL_ERR_SHAPE (formats or K differ), QL_ERR_ALIGN,
 * QL_ERR_UNSUPPORTED, QL_ERR_CUDA. */
ql_status qlinear_concat_n(const ql_desc *a, const ql_packed_const *wa,
                           const ql_desc *b, const ql_packed_const *wb,
                           const ql_packed *out, ql_stream_t stream);

/* qlinear_gemm for callers that may not allocate device memory at all --
 * e.g. an op behind a runtime's plug-in interface, which receives its input
 * and output pointers but no allocator, or a serving process that has
 * reserved all of HBM for its own pool, where cudaMalloc would fail or stall
 * the device.  (The pages describe no such entry point; it serves deployment
 * only.)  Same arguments, result and errors as qlinear_gemm, minus the
 * workspace: the library takes it from one fixed 32 MiB array in device
 * memory that exists on every GPU that loads the library, until the process
 * exits.  No call allocates or frees anything.
 *  - Limit: the call is accepted while qlinear_gemm_workspace_bytes(desc, M)
 *    is at most 33554432 bytes (about M*K <= 16.7 million for small N);
 *    larger problems return QL_ERR_RANGE before anything is enqueued.
 *  - The first call on a device looks up that device's address of the array
 *    (cudaGetSymbolAddress, with the device current) and caches it; make that
 *    first call before any stream capture.  With lazy module loading (the
 *    default of recent CUDA releases) the array and the library's kernels
 *    are only placed on a device when the library is first used there, so a
 *    process that reserves nearly all of HBM should make this first call on
 *    each device before it reserves its pool.
 *  - All calls on a device share the one array, which keeps whatever the last
 *    call left in it; nothing in it needs to start at zero, because each call
 *    writes every element of it that its kernels read.  Calls whose work
 *    overlaps on the GPU (other streams, or other threads) race on the array:
 *    order them. */
ql_status qlinear_gemm_noalloc(const ql_desc *desc, const ql_packed_const *w,
                               const void *x, int64_t M, void *y,
                               ql_stream_t stream);

/* Synchronise `stream`, then read and clear the current device's status
 * word: QL_ERR_TIMEOUT if a kernel's bounded wait gave up since the last
 * call, QL_ERR_RANGE if qlinear_quantize_meta met an input outside its
 * domain (the loud failure the ExecuTorch review's "Correctness" note 1 asks
 * of the metadata encoder, instead of a silent clamp), QL_ERR_CUDA if the
 * synchronisation failed, else QL_OK.  The word is per device and shared by
 * every stream: a status may come from work enqueued on another stream. */
ql_status qlinear_sync_status(ql_stream_t stream);

/* Every device-side wait of this library's kernels for another role or for
 * data is bounded (2e9 SM clock cycles, about 1 s at the B200's clock).  A
 * kernel whose wait runs out sets the device status word (qlinear_sync_status
 * then returns QL_ERR_TIMEOUT), makes its other roles leave their loops, waits
 * (bounded) for the copies and MMAs it has in flight, frees its tensor memory
 * and returns.  on != 0 makes the current device's kernels start no copies at
 * all, so their first wait for data is certain to run out (after about 1 s);
 * 0 restores normal operation.  It exists so that tests can drive that
 * give-up path; callers normally never change it.  (The pages have no
 * counterpart.)  Synchronous; do not call it while this library's kernels
 * run.  Errors: QL_ERR_CUDA. */
ql_status qlinear_set_withhold_copies(int32_t on);

/* Static, never NULL. */
const char *qlinear_status_string(ql_status status);

/* Library version, e.g. 1 */
int32_t qlinear_version(void);

#ifdef __cplusplus
}
#endif
#endif /* QLINEAR_H */
