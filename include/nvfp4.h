/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 / MXFP8 / MXFP4 block-scaled
 * quantize, dequantize and quantized matmuls on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *  [P1] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 8: ops.cpp validate_global_scale,
 *       validate_qqmm_inputs, qqmm, fp_quantize, fp_dequantize; qqmm_utils.h
 *       get_padded_scale_dims, pad_and_swizzle_scales.
 *  [P2] "mlx 0.30.7.2 -> 0.30.7.6" diff, page 7: fp_quantize.cu kernels
 *       fp_quantize_dequantize, fp_quantize_rowwise, fp_dequantize; qqmm.cpp
 *       QQMatmul::eval_gpu; qqmm_impl.h GemmScalars; qqmm_utils.cu
 *       compute_qqmm_pointers.
 *  [P3] "[Metal] global scale for qmm" (ml-explore/mlx pull 4458): gather_qmm
 *       with per-expert global scales; worked example.
 *  [P4] osaurus-ai/mlx pull 31: "The fix" (global scale per block scale).
 *  [P5] "mlx 0.30.7" diff, page 71: qqmm_utils.cu swizzle_scales, 128x4 tiles.
 *
 * Conventions for every call
 *  - Ownership: the caller allocates every buffer; all tensor pointers are
 *    DEVICE pointers on the current CUDA device.  The library allocates no
 *    device memory and never synchronizes; each call only enqueues kernels on
 *    `stream` (NULL = legacy default stream) and returns.
 *  - Layout: row-major, contiguous.  Every tensor pointer must be 16-byte
 *    aligned.  Codes of NVFP4 and MXFP4 are uint32 words holding 8 e2m1
 *    codes, element 8w+i of a row in bits 4i..4i+3 of word w; codes of MXFP8
 *    hold 4 e4m3 bytes, element 4w+i in byte i.
 *  - Scale layouts: NVFP4_LAYOUT_LINEAR is [rows, K/group] uint8.
 *    NVFP4_LAYOUT_SWIZZLED is the 128x4-tile layout the block-scaled MMA
 *    reads ([P5]; [P1] pad_and_swizzle_scales): a [ceil128(rows),
 *    ceil4(K/group)] buffer where linear scale (r, c) sits at byte
 *      ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4,
 *    Cp = ceil4(K/group), and every padding byte is 0.
 *  - Global scales g, g_x, g_w are `const float*` device pointers to one
 *    fp32 (as the device alpha of [P2] GemmScalars); NULL means none (encode
 *    and decode factors 1).  They are meaningful for NVFP4 only ([P1]
 *    validate_global_scale) and must be finite and > 0.
 *  - Inputs are finite: the codes, scales and outputs of a block holding a
 *    NaN or an infinity are unspecified (the pages do not define them).
 *  - Errors: every call returns an nvfp4_status and never throws.  Argument
 *    checks happen on the host before anything is enqueued; on failure
 *    nothing is enqueued and nvfp4_last_error_message() explains.
 *    NVFP4_ERR_CUDA reports a launch error.  Device-side checks (an expert
 *    index out of range in gather_qmm; a bounded wait that gave up in the
 *    tensor-core GEMM) set a device error word instead of trapping; read it
 *    with nvfp4_check_device_errors().
 *  - Empty outputs: a call whose output has no element (rows, N, M or T is
 *    0, or K is 0 for the quantizers) returns NVFP4_OK after its argument
 *    checks without querying or touching the device; its pointers may then
 *    be NULL.  nvfp4_amax is the exception: it writes *g_out = 0 for n = 0.
 *    The GEMMs (qqmm, gather_qmm, gather_qmm_kn) reject K = 0 with a
 *    non-empty output (NVFP4_ERR_INVALID_ARG); qmv needs K >= 32.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* bad shape, mode, pointer alignment, scale combination */
  NVFP4_ERR_UNSUPPORTED = 2, /* device is not sm_100, dtype or size not supported */
  NVFP4_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  NVFP4_ERR_TIMEOUT = 4,     /* a kernel gave up a bounded wait (device error word) */
  NVFP4_ERR_DEVICE_INDEX = 5 /* a kernel saw an index out of range (device error word) */
} nvfp4_status;

typedef enum { NVFP4_DT_F32 = 0, NVFP4_DT_F16 = 1, NVFP4_DT_BF16 = 2 } nvfp4_dtype;
typedef enum { NVFP4_LAYOUT_LINEAR = 0, NVFP4_LAYOUT_SWIZZLED = 1 } nvfp4_layout;
typedef enum { NVFP4_MODE_NVFP4 = 0, NVFP4_MODE_MXFP8 = 1, NVFP4_MODE_MXFP4 = 2 } nvfp4_mode;

/* Short text of a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status s);

/* Message of the last failed call on this host thread ("" if none).  The
 * texts of the argument checks follow [P1] (e.g. "[qqmm] For nvfp4 mode,
 * either both global_scale_x and global_scale_w must be provided, or
 * neither."). */
NVFP4_API const char* nvfp4_last_error_message(void);

/* Synchronizes `stream`, then reads and clears the device error word.
 * Returns NVFP4_OK, NVFP4_ERR_TIMEOUT, NVFP4_ERR_DEVICE_INDEX or
 * NVFP4_ERR_CUDA.  This is the only call that synchronizes. */
NVFP4_API nvfp4_status nvfp4_check_device_errors(nvfp4_stream_t stream);

/* Bytes of a scale buffer for `rows` x `cols` scales in `layout`
 * ([P1] get_padded_scale_dims for SWIZZLED). */
NVFP4_API size_t nvfp4_scale_bytes(int64_t rows, int64_t cols, nvfp4_layout layout);

/* a1 -- tensor amax: *g_out = max |x| over n elements, fp32.  This is the
 * global scale g the method uses ([P1] QQMatmul::vjp: astype(max(abs(cotan)),
 * float32); [P2] compute_qqmm_pointers names its inputs tensor_amax_x/_w).
 * x: [n] of dt.  g_out: device fp32, overwritten (zeroed then reduced). */
NVFP4_API nvfp4_status nvfp4_amax(const void* x, nvfp4_dtype dt, int64_t n, float* g_out,
                        nvfp4_stream_t stream);

/* a1 for several tensors in one launch: the raw-operand qqmm takes the amax
 * of both operands before quantizing them ([P1] qqmm; [P2]
 * compute_qqmm_pointers reads tensor_amax_x and tensor_amax_w).  items[i]
 * holds x (n elements of dt, 16-byte aligned) and g_out (device fp32,
 * overwritten with max |x|, 0 for n = 0); 1 <= count <= 4; the outputs must
 * be distinct (one memset clears them when they are consecutive floats).
 * The items array is read on the host during the call.  Same checks and
 * errors as nvfp4_amax, per item. */
typedef struct {
  const void* x;
  int64_t n;
  float* g_out;
} nvfp4_amax_item;

NVFP4_API nvfp4_status nvfp4_amax_multi(const nvfp4_amax_item* items, int count, nvfp4_dtype dt,
                                        nvfp4_stream_t stream);

/* a2-a4 -- NVFP4 two-level quantize ([P2] fp_quantize_rowwise with global
 * scale).  Per row, per 16-element block along K:
 *   E = 2688 / g (1 if g == NULL);  s = e4m3_rne_satfinite((amax/6) * E);
 *   q_i = e2m1_rne_satfinite(x_i * (E / f8(s)));  a block with s == 0 stores
 *   zero codes.
 * x: [rows, K] of dt (fp32, fp16, bf16), K % 16 == 0.
 * codes: [rows, K/8] uint32 (written).  scales: e4m3 bytes in `layout`
 * (written, padding included): nvfp4_scale_bytes(rows, K/16, layout). */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K,
                            const float* g, uint32_t* codes, uint8_t* scales,
                            nvfp4_layout layout, nvfp4_stream_t stream);

/* a5 -- NVFP4 dequantize ([P2] fp_dequantize with global scale):
 *   out = T(e2m1(q) * (f8(s) * g / 2688)),  products in fp32.
 * codes [rows, K/8], scales in `layout`, out [rows, K] of out_dt. */
NVFP4_API nvfp4_status nvfp4_dequantize(const uint32_t* codes, const uint8_t* scales,
                              nvfp4_layout layout, int64_t rows, int64_t K, const float* g,
                              void* out, nvfp4_dtype out_dt, nvfp4_stream_t stream);

/* nvfp4_quantize of several tensors in one launch (the raw-operand qqmm
 * quantizes x and w, [P1] qqmm).  items[i] holds the arguments of one
 * nvfp4_quantize call (x [rows, K] of dt, g, codes, scales, layout); every
 * item gets exactly the codes and scales nvfp4_quantize would write.
 * 1 <= count <= 4; items must not write overlapping buffers.  The items
 * array is read on the host during the call.  Each item is checked as
 * nvfp4_quantize checks its arguments; items with no element are skipped. */
typedef struct {
  const void* x;
  int64_t rows;
  int64_t K;
  const float* g;
  uint32_t* codes;
  uint8_t* scales;
  nvfp4_layout layout;
} nvfp4_quantize_item;

NVFP4_API nvfp4_status nvfp4_quantize_multi(const nvfp4_quantize_item* items, int count, nvfp4_dtype dt,
                                            nvfp4_stream_t stream);

/* f1 -- column-wise NVFP4 quantize ([P2] fp_quantize_columnwise: an M-major
 * matrix quantized along its last dimension): x [rows, cols] row-major is
 * quantized as x^T [cols, rows] along rows, block by block exactly as
 * nvfp4_quantize does (so the result equals nvfp4_quantize of the
 * transposed, contiguous matrix).  The backward pass of qqmm quantizes w^T,
 * x^T and the transposed upstream gradient this way ([P1] QQMatmul::vjp).
 * rows % 16 == 0; codes [cols, rows/8] uint32; scales for [cols, rows/16]
 * in `layout` (SWIZZLED: [ceil128(cols), ceil4(rows/16)], zero padding);
 * g as in nvfp4_quantize. */
NVFP4_API nvfp4_status nvfp4_quantize_columnwise(const void* x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                                                 const float* g, uint32_t* codes, uint8_t* scales,
                                                 nvfp4_layout layout, nvfp4_stream_t stream);

/* nvfp4_quantize_columnwise with stochastic rounding of the codes: equal to
 * nvfp4_quantize_sr of the transposed, contiguous matrix x^T [cols, rows]
 * with the same seed (its random bits indexed by the flat position in x^T).
 * The backward pass quantizes the transposed upstream gradient this way
 * ([P1] QQMatmul::vjp).  Arguments and errors as nvfp4_quantize_columnwise,
 * plus the 64-bit seed. */
NVFP4_API nvfp4_status nvfp4_quantize_columnwise_sr(const void* x, nvfp4_dtype dt, int64_t rows, int64_t cols,
                                                    const float* g, uint64_t seed, uint32_t* codes, uint8_t* scales,
                                                    nvfp4_layout layout, nvfp4_stream_t stream);

/* f4 -- NVFP4 quantize with stochastic rounding of the codes (the pages
 * reserve it: [P2] fp_quantize_rowwise<..., USE_SR> with rbits "reserved for
 * future use"; this library's reading).  Scales exactly as nvfp4_quantize;
 * each scaled value t = x * E / f8(s) (fp32) goes to one of its two e2m1
 * neighbours lo <= |t| <= hi: up iff b * 2^-8 < (|t| - lo) / (hi - lo)
 * (|t| >= 6 gives 6, grid values are kept, the sign is kept), with b byte
 * i % 4 of the 32-bit word w = i / 4 (one word per 4 values, as [P2] passes
 * rbits to each 4-value conversion), word w being output w % 4 of
 * Philox4x32-10 (Salmon et al., SC 2011) at counter (w / 4 as 64 bits, 0,
 * 0) and key (seed), i = row * K + k.  Same arguments, layouts and errors
 * as nvfp4_quantize, plus the 64-bit seed. */
NVFP4_API nvfp4_status nvfp4_quantize_sr(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K,
                                         const float* g, uint64_t seed, uint32_t* codes, uint8_t* scales,
                                         nvfp4_layout layout, nvfp4_stream_t stream);

/* a11 -- MXFP8 quantize ([P2] fp_quantize_rowwise with 8 bits and the e8m0
 * scale; group size 32, [P1] fp_quantize; the E8M0 scale is rounded up, [P3]
 * mlxcel note).  Per 32-block: s = ue8m0_round_up(amax / 448);
 *   q_i = e4m3_rne_satfinite(x_i / 2^(s-127)).
 * x [rows, K] of dt, K % 32 == 0; codes [rows, K/4] uint32; scales e8m0
 * bytes in `layout`: nvfp4_scale_bytes(rows, K/32, layout). */
NVFP4_API nvfp4_status mxfp8_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K,
                            uint32_t* codes, uint8_t* scales, nvfp4_layout layout,
                            nvfp4_stream_t stream);

/* MXFP8 dequantize ([P1] fp_dequantize fallback, e8m0 branch):
 *   out = T(e4m3(q) * 2^(s-127)). */
NVFP4_API nvfp4_status mxfp8_dequantize(const uint32_t* codes, const uint8_t* scales,
                              nvfp4_layout layout, int64_t rows, int64_t K, void* out,
                              nvfp4_dtype out_dt, nvfp4_stream_t stream);

/* f3 -- MXFP4 quantize ([P2] fp_quantize_rowwise with 4 bits and the e8m0
 * (mx) scale; group size 32; the E8M0 scale rounded up as for MXFP8, [P3]).
 * Per 32-block: s = ue8m0_round_up(amax / 6);
 *   q_i = e2m1_rne_satfinite(x_i / 2^(s-127)), 8 codes per uint32 as NVFP4.
 * x [rows, K] of dt, K % 32 == 0; codes [rows, K/8] uint32; scales e8m0
 * bytes in `layout`: nvfp4_scale_bytes(rows, K/32, layout).  No global
 * scale.  Errors as nvfp4_quantize. */
NVFP4_API nvfp4_status mxfp4_quantize(const void* x, nvfp4_dtype dt, int64_t rows, int64_t K,
                                      uint32_t* codes, uint8_t* scales, nvfp4_layout layout,
                                      nvfp4_stream_t stream);

/* MXFP4 dequantize ([P1] fp_dequantize fallback, e8m0 branch with 4-bit
 * codes): out = T(e2m1(q) * 2^(s-127)).  codes [rows, K/8], scales as
 * produced by mxfp4_quantize in `layout`, out [rows, K] of out_dt. */
NVFP4_API nvfp4_status mxfp4_dequantize(const uint32_t* codes, const uint8_t* scales,
                                        nvfp4_layout layout, int64_t rows, int64_t K, void* out,
                                        nvfp4_dtype out_dt, nvfp4_stream_t stream);

/* a4 -- LINEAR -> SWIZZLED re-layout of a [rows, cols] uint8 scale matrix
 * ([P5] swizzle_scales; [P1] pad_and_swizzle_scales), for scales produced
 * elsewhere.  swz: nvfp4_scale_bytes(rows, cols, SWIZZLED) bytes, all
 * written (padding zero). */
NVFP4_API nvfp4_status nvfp4_swizzle_scales(const uint8_t* lin, int64_t rows, int64_t cols,
                                  uint8_t* swz, nvfp4_stream_t stream);

/* a8-a9, a12 -- dense block-scaled quantized matmul y = x_hat . w_hat^T
 * ([P2] QQMatmul::eval_gpu dense route; [P1] validate_qqmm_inputs).
 *  mode NVFP4: a_codes [M, K/8], b_codes [N, K/8], e4m3 scales SWIZZLED
 *    (nvfp4_scale_bytes(M, K/16, SWIZZLED) and (N, K/16)); optional g_x, g_w
 *    (both or neither); y = alpha * sum_b f8(sx) f8(sw) sum_k e2m1 e2m1 with
 *    alpha = (g_x / 2688) * (g_w / 2688) ([P2] compute_qqmm_pointers).
 *  mode MXFP8: a_codes [M, K/4], b_codes [N, K/4], e8m0 scales SWIZZLED
 *    (K/32 per row); g_x, g_w must be NULL.
 *  mode MXFP4: a_codes [M, K/8], b_codes [N, K/8] (mxfp4_quantize), e8m0
 *    scales SWIZZLED (K/32 per row); g_x, g_w must be NULL;
 *    y = sum_b 2^(sx-127) 2^(sw-127) sum_k e2m1 e2m1.
 *  K % 32 == 0 (NVFP4: K % 64 recommended; a ragged last 64-block is zero
 *  padded by the kernel).  y: [M, N] of y_dt (fp32, fp16 or bf16), written. */
NVFP4_API nvfp4_status qqmm(nvfp4_mode mode, int64_t M, int64_t N, int64_t K, const uint32_t* a_codes,
                  const uint8_t* a_scales, const uint32_t* b_codes, const uint8_t* b_scales,
                  const float* g_x, const float* g_w, void* y, nvfp4_dtype y_dt,
                  nvfp4_stream_t stream);

/* a6-a7 -- qmv, the small-M route of qqmm with a pre-quantized NVFP4 weight
 * ([P2] QQMatmul::eval_gpu, M = 1 branch: fp_quantize_dequantize then
 * fp_qmv):  x_hat = quantize-dequantize(x, g_x) in x's type;
 *   y[m,n] = T(sum_k x_hat[m,k] * e2m1(q[n,k]) * sd[n,k/16]), fp32
 *   accumulation, sd = f8(s) * (g_w / 2688) in fp32: the global scale is
 *   applied to each block scale ([P4] "The fix"), and the weight is not
 *   rounded to T on this path.
 * x [M, K] of x_dt, 1 <= M <= 8, K % 32 == 0, M*K*4 bytes <= 160 KiB;
 * w_codes [N, K/8]; w_scales LINEAR [N, K/16]; y [M, N] of x_dt. */
NVFP4_API nvfp4_status qmv(const void* x, nvfp4_dtype x_dt, const float* g_x, const uint32_t* w_codes,
                 const uint8_t* w_scales, const float* g_w, int64_t M, int64_t N, int64_t K,
                 void* y, nvfp4_stream_t stream);

/* f3 -- qmv in the MX modes ([P2] QQMatmul::eval_gpu, M = 1 branch, which
 * quantize-dequantizes x with the mode's group size and bits before fp_qmv):
 *   x_hat = T(code(q) * 2^(s-127)) per 32-block of x (s = ue8m0_round_up(
 *   amax / 448) for MXFP8, amax / 6 for MXFP4, codes as mxfp8_quantize /
 *   mxfp4_quantize);  y[m,n] = T(sum_k x_hat[m,k] * code(q[n,k]) *
 *   2^(sw[n,k/32]-127)), fp32 accumulation.  No global scales ([P1]
 *   validate_global_scale: nvfp4 only).
 * mode NVFP4_MODE_MXFP8 (w_codes [N, K/4], e4m3 bytes) or NVFP4_MODE_MXFP4
 * (w_codes [N, K/8], e2m1 nibbles); w_scales LINEAR e8m0 [N, K/32]; x [M, K]
 * of x_dt, 1 <= M <= 8, K % 32 == 0, M*K*4 bytes <= 160 KiB; y [M, N] of
 * x_dt.  A SIMT kernel (a warp per weight row). */
NVFP4_API nvfp4_status qmv_mx(nvfp4_mode mode, const void* x, nvfp4_dtype x_dt, const uint32_t* w_codes,
                              const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* y,
                              nvfp4_stream_t stream);

/* qmv for chains of decode calls whose weights stay fixed (the layers of a
 * model at decode time): the same arguments, checks and result as qmv, but
 * launched with programmatic dependent launch.  The kernel starts streaming
 * w_codes and w_scales (and reads g_w) before the kernel before it on the
 * stream has finished; it reads x and g_x and writes y only after that
 * kernel has completed and its writes are visible.  Each call lets the next
 * launch start at once, so back-to-back calls overlap one weight stream
 * with the previous call's tail.
 * Precondition: w_codes, w_scales and g_w are not written by any work still
 * pending on the device when the call is enqueued (e.g. they were written
 * and the writer synchronized before, as for weights loaded once).  Sizes
 * the tensor-core path does not take (see qmv) run the SIMT kernel in plain
 * stream order. */
NVFP4_API nvfp4_status qmv_pdl(const void* x, nvfp4_dtype x_dt, const float* g_x, const uint32_t* w_codes,
                               const uint8_t* w_scales, const float* g_w, int64_t M, int64_t N, int64_t K,
                               void* y, nvfp4_stream_t stream);

/* a10 -- gather_qmm: MoE matmul with per-expert NVFP4 weights and per-expert
 * global scales ([P3]: the global scale multiplies each fp8 block scale
 * inside the dequantization, before the cast to bf16; weights transposed).
 *   y[t, j, :] = x[t, :] . w_hat_e^T,  e = idx[t, j],
 *   w_hat_e = bf16(e2m1(q) * (f8(s) * g[e] / 2688)),  fp32 accumulation.
 * x [T, K] bf16; w_codes [E, N, K/8]; w_scales LINEAR [E, N, K/16];
 * g [E] fp32 or NULL; idx [T, topk] int32 in [0, E) (checked on the device:
 * out-of-range entries set NVFP4_ERR_DEVICE_INDEX and produce zero rows);
 * y [T, topk, N] bf16.  K % 64 == 0, N % 16 == 0; T*topk, N and K at most
 * 2^30; 1 <= E <= 1024 and E*N < 2^31 (E*K for gather_qmm_kn), the
 * weight rows a 32-bit TMA coordinate reaches (beyond: NVFP4_ERR_UNSUPPORTED).
 * workspace: device scratch of at least gather_qmm_workspace_size(T, topk, E)
 * bytes, 16-byte aligned, contents undefined on entry and exit.  With at
 * least gather_qmm_staged_workspace_size(T, topk, E, K) bytes, calls with
 * T > 16 first copy the routed x rows, grouped by expert, into the
 * workspace and run the SM-pair tensor-core kernel on that copy; with less
 * they run the single-SM kernel that gathers x rows itself.  Both compute
 * the same result (the fp32 sums may differ in rounding order only). */
NVFP4_API nvfp4_status gather_qmm(const void* x, const uint32_t* w_codes, const uint8_t* w_scales,
                        const float* g, const int32_t* idx, int64_t T, int64_t topk,
                        int64_t E, int64_t N, int64_t K, void* y, void* workspace,
                        size_t workspace_bytes, nvfp4_stream_t stream);

/* f2 -- gather_qmm with transpose=False ([P3] tests loop over both layouts):
 * the weights stored [K, N] per expert and quantized along N.
 *   y[t, j, :] = x[t, :] . w_hat_e,  e = idx[t, j],
 *   w_hat_e[k, n] = bf16(e2m1(q[e,k,n]) * (f8(s[e,k,n/16]) * g[e] / 2688)).
 * x [T, K] bf16; w_codes [E, K, N/8]; w_scales LINEAR [E, K, N/16]; g, idx,
 * y, workspace and errors as gather_qmm.  K % 64 == 0, N % 32 == 0.  Every
 * T runs the tensor-core kernel (no separate decode path for this layout). */
NVFP4_API nvfp4_status gather_qmm_kn(const void* x, const uint32_t* w_codes, const uint8_t* w_scales,
                        const float* g, const int32_t* idx, int64_t T, int64_t topk,
                        int64_t E, int64_t N, int64_t K, void* y, void* workspace,
                        size_t workspace_bytes, nvfp4_stream_t stream);

/* Bytes of workspace gather_qmm and gather_qmm_kn need for (T, topk, E);
 * 0 for a triple they reject (T < 0, topk < 1, E outside [1, 1024],
 * T*topk > 2^30).  Host only. */
NVFP4_API size_t gather_qmm_workspace_size(int64_t T, int64_t topk, int64_t E);

/* Bytes of workspace with which gather_qmm stages the routed x rows (see
 * gather_qmm): gather_qmm_workspace_size(T, topk, E) rounded up to 256,
 * plus T*topk*K*2 bytes for the bf16 copy.  0 for arguments gather_qmm
 * rejects (as above, and K outside [0, 2^30]).  Host only. */
NVFP4_API size_t gather_qmm_staged_workspace_size(int64_t T, int64_t topk, int64_t E, int64_t K);

/* gather_qmm without a workspace argument; the pages have no counterpart of
 * this entry point.  It is for callers that cannot allocate device memory
 * themselves: code embedded in a host program that owns the device memory
 * budget and forbids growth after start-up, plugin code that has no handle
 * on its host framework's allocator, or a latency-critical loop where an
 * allocation could block on the device.  It computes exactly what
 * gather_qmm computes, with the same arguments minus the workspace.
 *
 * Scratch: a 1 MiB array inside the library (a static device variable,
 * 256-byte aligned), present on every GPU that loads the library until the
 * process exits.  Calls whose gather_qmm_workspace_size(T, topk, E) exceeds
 * 1 MiB are rejected with NVFP4_ERR_UNSUPPORTED (e.g. T = 4096 tokens, top-8,
 * 64 experts needs about 135 KB).  The call allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the
 * identity of the device's context; make that first call before any stream
 * capture.  A later context on the device (after cudaDeviceReset, which
 * unloads the array) makes the next call look the address up again, so
 * that call too belongs outside a capture.  All calls on a device share the
 * one array, which keeps the previous call's contents (each call rewrites
 * every entry it reads, so nothing has to be cleared); two calls whose
 * kernels overlap on the GPU -- on different streams, or from different
 * host threads -- race on it and must be serialized by the caller. */
NVFP4_API nvfp4_status gather_qmm_noalloc(const void* x, const uint32_t* w_codes, const uint8_t* w_scales,
                                          const float* g, const int32_t* idx, int64_t T, int64_t topk,
                                          int64_t E, int64_t N, int64_t K, void* y, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
