/*
 * w4a4.h -- C ABI of libw4a4, the DSFQ W4A4 quantized linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * DSFQ = Dual-Smoothed Fine-Grained Quantization, the quantizer of QuantVGGT.
 * Sources (page "十亿参数的三维重建模型，能塞进手机吗？", a translation of the
 * QuantVGGT paper):
 *   [PTQ]    section 训练后量化（PTQ）: symmetric N-bit quantizer,
 *            q = clamp(round(x / delta), -2^(N-1), 2^(N-1) - 1); here N = 4.
 *   [ROT]    section 预全局旋转（Pre-Global-Rotation）: Hadamard rotation of
 *            activations and weights along the input features, H H^T = I.
 *   [SMOOTH] section 后局部平滑（Post-Local-Smooth）: per-channel smoothing
 *            factors computed in the rotated space, alpha = 0.5, applied
 *            after the rotation and folded into the weights.
 *   [GRAN]   section 细粒度量化粒度: read as one step per token for
 *            activations and one step per output channel for weights.
 *
 * Per layer, with X [M, K] bf16 activations and W [N, K] bf16 weights:
 *   offline : Wt = W H/sqrt(K); s_j = max|Xt_calib[:,j]|^a / max|Wt[:,j]|^(1-a);
 *             W^ = Wt diag(s); qw[n,:] = int4(W^[n,:]), delta_ch[n] = max|W^[n,:]|/7
 *   online  : X^ = (X H/sqrt(K)) diag(s)^-1; qx[m,:] = int4(X^[m,:]),
 *             delta_tok[m] = max|X^[m,:]|/7;
 *             Y[m,n] = bf16( (sum_k qx[m,k] qw[n,k]) * delta_tok[m] * delta_ch[n] + b[n] )
 *   int4(v) = round-half-even(v / delta) with delta = max|v| / 7 (codes in [-7, 7];
 *   an all-zero row has delta = 0 and zero codes).  H is the Sylvester
 *   Hadamard matrix in natural order, K in {1024, 4096}.
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     allocates nothing and keeps no pointer after a call returns.
 *   - Arrays are row-major and contiguous.  bf16 values are passed as their
 *     raw 16-bit patterns (uint16_t).
 *   - Packed int4 codes: two per byte, element 2i in the low nibble, element
 *     2i+1 in the high nibble, each nibble the 4-bit two's complement code.
 *   - Alignment: every array pointer and the workspace must be 16-byte
 *     aligned (the kernels use 16-byte vector accesses and TMA).  Violations
 *     return W4A4_ERR_ALIGN.
 *   - Shapes: K must be 1024 or 4096 (W4A4_ERR_UNSUPPORTED otherwise); N must
 *     be a positive multiple of 256 (W4A4_ERR_SHAPE); M >= 0, and M = 0 is a
 *     no-op that returns W4A4_OK once the shape, flag and weight checks pass
 *     (the M-sized pointers may then be NULL).  M must stay below 2^31.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns without synchronizing, except
 *     w4a4_get_device_status.  Launch failures return W4A4_ERR_CUDA.
 *   - Argument checks happen on the host before anything is enqueued; a call
 *     that returns an error enqueued nothing.
 *   - Kernels never trap.  Every wait inside a kernel is bounded; a wait that
 *     runs out sets W4A4_DEV_TIMEOUT in the device status word (read it with
 *     w4a4_get_device_status) and the kernel returns early, leaving its output
 *     undefined.
 *   - Calls on the same stream are ordered; the library holds no state
 *     between calls except the device status word.
 */
#ifndef W4A4_H_
#define W4A4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    W4A4_OK = 0,
    W4A4_ERR_ARG = 1,          /* null pointer or invalid scalar argument */
    W4A4_ERR_SHAPE = 2,        /* M, N or workspace size not accepted */
    W4A4_ERR_ALIGN = 3,        /* pointer not aligned as required */
    W4A4_ERR_UNSUPPORTED = 4,  /* K not in {1024, 4096}, or unknown flag */
    W4A4_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed */
    W4A4_ERR_TIMEOUT = 6       /* a kernel reported a bounded wait running out */
} w4a4_status;

/* Bits of the device status word (w4a4_get_device_status). */
#define W4A4_DEV_TIMEOUT 0x1u

/* Flags. */
#define W4A4_FLAG_GELU  0x1u  /* quantize_act / linear_fused: apply exact-erf GELU
                                 to X (rounded to bf16) before the rotation; the
                                 input of an MLP's second linear.  The value is
                                 the exact GELU rounded to bf16 for every bf16 x
                                 with 1e-30 <= |x| <= 5.9375; x itself above
                                 5.9375; -8.6e-9 below -5.9375 (the exact values
                                 lie between it and 0); x/2 within one bf16 step
                                 for |x| < 1e-30 */
#define W4A4_FLAG_PLAIN 0x2u  /* no rotation and no smoothing: plain per-token /
                                 per-channel int4 quantization (the baseline that
                                 DSFQ is measured against); must match between
                                 prepare_weights and the activation calls */
#define W4A4_FLAG_INT8  0x4u  /* the W8A8 setting (reported beside W4A4 in the
                                 results of the summary page of "量化視覺幾何基礎變換器",
                                 lsdiaocha.cn, camera-pose paragraph): the same
                                 steps with the symmetric 8-bit quantizer of [PTQ],
                                 delta = absmax/127, one signed int8 code per byte
                                 in natural order, for activations and weights;
                                 must match between prepare_weights and the
                                 activation calls */
#define W4A4_FLAG_UNPACKED 0x8u  /* quantize_act / linear_ex: the int4 codes one per
                                 byte (int8 values in [-7, 7]) instead of two per
                                 byte, in the operand order of w4a4_expand_weights
                                 (within every 8 elements: 0, 2, 4, 6, 1, 3, 5, 7).
                                 Not on the pages: the tensor cores multiply 8-bit
                                 operands, and codes that arrive one per byte need
                                 no widening in the GEMM (which otherwise widens
                                 every activation tile once per output tile).
                                 Not with W4A4_FLAG_INT8. */
#define W4A4_FLAG_GELU_OUT 0x10u  /* linear_ex / linear_fused: Y = bf16(GELU(y)) of
                                 the bf16-rounded output y, the same exact-erf GELU
                                 as W4A4_FLAG_GELU, applied by the GEMM epilogue
                                 to the output of an MLP's first linear instead of
                                 by the quantize kernel to the input of its second
                                 (both give the same bf16 values: the MLP block of
                                 page "十亿参数的三维重建模型，能塞进手机吗？",
                                 section 视觉几何基础 Transformer（VGGT）, with its
                                 activation placed where it costs least). */

#define W4A4_FLAG_FWHT 0x100u  /* quantize_act / linear_fused: rotate the activations
                                 with the CUDA-core fast Walsh-Hadamard transform
                                 instead of the tensor cores.  The same method either
                                 way ([ROT]: x H / sqrt(K)); the two differ only in
                                 fp32 rounding, so codes may differ at rounding ties.
                                 By default the DSFQ path (no W4A4_FLAG_PLAIN, no
                                 W4A4_FLAG_GELU) uses the tensor cores, via
                                 H_K = H_128 (x) H_(K/128): the 128-point factor as a
                                 bf16 product (exact inputs, fp32 sums), the small
                                 factor in fp32 registers; W4A4_FLAG_PLAIN has no
                                 rotation and W4A4_FLAG_GELU inputs use the CUDA-core
                                 transform. */

/* Prepared weights of one linear layer.  The caller allocates every array
 * (device memory) with the sizes given and keeps ownership. */
typedef struct {
    int32_t N;            /* output features, multiple of 256 */
    int32_t K;            /* input features, 1024 or 4096 */
    uint8_t *qw;          /* [N, K/2] packed int4 codes of W^ */
    float *scale_ch;      /* [N] delta_ch */
    float *bias;          /* [N] fp32 bias (zeros when the layer has none) */
    float *smooth;        /* [K] s */
    float *inv_smooth;    /* [K] 1/s (what the activation quantizer multiplies by) */
    int8_t *qw8;          /* optional [N, K] int8: the codes of qw widened to 8 bits in the
                             order the tensor-core kernel consumes them (see
                             w4a4_expand_weights).  NULL: the GEMM widens the packed qw on
                             every tile instead (no extra memory, lower throughput).
                             With W4A4_FLAG_INT8: required, the [N, K] 8-bit codes of W^
                             in natural order (qw and colsum are then unused, may be NULL) */
    int32_t *colsum;      /* [N] sum over k of the int4 codes of row n; required when qw8
                             is set (NULL otherwise) */
    uint32_t flags;       /* W4A4_FLAG_PLAIN when prepared without DSFQ, W4A4_FLAG_INT8 for
                             8-bit codes */
} w4a4_weights_t;

/* Bytes of one device allocation that holds every array of a prepared layer
 * [PTQ][GRAN] (what w4a4_weights_bind lays out in it), each array starting at
 * a 256-byte boundary:
 *   flags 0:                    qw [N, K/2] packed int4 codes, scale_ch [N],
 *                               bias [N], smooth [K], inv_smooth [K];
 *   + W4A4_FLAG_UNPACKED:       also qw8 [N, K] (the codes widened to one per
 *                               byte in operand order, w4a4_expand_weights) and
 *                               colsum [N] (the tensor-core GEMM's fast route);
 *   W4A4_FLAG_INT8:             qw8 [N, K] 8-bit codes, scale_ch, bias, smooth,
 *                               inv_smooth (no qw, no colsum).
 * W4A4_FLAG_PLAIN may be given and changes nothing.  About N*K/2 + 12 N + 8 K
 * bytes for packed int4 weights, against 2 N K + 2 N for bf16 weights and bias.
 * Returns 0 for an unsupported K, an N that is not a positive multiple of 256,
 * or another flag. */
size_t w4a4_weights_bytes(int32_t N, int32_t K, uint32_t flags);

/* Points out's arrays into `base` (device memory of at least
 * w4a4_weights_bytes(N, K, flags) bytes, 16-byte aligned, owned by the caller)
 * in the layout w4a4_weights_bytes describes and sets out->N, out->K; pointers
 * the layout does not use are set to NULL, out->flags to 0.  Reads and writes
 * no device memory: fill the arrays with w4a4_prepare_weights (same flags
 * minus W4A4_FLAG_UNPACKED).  W4A4_ERR_ARG for NULL base or out,
 * W4A4_ERR_ALIGN for a misaligned base, W4A4_ERR_SHAPE when `bytes` is too
 * small or N, K are not accepted, W4A4_ERR_UNSUPPORTED for another flag. */
w4a4_status w4a4_weights_bind(void *base, size_t bytes, int32_t N, int32_t K, uint32_t flags,
                              w4a4_weights_t *out);

/* Bytes of workspace that let w4a4_linear_fused take its fastest route for M
 * tokens of width K, whatever the weights and flags: activation codes one per
 * byte (M*K, rounded up to 256) followed by the per-token steps (4*M).
 * Returns 0 for an unsupported K. */
size_t w4a4_workspace_bytes(int64_t M, int32_t K);

/* The least workspace w4a4_linear_fused accepts for these flags: codes two per
 * byte (M*K/2 rounded up to 256, + 4*M) for 4-bit weights, one per byte
 * (M*K ...) with W4A4_FLAG_INT8 or W4A4_FLAG_UNPACKED.  Returns 0 for an
 * unsupported K or an unknown flag. */
size_t w4a4_workspace_bytes_min(int64_t M, int32_t K, uint32_t flags);

/* Offline weight preparation [ROT][SMOOTH][PTQ][GRAN].
 *   W       [N, K] bf16 weights; bias [N] bf16 or NULL;
 *   X_calib [M_calib, K] bf16 calibration activations (M_calib >= 1), used
 *           only for the per-channel activation maxima of the smoothing step;
 *   alpha   smoothing exponent in [0, 1] (the page uses 0.5);
 *   flags   0, W4A4_FLAG_PLAIN (then s = 1 and no rotation; X_calib may be
 *           NULL) and/or W4A4_FLAG_INT8 (8-bit codes into out->qw8);
 *   out     caller-allocated arrays to fill; out->N and out->K must equal N
 *           and K; out->flags is set to (flags & (W4A4_FLAG_PLAIN |
 *           W4A4_FLAG_INT8)); for 4-bit codes, when out->qw8 is set, qw8 and
 *           colsum are filled too (w4a4_expand_weights).
 * Rounding decisions are taken in binary32.  A channel whose activation or
 * weight maximum is zero gets s_j = 1. */
w4a4_status w4a4_prepare_weights(const uint16_t *W, const uint16_t *bias, int32_t N, int32_t K,
                                 const uint16_t *X_calib, int64_t M_calib, float alpha,
                                 uint32_t flags, w4a4_weights_t *out, void *stream);

/* Widens the packed codes w->qw into w->qw8 (the tensor-core operand order:
 * within every group of 8 consecutive codes k = 8g..8g+7 the bytes hold codes
 * 8g+0, 2, 4, 6, 1, 3, 5, 7, as signed int8) and writes w->colsum[n] =
 * sum_k code[n, k].  Both arrays must be set.  Not on the pages: weights are
 * static, so the per-tile widening of B is hoisted to preparation time.
 * W4A4_ERR_ARG for weights prepared with W4A4_FLAG_INT8 (nothing to widen). */
w4a4_status w4a4_expand_weights(w4a4_weights_t *w, void *stream);

/* Online activation quantizer [ROT][SMOOTH][PTQ][GRAN]: for each of the M
 * rows of X [M, K] bf16: optional GELU (W4A4_FLAG_GELU), rotation X H/sqrt(K),
 * multiplication by inv_smooth [K], per-token step delta = absmax/7 written to
 * scale_tok [M] (fp32), codes round-half-even(x / delta) packed into qx
 * [M, K/2].  With W4A4_FLAG_PLAIN the rotation and smoothing are skipped
 * (inv_smooth may then be NULL).  With W4A4_FLAG_INT8, delta = absmax/127 and
 * qx [M, K] holds one int8 code per element; with W4A4_FLAG_UNPACKED, qx [M, K]
 * holds the int4 codes one per byte in operand order.  Inputs must be finite. */
w4a4_status w4a4_quantize_act(const uint16_t *X, int64_t M, int32_t K, const float *inv_smooth,
                              uint8_t *qx, float *scale_tok, uint32_t flags, void *stream);

/* Quantized linear from codes: Y [M, N] bf16 =
 *   round-to-nearest-even( (qx qw^T)[m,n] * scale_tok[m] * w->scale_ch[n] + w->bias[n] ).
 * The integer product is exact (int32 accumulation on the tensor cores); the
 * epilogue is fp32.  For weights prepared with W4A4_FLAG_INT8, qx is [M, K]
 * int8 (w4a4_quantize_act with W4A4_FLAG_INT8). */
w4a4_status w4a4_linear(const uint8_t *qx, const float *scale_tok, int64_t M,
                        const w4a4_weights_t *w, uint16_t *Y, void *stream);

/* w4a4_linear with the code layout of qx given by flags: 0 (as w4a4_linear)
 * or W4A4_FLAG_UNPACKED for 4-bit weights that carry qw8 (then qx [M, K] holds
 * the int4 codes one per byte in operand order, as w4a4_quantize_act writes
 * them with that flag; W4A4_ERR_ARG without qw8); W4A4_FLAG_GELU_OUT may be
 * added (the GELU on the output).  Other flags: W4A4_ERR_UNSUPPORTED. */
w4a4_status w4a4_linear_ex(const uint8_t *qx, const float *scale_tok, int64_t M,
                           const w4a4_weights_t *w, uint16_t *Y, uint32_t flags, void *stream);

/* Quantized linear from bf16 activations: w4a4_quantize_act (with
 * w->inv_smooth and the given flags) into `workspace`, then w4a4_linear_ex.
 * workspace_bytes says how many bytes workspace holds: at least
 * w4a4_workspace_bytes_min(M, w->K, flags) (W4A4_ERR_SHAPE otherwise).  For
 * 4-bit weights with qw8 and a workspace of w4a4_workspace_bytes(M, w->K)
 * bytes the codes go one per byte (W4A4_FLAG_UNPACKED layout) and the GEMM
 * reads them without widening; otherwise they are packed two per byte.  The
 * workspace afterwards holds those codes, then (at the next 256-byte boundary)
 * the steps.  flags must carry the same W4A4_FLAG_PLAIN and W4A4_FLAG_INT8
 * bits as w->flags (W4A4_ERR_ARG otherwise); W4A4_FLAG_GELU applies the GELU
 * to X, W4A4_FLAG_GELU_OUT to Y (both may be given); W4A4_FLAG_UNPACKED is not
 * a flag of this call (W4A4_ERR_UNSUPPORTED). */
w4a4_status w4a4_linear_fused(const uint16_t *X, int64_t M, const w4a4_weights_t *w, uint16_t *Y,
                              void *workspace, size_t workspace_bytes, uint32_t flags,
                              void *stream);

/* Size of the scratch array built into the library for
 * w4a4_linear_fused_noalloc (8 MiB on every GPU that loads the library). */
#define W4A4_NOALLOC_SCRATCH_BYTES (8u << 20)

/* w4a4_linear_fused for callers that cannot allocate device memory.  No page
 * describes this; it serves callers that may not call cudaMalloc / cudaFree
 * where they run (cudaFree synchronizes the whole device; a serving loop with a
 * fixed memory budget or a plugin host's enqueue callback may forbid any
 * allocation after start-up) or that only hold the input and output buffers
 * another runtime handed them.  Same arguments and result as
 * w4a4_linear_fused without the workspace: the codes and steps go to a scratch
 * array of W4A4_NOALLOC_SCRATCH_BYTES inside the library instead, so the call
 * allocates nothing.
 *   - Accepts M with w4a4_workspace_bytes_min(M, w->K, flags) <=
 *     W4A4_NOALLOC_SCRATCH_BYTES (4-bit codes: M <= 16256 tokens at K = 1024,
 *     M <= 4088 at K = 4096; 8-bit codes: about half of that); larger M
 *     returns W4A4_ERR_SHAPE.  Up to about half those sizes the codes go one
 *     per byte (the faster route of w4a4_linear_fused).
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept per CUDA context: after
 *     cudaDeviceReset, or under another context of the same device, the next
 *     call looks it up again (make that call, too, outside a capture).
 *   - Every call on a device shares the one scratch array, which keeps the
 *     last call's contents: calls that may overlap on the GPU (different
 *     streams without ordering between them) race on it and must not be
 *     issued. */
w4a4_status w4a4_linear_fused_noalloc(const uint16_t *X, int64_t M, const w4a4_weights_t *w,
                                      uint16_t *Y, uint32_t flags, void *stream);

/* ---------------------------------------------------------------------------
 * Host-buffer entry point.  No page describes one: it is the layer as a caller
 * with inputs and outputs in host memory uses it (the pages' deployment keeps
 * activations on the accelerator).  The M rows are processed in chunks of
 * chunk_rows; the host->device copy of a chunk, the two kernels of the
 * previous chunk and the device->host copy of the one before run at the same
 * time on three streams, so the call takes about as long as its larger copy
 * direction instead of the sum of both copies and the kernels.  Every row's
 * result is the same as w4a4_linear_fused's (rows are independent).
 * ------------------------------------------------------------------------- */

/* Chunk buffers in flight (per direction). */
#define W4A4_PIPE_DEPTH 2

/* The streams and events of the pipeline: created by w4a4_host_pipe_create on
 * the current device, owned by the caller, reusable across calls (calls on one
 * pipe must be issued from one host thread at a time). */
typedef struct w4a4_host_pipe w4a4_host_pipe_t;

/* Creates a pipe on the current device (two non-blocking streams and
 * 3 * W4A4_PIPE_DEPTH events without timing).  *out receives the handle;
 * W4A4_ERR_CUDA if a stream or event cannot be created. */
w4a4_status w4a4_host_pipe_create(w4a4_host_pipe_t **out);

/* Waits for the pipe's streams and frees it (NULL is a no-op). */
w4a4_status w4a4_host_pipe_destroy(w4a4_host_pipe_t *pipe);

/* Device workspace for w4a4_linear_fused_host: W4A4_PIPE_DEPTH slots, each
 * holding one chunk's X (2 chunk_rows K bytes), Y (2 chunk_rows N bytes),
 * codes and steps (w4a4_workspace_bytes(chunk_rows, K)), each part 256-byte
 * aligned. */
size_t w4a4_host_workspace_bytes(int64_t chunk_rows, int32_t K, int32_t N);

/* Flags of w4a4_linear_fused_host only: X_host (W4A4_FLAG_X_DEVICE) or Y_host
 * (W4A4_FLAG_Y_DEVICE) is a device pointer (16-byte aligned) instead, read or
 * written in place without copies -- the first or last layer of a stack whose
 * other layers run on the device. */
#define W4A4_FLAG_X_DEVICE 0x20u
#define W4A4_FLAG_Y_DEVICE 0x40u

/* Y_host [M, N] bf16 = w4a4_linear_fused(X_host [M, K] bf16) with X_host and
 * Y_host in host memory (page-locked memory for the copies to overlap; pageable
 * memory works but serializes), unless flagged as device memory above.  workspace: device memory of at least
 * w4a4_host_workspace_bytes(chunk_rows, w->K, w->N) bytes, 16-byte aligned;
 * chunk_rows > 0 (a multiple of 128 uses whole GEMM tiles).  The call enqueues
 * the work and returns; `stream` (the compute stream; NULL = legacy default
 * stream) is made to wait for the last copy, so work enqueued on it afterwards,
 * or a synchronize of it, sees Y_host complete.  Flags and errors as
 * w4a4_linear_fused, plus W4A4_FLAG_X_DEVICE / W4A4_FLAG_Y_DEVICE; M = 0 is a
 * no-op. */
w4a4_status w4a4_linear_fused_host(const uint16_t *X_host, int64_t M, const w4a4_weights_t *w,
                                   uint16_t *Y_host, int64_t chunk_rows, void *workspace,
                                   size_t workspace_bytes, w4a4_host_pipe_t *pipe,
                                   uint32_t flags, void *stream);

/* Integer product only: acc [M, N] int32 = sum_k qx[m, k] * code_w[n, k] for
 * packed activation codes qx [M, K/2] and the weight codes of *w (w->qw8 and
 * w->colsum when set, else the packed w->qw; scale_ch, bias and the smoothing
 * arrays are not used and may be NULL); for weights with W4A4_FLAG_INT8, qx
 * [M, K] and w->qw8 hold int8 codes.  Same tensor-core kernel as
 * w4a4_linear with the raw accumulators written out: the integer product is
 * exact. */
w4a4_status w4a4_gemm_s32(const uint8_t *qx, int64_t M, const w4a4_weights_t *w, int32_t *acc,
                          void *stream);

/* Failure-path test of the bounded waits (include/w4a4.h conventions): with
 * this bit, w4a4_gemm_s32_ex launches the GEMM with its TMA producer issuing
 * no copy and every bounded wait limited to 1 ms, so the consumers' waits run
 * out: the kernel sets W4A4_DEV_TIMEOUT in the device status word, drains,
 * frees its tensor memory and returns, leaving acc undefined.  Not for
 * computing anything. */
#define W4A4_DEBUG_STALL 0x80000000u

/* w4a4_gemm_s32 with flags: 0; W4A4_FLAG_UNPACKED (qx [M, K] holds the int4
 * codes one per byte in operand order, the layout w4a4_quantize_act writes with
 * that flag; the weights must carry qw8); W4A4_DEBUG_STALL may be added.
 * Other flags: W4A4_ERR_UNSUPPORTED. */
w4a4_status w4a4_gemm_s32_ex(const uint8_t *qx, int64_t M, const w4a4_weights_t *w, int32_t *acc,
                             uint32_t flags, void *stream);

/* Synchronizes `stream`, then copies the device status word (bits
 * W4A4_DEV_*) of the current device into *status.  Returns W4A4_ERR_TIMEOUT
 * when a bit is set, W4A4_OK otherwise. */
w4a4_status w4a4_get_device_status(void *stream, uint32_t *status);

/* Clears the device status word of the current device (enqueued on stream). */
w4a4_status w4a4_clear_device_status(void *stream);

/* Human-readable name of a status code (static string). */
const char *w4a4_status_string(w4a4_status s);

/* Library version string. */
const char *w4a4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* W4A4_H_ */
