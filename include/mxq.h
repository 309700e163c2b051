/*
 * mxq.h -- C ABI of the B200 (sm_100a) microscaling W4A4 linear-layer library (libmxq.so).
 *
 * The library implements the hot path of a block-scaled quantized linear layer,
 * Out = A * W^T with A [M, K] activations and W [N, K] weights (nn.Linear layout):
 *   - MXFP4: E2M1 elements in blocks of 32 along K with one E8M0 (power-of-two) scale per block,
 *     the EVEN rule for weights and the CEIL rule for per-token dynamic activation quantization
 *     ("Qwen3.5-27B-MXFP4-QAD-W4A4-LR1e-5-s1000", "How this checkpoint was produced", Training row;
 *      "Qwen3.5-9B-MXFP4-QAD-W4A4-LR1e-5-s3000", "Training mode" paragraph);
 *   - NVFP4: E2M1 elements, blocks of 16 with an E4M3 scale, and one fp32 per-tensor global scale
 *     ("Qwen3.5-27B-NVFP4-RTN-weight-only", first paragraph; "Qwen3.5-27B-NVFP4-GPTQ", Recipe row);
 *   - MXFP8: E4M3 elements, blocks of 32 with an E8M0 scale
 *     ("intel-ai/Qwen3.8-27B-MXFP4-AutoRound", section 1 and section 7, OCP MX).
 *
 * Scale rules (block amax over |x|, e clamped to [-127, 127], amax = 0 gives e = -127):
 *   EVEN  e = floor(log2 amax) - emax_elem           (emax_elem 2 for E2M1, 8 for E4M3)
 *   CEIL  e = least integer with amax <= elem_max * 2^e   (elem_max 6 for E2M1, 448 for E4M3)
 * MX elements are RNE(x / 2^e) on the element grid, saturating at +-elem_max.
 * NVFP4 (fp32 IEEE, g = global scale in the decode direction, x ~ q * s * g):
 *   s = RNE_E4M3_satfinite(fl(fl(amax/6) / g)) (0 for an all-zero block), d = fl(dec(s) * g),
 *   q_i = RNE_E2M1_sat(fl(x_i * fl(1/d))); when d == 0 every code is a zero that keeps x_i's sign.
 *   Where fl(1/d) overflows to +inf (d < 2^-128, only with an fp32-subnormal g), a nonzero x_i
 *   saturates to +-6 and a zero x_i stays a zero with its sign (0 * inf has no E2M1 code).
 *
 * Conventions for every call:
 *   - Pointers marked (device) are device memory of the current CUDA device; the caller owns and
 *     allocates every buffer.  The compute calls allocate nothing.
 *   - Calls are asynchronous and stream-ordered on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Return MXQ_OK (0) or a negative MXQ_ERR_* code.  Argument errors are detected on the host
 *     before anything is launched; MXQ_ERR_CUDA reports a failed launch.
 *   - Device pointers must be 16-byte aligned.
 *   - Quantized FP4 data: [rows, K/2] bytes, element 2i in bits 0-3 and element 2i+1 in bits 4-7
 *     of byte i of the row.  MXFP8 data: [rows, K] bytes of E4M3 codes.
 *   - Row-major scales: [rows, K/bs] bytes.  Swizzled scales (what the GEMM consumes): tiles of
 *     128 rows x 4 scale columns, 512 bytes each, ordered [ceil(rows/128)][ceil((K/bs)/4)]; inside a
 *     tile, scale (r, c) sits at byte (r%32)*16 + ((r%128)/32)*4 + c%4.  Padding bytes are zero.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mxq_stream_t; /* same type as cudaStream_t */

typedef enum { MXQ_MXFP4 = 0, MXQ_NVFP4 = 1, MXQ_MXFP8 = 2 } mxq_fmt;
typedef enum { MXQ_RULE_EVEN = 0, MXQ_RULE_CEIL = 1 } mxq_rule; /* ignored for NVFP4 */
typedef enum { MXQ_OUT_BF16 = 0, MXQ_OUT_FP32 = 1 } mxq_out;
typedef enum { MXQ_SF_ROWMAJOR = 0, MXQ_SF_SWIZZLED = 1 } mxq_sf_layout;

#define MXQ_OK 0
#define MXQ_ERR_NULL (-1)        /* a required pointer is NULL */
#define MXQ_ERR_SHAPE (-2)       /* M, N or K out of range, or K not a multiple of what fmt needs */
#define MXQ_ERR_ALIGN (-3)       /* a pointer is not 16-byte aligned */
#define MXQ_ERR_UNSUPPORTED (-4) /* unknown fmt / rule / out / layout */
#define MXQ_ERR_WORKSPACE (-5)   /* workspace smaller than mxq_linear_workspace_size() */
#define MXQ_ERR_CUDA (-6)        /* a CUDA launch or query failed */
#define MXQ_ERR_TIMEOUT (-7)     /* a kernel gave up on a bounded wait (see mxq_device_status) */
#define MXQ_ERR_DEVICE (-8)      /* the current device is not sm_100 */

/* Block size along K: 32 for MXFP4/MXFP8, 16 for NVFP4. */
int mxq_block_size(mxq_fmt fmt);

/* Bytes of quantized element data for a [rows, K] matrix (rows*K/2 for FP4, rows*K for MXFP8). */
int mxq_q_bytes(int64_t rows, int64_t K, mxq_fmt fmt, size_t* bytes);

/* Bytes of the scale tensor for a [rows, K] matrix in the given layout (swizzled is padded). */
int mxq_sf_bytes(int64_t rows, int64_t K, mxq_fmt fmt, mxq_sf_layout layout, size_t* bytes);

/*
 * Quantize x [M, K] bf16 (device, row-major, K contiguous) along K.
 *   fmt, rule     element format and MX scale rule (rule ignored for NVFP4).
 *   global_scale  (device) fp32[1], the NVFP4 decode-direction global scale g > 0; NULL otherwise.
 *   q_out         (device) mxq_q_bytes() bytes; sf_out (device) mxq_sf_bytes(layout) bytes.
 * Requires M >= 1 and K >= bs with K % bs == 0.  The activation path ("Qwen3.5-9B-MXFP4-QAD-W4A4-
 * LR1e-5-s3000", "Training mode") is fmt=MXFP4, rule=CEIL; the RTN weight export
 * ("Qwen3.5-27B-NVFP4-RTN-weight-only", Training row: round-to-nearest) is rule=EVEN.
 */
int mxq_quantize(const void* x_bf16, int64_t M, int64_t K, mxq_fmt fmt, mxq_rule rule,
                 const float* global_scale, void* q_out, void* sf_out, mxq_sf_layout layout,
                 mxq_stream_t stream);

/*
 * NVFP4 quantization with a running-max activation global scale, the observer fused into the
 * quantizer ("Qwen3.5-27B-NVFP4-GPTQ", Serving-KL table and caveat: the RTN export's running-max
 * input scales).  The block scales use g = fl(*amax_in / (6 * 448)), the running state from earlier
 * batches (device fp32[1], positive); in the same pass *amax_out receives max(*amax_in, max |x|),
 * the state for the next call.  amax_in and amax_out must be different buffers (swap them between
 * calls).  Other arguments as mxq_quantize with fmt = NVFP4.
 */
int mxq_quantize_running(const void* x_bf16, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q_out,
                         void* sf_out, mxq_sf_layout layout, mxq_stream_t stream);

/*
 * Fake quantization (quantize, then dequantize back to bf16): y = bf16(dq(Q(x))) with exactly the
 * codes and scales mxq_quantize produces, decoded in the format's precision (MX: elem * 2^e, exact;
 * NVFP4: fl32(elem * d), d = fl32(dec(s) * g)) and rounded once to bf16 (RNE).  This is the
 * fake-quantized forward of quantization-aware training, bit-identical to the serving quantizer
 * ("Qwen3.5-9B-MXFP4-QAD-W4A4-LR1e-5-s3000", "Training mode": W4A4 fake-quant, EVEN weights, CEIL
 * activations).  x, y: [M, K] bf16 (device); y may be x (in place).  Arguments as mxq_quantize.
 */
int mxq_fake_quantize(const void* x_bf16, int64_t M, int64_t K, mxq_fmt fmt, mxq_rule rule, const float* global_scale,
                      void* y_bf16, mxq_stream_t stream);

/*
 * Re-lay row-major scales [rows, kblocks] (device) into the swizzled tensor-core layout
 * (device, mxq_sf_bytes(SWIZZLED) bytes, padding zeroed).  Pure byte permutation.
 * The pages do not describe this layout: they only store the scales as U8 tensors
 * ("intel-ai/Qwen3.8-27B-MXFP4-AutoRound", section 1 "Model summary", Weight dtype row) that the
 * serving FP4 kernel consumes.  The layout is
 * the one the tcgen05 block-scaled MMA reads its scale factors in (128-row x 4-column tiles, see the
 * conventions above); this library's own reading, confirmed end to end by the GEMM parity tests.
 *   sf_rowmajor  (device) rows * kblocks bytes, read only.
 *   sf_swizzled  (device) mxq_sf_bytes(rows, K, fmt, MXQ_SF_SWIZZLED) bytes, written whole.
 * Errors: MXQ_ERR_NULL for a NULL pointer, MXQ_ERR_SHAPE unless 1 <= rows < 2^31 and
 * 1 <= kblocks < 2^24; nothing is launched then.
 */
int mxq_swizzle_scales(const uint8_t* sf_rowmajor, int64_t rows, int64_t kblocks, uint8_t* sf_swizzled,
                       mxq_stream_t stream);

/*
 * NVFP4 per-tensor global scale of x (n bf16 values, device): amax_out = max |x| and
 * g_out = fl(amax / (6 * 448)) in fp32 (decode direction), both device fp32[1].  This is the
 * running-max form of input_global_scale ("Qwen3.5-27B-NVFP4-GPTQ", Serving-KL table, RTN row).
 */
int mxq_global_scale(const void* x_bf16, int64_t n, float* g_out, float* amax_out, mxq_stream_t stream);

/*
 * Tensor amax of x (n bf16 values, device, 16-byte aligned): *amax_out = max |x| (device fp32[1],
 * exact: a bf16 value is an fp32 value).  This is the tensor-max helper a caller uses to derive a
 * dynamic NVFP4 global scale or to feed a running-max observer ("Qwen3.5-27B-NVFP4-GPTQ",
 * Serving-KL table: running-max versus static input scales); mxq_global_scale is the same
 * reduction followed by g = fl(amax / (6 * 448)).  Errors: MXQ_ERR_NULL, MXQ_ERR_SHAPE (n < 1),
 * MXQ_ERR_ALIGN; nothing is launched then.  Stream-ordered; allocates nothing.
 */
int mxq_amax(const void* x_bf16, int64_t n, float* amax_out, mxq_stream_t stream);

/*
 * Block-scaled GEMM on the tcgen05 tensor cores: out[M, N] = alpha * dq(A) dq(B)^T, fp32
 * accumulation, alpha = g_A[0] * g_B[0] for NVFP4 and 1 otherwise ("Qwen3.5-9B-MXFP4-QAD-W4A4-
 * LR1e-5-s3000", Serving: FP4 GEMM on quantized activations and weights).
 *   A_q [M, K] and B_q [N, K] quantized data (device); A_sf, B_sf SWIZZLED scales (device).
 *   g_A, g_B  (device) fp32[1] NVFP4 global scales; ignored (may be NULL) for MX formats.
 *   out       (device) [M, N] bf16 (RNE) or fp32, row-major.
 * Requires M, N >= 1; K >= 64 with K % 64 == 0 for FP4 and K % 32 == 0 for MXFP8.  There is no
 * lower bound on N beyond 1.
 */
int mxq_gemm(const void* A_q, const uint8_t* A_sf, const void* B_q, const uint8_t* B_sf, const float* g_A,
             const float* g_B, int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_out out_type, void* out,
             mxq_stream_t stream);

/*
 * Weight-only (W4A16) GEMM: out[M, N] = alpha * A dq(W)^T with bf16 activations A and MXFP4 or
 * NVFP4 weights, alpha = g_W[0] for NVFP4 and 1 for MXFP4.  This is the weight-only serving mode:
 * "Qwen3.5-27B-NVFP4-RTN-weight-only" (activations run bf16, no input_global_scale) and the
 * Marlin mode of "Qwen3.5-27B-MXFP4-QAD-W4A4-LR1e-5-s1000" ("Evaluation results": one weight
 * artifact serves W4A4 and W4A16).  W is dequantized to bf16 inside the kernel and multiplied on
 * the tcgen05 tensor cores (bf16 x bf16, fp32 accumulation).
 *   A        (device) [M, K] bf16, row-major.
 *   W_q      (device) [N, K/2] packed E2M1 codes; W_sf (device) their SWIZZLED scales, the same
 *            bytes mxq_gemm and mxq_linear read.
 *   g_W      (device) fp32[1] NVFP4 global scale of W; ignored (may be NULL) for MXFP4.
 *   out      (device) [M, N] bf16 (RNE) or fp32, row-major.
 * Requires fmt MXQ_MXFP4 or MXQ_NVFP4 (else MXQ_ERR_UNSUPPORTED), M, N >= 1, K >= 64 with
 * K % 64 == 0, 16-byte aligned pointers.  The dequantized weights are exact in bf16 for every
 * scale the EVEN-rule weight quantizer emits (E8M0 codes up to 252, E4M3 codes up to 0x7E); larger
 * E8M0 codes can overflow and are outside the contract.  Stream-ordered; allocates nothing.
 */
int mxq_gemm_w4a16(const void* A, const void* W_q, const uint8_t* W_sf, const float* g_W, int64_t M, int64_t N,
                   int64_t K, mxq_fmt fmt, mxq_out out_type, void* out, mxq_stream_t stream);

/* Workspace bytes mxq_linear needs for M tokens of width K (quantized A plus swizzled scales). */
size_t mxq_linear_workspace_size(int64_t M, int64_t K, mxq_fmt fmt);

/*
 * Kernels one mxq_linear call launches for this problem on the current device: 1 when the GEMM
 * quantizes its own activations (up to 32 tokens with several K splits; the workspace then stays
 * unused), 2 otherwise (quantizer, then GEMM).  The shape checks of mxq_linear come first (negative
 * MXQ_ERR_* codes), then the device check (MXQ_ERR_DEVICE / MXQ_ERR_CUDA without a usable sm_100
 * device).  Useful to plan CUDA-graph capture and to count launches.
 */
int mxq_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxq_fmt fmt);

/*
 * Quantized linear layer, the W4A4 serving path: the activations are quantized dynamically per
 * token at run time and multiplied with the pre-quantized weights by an FP4 GEMM
 * ("Qwen3.5-9B-MXFP4-QAD-W4A4-LR1e-5-s3000", Serving, W4A4 bullet; the CEIL activation rule from its
 * "Training mode" paragraph).  out = dq(Q(x)) dq(W)^T * alpha with Q the quantizer of mxq_quantize.
 *   x_bf16     (device) [M, K] bf16 activations, row-major.
 *   W_q, W_sf  (device) the pre-quantized weights [N, K] (mxq_quantize output) with SWIZZLED scales.
 *   g_W, g_A   (device) fp32[1] NVFP4 global scales of W and of x (decode direction); ignored (may
 *              be NULL) for MX formats.
 *   act_rule   MX scale rule of the activations (ignored for NVFP4).
 *   workspace  (device) at least mxq_linear_workspace_size(M, K, fmt) bytes, caller-owned, 16-byte
 *              aligned: the quantized activations and their swizzled scales (up to 32 tokens the
 *              call may not touch it).
 *   out        (device) [M, N] bf16 (RNE) or fp32, row-major.
 * Requirements as mxq_gemm, plus M * K / 8 < 2^31.  The quantizer and the GEMM run back to back on
 * `stream` with programmatic dependent launch (one launch up to 32 tokens, see
 * mxq_linear_kernel_count); A is quantized once, not once per output tile.  Errors are checked in
 * this order before anything is launched: MXQ_ERR_UNSUPPORTED (fmt, act_rule, out_type),
 * MXQ_ERR_NULL, MXQ_ERR_SHAPE, MXQ_ERR_ALIGN, MXQ_ERR_WORKSPACE (ws_bytes too small),
 * MXQ_ERR_DEVICE; MXQ_ERR_CUDA reports a failed launch.
 */
int mxq_linear(const void* x_bf16, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
               int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_rule act_rule, mxq_out out_type,
               void* workspace, size_t ws_bytes, void* out, mxq_stream_t stream);

/*
 * mxq_linear without a caller-supplied workspace.  The pages have no counterpart: this call exists
 * for callers that are not allowed to allocate device memory -- e.g. plugins inside a host
 * framework that owns all device memory and passes only input and output buffers, or processes
 * under a fixed device-memory cap that must not grow (or synchronise the device through an
 * allocation) while serving.
 *
 * The activation workspace comes from a static array inside the library, MXQ_NOALLOC_SCRATCH_BYTES
 * bytes per GPU, held by every GPU that loads the library until the process exits.  Problems
 * whose mxq_linear_workspace_size(M, K, fmt) exceeds that size are rejected with
 * MXQ_ERR_WORKSPACE before anything is launched (8 MiB covers, e.g., up to 2048 tokens at K = 5120
 * for FP4).  Other arguments, requirements, error codes (in mxq_linear's order, the scratch limit
 * taking the place of the workspace size) and results are exactly those of mxq_linear: the same
 * kernels on the same bytes, so the output is bit-identical.  The caller still provides x, the
 * quantized weights and `out`.  The call allocates nothing.
 *
 * The first call on a device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture.  All calls share the one array
 * and it keeps the last call's contents (each call rewrites everything it reads), so calls whose
 * executions overlap on the GPU -- e.g. on two streams without ordering between them -- race.
 */
#define MXQ_NOALLOC_SCRATCH_BYTES (8u << 20)
int mxq_linear_noalloc(const void* x_bf16, const void* W_q, const uint8_t* W_sf, const float* g_W,
                       const float* g_A, int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_rule act_rule,
                       mxq_out out_type, void* out, mxq_stream_t stream);

/* Read the device status word that kernels set when a bounded wait gives up (0 = clean).
 * Synchronizes `stream`.  If reset != 0 the word is cleared afterwards. */
int mxq_device_status(int* status_out, int reset, mxq_stream_t stream);

/* Self-test of the bounded-wait path: launches one CTA that waits on a barrier nothing completes,
 * with a limit of timeout_ns; the kernel records MXQ_ERR_TIMEOUT in the status word and returns.
 * Returns MXQ_OK if the launch succeeded (read the outcome with mxq_device_status). */
int mxq_selftest_timeout(uint64_t timeout_ns, mxq_stream_t stream);

/* Human-readable name of an MXQ_* code. */
const char* mxq_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* MXQ_H */
