// mxq_internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "mxq.h"

namespace mxq {

// Device status word of the current device (kernels record bounded-wait timeouts there).
int* status_ptr();

// MXQ_OK if the current device is an sm_100 part, MXQ_ERR_DEVICE otherwise (MXQ_ERR_CUDA when the
// query fails); cached per device.
int check_device();

// Host-side argument checks of the linear layer, in mxq_linear's order (unsupported enum, NULL
// pointer, shape, alignment); the workspace pointer is checked only when the caller supplies one.
int validate_linear(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
                    int64_t M, int64_t N, int64_t K, int fmt, int act_rule, int out_type, const void* out,
                    bool caller_workspace, const void* workspace);

// The linear layer's launches on validated arguments: the one-launch few-token path, else the
// quantizer into `workspace` (mxq_linear_workspace_size bytes) followed by the GEMM.
int run_linear(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A, int64_t M,
               int64_t N, int64_t K, int fmt, int act_rule, int out_type, void* workspace, void* out,
               cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int sm_count();

// cuTensorMapEncodeTiled from the driver (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline int block_size(int fmt) { return fmt == MXQ_NVFP4 ? 16 : 32; }

inline int64_t swizzled_sf_bytes(int64_t rows, int64_t kblocks) {
    return ceil_div(rows, 128) * 128 * ceil_div(kblocks, 4) * 4;
}

// Quantizer launch (arguments already validated).  `pdl_primary` lets a dependent kernel launched
// with programmatic stream serialization start early.
cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, void* q,
                            void* sf, int layout, cudaStream_t stream);

cudaError_t launch_quantize_running(const void* x, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q,
                                   void* sf, int layout, cudaStream_t stream);

cudaError_t launch_fake_quantize(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, void* y,
                                 cudaStream_t stream);

cudaError_t launch_swizzle(const uint8_t* src, int64_t rows, int64_t kblocks, uint8_t* dst, cudaStream_t stream);

// Tensor amax of n bf16 values into *amax_out, then g = fl(amax / 2688) into *g_out (skipped when
// g_out is NULL).
cudaError_t launch_global_scale(const void* x, int64_t n, float* g_out, float* amax_out, cudaStream_t stream);

// GEMM launch.  `pdl_secondary` launches with programmatic stream serialization so that the
// kernel's prologue overlaps the tail of the preceding kernel on the stream.
int launch_gemm(const void* A_q, const uint8_t* A_sf, const void* B_q, const uint8_t* B_sf, const float* g_A,
                const float* g_B, int64_t M, int64_t N, int64_t K, int fmt, int out_type, void* out,
                cudaStream_t stream, bool pdl_secondary);

// Linear layer in one launch where the GEMM quantizes the bf16 activations x itself (rule `rule`
// for MX formats, global scale g_A for NVFP4) with the quantizer's arithmetic: the few-token kernel
// for up to 32 tokens (the result equals quantize-then-GEMM bit for bit), and the small-N kernel
// for more tokens and N <= 128.  Returns kNotFused (nothing launched) otherwise; arguments already
// validated.
constexpr int kNotFused = 1;
// K splits of the one-launch path for this problem on the current device (the few-token kernel
// quantizing up to 32 token rows, or the small-N kernel quantizing whole 128-row M tiles for N <= 128;
// 1 when that kernel runs without a K split), 0 when no one-launch path applies.
int linear_fused_splits(int64_t M, int64_t N, int64_t K, int fmt);
int launch_linear_fused(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
                        int64_t M, int64_t N, int64_t K, int fmt, int rule, int out_type, void* out,
                        cudaStream_t stream);

// Weight-only (W4A16) GEMM launch (arguments already validated).
int launch_w4a16(const void* A, const void* W_q, const uint8_t* W_sf, const float* g_W, int64_t M, int64_t N,
                 int64_t K, int fmt, int out_type, void* out, cudaStream_t stream);

cudaError_t launch_selftest_timeout(uint64_t timeout_ns, cudaStream_t stream);

}  // namespace mxq
