// api.cu -- the extern "C" entry points of libmxq.so: argument validation (before any launch),
// workspace layout, device status word, and dispatch to the kernels.
#include <cuda_runtime.h>

#include <atomic>

#include "mxq.h"
#include "mxq_internal.h"

// Status word: kernels record bounded-wait timeouts here (first writer wins).
__device__ int g_mxq_status;

namespace mxq {

namespace {
constexpr int kMaxDevices = 64;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_fmt(int fmt) { return fmt == MXQ_MXFP4 || fmt == MXQ_NVFP4 || fmt == MXQ_MXFP8; }
bool valid_rule(int rule) { return rule == MXQ_RULE_EVEN || rule == MXQ_RULE_CEIL; }
bool valid_out(int out) { return out == MXQ_OUT_BF16 || out == MXQ_OUT_FP32; }

}  // namespace

// Checks the current device is an sm_100 part (the library carries sm_100a code only).
int check_device() {
    static std::atomic<int> verdict[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return MXQ_ERR_CUDA;
    int v = verdict[dev].load();
    if (v == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return MXQ_ERR_CUDA;
        v = (major == 10 && minor == 0) ? 1 : 2;
        verdict[dev].store(v);
    }
    return v == 1 ? MXQ_OK : MXQ_ERR_DEVICE;
}

namespace {

// A dimension the library accepts: 1 <= v < 2^31 (products of two fit in 62 bits).
bool dim_ok(int64_t v) { return v >= 1 && v < (int64_t(1) << 31); }

int q_bytes(int64_t rows, int64_t K, int fmt, size_t* out) {
    if (!dim_ok(rows) || !dim_ok(K)) return MXQ_ERR_SHAPE;
    *out = static_cast<size_t>(rows) * static_cast<size_t>(fmt == MXQ_MXFP8 ? K : K / 2);
    return MXQ_OK;
}

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

int validate_quant(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, const void* q,
                   const void* sf, int layout) {
    if (!valid_fmt(fmt) || (fmt != MXQ_NVFP4 && !valid_rule(rule)) ||
        (layout != MXQ_SF_ROWMAJOR && layout != MXQ_SF_SWIZZLED))
        return MXQ_ERR_UNSUPPORTED;
    if (!x || !q || !sf || (fmt == MXQ_NVFP4 && !g)) return MXQ_ERR_NULL;
    const int bs = block_size(fmt);
    if (!dim_ok(M) || !dim_ok(K) || K < bs || K % bs != 0) return MXQ_ERR_SHAPE;
    if (M * K / 8 >= (int64_t(1) << 31)) return MXQ_ERR_SHAPE;  // block indices are 32-bit
    if (!aligned16(x) || !aligned16(q) || !aligned16(sf) || (g && (reinterpret_cast<uintptr_t>(g) & 3u)))
        return MXQ_ERR_ALIGN;
    return MXQ_OK;
}

int validate_gemm_shape(int64_t M, int64_t N, int64_t K, int fmt) {
    if (M < 1 || N < 1 || M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return MXQ_ERR_SHAPE;
    const int kstep = fmt == MXQ_MXFP8 ? 32 : 64;
    if (K < kstep || K % kstep != 0 || K >= (int64_t(1) << 31)) return MXQ_ERR_SHAPE;
    return MXQ_OK;
}
}  // namespace

int* status_ptr() {
    static std::atomic<int*> ptrs[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    int* p = ptrs[dev].load();
    if (!p) {
        void* sym = nullptr;
        if (cudaGetSymbolAddress(&sym, g_mxq_status) != cudaSuccess) return nullptr;
        p = static_cast<int*>(sym);
        ptrs[dev].store(p);
    }
    return p;
}

int sm_count() {
    static std::atomic<int> counts[kMaxDevices];
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int c = counts[dev].load();
    if (c == 0) {
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
        counts[dev].store(c);
    }
    return c;
}

int validate_linear(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
                    int64_t M, int64_t N, int64_t K, int fmt, int act_rule, int out_type, const void* out,
                    bool caller_workspace, const void* workspace) {
    if (!valid_fmt(fmt) || !valid_out(out_type) || (fmt != MXQ_NVFP4 && !valid_rule(act_rule)))
        return MXQ_ERR_UNSUPPORTED;
    if (!x || !W_q || !W_sf || !out || (caller_workspace && !workspace) || (fmt == MXQ_NVFP4 && (!g_W || !g_A)))
        return MXQ_ERR_NULL;
    int rc = validate_gemm_shape(M, N, K, fmt);
    if (rc != MXQ_OK) return rc;
    if (M * K / 8 >= (int64_t(1) << 31)) return MXQ_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(W_q) || !aligned16(W_sf) || !aligned16(out) ||
        (caller_workspace && !aligned16(workspace)))
        return MXQ_ERR_ALIGN;
    return MXQ_OK;
}

int run_linear(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A, int64_t M,
               int64_t N, int64_t K, int fmt, int act_rule, int out_type, void* workspace, void* out,
               cudaStream_t st) {
    size_t qb = 0;
    q_bytes(M, K, fmt, &qb);
    uint8_t* a_q = static_cast<uint8_t*>(workspace);
    uint8_t* a_sf = a_q + round256(qb);
    // few tokens: one launch, the GEMM quantizing its own activations (the workspace stays unused)
    int rc = launch_linear_fused(x, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, out, st);
    if (rc != kNotFused) return rc;
    if (launch_quantize(x, M, K, fmt, act_rule, g_A, a_q, a_sf, MXQ_SF_SWIZZLED, st) != cudaSuccess)
        return MXQ_ERR_CUDA;
    return launch_gemm(a_q, a_sf, W_q, W_sf, g_A, g_W, M, N, K, fmt, out_type, out, st, true);
}

}  // namespace mxq

using namespace mxq;

extern "C" {

int mxq_block_size(mxq_fmt fmt) { return valid_fmt(fmt) ? block_size(fmt) : MXQ_ERR_UNSUPPORTED; }

int mxq_q_bytes(int64_t rows, int64_t K, mxq_fmt fmt, size_t* bytes) {
    if (!valid_fmt(fmt)) return MXQ_ERR_UNSUPPORTED;
    if (!bytes) return MXQ_ERR_NULL;
    if (K % block_size(fmt) != 0) return MXQ_ERR_SHAPE;
    return q_bytes(rows, K, fmt, bytes);
}

int mxq_sf_bytes(int64_t rows, int64_t K, mxq_fmt fmt, mxq_sf_layout layout, size_t* bytes) {
    if (!valid_fmt(fmt) || (layout != MXQ_SF_ROWMAJOR && layout != MXQ_SF_SWIZZLED)) return MXQ_ERR_UNSUPPORTED;
    if (!bytes) return MXQ_ERR_NULL;
    const int bs = block_size(fmt);
    if (!dim_ok(rows) || !dim_ok(K) || K < bs || K % bs != 0) return MXQ_ERR_SHAPE;
    const int64_t kb = K / bs;
    *bytes = static_cast<size_t>(layout == MXQ_SF_SWIZZLED ? swizzled_sf_bytes(rows, kb) : rows * kb);
    return MXQ_OK;
}

int mxq_quantize(const void* x_bf16, int64_t M, int64_t K, mxq_fmt fmt, mxq_rule rule, const float* global_scale,
                 void* q_out, void* sf_out, mxq_sf_layout layout, mxq_stream_t stream) {
    int rc = validate_quant(x_bf16, M, K, fmt, rule, global_scale, q_out, sf_out, layout);
    if (rc != MXQ_OK) return rc;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return launch_quantize(x_bf16, M, K, fmt, rule, global_scale, q_out, sf_out, layout,
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_quantize_running(const void* x_bf16, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q_out,
                         void* sf_out, mxq_sf_layout layout, mxq_stream_t stream) {
    if (!amax_out) return MXQ_ERR_NULL;
    int rc = validate_quant(x_bf16, M, K, MXQ_NVFP4, 0, amax_in, q_out, sf_out, layout);
    if (rc != MXQ_OK) return rc;
    if (reinterpret_cast<uintptr_t>(amax_out) & 3u) return MXQ_ERR_ALIGN;
    if (static_cast<const void*>(amax_in) == static_cast<const void*>(amax_out)) return MXQ_ERR_UNSUPPORTED;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return launch_quantize_running(x_bf16, M, K, amax_in, amax_out, q_out, sf_out, layout,
                                   reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_fake_quantize(const void* x_bf16, int64_t M, int64_t K, mxq_fmt fmt, mxq_rule rule, const float* global_scale,
                      void* y_bf16, mxq_stream_t stream) {
    // same argument rules as mxq_quantize; y takes the place of the codes (and may equal x)
    int rc = validate_quant(x_bf16, M, K, fmt, rule, global_scale, y_bf16, y_bf16, MXQ_SF_ROWMAJOR);
    if (rc != MXQ_OK) return rc;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return launch_fake_quantize(x_bf16, M, K, fmt, rule, global_scale, y_bf16, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_swizzle_scales(const uint8_t* sf_rowmajor, int64_t rows, int64_t kblocks, uint8_t* sf_swizzled,
                       mxq_stream_t stream) {
    if (!sf_rowmajor || !sf_swizzled) return MXQ_ERR_NULL;
    if (rows < 1 || kblocks < 1 || rows >= (int64_t(1) << 31) || kblocks >= (int64_t(1) << 24)) return MXQ_ERR_SHAPE;
    int rc = check_device();
    if (rc != MXQ_OK) return rc;
    return launch_swizzle(sf_rowmajor, rows, kblocks, sf_swizzled, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_global_scale(const void* x_bf16, int64_t n, float* g_out, float* amax_out, mxq_stream_t stream) {
    if (!x_bf16 || !g_out || !amax_out) return MXQ_ERR_NULL;
    if (n < 1) return MXQ_ERR_SHAPE;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(g_out) & 3u) || (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return MXQ_ERR_ALIGN;
    int rc = check_device();
    if (rc != MXQ_OK) return rc;
    return launch_global_scale(x_bf16, n, g_out, amax_out, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_amax(const void* x_bf16, int64_t n, float* amax_out, mxq_stream_t stream) {
    if (!x_bf16 || !amax_out) return MXQ_ERR_NULL;
    if (n < 1) return MXQ_ERR_SHAPE;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(amax_out) & 3u)) return MXQ_ERR_ALIGN;
    int rc = check_device();
    if (rc != MXQ_OK) return rc;
    return launch_global_scale(x_bf16, n, nullptr, amax_out, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MXQ_OK
               : MXQ_ERR_CUDA;
}

int mxq_gemm(const void* A_q, const uint8_t* A_sf, const void* B_q, const uint8_t* B_sf, const float* g_A,
             const float* g_B, int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_out out_type, void* out,
             mxq_stream_t stream) {
    if (!valid_fmt(fmt) || !valid_out(out_type)) return MXQ_ERR_UNSUPPORTED;
    if (!A_q || !A_sf || !B_q || !B_sf || !out || (fmt == MXQ_NVFP4 && (!g_A || !g_B))) return MXQ_ERR_NULL;
    int rc = validate_gemm_shape(M, N, K, fmt);
    if (rc != MXQ_OK) return rc;
    if (!aligned16(A_q) || !aligned16(A_sf) || !aligned16(B_q) || !aligned16(B_sf) || !aligned16(out))
        return MXQ_ERR_ALIGN;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return launch_gemm(A_q, A_sf, B_q, B_sf, g_A, g_B, M, N, K, fmt, out_type, out,
                       reinterpret_cast<cudaStream_t>(stream), true);
}

int mxq_gemm_w4a16(const void* A, const void* W_q, const uint8_t* W_sf, const float* g_W, int64_t M, int64_t N,
                   int64_t K, mxq_fmt fmt, mxq_out out_type, void* out, mxq_stream_t stream) {
    if ((fmt != MXQ_MXFP4 && fmt != MXQ_NVFP4) || !valid_out(out_type)) return MXQ_ERR_UNSUPPORTED;
    if (!A || !W_q || !W_sf || !out || (fmt == MXQ_NVFP4 && !g_W)) return MXQ_ERR_NULL;
    int rc = validate_gemm_shape(M, N, K, fmt);
    if (rc != MXQ_OK) return rc;
    if (!aligned16(A) || !aligned16(W_q) || !aligned16(W_sf) || !aligned16(out)) return MXQ_ERR_ALIGN;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return launch_w4a16(A, W_q, W_sf, g_W, M, N, K, fmt, out_type, out, reinterpret_cast<cudaStream_t>(stream));
}

int mxq_linear_kernel_count(int64_t M, int64_t N, int64_t K, mxq_fmt fmt) {
    if (!valid_fmt(fmt)) return MXQ_ERR_UNSUPPORTED;
    int rc = validate_gemm_shape(M, N, K, fmt);
    if (rc != MXQ_OK) return rc;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return linear_fused_splits(M, N, K, fmt) > 0 ? 1 : 2;
}

size_t mxq_linear_workspace_size(int64_t M, int64_t K, mxq_fmt fmt) {
    if (!valid_fmt(fmt) || !dim_ok(M) || !dim_ok(K) || K % block_size(fmt) != 0) return 0;
    size_t qb = 0;
    q_bytes(M, K, fmt, &qb);
    return round256(qb) + static_cast<size_t>(swizzled_sf_bytes(M, K / block_size(fmt)));
}

int mxq_linear(const void* x_bf16, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
               int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_rule act_rule, mxq_out out_type, void* workspace,
               size_t ws_bytes, void* out, mxq_stream_t stream) {
    int rc = validate_linear(x_bf16, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, out, true, workspace);
    if (rc != MXQ_OK) return rc;
    if (ws_bytes < mxq_linear_workspace_size(M, K, fmt)) return MXQ_ERR_WORKSPACE;
    if ((rc = check_device()) != MXQ_OK) return rc;
    return run_linear(x_bf16, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, workspace, out,
                      reinterpret_cast<cudaStream_t>(stream));
}

int mxq_device_status(int* status_out, int reset, mxq_stream_t stream) {
    if (!status_out) return MXQ_ERR_NULL;
    int* p = status_ptr();
    if (!p) return MXQ_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, p, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MXQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MXQ_ERR_CUDA;
    if (reset) {
        if (cudaMemsetAsync(p, 0, sizeof(int), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
            return MXQ_ERR_CUDA;
    }
    *status_out = v;
    return MXQ_OK;
}

int mxq_selftest_timeout(uint64_t timeout_ns, mxq_stream_t stream) {
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return MXQ_ERR_SHAPE;
    int rc = check_device();
    if (rc != MXQ_OK) return rc;
    return launch_selftest_timeout(timeout_ns, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? MXQ_OK
                                                                                                       : MXQ_ERR_CUDA;
}

const char* mxq_strerror(int code) {
    switch (code) {
        case MXQ_OK: return "ok";
        case MXQ_ERR_NULL: return "null pointer argument";
        case MXQ_ERR_SHAPE: return "shape out of range or not a multiple of the block / MMA step";
        case MXQ_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MXQ_ERR_UNSUPPORTED: return "unsupported format, rule, output type or layout";
        case MXQ_ERR_WORKSPACE: return "workspace too small";
        case MXQ_ERR_CUDA: return "CUDA launch or query failed";
        case MXQ_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
        case MXQ_ERR_DEVICE: return "device is not sm_100 (B200)";
        default: return "unknown mxq error";
    }
}

}  // extern "C"
