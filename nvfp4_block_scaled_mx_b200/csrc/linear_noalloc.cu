// linear_noalloc.cu -- mxq_linear_noalloc: the quantized linear layer for callers that cannot
// allocate device memory.
//
// Some host programs own every byte of device memory themselves and hand a kernel library only
// its input and output buffers: inference-server plugins that receive no workspace, processes
// running under a hard device-memory cap that must not grow at serving time, or code paths where
// an allocation's implicit device synchronisation is not allowed.  mxq_linear needs a workspace
// for the quantized activations; this entry point takes that workspace from a fixed array that
// lives in the library's own device memory instead of asking the caller for one.
//
// The array is a file-scope static __device__ array of MXQ_NOALLOC_SCRATCH_BYTES bytes.  Every GPU
// that loads this library holds it until the process exits.  Host code cannot use the array's
// name as a device address (on the host it names a stand-in object), so the device address is
// looked up once per device with cudaGetSymbolAddress while that device is current, cached, and
// handed to the kernels as a plain pointer.
#include <cuda_runtime.h>

#include <atomic>

#include "mxq.h"
#include "mxq_internal.h"

static __device__ __align__(256) uint8_t mxq_noalloc_scratch[MXQ_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (set-up on first use per device).
int scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MXQ_ERR_CUDA;
    void* p = g_scratch_addr[dev].load();
    if (p == nullptr) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, mxq_noalloc_scratch) != cudaSuccess || addr == nullptr) {
            (void)cudaGetLastError();  // clear the runtime's last error: the return code reports it
            return MXQ_ERR_CUDA;
        }
        g_scratch_addr[dev].store(addr);
        p = addr;
    }
    *out = p;
    return MXQ_OK;
}

}  // namespace

extern "C" int mxq_linear_noalloc(const void* x_bf16, const void* W_q, const uint8_t* W_sf, const float* g_W,
                                  const float* g_A, int64_t M, int64_t N, int64_t K, mxq_fmt fmt, mxq_rule act_rule,
                                  mxq_out out_type, void* out, mxq_stream_t stream) {
    // the argument checks of mxq_linear, in its order, then the scratch limit in place of the
    // caller's workspace size, then the device: the same codes mxq_linear returns for the same inputs
    int rc = mxq::validate_linear(x_bf16, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, out, false, nullptr);
    if (rc != MXQ_OK) return rc;
    if (mxq_linear_workspace_size(M, K, fmt) > static_cast<size_t>(MXQ_NOALLOC_SCRATCH_BYTES)) return MXQ_ERR_WORKSPACE;
    if ((rc = mxq::check_device()) != MXQ_OK) return rc;
    void* ws = nullptr;
    if ((rc = scratch_address(&ws)) != MXQ_OK) return rc;
    // Everything the GEMM reads from the scratch is rewritten by this call's quantizer (codes of
    // all M rows, scales including their zero padding), so the previous call's contents never leak
    // into the result.
    return mxq::run_linear(x_bf16, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, ws, out,
                           reinterpret_cast<cudaStream_t>(stream));
}
