// no_alloc.cu -- a backward-pass entry point for callers that cannot allocate device memory.
//
// skiparse2d_attn_bwd needs a (B, T, H, W, heads) fp32 workspace, which its caller allocates.
// Some callers cannot: a host framework or plugin interface that hands a library only the
// tensors of the operation and owns every allocation itself; a latency-critical loop that must
// not call cudaMalloc (it can synchronize the whole device); a deployment that pre-reserves its
// whole memory budget up front. skiparse2d_attn_bwd_noalloc serves them: it keeps the workspace
// in a fixed-size array that belongs to this library (kNoAllocMaxRows fp32 values, 16 MiB, held
// on every device that loads the library until the process exits) and otherwise runs exactly
// the kernels of skiparse2d_attn_bwd.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/skiparse.h"

namespace {

// Largest B*T*H*W*heads the workspace holds (4,194,304 rows of one fp32 each = 16 MiB).
constexpr long long kNoAllocMaxRows = 1LL << 22;

static __device__ __align__(256) float g_bwd_workspace[kNoAllocMaxRows];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_workspace_ptr[kMaxDevices] = {nullptr};

// Device address of the workspace on the current device. In host code the array's name is only
// a stand-in for the symbol, never a device address, so the address is asked for once per
// device (with that device current) and cached.
int workspace_on_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return SKIPARSE_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return SKIPARSE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_workspace_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_bwd_workspace) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return SKIPARSE_ERR_CUDA;
        }
        g_workspace_ptr[dev] = static_cast<float*>(ptr);
    }
    *out = g_workspace_ptr[dev];
    return SKIPARSE_OK;
}

}  // namespace

extern "C" int skiparse2d_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                           const void* out, const void* dout, const float* lse,
                                           void* dq, void* dk, void* dv, int B, int T, int H,
                                           int W, int heads, int d, int P, int mode,
                                           skiparse_stream_t stream) {
    if (B > 0 && T > 0 && H > 0 && W > 0 && heads > 0) {
        const long long rows = static_cast<long long>(B) * T * H * W * heads;
        if (rows > kNoAllocMaxRows) return SKIPARSE_ERR_UNSUPPORTED;  // workspace too small
    }
    float* workspace = nullptr;
    const int st = workspace_on_current_device(&workspace);
    if (st != SKIPARSE_OK) return st;
    // The workspace is written in full by the first of the backward's launches before anything
    // reads it, so the previous call's contents never matter and nothing needs clearing.
    return skiparse2d_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace, B, T, H, W, heads,
                               d, P, mode, stream);
}
