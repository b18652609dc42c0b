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

#include "../../include/skiparse.h"

namespace {

// Largest B*T*H*W*heads the workspace holds (4,194,304 rows of one fp32 each = 16 MiB).
constexpr long long kNoAllocMaxRows = 1LL << 22;

static __device__ __align__(256) float g_bwd_workspace[kNoAllocMaxRows];

// Device address of the workspace in the current device's context. In host code the array's
// name is only a stand-in for the symbol, never a device address, so the address is asked for
// on every call: a cached address could belong to a context that cudaDeviceReset has since
// destroyed, or to another context the caller made current. The lookup allocates nothing.
int workspace_in_current_context(float** out) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_workspace) != cudaSuccess || !ptr) {
        cudaGetLastError();
        return SKIPARSE_ERR_CUDA;
    }
    *out = static_cast<float*>(ptr);
    return SKIPARSE_OK;
}

}  // namespace

extern "C" int skiparse2d_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                           const void* out, const void* dout, const float* lse,
                                           void* dq, void* dk, void* dv, int B, int T, int H,
                                           int W, int heads, int d, int P, int mode,
                                           skiparse_stream_t stream) {
    // Argument errors first, before any CUDA call, in the order and with the codes of
    // skiparse2d_attn_bwd (which checks the rest -- alignment, overlaps -- before it launches).
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return SKIPARSE_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || P < 1) return SKIPARSE_ERR_INVALID_ARG;
    if (mode != SKIPARSE_TOKEN_WISE && mode != SKIPARSE_GROUP_WISE) return SKIPARSE_ERR_INVALID_ARG;
    if (P > 8 || (d != 32 && d != 64 && d != 128)) return SKIPARSE_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(B) * T * H * W * heads;
    if (rows > kNoAllocMaxRows) return SKIPARSE_ERR_UNSUPPORTED;  // workspace too small
    float* workspace = nullptr;
    const int st = workspace_in_current_context(&workspace);
    if (st != SKIPARSE_OK) return st;
    // The workspace is written in full by the first of the backward's launches before anything
    // reads it, so the previous call's contents never matter and nothing needs clearing.
    return skiparse2d_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace, B, T, H, W, heads,
                               d, P, mode, stream);
}
