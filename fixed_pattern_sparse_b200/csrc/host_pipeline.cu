// host_pipeline.cu -- the attention forward called with HOST buffers: host->device copies, the
// fused kernel and device->host copies of one call, overlapped across groups of heads.
//
// Heads are independent in every step of the method (each (class, head) subsequence attends on
// its own), so a call is cut into groups of `heads_per_group` heads. A group's q, k, v rows are
// copied (one pitched copy per tensor: the group's heads are a contiguous run inside every token
// row) into a compact (B, T, H, W, group_heads, d) device buffer, the unmodified fused kernel runs
// on it, and its output rows are copied back into the group's heads of the host output. Three
// library-owned streams per device -- copies in, kernels, copies out -- and two workspace buffer
// sets let group g's kernel run while group g+1 is copied in and group g-1 is copied out. The
// call is ordered after earlier work on the caller's stream and later work on that stream waits
// for it, as for every other entry point.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/skiparse.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSets = 2;  // workspace buffer sets (double buffering)

struct DeviceQueues {
    bool ready = false;
    cudaStream_t in = nullptr, run = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in_ready[kSets] = {}, in_free[kSets] = {}, out_ready[kSets] = {}, out_free[kSets] = {};
};

std::mutex g_queue_mutex;
DeviceQueues g_queues[kMaxDevices];

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return SKIPARSE_OK;
    cudaGetLastError();
    return SKIPARSE_ERR_CUDA;
}

// Streams and events of the current device, created on first use (the caller holds the mutex).
int queues_for_current_device(DeviceQueues** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
    if (dev < 0 || dev >= kMaxDevices) return SKIPARSE_ERR_UNSUPPORTED;
    DeviceQueues& q = g_queues[dev];
    if (!q.ready) {
        const unsigned ev_flags = cudaEventDisableTiming;
        cudaError_t e = cudaStreamCreateWithFlags(&q.in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&q.run, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&q.out, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.start, ev_flags);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.done, ev_flags);
        for (int s = 0; s < kSets && e == cudaSuccess; ++s) {
            e = cudaEventCreateWithFlags(&q.in_ready[s], ev_flags);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.in_free[s], ev_flags);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.out_ready[s], ev_flags);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&q.out_free[s], ev_flags);
        }
        if (e != cudaSuccess) return cuda_status(e);
        q.ready = true;
    }
    *out = &q;
    return SKIPARSE_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Bytes of one (B,T,H,W,group_heads,d) bf16 buffer.
size_t group_buffer_bytes(long long ntok, int group_heads, int d) {
    return align256(static_cast<size_t>(ntok) * group_heads * d * 2);
}

using AttnFn = int (*)(const void*, const void*, const void*, void*, int, int, int, int, int, int,
                       int, int, skiparse_stream_t);
using NumelFn = long long (*)(int, int, int, int, int, int, int);

int attn_fwd_host_common(AttnFn attn, NumelFn numel, const void* q, const void* k, const void* v, void* out,
                         int B, int T, int H, int W, int heads, int d, int P, int mode,
                         int heads_per_group, void* workspace, size_t workspace_bytes,
                         skiparse_stream_t stream) {
    if (!q || !k || !v || !out || !workspace) return SKIPARSE_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || P < 1) return SKIPARSE_ERR_INVALID_ARG;
    if (heads_per_group < 1 || heads_per_group > heads) return SKIPARSE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SKIPARSE_ERR_MISALIGNED;
    const long long ntok = static_cast<long long>(B) * T * H * W;
    const long long need = skiparse_attn_fwd_host_workspace_bytes(B, T, H, W, heads, d, heads_per_group);
    if (need < 0) return SKIPARSE_ERR_INVALID_ARG;
    if (workspace_bytes < static_cast<size_t>(need)) return SKIPARSE_ERR_INVALID_ARG;
    if (mode != SKIPARSE_TOKEN_WISE && mode != SKIPARSE_GROUP_WISE) return SKIPARSE_ERR_INVALID_ARG;
    // d, P and the sizes of one group, checked before anything is enqueued
    if (numel(B, T, H, W, heads_per_group, d, P) < 0) return SKIPARSE_ERR_UNSUPPORTED;
    const size_t tensor_bytes = static_cast<size_t>(ntok) * heads * d * 2;
    const void* ins[3] = {q, k, v};
    for (const void* in : ins) {
        const uintptr_t a = reinterpret_cast<uintptr_t>(out), b = reinterpret_cast<uintptr_t>(in);
        if (a < b + tensor_bytes && b < a + tensor_bytes) return SKIPARSE_ERR_INVALID_ARG;
    }
    const size_t buf = group_buffer_bytes(ntok, heads_per_group, d);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    std::lock_guard<std::mutex> lock(g_queue_mutex);
    DeviceQueues* dq = nullptr;
    int st = queues_for_current_device(&dq);
    if (st != SKIPARSE_OK) return st;
    cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaEventRecord(dq->start, user);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(dq->in, dq->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(dq->run, dq->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(dq->out, dq->start, 0);
    if (e != cudaSuccess) return cuda_status(e);

    const size_t row_bytes = static_cast<size_t>(heads) * d * 2;  // one token row on the host
    const int ngroups = (heads + heads_per_group - 1) / heads_per_group;
    for (int g = 0; g < ngroups && e == cudaSuccess; ++g) {
        const int s = g % kSets;
        const int h0 = g * heads_per_group;
        const int hg = heads - h0 < heads_per_group ? heads - h0 : heads_per_group;
        const size_t grp_bytes = static_cast<size_t>(hg) * d * 2;   // the group's part of a row
        const size_t host_off = static_cast<size_t>(h0) * d * 2;
        uint8_t* set = ws + static_cast<size_t>(s) * 4 * buf;
        uint8_t* dbuf[4] = {set, set + buf, set + 2 * buf, set + 3 * buf};  // q, k, v, out
        const void* hin[3] = {q, k, v};
        // copies in: the group's heads of every token row -> a compact device tensor
        if (g >= kSets) e = cudaStreamWaitEvent(dq->in, dq->in_free[s], 0);
        for (int t = 0; t < 3 && e == cudaSuccess; ++t)
            e = cudaMemcpy2DAsync(dbuf[t], grp_bytes, static_cast<const uint8_t*>(hin[t]) + host_off,
                                  row_bytes, grp_bytes, static_cast<size_t>(ntok),
                                  cudaMemcpyHostToDevice, dq->in);
        if (e == cudaSuccess) e = cudaEventRecord(dq->in_ready[s], dq->in);
        // the fused kernel on the group
        if (e == cudaSuccess) e = cudaStreamWaitEvent(dq->run, dq->in_ready[s], 0);
        if (e == cudaSuccess && g >= kSets) e = cudaStreamWaitEvent(dq->run, dq->out_free[s], 0);
        if (e != cudaSuccess) break;
        st = attn(dbuf[0], dbuf[1], dbuf[2], dbuf[3], B, T, H, W, hg, d, P, mode,
                  reinterpret_cast<skiparse_stream_t>(dq->run));
        if (st != SKIPARSE_OK) break;
        e = cudaEventRecord(dq->in_free[s], dq->run);
        if (e == cudaSuccess) e = cudaEventRecord(dq->out_ready[s], dq->run);
        // copies out: the compact output -> the group's heads of the host rows
        if (e == cudaSuccess) e = cudaStreamWaitEvent(dq->out, dq->out_ready[s], 0);
        if (e == cudaSuccess)
            e = cudaMemcpy2DAsync(static_cast<uint8_t*>(out) + host_off, row_bytes, dbuf[3], grp_bytes,
                                  grp_bytes, static_cast<size_t>(ntok), cudaMemcpyDeviceToHost, dq->out);
        if (e == cudaSuccess) e = cudaEventRecord(dq->out_free[s], dq->out);
    }
    // Later work on the caller's stream waits for everything enqueued above (the copies out
    // follow every kernel and the copies in precede them), also after a failure part-way.
    cudaError_t e2 = cudaEventRecord(dq->done, dq->out);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(user, dq->done, 0);
    if (st != SKIPARSE_OK) return st;
    return cuda_status(e != cudaSuccess ? e : e2);
}

}  // namespace

extern "C" long long skiparse_attn_fwd_host_workspace_bytes(int B, int T, int H, int W, int heads,
                                                            int d, int heads_per_group) {
    if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || d < 1) return -1;
    if (heads_per_group < 1 || heads_per_group > heads) return -1;
    const long long ntok = static_cast<long long>(B) * T * H * W;
    if (ntok * heads >= (1LL << 31)) return -1;
    return static_cast<long long>(kSets) * 4 * static_cast<long long>(group_buffer_bytes(ntok, heads_per_group, d));
}

extern "C" int skiparse2d_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                        int B, int T, int H, int W, int heads, int d, int P,
                                        int mode, int heads_per_group, void* workspace,
                                        size_t workspace_bytes, skiparse_stream_t stream) {
    return attn_fwd_host_common(skiparse2d_attn_fwd, skiparse_rearranged_numel, q, k, v, out, B, T, H, W, heads, d, P, mode,
                                heads_per_group, workspace, workspace_bytes, stream);
}

extern "C" int skiparse1d_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                        int B, int T, int H, int W, int heads, int d, int P,
                                        int mode, int heads_per_group, void* workspace,
                                        size_t workspace_bytes, skiparse_stream_t stream) {
    return attn_fwd_host_common(skiparse1d_attn_fwd, skiparse1d_rearranged_numel, q, k, v, out, B, T, H, W, heads, d, P, mode,
                                heads_per_group, workspace, workspace_bytes, stream);
}
