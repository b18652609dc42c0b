// skiparse_api.cu -- the C ABI of libskiparse.so (declared in include/skiparse.h):
// argument validation, Skiparse-2D and Skiparse-1D geometry, kernel launch and the per-device
// status word.
// Nothing here allocates device memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/skiparse.h"
#include "skiparse_internal.cuh"

namespace {

using skiparse::Geometry;

__device__ int g_skiparse_status = 0;  // one error word per device

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
thread_local const char* t_last_cuda_error = "no error";

// Records a failed CUDA call's message for skiparse_last_error_string(); returns the status.
int cuda_fail(int err) {
    t_last_cuda_error = cudaGetErrorString(static_cast<cudaError_t>(err));
    return SKIPARSE_ERR_CUDA;
}
std::atomic<int> g_fault{0};
// Debug builds: rows by which the next launch's bounds are declared smaller than its tensors
// (skiparse_debug_shrink_bounds), so that a test sees the bounds check report without any
// access leaving a tensor. Consumed by the next launch.
std::atomic<long long> g_bounds_shrink{0};

long long checked_bound(long long rows) {
    const long long shrink = g_bounds_shrink.exchange(0);
    return SKIPARSE_DEBUG ? rows - shrink : rows;
}

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

int padded(int X, int P) { return ((X + P * P - 1) / (P * P)) * (P * P); }

// Real (unpadded) positions of class c along an axis of X real positions with P classes: the
// sub-grid positions whose coordinate (axis_coord) is below X. Token-wise the coordinates are
// c, c+P, c+2P, ...; group-wise every full P^2 block gives each class P positions and the last,
// partial block gives class c the part of [c*P, c*P+P) below X's remainder.
int axis_real_count(int X, int c, int P, int mode) {
    if (mode == SKIPARSE_TOKEN_WISE) return c < X ? (X - c + P - 1) / P : 0;
    const int q = P * P, rem = X % q - c * P;
    return (X / q) * P + (rem < 0 ? 0 : rem > P ? P : rem);
}

// Validates the shared shape arguments and fills the geometry of Skiparse-2D (dims 2) or
// Skiparse-1D (dims 1). Returns a status code.
int make_geometry(int dims, int B, int T, int H, int W, int heads, int d, int P, int mode,
                  Geometry& g) {
    if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || P < 1) return SKIPARSE_ERR_INVALID_ARG;
    if (mode != SKIPARSE_TOKEN_WISE && mode != SKIPARSE_GROUP_WISE) return SKIPARSE_ERR_INVALID_ARG;
    if (P > skiparse::kMaxP) return SKIPARSE_ERR_UNSUPPORTED;
    if (d != 32 && d != 64 && d != 128) return SKIPARSE_ERR_UNSUPPORTED;
    const long long q2 = static_cast<long long>(P) * P;
    if (H > (1 << 24) || W > (1 << 24)) return SKIPARSE_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(B) * T * H * W * heads;       // original rows
    if (rows >= (1ll << 31)) return SKIPARSE_ERR_UNSUPPORTED;
    // The frame axes the class rule runs on and the class count along each.
    const long long Hax = dims == 2 ? H : 1, Wax = dims == 2 ? W : static_cast<long long>(H) * W;
    const long long Ph = dims == 2 ? P : 1, Pw = dims == 2 ? P : q2;
    const long long Hp = (Hax + Ph * Ph - 1) / (Ph * Ph) * (Ph * Ph);
    const long long Wp = (Wax + Pw * Pw - 1) / (Pw * Pw) * (Pw * Pw);
    const long long prow = static_cast<long long>(B) * T * Hp * Wp * heads;     // rearranged rows
    if (prow >= (1ll << 31)) return SKIPARSE_ERR_UNSUPPORTED;
    if (heads > 65535 || B * q2 > 65535) return SKIPARSE_ERR_UNSUPPORTED;
    g.B = B; g.T = T; g.heads = heads; g.d = d; g.P = P; g.mode = mode;
    g.H = static_cast<int>(Hax);
    g.W = static_cast<int>(Wax);
    g.Ph = static_cast<int>(Ph);
    g.Pw = static_cast<int>(Pw);
    g.Hp = static_cast<int>(Hp);
    g.Wp = static_cast<int>(Wp);
    g.R = g.Hp / g.Ph;
    g.S = g.Wp / g.Pw;
    g.n = static_cast<long long>(T) * g.R * g.S;
    for (int c = 0; c < skiparse::kMaxAxisClasses; ++c) {
        g.Rc[c] = c < g.Ph ? axis_real_count(g.H, c, g.Ph, mode) : 0;
        g.Sc[c] = c < g.Pw ? axis_real_count(g.W, c, g.Pw, mode) : 0;
    }
    return SKIPARSE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t abytes, const void* b, size_t bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bbytes && b0 < a0 + abytes;
}

int* status_ptr() {
    int* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_skiparse_status);
    if (e != cudaSuccess) {
        cudaGetLastError();
        cuda_fail(e);
        return nullptr;
    }
    return p;
}

}  // namespace

extern "C" {

const char* skiparse_status_string(int status) {
    switch (status) {
        case SKIPARSE_OK: return "SKIPARSE_OK";
        case SKIPARSE_ERR_INVALID_ARG: return "SKIPARSE_ERR_INVALID_ARG";
        case SKIPARSE_ERR_UNSUPPORTED: return "SKIPARSE_ERR_UNSUPPORTED";
        case SKIPARSE_ERR_MISALIGNED: return "SKIPARSE_ERR_MISALIGNED";
        case SKIPARSE_ERR_CUDA: return "SKIPARSE_ERR_CUDA";
        case SKIPARSE_ERR_TIMEOUT: return "SKIPARSE_ERR_TIMEOUT";
        case SKIPARSE_ERR_BOUNDS: return "SKIPARSE_ERR_BOUNDS";
        default: return "SKIPARSE_ERR_UNKNOWN";
    }
}

const char* skiparse_version(void) {
    return SKIPARSE_DEBUG ? "skiparse-b200 0.1 (sm_100a, tcgen05; debug build: row bounds checked)"
                          : "skiparse-b200 0.1 (sm_100a, tcgen05)";
}

const char* skiparse_last_error_string(void) { return t_last_cuda_error; }

int skiparse_padded_extent(int X, int P) {
    if (X < 1 || P < 1 || P > skiparse::kMaxP) return -1;
    return padded(X, P);
}

long long skiparse_subseq_len(int T, int H, int W, int P) {
    if (T < 1 || H < 1 || W < 1 || P < 1 || P > skiparse::kMaxP) return -1;
    return static_cast<long long>(T) * (padded(H, P) / P) * (padded(W, P) / P);
}

long long skiparse_class_len(int T, int H, int W, int P, int mode, int ci, int cj) {
    Geometry g;
    if (make_geometry(2, 1, T, H, W, 1, 32, P, mode, g) != SKIPARSE_OK) return -1;
    if (ci < 0 || cj < 0 || ci >= P || cj >= P) return -1;
    return static_cast<long long>(T) * g.Rc[ci] * g.Sc[cj];
}

long long skiparse_rearranged_numel(int B, int T, int H, int W, int heads, int d, int P) {
    Geometry g;
    if (make_geometry(2, B, T, H, W, heads, d, P, SKIPARSE_TOKEN_WISE, g) != SKIPARSE_OK) return -1;
    return static_cast<long long>(B) * P * P * g.n * heads * d;
}

long long skiparse1d_padded_length(long long L, int P) {
    if (L < 1 || P < 1 || P > skiparse::kMaxP) return -1;
    const long long q4 = static_cast<long long>(P) * P * P * P;
    return (L + q4 - 1) / q4 * q4;
}

long long skiparse1d_subseq_len(int T, int H, int W, int P) {
    Geometry g;
    if (make_geometry(1, 1, T, H, W, 1, 32, P, SKIPARSE_TOKEN_WISE, g) != SKIPARSE_OK) return -1;
    return g.n;
}

long long skiparse1d_class_len(int T, int H, int W, int P, int mode, int c) {
    Geometry g;
    if (make_geometry(1, 1, T, H, W, 1, 32, P, mode, g) != SKIPARSE_OK) return -1;
    if (c < 0 || c >= P * P) return -1;
    return static_cast<long long>(T) * g.Sc[c];
}

long long skiparse1d_rearranged_numel(int B, int T, int H, int W, int heads, int d, int P) {
    Geometry g;
    if (make_geometry(1, B, T, H, W, heads, d, P, SKIPARSE_TOKEN_WISE, g) != SKIPARSE_OK) return -1;
    return static_cast<long long>(B) * P * P * g.n * heads * d;
}

unsigned long long skiparse_set_wait_limit_ns(unsigned long long ns) {
    return g_wait_limit_ns.exchange(ns == 0 ? kDefaultWaitNs : ns);
}

// A pending fault of `kind`, consumed (one launch) by the entry point it concerns only.
static int take_fault(int kind) {
    int expected = kind;
    return g_fault.compare_exchange_strong(expected, 0) ? 1 : 0;
}

int skiparse_debug_inject_fault(int kind) {
    if (kind != 0 && kind != 1 && kind != 2) return SKIPARSE_ERR_INVALID_ARG;
    g_fault.store(kind);
    return SKIPARSE_OK;
}

int skiparse_debug_shrink_bounds(long long rows) {
    if (!SKIPARSE_DEBUG) return SKIPARSE_ERR_UNSUPPORTED;
    if (rows < 0) return SKIPARSE_ERR_INVALID_ARG;
    g_bounds_shrink.store(rows);
    return SKIPARSE_OK;
}

int skiparse_debug_exp2(const float* x, float* y, long long n, int method,
                        skiparse_stream_t stream) {
    if (n < 0 || (n > 0 && (!x || !y)) || method != 0) return SKIPARSE_ERR_INVALID_ARG;
    if (n >= (1ll << 40)) return SKIPARSE_ERR_UNSUPPORTED;
    const int e = skiparse::launch_exp2(x, y, n, stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse_debug_mma_rate(int pattern, int groups, long long* clocks, int n_clocks,
                            skiparse_stream_t stream) {
    if (pattern < 0 || pattern > 6 || groups < 1 || n_clocks < 1 || !clocks) return SKIPARSE_ERR_INVALID_ARG;
    if (groups > 65536 || n_clocks > 4096) return SKIPARSE_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(clocks) & 7u) return SKIPARSE_ERR_MISALIGNED;
    const int e = skiparse::launch_mma_rate(clocks, n_clocks, pattern, groups, g_wait_limit_ns.load(), stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse_debug_softmax_rate(int warps_per_subpartition, int reps, long long* clocks, int n_ctas,
                                skiparse_stream_t stream) {
    const int wps = warps_per_subpartition;
    if ((wps != 1 && wps != 2 && wps != 4) || reps < 1 || n_ctas < 1 || !clocks) return SKIPARSE_ERR_INVALID_ARG;
    if (reps > 65536 || n_ctas > 1024) return SKIPARSE_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(clocks) & 7u) return SKIPARSE_ERR_MISALIGNED;
    const int e = skiparse::launch_softmax_rate(clocks, n_ctas, wps, reps, stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse_get_device_status(skiparse_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e);
    }
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_skiparse_status, sizeof(int));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e);
    }
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_skiparse_status, &zero, sizeof(int));
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e);
        }
    }
    return v;
}

static int attn_fwd_common(int dims, const void* q, const void* k, const void* v, void* out,
                           float* lse, int B, int T, int H, int W, int heads, int d, int P,
                           int mode, skiparse_stream_t stream) {
    if (!q || !k || !v || !out) return SKIPARSE_ERR_INVALID_ARG;
    Geometry g;
    int st = make_geometry(dims, B, T, H, W, heads, d, P, mode, g);
    if (st != SKIPARSE_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SKIPARSE_ERR_MISALIGNED;
    const long long rows = static_cast<long long>(B) * T * H * W * heads;
    const size_t bytes = static_cast<size_t>(rows) * d * 2;
    if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) || overlaps(out, bytes, v, bytes))
        return SKIPARSE_ERR_INVALID_ARG;
    if (lse) {
        if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return SKIPARSE_ERR_MISALIGNED;
        const size_t lbytes = static_cast<size_t>(rows) * 4;
        if (overlaps(lse, lbytes, q, bytes) || overlaps(lse, lbytes, k, bytes) ||
            overlaps(lse, lbytes, v, bytes) || overlaps(lse, lbytes, out, bytes))
            return SKIPARSE_ERR_INVALID_ARG;
    }
    skiparse::AttnParams p{};
    p.q = static_cast<const uint16_t*>(q);
    p.k = static_cast<const uint16_t*>(k);
    p.v = static_cast<const uint16_t*>(v);
    p.out = static_cast<uint16_t*>(out);
    p.lse = lse;
    p.status = status_ptr();
    if (!p.status) return SKIPARSE_ERR_CUDA;
    p.T = T; p.H = g.H; p.W = g.W; p.heads = heads; p.Ph = g.Ph; p.Pw = g.Pw; p.mode = mode;
    for (int c = 0; c < skiparse::kMaxAxisClasses; ++c) {
        p.Rc[c] = g.Rc[c];
        p.Sc[c] = g.Sc[c];
    }
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.fault = take_fault(1);
    p.nrows = checked_bound(rows);
    const int e = skiparse::launch_attn_fwd(p, g, stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse2d_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int T,
                        int H, int W, int heads, int d, int P, int mode, skiparse_stream_t stream) {
    return attn_fwd_common(2, q, k, v, out, nullptr, B, T, H, W, heads, d, P, mode, stream);
}

int skiparse2d_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int T, int H, int W, int heads, int d, int P, int mode,
                            skiparse_stream_t stream) {
    if (!lse) return SKIPARSE_ERR_INVALID_ARG;
    return attn_fwd_common(2, q, k, v, out, lse, B, T, H, W, heads, d, P, mode, stream);
}

int skiparse1d_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int T,
                        int H, int W, int heads, int d, int P, int mode, skiparse_stream_t stream) {
    return attn_fwd_common(1, q, k, v, out, nullptr, B, T, H, W, heads, d, P, mode, stream);
}

int skiparse1d_attn_fwd_lse(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int T, int H, int W, int heads, int d, int P, int mode,
                            skiparse_stream_t stream) {
    if (!lse) return SKIPARSE_ERR_INVALID_ARG;
    return attn_fwd_common(1, q, k, v, out, lse, B, T, H, W, heads, d, P, mode, stream);
}

static int attn_bwd_common(int dims, const void* q, const void* k, const void* v, const void* out,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           float* delta, int B, int T, int H, int W, int heads, int d, int P,
                           int mode, skiparse_stream_t stream) {
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !delta) return SKIPARSE_ERR_INVALID_ARG;
    Geometry g;
    int st = make_geometry(dims, B, T, H, W, heads, d, P, mode, g);
    if (st != SKIPARSE_OK) return st;
    const void* bf[8] = {q, k, v, out, dout, dq, dk, dv};
    for (const void* ptr : bf)
        if (!aligned16(ptr)) return SKIPARSE_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(delta) & 3u))
        return SKIPARSE_ERR_MISALIGNED;
    const long long rows = static_cast<long long>(B) * T * H * W * heads;
    const size_t tb = static_cast<size_t>(rows) * d * 2, vb = static_cast<size_t>(rows) * 4;
    const void* outs[4] = {dq, dk, dv, delta};
    const size_t out_bytes[4] = {tb, tb, tb, vb};
    const void* ins[6] = {q, k, v, out, dout, lse};
    const size_t in_bytes[6] = {tb, tb, tb, tb, tb, vb};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 6; ++j)
            if (overlaps(outs[i], out_bytes[i], ins[j], in_bytes[j])) return SKIPARSE_ERR_INVALID_ARG;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], out_bytes[i], outs[j], out_bytes[j])) return SKIPARSE_ERR_INVALID_ARG;
    }
    skiparse::BwdParams p{};
    p.q = static_cast<const uint16_t*>(q);
    p.k = static_cast<const uint16_t*>(k);
    p.v = static_cast<const uint16_t*>(v);
    p.out = static_cast<const uint16_t*>(out);
    p.dout = static_cast<const uint16_t*>(dout);
    p.lse = lse;
    p.delta = delta;
    p.dq = static_cast<uint16_t*>(dq);
    p.dk = static_cast<uint16_t*>(dk);
    p.dv = static_cast<uint16_t*>(dv);
    p.status = status_ptr();
    if (!p.status) return SKIPARSE_ERR_CUDA;
    p.T = T; p.H = g.H; p.W = g.W; p.heads = heads; p.Ph = g.Ph; p.Pw = g.Pw; p.mode = mode;
    for (int c = 0; c < skiparse::kMaxAxisClasses; ++c) {
        p.Rc[c] = g.Rc[c];
        p.Sc[c] = g.Sc[c];
    }
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.nrows = checked_bound(rows);
    p.fault = take_fault(2);
    const int e = skiparse::launch_attn_bwd(p, g, stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse2d_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, float* delta,
                        int B, int T, int H, int W, int heads, int d, int P, int mode,
                        skiparse_stream_t stream) {
    return attn_bwd_common(2, q, k, v, out, dout, lse, dq, dk, dv, delta, B, T, H, W, heads, d, P,
                           mode, stream);
}

int skiparse1d_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, float* delta,
                        int B, int T, int H, int W, int heads, int d, int P, int mode,
                        skiparse_stream_t stream) {
    return attn_bwd_common(1, q, k, v, out, dout, lse, dq, dk, dv, delta, B, T, H, W, heads, d, P,
                           mode, stream);
}

static int rearrange_common(int dims, const void* src, void* dst, int B, int T, int H, int W,
                            int heads, int d, int P, int mode, skiparse_stream_t stream, int kind) {
    if (!src || !dst) return SKIPARSE_ERR_INVALID_ARG;
    Geometry g;
    int st = make_geometry(dims, B, T, H, W, heads, d, P, mode, g);
    if (st != SKIPARSE_OK) return st;
    if (!aligned16(src) || !aligned16(dst)) return SKIPARSE_ERR_MISALIGNED;
    const long long row_bytes = static_cast<long long>(heads) * d * 2;
    const long long ntok = static_cast<long long>(B) * T * H * W;
    const long long nslot = static_cast<long long>(B) * P * P * g.n;
    const size_t orig_bytes = static_cast<size_t>(ntok * row_bytes);
    const size_t rear_bytes = static_cast<size_t>(nslot * row_bytes);
    const size_t src_bytes = kind == 0 ? orig_bytes : rear_bytes;
    const size_t dst_bytes = kind == 1 ? orig_bytes : rear_bytes;
    if (overlaps(src, src_bytes, dst, dst_bytes)) return SKIPARSE_ERR_INVALID_ARG;
    skiparse::RearrangeParams p{};
    p.src = src;
    p.dst = dst;
    p.B = B; p.T = T; p.H = g.H; p.W = g.W; p.Ph = g.Ph; p.Pw = g.Pw; p.mode = mode;
    p.R = g.R; p.S = g.S;
    p.n = g.n;
    p.row_chunks = static_cast<int>(row_bytes / 16);
    p.nrows = kind == 1 ? ntok : nslot;
    p.src_rows = checked_bound(kind == 0 ? ntok : nslot);
    p.status = status_ptr();
    if (!p.status) return SKIPARSE_ERR_CUDA;
    const int e = skiparse::launch_rearrange(p, kind, stream);
    return e == 0 ? SKIPARSE_OK : cuda_fail(e);
}

int skiparse_rearrange(const void* x, void* y, int B, int T, int H, int W, int heads, int d, int P,
                       int mode, skiparse_stream_t stream) {
    return rearrange_common(2, x, y, B, T, H, W, heads, d, P, mode, stream, 0);
}

int skiparse_unrearrange(const void* y, void* x, int B, int T, int H, int W, int heads, int d,
                         int P, int mode, skiparse_stream_t stream) {
    return rearrange_common(2, y, x, B, T, H, W, heads, d, P, mode, stream, 1);
}

int skiparse_switch_mode(const void* y_src, void* y_dst, int B, int T, int H, int W, int heads,
                         int d, int P, int src_mode, skiparse_stream_t stream) {
    return rearrange_common(2, y_src, y_dst, B, T, H, W, heads, d, P, src_mode, stream, 2);
}

int skiparse1d_rearrange(const void* x, void* y, int B, int T, int H, int W, int heads, int d,
                         int P, int mode, skiparse_stream_t stream) {
    return rearrange_common(1, x, y, B, T, H, W, heads, d, P, mode, stream, 0);
}

int skiparse1d_unrearrange(const void* y, void* x, int B, int T, int H, int W, int heads, int d,
                           int P, int mode, skiparse_stream_t stream) {
    return rearrange_common(1, y, x, B, T, H, W, heads, d, P, mode, stream, 1);
}

int skiparse1d_switch_mode(const void* y_src, void* y_dst, int B, int T, int H, int W, int heads,
                           int d, int P, int src_mode, skiparse_stream_t stream) {
    return rearrange_common(1, y_src, y_dst, B, T, H, W, heads, d, P, src_mode, stream, 2);
}

}  // extern "C"
