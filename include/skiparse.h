/*
 * skiparse.h -- C ABI of libskiparse.so: Skiparse-2D (and Skiparse-1D) sparse attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method (paper.rainbus.top summary of "OSP-Next: Efficient High-Quality Video Generation
 * with Sparse Sequence Parallelism, HiF8 Quantization, and Reinforcement Learning", sections
 * 核心方法 (core method) and 方法步骤详情 (method step details)):
 *   video tokens of shape (B, T, H, W, C) with C = heads*d are split into P^2 subsequences;
 *   token-wise mode (pixel-unshuffle-like) puts token (h, w) in class (h mod P, w mod P),
 *   group-wise mode (patch-unshuffle-like) puts it in class ((h div P) mod P, (w div P) mod P);
 *   when H or W is not a multiple of P^2 the grid is padded up to the next multiple and the
 *   padded keys are masked; every subsequence runs dense softmax attention; the result is
 *   rearranged back to the original layout.
 *
 * Conventions shared by every entry point
 *   - Tensors are bfloat16, contiguous (row-major), device pointers, 16-byte aligned.
 *   - Original layout: (B, T, H, W, heads, d). Rearranged layout: (B*P*P, n, heads, d) with
 *     n = T * (Hp/P) * (Wp/P), Hp = ceil(H/P^2)*P^2, Wp = ceil(W/P^2)*P^2; subsequence index
 *     b*P*P + ci*P + cj; inside a subsequence tokens are in (t, r, s) raster order, where (r, s)
 *     is the token's position in its class's sub-grid: r = h div P (token-wise) or
 *     (h div P^2)*P + h mod P (group-wise), and s likewise from w. Padding is at the
 *     bottom/right of each frame.
 *   - Softmax scale is 1/sqrt(d); no causal mask, no dropout, no bias.
 *   - Ownership: the caller allocates and owns every buffer. The library allocates no device
 *     memory per call. Its device state: one status word per device, and the fixed workspace
 *     of skiparse2d_attn_bwd_noalloc (a static 16 MiB array on every device that loads the
 *     library); the host-buffer entry points also create three streams and a few events per
 *     device on their first call there.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *     Argument errors are reported synchronously, before any launch, and nothing is launched.
 *     No function throws across the ABI.
 *   - Supported: 1 <= B, T, H, W, heads; d in {32, 64, 128}; 1 <= P <= 8;
 *     mode in {SKIPARSE_TOKEN_WISE, SKIPARSE_GROUP_WISE}; B*T*H*W*heads < 2^31.
 */
#ifndef SKIPARSE_H
#define SKIPARSE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SKIPARSE_API __attribute__((visibility("default")))
#else
#define SKIPARSE_API
#endif

/* Opaque CUDA stream handle; identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* skiparse_stream_t;

enum { SKIPARSE_TOKEN_WISE = 0, SKIPARSE_GROUP_WISE = 1 };

enum {
    SKIPARSE_OK = 0,
    SKIPARSE_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad mode, aliasing */
    SKIPARSE_ERR_UNSUPPORTED = 2, /* valid but outside the supported set (d, P, size) */
    SKIPARSE_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
    SKIPARSE_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, tensor map) */
    SKIPARSE_ERR_TIMEOUT = 5,     /* a kernel's bounded wait expired; its output is invalid */
    SKIPARSE_ERR_BOUNDS = 6       /* debug build only: a kernel computed a token row outside its
                                     tensor; the access was skipped and the output is invalid */
};

/*
 * Skiparse-2D attention forward, fused: the class rearrange, the pad-key mask, the dense
 * attention of every subsequence and the inverse rearrange, in one kernel launch.
 * (核心方法 and 方法步骤详情 on the summary page; the English abstract on chatpaper.ai.)
 *
 *   q, k, v : (B, T, H, W, heads, d) bf16, read-only.
 *   out     : (B, T, H, W, heads, d) bf16, written entirely (every real token has an output).
 *             Must not overlap q, k or v (SKIPARSE_ERR_INVALID_ARG).
 *   For every real query token x of class c in batch b and every head:
 *     out[x] = sum_y softmax_y(q[x].k[y] / sqrt(d)) v[y] over the real tokens y of class c,
 *   accumulated in fp32, rounded once to bf16. P = 1 is dense full attention.
 * Returns SKIPARSE_OK once the kernel is queued. Device-side failures (a bounded wait that
 * expired) are reported by skiparse_get_device_status().
 */
SKIPARSE_API int skiparse2d_attn_fwd(const void* q, const void* k, const void* v, void* out,
                        int B, int T, int H, int W, int heads, int d, int P, int mode,
                        skiparse_stream_t stream);

/*
 * Forward as skiparse2d_attn_fwd that also writes, for the backward pass,
 *   lse : (B, T, H, W, heads) fp32, 4-byte aligned, written for every real token:
 *         lse[x] = log sum_y exp(q[x].k[y] / sqrt(d)) over the keys y of x's class (natural log).
 * lse must not overlap q, k, v or out.
 */
SKIPARSE_API int skiparse2d_attn_fwd_lse(const void* q, const void* k, const void* v, void* out,
                                         float* lse, int B, int T, int H, int W, int heads, int d,
                                         int P, int mode, skiparse_stream_t stream);

/*
 * Backward pass of skiparse2d_attn_fwd (for fine-tuning the sparse model). With, inside each
 * class subsequence, P = softmax(q.k^T/sqrt(d)) and D_x = dout[x].out[x]:
 *   dv = P^T dout,  dS = P o (dout v^T - D),  dq = dS k / sqrt(d),  dk = dS^T q / sqrt(d).
 *   q, k, v, out, dout : (B, T, H, W, heads, d) bf16, read-only; out is the forward's output.
 *   lse                : (B, T, H, W, heads) fp32 from skiparse2d_attn_fwd_lse, read-only.
 *   dq, dk, dv         : (B, T, H, W, heads, d) bf16, written entirely.
 *   delta              : (B, T, H, W, heads) fp32 workspace owned by the caller; on return it
 *                        holds D. 4-byte aligned.
 * None of dq, dk, dv, delta may overlap each other or an input. Three kernel launches (D, then
 * the key-tile-major dk/dv kernel, then the query-tile-major dq kernel); no atomics, results
 * are deterministic.
 */
SKIPARSE_API int skiparse2d_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                                     const void* dout, const float* lse, void* dq, void* dk,
                                     void* dv, float* delta, int B, int T, int H, int W, int heads,
                                     int d, int P, int mode, skiparse_stream_t stream);

/*
 * Backward pass for callers that cannot allocate device memory (the pages have no counterpart:
 * this is an interface convenience). Same arguments, kernels and results as skiparse2d_attn_bwd
 * without `delta`: the D workspace lives in a fixed array owned by the library instead -- 2^22
 * fp32 values (16 MiB) that every device loading the library holds until the process exits.
 * For callers whose host framework owns all device memory, or that must not call the allocator.
 *   - B*T*H*W*heads must be at most 4,194,304; larger problems get SKIPARSE_ERR_UNSUPPORTED
 *     before anything is launched (use skiparse2d_attn_bwd with your own workspace instead).
 *   - Allocates nothing: no cudaMalloc or cudaFree, no allocating library call.
 *   - Argument errors are reported first, before any CUDA call, with the codes of
 *     skiparse2d_attn_bwd.
 *   - Every call looks up the workspace's device address in the current context
 *     (cudaGetSymbolAddress, which allocates nothing), so a reset device or another current
 *     context never sees a stale address. The first use of the library on a device loads its
 *     kernels and this array there: make a first call on each device before any stream capture.
 *   - All calls share the one workspace per device: calls that can run at the same time on
 *     the GPU (on different streams) race on it and must be ordered by the caller. The
 *     previous call's contents never matter; nothing needs clearing between calls.
 */
SKIPARSE_API int skiparse2d_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                             const void* out, const void* dout, const float* lse,
                                             void* dq, void* dk, void* dv, int B, int T, int H,
                                             int W, int heads, int d, int P, int mode,
                                             skiparse_stream_t stream);

/*
 * Rearrange (方法步骤详情: the rearrange that forms the P^2 subsequences, with padding).
 *   x : (B, T, H, W, heads, d) bf16, read-only.
 *   y : (B*P*P, n, heads, d) bf16, skiparse_rearranged_numel() elements, written entirely;
 *       pad slots are written as +0.0. Must not overlap x.
 * A bit-exact permutation of whole (heads*d) token rows.
 */
SKIPARSE_API int skiparse_rearrange(const void* x, void* y, int B, int T, int H, int W, int heads, int d,
                       int P, int mode, skiparse_stream_t stream);

/*
 * Inverse rearrange (方法步骤详情: rearranged back to the original layout).
 *   y : (B*P*P, n, heads, d) bf16, read-only; pad slots are ignored.
 *   x : (B, T, H, W, heads, d) bf16, written entirely. Must not overlap y.
 */
SKIPARSE_API int skiparse_unrearrange(const void* y, void* x, int B, int T, int H, int W, int heads, int d,
                         int P, int mode, skiparse_stream_t stream);

/*
 * Pattern switch (核心方法: token-wise and group-wise layers alternate; under sequence
 * parallelism a switch is a local rearrange plus one exchange -- this is that local step).
 *   y_src : (B*P*P, n, heads, d) bf16 in src_mode's rearranged layout, read-only; its pad slots
 *           are ignored.
 *   y_dst : (B*P*P, n, heads, d) bf16, written entirely in the other mode's rearranged layout;
 *           pad slots are +0.0. Must not overlap y_src.
 * Equal, bit for bit, to skiparse_unrearrange(src_mode) followed by skiparse_rearrange of the
 * other mode, in one pass over HBM.
 */
SKIPARSE_API int skiparse_switch_mode(const void* y_src, void* y_dst, int B, int T, int H, int W,
                                      int heads, int d, int P, int src_mode,
                                      skiparse_stream_t stream);

/* Number of elements of the rearranged tensor, B*P*P*n*heads*d; -1 on invalid arguments. */
SKIPARSE_API long long skiparse_rearranged_numel(int B, int T, int H, int W, int heads, int d, int P);

/* H or W padded to the next multiple of P*P; -1 on invalid arguments. */
SKIPARSE_API int skiparse_padded_extent(int X, int P);

/* Padded subsequence length n = T*(Hp/P)*(Wp/P); -1 on invalid arguments. */
SKIPARSE_API long long skiparse_subseq_len(int T, int H, int W, int P);

/* Number of real tokens of class (ci, cj) in one batch element; -1 on invalid arguments. */
SKIPARSE_API long long skiparse_class_len(int T, int H, int W, int P, int mode, int ci, int cj);

/*
 * The forward called with HOST buffers: q, k, v are read from host memory and out is written to
 * host memory within the call (the same layouts and results as skiparse2d_attn_fwd). Heads are
 * independent in the method (every (class, head) subsequence attends on its own), so the call is
 * cut into groups of `heads_per_group` heads: a group's rows are copied in (one pitched copy per
 * tensor), the fused kernel runs on it, and its output is copied out, with the copies of one
 * group overlapping the kernel of another (library-owned streams, two workspace buffer sets).
 *   q, k, v, out    : host pointers, (B, T, H, W, heads, d) bf16. Pinned (page-locked) memory
 *                     lets the copies overlap; pageable memory gives the same results, slower.
 *                     out must not overlap q, k or v.
 *   heads_per_group : 1 <= heads_per_group <= heads; the last group may be smaller.
 *   workspace       : device memory owned by the caller, 256-byte aligned, of at least
 *                     skiparse_attn_fwd_host_workspace_bytes(B, T, H, W, heads, d,
 *                     heads_per_group) bytes; it must not be used by anything else until the
 *                     call has completed on `stream`.
 * Asynchronous on `stream` like every entry point: the call starts after earlier work on
 * `stream` and later work on `stream` (e.g. a synchronize) sees out written. Calls on one
 * device are enqueued under a lock and run on the same internal streams, one after another.
 * Errors: as skiparse2d_attn_fwd, plus SKIPARSE_ERR_INVALID_ARG for a bad group size or a small
 * workspace, SKIPARSE_ERR_MISALIGNED for an unaligned workspace.
 */
SKIPARSE_API int skiparse2d_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                          int B, int T, int H, int W, int heads, int d, int P,
                                          int mode, int heads_per_group, void* workspace,
                                          size_t workspace_bytes, skiparse_stream_t stream);

/* Device workspace bytes for skiparse2d_attn_fwd_host / skiparse1d_attn_fwd_host: two sets of
 * four (B, T, H, W, heads_per_group, d) bf16 buffers; -1 on invalid arguments. */
SKIPARSE_API long long skiparse_attn_fwd_host_workspace_bytes(int B, int T, int H, int W, int heads,
                                                              int d, int heads_per_group);

/*
 * ---- Skiparse-1D ------------------------------------------------------------------------
 * The 1D skip pattern on the flattened sequence, the variant that the summary page's sections
 * 技术新颖性 (novelty) and 实验结果 (results) compare Skiparse-2D with; the pages give no formula
 * for it. The reading implemented here: the in-frame index x = h*W + w with ratio P^2, so that
 * there are P^2 subsequences as in Skiparse-2D --
 *   token-wise class x mod P^2,              position in the class x div P^2;
 *   group-wise class (x div P^2) mod P^2,    position (x div P^4)*P^2 + x mod P^2
 *   (runs of P^2 consecutive tokens stay together);
 * each frame's H*W positions are padded at the end to Lp, the next multiple of P^4, and the
 * padded keys are masked. Rearranged layout: (B*P*P, n, heads, d) with n = T * Lp / P^2,
 * subsequence b*P^2 + class, tokens in (t, position-in-class) order.
 * Every function below takes the same arguments, with the same layout, ownership, alignment,
 * aliasing and error rules, as the Skiparse-2D function of the same name; only the class rule
 * differs. Supported sizes as above (1 <= P <= 8; B*T*Lp*heads < 2^31).
 */
SKIPARSE_API int skiparse1d_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                     int B, int T, int H, int W, int heads, int d, int P, int mode,
                                     skiparse_stream_t stream);
SKIPARSE_API int skiparse1d_attn_fwd_lse(const void* q, const void* k, const void* v, void* out,
                                         float* lse, int B, int T, int H, int W, int heads, int d,
                                         int P, int mode, skiparse_stream_t stream);
SKIPARSE_API int skiparse1d_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                                          int B, int T, int H, int W, int heads, int d, int P,
                                          int mode, int heads_per_group, void* workspace,
                                          size_t workspace_bytes, skiparse_stream_t stream);
SKIPARSE_API int skiparse1d_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                                     const void* dout, const float* lse, void* dq, void* dk,
                                     void* dv, float* delta, int B, int T, int H, int W, int heads,
                                     int d, int P, int mode, skiparse_stream_t stream);
/* x (B,T,H,W,heads,d) -> y (B*P*P, n, heads, d), pad slots +0.0; bit-exact row permutation. */
SKIPARSE_API int skiparse1d_rearrange(const void* x, void* y, int B, int T, int H, int W, int heads,
                                      int d, int P, int mode, skiparse_stream_t stream);
/* y (B*P*P, n, heads, d) -> x (B,T,H,W,heads,d); pad slots ignored. */
SKIPARSE_API int skiparse1d_unrearrange(const void* y, void* x, int B, int T, int H, int W,
                                        int heads, int d, int P, int mode,
                                        skiparse_stream_t stream);
/* src_mode's Skiparse-1D rearranged layout -> the other mode's, in one pass; pad slots +0.0. */
SKIPARSE_API int skiparse1d_switch_mode(const void* y_src, void* y_dst, int B, int T, int H,
                                        int W, int heads, int d, int P, int src_mode,
                                        skiparse_stream_t stream);
/* Per-frame length L padded to the next multiple of P^4; -1 on invalid arguments. */
SKIPARSE_API long long skiparse1d_padded_length(long long L, int P);
/* Padded subsequence length n = T * Lp / P^2; -1 on invalid arguments. */
SKIPARSE_API long long skiparse1d_subseq_len(int T, int H, int W, int P);
/* Real tokens of class c (0 <= c < P^2) in one batch element; -1 on invalid arguments. */
SKIPARSE_API long long skiparse1d_class_len(int T, int H, int W, int P, int mode, int c);
/* Elements of the Skiparse-1D rearranged tensor, B*P*P*n*heads*d; -1 on invalid arguments. */
SKIPARSE_API long long skiparse1d_rearranged_numel(int B, int T, int H, int W, int heads, int d,
                                                   int P);

/*
 * Synchronizes `stream`, then returns and clears the current device's error word: SKIPARSE_OK,
 * or SKIPARSE_ERR_TIMEOUT if any kernel since the last call gave up on a bounded wait (its
 * output is then invalid), or SKIPARSE_ERR_BOUNDS (debug build only) if a kernel computed a
 * token row outside its tensor, or SKIPARSE_ERR_CUDA if the synchronization itself failed.
 */
SKIPARSE_API int skiparse_get_device_status(skiparse_stream_t stream);

/* Static, human-readable name of a status code. Never NULL. */
SKIPARSE_API const char* skiparse_status_string(int status);

/* Message of the last CUDA failure reported as SKIPARSE_ERR_CUDA on this host thread
 * ("no error" if none). Static storage; never NULL. */
SKIPARSE_API const char* skiparse_last_error_string(void);

/* Library version string, static. */
SKIPARSE_API const char* skiparse_version(void);

/*
 * Bound, in nanoseconds, on every wait inside a kernel (default 2e9 = 2 s). After the bound a
 * kernel records SKIPARSE_ERR_TIMEOUT and returns instead of hanging. Applies to later
 * launches from any thread. ns == 0 restores the default. Returns the previous value.
 */
SKIPARSE_API unsigned long long skiparse_set_wait_limit_ns(unsigned long long ns);

/*
 * Test hook for failure detection. kind = 1 makes the next forward launch of this process
 * (skiparse2d_attn_fwd and the other forward entry points) lose one arrival on its first K-tile
 * barrier (one producer thread never signals it); kind = 2 does the same to the next backward
 * call's key-major kernel on its first streamed tile. The consumer's bounded wait then expires
 * and the kernel reports SKIPARSE_ERR_TIMEOUT without faulting or hanging the GPU. kind = 0
 * clears it. A hook is consumed by one launch of the entry point it concerns. Returns
 * SKIPARSE_OK or SKIPARSE_ERR_INVALID_ARG.
 */
SKIPARSE_API int skiparse_debug_inject_fault(int kind);

/*
 * Debug build (libskiparse_debug.so, compiled with SKIPARSE_DEBUG=1; no counterpart on the
 * pages). Its kernels check every token row index they compute for a global load or store
 * against the row count of the tensor; an index outside is recorded as SKIPARSE_ERR_BOUNDS in
 * the device error word and the access is skipped (a load reads row 0, a store is dropped),
 * so the check itself never leaves a tensor. This hook declares the next launch's row counts
 * `rows` smaller than the tensors really are, so that a test can see the check report while
 * every actual access stays inside the tensors. Consumed by the next launch of any entry point.
 * Returns SKIPARSE_OK (debug build), SKIPARSE_ERR_UNSUPPORTED (release build, which has no
 * checks) or SKIPARSE_ERR_INVALID_ARG (rows < 0).
 */
SKIPARSE_API int skiparse_debug_shrink_bounds(long long rows);

/*
 * Diagnostic (no counterpart on the pages): y[i] = 2^x[i] for n fp32 device values, evaluated
 * exactly as the attention softmax does, with the MUFU ex2.approx instruction (method must be
 * 0; other values are SKIPARSE_ERR_INVALID_ARG). x and y are device pointers, n >= 0;
 * asynchronous on `stream`. Returns SKIPARSE_OK, SKIPARSE_ERR_INVALID_ARG or SKIPARSE_ERR_CUDA.
 */
SKIPARSE_API int skiparse_debug_exp2(const float* x, float* y, long long n, int method,
                                     skiparse_stream_t stream);

/*
 * Diagnostic (no counterpart on the pages): the tensor-core rate behind the kernels' design.
 * Launches n_clocks CTAs (pass the SM count: one per SM); in each, one thread issues `groups`
 * groups of 8 tcgen05.mma K-steps (K = 16, bf16 in, fp32 accumulator in TMEM) in an unrolled
 * stream, as the attention kernels' MMA warp does, and writes the SM clocks from the first issue
 * to completion to clocks[cta] (-1 if its bounded wait ran out). Patterns: 0 = A and B in shared
 * memory, M = 128, N = 128; 1 = A in TMEM, M = N = 128; 2 = shared memory, N = 256;
 * 3 = shared memory, N = 64; 4, 5, 6 = pattern 0 while 8 more warps of the CTA (2 per SM
 * sub-partition) run independent FFMA chains (4), the backward's dS arithmetic (5: FADD, FMUL,
 * bf16 pack) or the forward softmax's exponential loop (6) until the stream is done. One group
 * is 8 x 2 x 128 x N x 16 FLOP; the nominal dense bf16 rate of an SM is 8192 FLOP per clock.
 *   clocks : device pointer to n_clocks int64, 8-byte aligned. 1 <= n_clocks <= 4096,
 *            1 <= groups <= 65536, 0 <= pattern <= 6.
 * Asynchronous on `stream`. Returns SKIPARSE_OK, SKIPARSE_ERR_INVALID_ARG, _UNSUPPORTED,
 * _MISALIGNED or SKIPARSE_ERR_CUDA.
 */
SKIPARSE_API int skiparse_debug_mma_rate(int pattern, int groups, long long* clocks, int n_clocks,
                                         skiparse_stream_t stream);

/*
 * Diagnostic (no counterpart on the pages): the rate of the forward softmax's exponential loop,
 * with no tensor core or loads beside it. Launches n_ctas CTAs (pass the SM count: one
 * per SM) of 4 x warps_per_subpartition warps; every warp runs `reps` passes of the softmax's
 * loop body over 64 scores per thread (exponent by FFMA, ex2.approx, four running sums, bf16
 * pack: 64 exponentials per thread per pass) and writes its SM clocks to
 * clocks[cta * 4 * warps_per_subpartition + warp].
 *   clocks : device pointer to n_ctas * 4 * warps_per_subpartition int64, 8-byte aligned.
 *            warps_per_subpartition in {1, 2, 4}, 1 <= reps <= 65536, 1 <= n_ctas <= 1024.
 * Asynchronous on `stream`. Returns SKIPARSE_OK, SKIPARSE_ERR_INVALID_ARG, _UNSUPPORTED,
 * _MISALIGNED or SKIPARSE_ERR_CUDA.
 */
SKIPARSE_API int skiparse_debug_softmax_rate(int warps_per_subpartition, int reps, long long* clocks,
                                             int n_ctas, skiparse_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SKIPARSE_H */
