// rearrange.cu -- standalone Skiparse rearrange, inverse rearrange and pattern switch for B200
// (sm_100a).
//
// Summary page of OSP-Next, 方法步骤详情 (method step details): the (B,T,H,W,C) tokens are
// rearranged into P^2 subsequences of length N/P^2 (padding H and W up to multiples of P^2),
// and the attention result is rearranged back to the original layout; 核心方法 (core method):
// token-wise and group-wise layers alternate, and under sequence parallelism a pattern switch is
// a local rearrange plus one exchange -- the switch kernel here is that local step, from one
// mode's rearranged layout straight to the other's. All three are permutations of whole token
// rows of heads*d bf16 values (contiguous in every layout), so the kernels are pure HBM copies:
// one warp moves one row with 16-byte loads and stores, several chunks in flight per lane; pad
// rows of a rearranged result are written as zero. Skiparse-1D uses the same kernels on a
// (1, H*W) frame with (1, P^2) classes.
#include <cuda_runtime.h>

#include <cstdint>

#include "skiparse_internal.cuh"

namespace skiparse {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// kKind 0 (rearrange): row is a slot (seq*n + pos) of the rearranged tensor (mode p.mode).
// kKind 1 (inverse)  : row is a token ((b*T + t)*H + h)*W + w of the original tensor.
// kKind 2 (switch)   : row is a slot of the other mode's rearranged tensor; the source is the
//                      same token's slot in mode p.mode's rearranged tensor.
template <int kKind>
__global__ void __launch_bounds__(kThreads) skiparse_rearrange_kernel(const RearrangeParams p) {
    const int lane = threadIdx.x & 31;
    const long long warp0 = (static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const long long nwarps = (static_cast<long long>(gridDim.x) * kThreads) >> 5;
    const int q2 = p.Ph * p.Pw;
    const uint4* src = static_cast<const uint4*>(p.src);
    uint4* dst = static_cast<uint4*>(p.dst);
    for (long long row = warp0; row < p.nrows; row += nwarps) {
        long long src_row;
        bool real = true;
        if (kKind == 0 || kKind == 2) {
            const int out_mode = kKind == 0 ? p.mode : 1 - p.mode;
            const long long seq = row / p.n;
            const long long pos = row - seq * p.n;
            const int b = static_cast<int>(seq / q2);
            const int c = static_cast<int>(seq - static_cast<long long>(b) * q2);
            const int s = static_cast<int>(pos % p.S);
            const long long tr = pos / p.S;
            const int r = static_cast<int>(tr % p.R);
            const int t = static_cast<int>(tr / p.R);
            const int h = axis_coord(r, c / p.Pw, p.Ph, out_mode);
            const int w = axis_coord(s, c % p.Pw, p.Pw, out_mode);
            real = h < p.H && w < p.W;
            if (kKind == 0) {
                src_row = ((static_cast<long long>(b) * p.T + t) * p.H + h) * p.W + w;
            } else {
                int ci = 0, r2 = 0, cj = 0, s2 = 0;
                if (real) {
                    axis_class(h, p.Ph, p.mode, ci, r2);
                    axis_class(w, p.Pw, p.mode, cj, s2);
                }
                const long long sseq = static_cast<long long>(b) * q2 + ci * p.Pw + cj;
                src_row = sseq * p.n + (static_cast<long long>(t) * p.R + r2) * p.S + s2;
            }
        } else {
            long long tok = row;
            const int w = static_cast<int>(tok % p.W);
            tok /= p.W;
            const int h = static_cast<int>(tok % p.H);
            tok /= p.H;
            const int t = static_cast<int>(tok % p.T);
            const int b = static_cast<int>(tok / p.T);
            int ci, r, cj, s;
            axis_class(h, p.Ph, p.mode, ci, r);
            axis_class(w, p.Pw, p.mode, cj, s);
            const long long seq = static_cast<long long>(b) * q2 + ci * p.Pw + cj;
            src_row = seq * p.n + (static_cast<long long>(t) * p.R + r) * p.S + s;
        }
        if (real && !row_ok(src_row, p.src_rows, p.status)) real = false;  // debug builds
        const uint4* s_row = src + (real ? src_row : 0) * p.row_chunks;
        uint4* d_row = dst + row * p.row_chunks;
        for (int k = lane; k < p.row_chunks; k += 32 * kUnroll) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int idx = k + 32 * u;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (real && idx < p.row_chunks) v[u] = ld_stream(s_row + idx);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int idx = k + 32 * u;
                if (idx < p.row_chunks) st_stream(d_row + idx, v[u]);
            }
        }
    }
}

}  // namespace

int launch_rearrange(const RearrangeParams& p, int kind, void* stream) {
    if (p.nrows <= 0) return static_cast<int>(cudaSuccess);
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return static_cast<int>(e);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long warps_needed = p.nrows;
    const long long blocks_needed = (warps_needed * 32 + kThreads - 1) / kThreads;
    const long long max_blocks = static_cast<long long>(sms) * 8;  // 8 x 256 threads per SM
    const int blocks = static_cast<int>(blocks_needed < max_blocks ? blocks_needed : max_blocks);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == 0)
        skiparse_rearrange_kernel<0><<<blocks, kThreads, 0, st>>>(p);
    else if (kind == 1)
        skiparse_rearrange_kernel<1><<<blocks, kThreads, 0, st>>>(p);
    else
        skiparse_rearrange_kernel<2><<<blocks, kThreads, 0, st>>>(p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace skiparse
