// diag_sm100.cu -- diagnostic microbenchmark of the tensor-core issue patterns the attention
// kernels use (no counterpart on the pages): how many SM clocks a tcgen05.mma of each shape takes
// when one thread issues a long unrolled stream of them, the way the kernels' MMA warp does.
//
// Every CTA (one per SM: it allocates all 512 TMEM columns and holds 100 KB of shared memory)
// fills an A tile (128 x 128 bf16) and a B tile (256 x 128 bf16) in shared memory, then lane 0 of
// warp 0 issues `groups` groups of 8 K-steps (K = 16 each) into one fp32 accumulator in TMEM,
// commits, and waits (bounded) for completion; the SM clocks from the first issue to completion
// go to clocks[blockIdx.x]. Patterns:
//   0: A and B from shared memory, M = 128, N = 128  (S = Q K^T)
//   1: A from TMEM,                M = 128, N = 128  (O += P V with P in TMEM)
//   2: A and B from shared memory, M = 128, N = 256
//   3: A and B from shared memory, M = 128, N = 64
//   4, 5, 6: pattern 0 while 8 more warps of the CTA (2 per SM sub-partition, including the
//      issuing thread's) run, until the stream is done, a loop of independent FFMA chains (4),
//      the backward's dS arithmetic (5: FADD, FMUL, bf16 pack, no MUFU) or the forward
//      softmax's exponential loop (6: FFMA, ex2, FADD, bf16 pack): how much the tensor pipe
//      loses when its issuing thread shares a sub-partition with warps that never stall.
// Work per group: 8 x 2 x 128 x N x 16 FLOP. A wait that runs out leaves clocks = -1.
//
// A second diagnostic times the forward softmax's exponential loop alone (no tensor core, no
// loads): skiparse_softmax_rate_kernel runs, in every warp of a CTA that owns its SM, `reps`
// passes over 64 scores per thread of the loop body the attention softmax uses (exponent by
// FFMA, ex2.approx, four running sums, bf16 pack), with 1, 2 or 4 warps per SM sub-partition,
// and writes each warp's SM clocks to clocks[cta * warps + warp].
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_common.cuh"

namespace skiparse {
namespace {

constexpr int kDiagBox = 128 * 128;           // 128 rows x 64 bf16, 128-byte swizzle
constexpr int kDiagA = 2 * kDiagBox;          // 128 x 128 bf16
constexpr int kDiagB = 2 * 256 * 128;         // 256 x 128 bf16
constexpr int kDiagSmem = 100 * 1024;         // > 227 KB / 3: at most two CTAs per SM by shared
                                              // memory; TMEM (512 columns each) admits one

template <int PATTERN>
__global__ void __launch_bounds__(128, 1) skiparse_mma_rate_kernel(long long* clocks, int groups,
                                                                    unsigned long long wait_ns) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) unsigned long long done_bar;
    __shared__ uint32_t tmem_slot;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t a_s = raw + pad, b_s = a_s + kDiagA;
    // bf16 1.0 / 0.5 / -1.0 / 0.25 patterns: finite values, the contents do not matter
    for (int i = threadIdx.x; i < (kDiagA + kDiagB) / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0x3f003f00u, 0xbf80bf80u, 0x3e803e80u);
    const uint32_t bar = ptx::smem_u32(&done_bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        ptx::tmem_alloc(ptx::smem_u32(&tmem_slot), 512);
        ptx::tmem_relinquish();
    }
    fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (threadIdx.x == 0) {
        const uint64_t ad = ptx::smem_desc(a_s, 16, 1024, 2);
        const uint64_t bd = ptx::smem_desc(b_s, 16, 1024, 2);
        constexpr int N = PATTERN == 2 ? 256 : PATTERN == 3 ? 64 : 128;
        constexpr int B_BOX = 256 * 128;  // B boxes are laid out for 256 rows
        const uint32_t idesc = ptx::idesc_bf16_f32(128, N, false);
        const long long t0 = clock64();
        for (int g = 0; g < groups; ++g) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a_off = ((kk / 4) * kDiagBox + (kk % 4) * 32) >> 4;
                const uint32_t b_off = ((kk / 4) * B_BOX + (kk % 4) * 32) >> 4;
                if (PATTERN == 1) {
                    // A: 128 x 16 bf16 in TMEM columns 384 + 8 kk (never written: the values do
                    // not matter for timing), accumulator at column 0
                    ptx::mma_ts(tmem, tmem + 384 + 8 * kk, bd + b_off, idesc, (g | kk) != 0);
                } else {
                    ptx::mma_ss(tmem, ad + a_off, bd + b_off, idesc, (g | kk) != 0);
                }
            }
        }
        ptx::mma_commit(bar);
        volatile int never = 0;
        const bool ok = ptx::mbar_wait(bar, 0, &never, wait_ns);
        clocks[blockIdx.x] = ok ? clock64() - t0 : -1;
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

template <int PATTERN>
int launch_pattern(long long* clocks, int ctas, int groups, unsigned long long wait_ns, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(skiparse_mma_rate_kernel<PATTERN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDiagSmem);
    if (e != cudaSuccess) return static_cast<int>(e);
    skiparse_mma_rate_kernel<PATTERN><<<ctas, 128, kDiagSmem, st>>>(clocks, groups, wait_ns);
    return static_cast<int>(cudaGetLastError());
}

__global__ void __launch_bounds__(512, 1) skiparse_softmax_rate_kernel(long long* clocks, int reps, float sl2) {
    // scores of a plausible range (the values do not change the instruction stream)
    float sc[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) sc[e] = -0.03125f * static_cast<float>((threadIdx.x * 7 + e * 3) & 63);
    float neg = -1.f;
    float sum0 = 0.f, sum1 = 0.f, sum2 = 0.f, sum3 = 0.f;
    uint32_t packs = 0;
    __syncthreads();
    const long long t0 = clock64();
    for (int r = 0; r < reps; ++r) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const float p0 = ptx::ex2_approx(fmaf(sc[2 * e], sl2, neg));
            const float p1 = ptx::ex2_approx(fmaf(sc[2 * e + 1], sl2, neg));
            if (e & 1) {
                sum2 += p0;
                sum3 += p1;
            } else {
                sum0 += p0;
                sum1 += p1;
            }
            packs ^= ptx::pack_bf16x2(p0, p1);
        }
        neg -= 1.0e-7f;  // a new exponent offset per pass, as a new running maximum would be
    }
    // the results are complete before the second clock read (the compiler may not move the
    // loop's work past it)
    asm volatile("" ::"f"(sum0), "f"(sum1), "f"(sum2), "f"(sum3), "r"(packs) : "memory");
    const long long t1 = clock64();
    // the results feed the output (a NaN pattern no finite sum produces adds one clock), so the
    // loop cannot be removed
    const uint32_t bits = __float_as_uint((sum0 + sum1) + (sum2 + sum3)) ^ packs;
    if ((threadIdx.x & 31) == 0)
        clocks[static_cast<size_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)] =
            t1 - t0 + (bits == 0x7fc00001u ? 1 : 0);
}

// Patterns 4-6: warp 0's lane 0 issues pattern 0's stream; warps 4-11 run background loop BG
// (0 FFMA chains, 1 dS arithmetic, 2 exponential loop) until the stream has completed (a flag
// in shared memory; at most 1 << 20 passes).
template <int BG>
__global__ void __launch_bounds__(384, 1) skiparse_mma_contended_kernel(long long* clocks, int groups,
                                                                         unsigned long long wait_ns) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(8) unsigned long long done_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile int stop;
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t a_s = raw + pad, b_s = a_s + kDiagA;
    for (int i = threadIdx.x; i < (kDiagA + kDiagB) / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0x3f003f00u, 0xbf80bf80u, 0x3e803e80u);
    const uint32_t bar = ptx::smem_u32(&done_bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        stop = 0;
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
        ptx::tmem_alloc(ptx::smem_u32(&tmem_slot), 512);
        ptx::tmem_relinquish();
    }
    fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (warp == 0) {
        if (threadIdx.x == 0) {
            const uint64_t ad = ptx::smem_desc(a_s, 16, 1024, 2);
            const uint64_t bd = ptx::smem_desc(b_s, 16, 1024, 2);
            constexpr int B_BOX = 256 * 128;
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 128, false);
            const long long t0 = clock64();
            for (int g = 0; g < groups; ++g) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a_off = ((kk / 4) * kDiagBox + (kk % 4) * 32) >> 4;
                    const uint32_t b_off = ((kk / 4) * B_BOX + (kk % 4) * 32) >> 4;
                    ptx::mma_ss(tmem, ad + a_off, bd + b_off, idesc, (g | kk) != 0);
                }
            }
            ptx::mma_commit(bar);
            volatile int never = 0;
            const bool ok = ptx::mbar_wait(bar, 0, &never, wait_ns);
            clocks[blockIdx.x] = ok ? clock64() - t0 : -1;
            stop = 1;
        }
        __syncwarp();
    } else if (warp >= 4) {
        float x0 = 0.001f * threadIdx.x, x1 = x0 + 0.25f, x2 = x0 + 0.5f, x3 = x0 + 0.75f;
        uint32_t acc = 0;
        for (int it = 0; it < (1 << 20) && !stop; ++it) {
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                if (BG == 0) {
                    x0 = fmaf(x0, 0.999f, 0.001f);
                    x1 = fmaf(x1, 0.999f, 0.001f);
                    x2 = fmaf(x2, 0.999f, 0.001f);
                    x3 = fmaf(x3, 0.999f, 0.001f);
                } else if (BG == 1) {
                    const float s0 = x0 * (x1 - 0.5f), s1 = x1 * (x2 - 0.25f);
                    const float s2 = x2 * (x3 - 0.125f), s3 = x3 * (x0 - 0.0625f);
                    acc ^= ptx::pack_bf16x2(s0, s1) ^ ptx::pack_bf16x2(s2, s3);
                    x0 += 1e-3f;
                    x1 += 1e-3f;
                    x2 += 1e-3f;
                    x3 += 1e-3f;
                } else {
                    const float p0 = ptx::ex2_approx(fmaf(x0, 0.01f, -1.f));
                    const float p1 = ptx::ex2_approx(fmaf(x1, 0.01f, -1.f));
                    x2 += p0;
                    x3 += p1;
                    x0 += 1e-3f;
                    x1 += 1e-3f;
                    acc ^= ptx::pack_bf16x2(p0, p1);
                }
            }
        }
        // the loop's results feed a store that no real value triggers, so it cannot be removed
        if (__float_as_uint(x0 + x1 + x2 + x3) == 0x7fc00001u && acc == 0x12345u) clocks[blockIdx.x] = -3;
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

template <int BG>
int launch_contended(long long* clocks, int ctas, int groups, unsigned long long wait_ns, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(skiparse_mma_contended_kernel<BG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kDiagSmem);
    if (e != cudaSuccess) return static_cast<int>(e);
    skiparse_mma_contended_kernel<BG><<<ctas, 384, kDiagSmem, st>>>(clocks, groups, wait_ns);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace

static_assert(kDiagA + kDiagB + 1024 <= kDiagSmem, "diagnostic shared memory");

int launch_softmax_rate(long long* clocks, int ctas, int warps_per_subpartition, int reps, void* stream) {
    cudaError_t e = cudaFuncSetAttribute(skiparse_softmax_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDiagSmem);
    if (e != cudaSuccess) return static_cast<int>(e);
    // kDiagSmem of (unused) dynamic shared memory: one CTA per SM
    skiparse_softmax_rate_kernel<<<ctas, 128 * warps_per_subpartition, kDiagSmem, static_cast<cudaStream_t>(stream)>>>(
        clocks, reps, 1.4426950408889634f * 0.08838834764831845f);
    return static_cast<int>(cudaGetLastError());
}

int launch_mma_rate(long long* clocks, int ctas, int pattern, int groups, unsigned long long wait_ns,
                    void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pattern) {
        case 0: return launch_pattern<0>(clocks, ctas, groups, wait_ns, st);
        case 1: return launch_pattern<1>(clocks, ctas, groups, wait_ns, st);
        case 2: return launch_pattern<2>(clocks, ctas, groups, wait_ns, st);
        case 3: return launch_pattern<3>(clocks, ctas, groups, wait_ns, st);
        case 4: return launch_contended<0>(clocks, ctas, groups, wait_ns, st);
        case 5: return launch_contended<1>(clocks, ctas, groups, wait_ns, st);
        case 6: return launch_contended<2>(clocks, ctas, groups, wait_ns, st);
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
}

}  // namespace skiparse
