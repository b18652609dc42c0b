// attn_fwd_sm100.cu -- fused Skiparse-2D attention forward for B200 (sm_100a).
//
// What it computes (summary page of OSP-Next, 核心方法 / 方法步骤详情): for every batch b, class
// c = (ci, cj) and head, dense softmax attention among the real tokens of class c, with scale
// 1/sqrt(d); the result is written straight back to the original (B,T,H,W,heads,d) layout.
// The rearrange is never materialised: each tile's rows are gathered from the original tensor
// with TMA tile::gather4 loads whose row coordinates come from the class geometry, and the
// output rows are stored to their original positions. Only real tokens are enumerated, so
// the pad-key mask is needed on the last (ragged) key tile of a subsequence only.
//
// One CTA = one tile of 128 queries of one (b, class, head). Warp roles:
//   warps 0-3 : softmax (one query row per thread, TMEM lanes 0..127) and epilogue
//   warp  4   : producer (TMA gather4 of Q once, then K/V tiles into a 2-stage ring)
//   warp  5   : TMEM allocator; lane 0 issues tcgen05.mma and commits
// TMEM (512 columns): S0 [0,128) S1 [128,256) fp32 scores (double-buffered so Q*K_{j+1}^T
// runs while the softmax of tile j is busy), O [256,256+d) fp32, P [384,448) bf16 pairs --
// P is the A operand of O += P*V straight from TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx_sm100.cuh"
#include "skiparse_internal.cuh"

namespace skiparse {
namespace {

constexpr int kBM = 128;   // queries per tile == TMEM lanes
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

template <int D>
struct Cfg {
    static constexpr int SW = D >= 64 ? 128 : 64;         // swizzle span == bytes per box row
    static constexpr int BOX_COLS = SW / 2;               // bf16 columns per TMA box
    static constexpr int NBOX = D / BOX_COLS;
    static constexpr int BOX_BYTES = kBM * SW;            // one 128-row box
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;   // 128 rows x D bf16
    static constexpr int STAGES = 2;
    static constexpr uint32_t LAYOUT = SW == 128 ? 2u : 4u;  // descriptor swizzle code
    static constexpr int KSTEPS = D / 16;                 // MMA K-steps of Q*K^T
    static constexpr int KPB = BOX_COLS / 16;             // K-steps per box
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256, COL_P = 384;
    static constexpr uint32_t NCOLS = 512;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE_BYTES;
    static constexpr int OFF_V = TILE_BYTES * (1 + STAGES);
    static constexpr int OFF_BAR = TILE_BYTES * (1 + 2 * STAGES);
    // barrier indices
    static constexpr int B_Q = 0;
    static constexpr int B_KFULL = 1;
    static constexpr int B_VFULL = B_KFULL + STAGES;
    static constexpr int B_EMPTY = B_VFULL + STAGES;
    static constexpr int B_SFULL = B_EMPTY + STAGES;      // 2 of them
    static constexpr int B_PFULL = B_SFULL + 2;
    static constexpr int B_PVDONE = B_PFULL + 1;
    static constexpr int B_OFULL = B_PVDONE + 1;
    static constexpr int B_DRAIN = B_OFULL + 1;
    static constexpr int NBARS = B_DRAIN + 1;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + 8 * NBARS;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
    static constexpr int SMEM_USED = OFF_ABORT + 4;
    // + slack for 1024-byte alignment; at least 116 KB so that one CTA (and its 512 TMEM
    // columns) owns an SM even for small d
    static constexpr int SMEM_BYTES = SMEM_USED + 1024 > 118784 ? SMEM_USED + 1024 : 118784;
    static_assert(D % 32 == 0 && D <= 128, "d must be 32, 64 or 128");
    static_assert(COL_O + D <= COL_P, "TMEM regions overlap");
};

// Global row (token*heads + head) of the class-local real token i of (b, ci, cj).
struct RowMap {
    int T, H, W, heads, P, mode;
    int ci, cj, Rc, Sc, b, head;
    __device__ __forceinline__ int operator()(int i) const {
        const int s = i % Sc;
        const int tr = i / Sc;
        const int r = tr % Rc;
        const int t = tr / Rc;
        const int h = axis_coord(r, ci, P, mode);
        const int w = axis_coord(s, cj, P, mode);
        return (((b * T + t) * H + h) * W + w) * heads + head;
    }
};

__device__ __forceinline__ void record_abort(volatile int* abort, int* status) {
    *abort = 1;
    atomicExch(status, kErrTimeout);
}

// Gathers rows [first, first+128) of the class's real-token list (clamped to n_c-1) into a
// 128-row tile. Each lane gathers 4 consecutive rows per box.
template <int D>
__device__ __forceinline__ void gather_tile(const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                            const RowMap& rows, int first, int n_c, int lane) {
    using C = Cfg<D>;
    int r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int i = first + 4 * lane + u;
        i = i < n_c ? i : n_c - 1;
        r[u] = rows(i);
    }
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx)
        ptx::tma_gather4(dst + bx * C::BOX_BYTES + lane * 4 * C::SW, map, bar, bx * C::BOX_COLS,
                         r[0], r[1], r[2], r[3]);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    skiparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                             const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v, const AttnParams p) {
    using C = Cfg<D>;
    const int q_tile = blockIdx.x;
    const int head = blockIdx.y;
    const int seq = blockIdx.z;
    const int q2 = p.P * p.P;
    const int b = seq / q2, c = seq % q2, ci = c / p.P, cj = c % p.P;
    const int Rc = p.Rc[ci], Sc = p.Sc[cj];
    const int n_c = p.T * Rc * Sc;
    if (q_tile * kBM >= n_c) return;  // uniform over the CTA, before any shared state
    const int nkv = (n_c + kBN - 1) / kBN;
    const RowMap rows{p.T, p.H, p.W, p.heads, p.P, p.mode, ci, cj, Rc, Sc, b, head};

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_base = ptx::smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_base & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;
    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_SLOT);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint64_t lim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(C::B_Q), 1);
        for (int s = 0; s < C::STAGES; ++s) {
            ptx::mbar_init(bar(C::B_KFULL + s), 1);
            ptx::mbar_init(bar(C::B_VFULL + s), 1);
            ptx::mbar_init(bar(C::B_EMPTY + s), 1);
        }
        ptx::mbar_init(bar(C::B_SFULL + 0), 1);
        ptx::mbar_init(bar(C::B_SFULL + 1), 1);
        ptx::mbar_init(bar(C::B_PFULL), kBM);
        ptx::mbar_init(bar(C::B_PVDONE), 1);
        ptx::mbar_init(bar(C::B_OFULL), 1);
        ptx::mbar_init(bar(C::B_DRAIN), 1);
        *abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::NCOLS);
        ptx::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        ptx::prefetch_tensormap(&tmap_q);
        ptx::prefetch_tensormap(&tmap_k);
        ptx::prefetch_tensormap(&tmap_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    int issued = 0;  // producer: K/V tiles issued

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar(C::B_Q), C::TILE_BYTES);
        __syncwarp();
        gather_tile<D>(&tmap_q, sbase + C::OFF_Q, bar(C::B_Q), rows, q_tile * kBM, n_c, lane);
        for (int j = 0; j < nkv; ++j) {
            const int s = j % C::STAGES;
            if (j >= C::STAGES) {
                int ok = 1;
                if (lane == 0) {
                    ok = ptx::mbar_wait(bar(C::B_EMPTY + s), ((j / C::STAGES) - 1) & 1, abort, lim);
                    if (!ok) record_abort(abort, p.status);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
            if (lane == 0) {
                const uint32_t extra = (p.fault == 1 && j == 0) ? 16u : 0u;
                ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES + extra);
            }
            __syncwarp();
            gather_tile<D>(&tmap_k, sbase + C::OFF_K + s * C::TILE_BYTES, bar(C::B_KFULL + s), rows,
                           j * kBN, n_c, lane);
            if (lane == 0) ptx::mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::TILE_BYTES);
            __syncwarp();
            gather_tile<D>(&tmap_v, sbase + C::OFF_V + s * C::TILE_BYTES, bar(C::B_VFULL + s), rows,
                           j * kBN, n_c, lane);
            issued = j + 1;
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, kBN, false);
            const uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, D, true);
            bool ok = ptx::mbar_wait(bar(C::B_Q), 0, abort, lim);
            for (int j = 0; ok && j <= nkv; ++j) {
                if (j < nkv) {
                    const int s = j % C::STAGES;
                    if (!ptx::mbar_wait(bar(C::B_KFULL + s), (j / C::STAGES) & 1, abort, lim)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t d_s = tmem + ((j & 1) ? C::COL_S1 : C::COL_S0);
                    const uint32_t kbase = sbase + C::OFF_K + s * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::KSTEPS; ++kk) {
                        const uint32_t off = (kk / C::KPB) * C::BOX_BYTES + (kk % C::KPB) * 32;
                        const uint64_t ad = ptx::smem_desc(sbase + C::OFF_Q + off, 16, 8 * C::SW, C::LAYOUT);
                        const uint64_t bd = ptx::smem_desc(kbase + off, 16, 8 * C::SW, C::LAYOUT);
                        ptx::mma_ss(d_s, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(bar(C::B_SFULL + (j & 1)));
                }
                if (j >= 1) {
                    const int jj = j - 1;
                    const int s = jj % C::STAGES;
                    if (!ptx::mbar_wait(bar(C::B_PFULL), jj & 1, abort, lim) ||
                        !ptx::mbar_wait(bar(C::B_VFULL + s), (jj / C::STAGES) & 1, abort, lim)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t vbase = sbase + C::OFF_V + s * C::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk) {
                        const uint64_t bd = ptx::smem_desc(vbase + kk * 16 * C::SW, C::BOX_BYTES,
                                                           8 * C::SW, C::LAYOUT);
                        ptx::mma_ts(tmem + C::COL_O, tmem + C::COL_P + kk * 8, bd, idesc_o,
                                    (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(bar(C::B_EMPTY + s));
                    ptx::mma_commit(bar(C::B_PVDONE));
                }
            }
            if (ok) {
                ptx::mma_commit(bar(C::B_OFULL));
            } else {
                record_abort(abort, p.status);
            }
            // every MMA issued by this thread must finish before TMEM is released
            ptx::mma_commit(bar(C::B_DRAIN));
            volatile int never = 0;
            ptx::mbar_wait(bar(C::B_DRAIN), 0, &never, lim);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ softmax
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            if (!ptx::mbar_wait(bar(C::B_SFULL + (j & 1)), (j >> 1) & 1, abort, lim)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + ((j & 1) ? C::COL_S1 : C::COL_S0);
            uint32_t sv[4][32];
#pragma unroll
            for (int g = 0; g < 4; ++g) ptx::tmem_ld32(s_addr + 32 * g, sv[g]);
            ptx::tmem_wait_ld();
            float sc[kBN];
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int e = 0; e < 32; ++e) sc[32 * g + e] = __uint_as_float(sv[g][e]);
            if (j == nkv - 1) {
                const int valid = n_c - j * kBN;
#pragma unroll
                for (int e = 0; e < kBN; ++e)
                    if (e >= valid) sc[e] = -INFINITY;
            }
            float mx0 = sc[0], mx1 = sc[1], mx2 = sc[2], mx3 = sc[3];
#pragma unroll
            for (int e = 4; e < kBN; e += 4) {
                mx0 = fmaxf(mx0, sc[e]);
                mx1 = fmaxf(mx1, sc[e + 1]);
                mx2 = fmaxf(mx2, sc[e + 2]);
                mx3 = fmaxf(mx3, sc[e + 3]);
            }
            const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)));
            const float alpha = ptx::ex2_approx((m_run - m_new) * sl2);
            const float neg = -m_new * sl2;
            float sum0 = 0.f, sum1 = 0.f;
            uint32_t pk[kBN / 2];
#pragma unroll
            for (int e = 0; e < kBN / 2; ++e) {
                const float p0 = ptx::ex2_approx(fmaf(sc[2 * e], sl2, neg));
                const float p1 = ptx::ex2_approx(fmaf(sc[2 * e + 1], sl2, neg));
                sum0 += p0;
                sum1 += p1;
                pk[e] = ptx::pack_bf16x2(p0, p1);
            }
            l_run = l_run * alpha + (sum0 + sum1);
            if (j > 0) {
                // P_{j-1} and O are still being read/written by the previous P*V MMA
                if (!ptx::mbar_wait(bar(C::B_PVDONE), (j - 1) & 1, abort, lim)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int g = 0; g < D / 32; ++g) {
                        uint32_t ov[32];
                        const uint32_t o_addr = tmem + lane_base + C::COL_O + 32 * g;
                        ptx::tmem_ld32(o_addr, ov);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        ptx::tmem_st32(o_addr, ov);
                    }
                }
            }
            {
                uint32_t half[32];
#pragma unroll
                for (int h2 = 0; h2 < kBN / 64; ++h2) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) half[e] = pk[32 * h2 + e];
                    ptx::tmem_st32(tmem + lane_base + C::COL_P + 32 * h2, half);
                }
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(C::B_PFULL));
            m_run = m_new;
        }
        if (ok && ptx::mbar_wait(bar(C::B_OFULL), 0, abort, lim)) {
            ptx::tc_fence_after();
            const int qi = q_tile * kBM + static_cast<int>(threadIdx.x);
            const float inv_l = 1.f / l_run;
            uint4* dst = nullptr;
            if (qi < n_c) dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(rows(qi)) * D);
#pragma unroll
            for (int g = 0; g < D / 32; ++g) {
                uint32_t ov[32];
                ptx::tmem_ld32(tmem + lane_base + C::COL_O + 32 * g, ov);
                ptx::tmem_wait_ld();
                uint32_t pkd[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pkd[e] = ptx::pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l,
                                              __uint_as_float(ov[2 * e + 1]) * inv_l);
                if (dst) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[4 * g + v4] = make_uint4(pkd[4 * v4], pkd[4 * v4 + 1], pkd[4 * v4 + 2],
                                                     pkd[4 * v4 + 3]);
                }
            }
        } else if (!*abort) {
            record_abort(abort, p.status);
        }
    }

    __syncthreads();
    if (*abort && warp == kProducerWarp && lane == 0) {
        // Let any TMA copy this CTA issued land before its shared memory is released.
        volatile int never = 0;
        const uint64_t drain_ns = lim < 1000000ull ? lim : 1000000ull;
        ptx::mbar_wait(bar(C::B_Q), 0, &never, drain_ns);
        const int first = issued > C::STAGES ? issued - C::STAGES : 0;
        for (int j = first; j < issued; ++j) {
            const int s = j % C::STAGES;
            ptx::mbar_wait(bar(C::B_KFULL + s), (j / C::STAGES) & 1, &never, drain_ns);
            ptx::mbar_wait(bar(C::B_VFULL + s), (j / C::STAGES) & 1, &never, drain_ns);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::NCOLS);
    }
}

template <int D>
int launch_d(const void* tq, const void* tk, const void* tv, const AttnParams& p,
             const Geometry& g, cudaStream_t stream) {
    using C = Cfg<D>;
    static int attr_done_dev[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return static_cast<int>(e);
    if (dev >= 0 && dev < 64 && !attr_done_dev[dev]) {
        e = cudaFuncSetAttribute(skiparse_attn_fwd_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return static_cast<int>(e);
        attr_done_dev[dev] = 1;
    }
    int n_max = 0;
    for (int ci = 0; ci < g.P; ++ci)
        for (int cj = 0; cj < g.P; ++cj) {
            const int n_c = g.T * g.Rc[ci] * g.Sc[cj];
            n_max = n_c > n_max ? n_c : n_max;
        }
    dim3 grid((n_max + kBM - 1) / kBM, g.heads, g.B * g.P * g.P);
    skiparse_attn_fwd_kernel<D><<<grid, kThreads, C::SMEM_BYTES, stream>>>(
        *static_cast<const CUtensorMap*>(tq), *static_cast<const CUtensorMap*>(tk),
        *static_cast<const CUtensorMap*>(tv), p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace

int attn_smem_bytes(int d) {
    switch (d) {
        case 32: return Cfg<32>::SMEM_BYTES;
        case 64: return Cfg<64>::SMEM_BYTES;
        case 128: return Cfg<128>::SMEM_BYTES;
        default: return -1;
    }
}

int launch_attn_fwd(const void* tq, const void* tk, const void* tv, const AttnParams& p,
                    const Geometry& g, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (g.d) {
        case 32: return launch_d<32>(tq, tk, tv, p, g, st);
        case 64: return launch_d<64>(tq, tk, tv, p, g, st);
        case 128: return launch_d<128>(tq, tk, tv, p, g, st);
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
}

}  // namespace skiparse
