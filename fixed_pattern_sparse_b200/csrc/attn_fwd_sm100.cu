// attn_fwd_sm100.cu -- fused Skiparse-2D attention forward for B200 (sm_100a).
//
// What it computes (summary page of OSP-Next, 核心方法 / 方法步骤详情): for every batch b, class
// c = (ci, cj) and head, dense softmax attention among the real tokens of class c, scale
// 1/sqrt(d), written straight back to the original (B,T,H,W,heads,d) layout. The rearrange is
// never materialised: tile rows are gathered from the original tensor at addresses computed from
// the class geometry, and output rows are stored to their original positions. Only real tokens
// are enumerated, so the pad-key mask touches the last (ragged) key tile of a subsequence only.
//
// One CTA = 256 queries (two 128-row tiles Q0, Q1) of one (b, class, head); every K/V tile is
// shared by both query tiles. Warp roles (11 warps):
//   warps 0-3  : softmax of Q0 (one query row per thread = TMEM lanes 0..127), epilogue of Q0
//   warps 4-7  : softmax of Q1, epilogue of Q1
//   warps 8-9  : producers: 16-byte cp.async gathers of class rows into the UMMA 128-byte
//                swizzled K-major layout, one K ring and one V ring of 2 slots each
//   warp  10   : TMEM allocator; lane 0 issues tcgen05.mma and commits
// TMEM (512 columns): S0 [0,128) S1 [128,256) fp32 scores; O0, O1 fp32 [256, 256+2d).
// P_i (bf16 pairs) is written over the first 64 columns of S_i and is the A operand of
// O_i += P_i * V straight from TMEM. MMA order per key tile j:
//   O0 += P0(j) V_j ; S0(j+1) = Q0 K_{j+1}^T ; O1 += P1(j) V_j ; S1(j+1) = Q1 K_{j+1}^T
// so the softmax of one query tile overlaps the tensor-core work of the other.
// Softmax rescales O lazily: only when a row maximum grows by more than 2^8 (FlashAttention-4's
// lazy rescaling); the stale maximum keeps every p <= 256, exact after the final division.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx_sm100.cuh"
#include "skiparse_internal.cuh"

namespace skiparse {
namespace {

constexpr int kBM = 128;   // queries per tile == TMEM lanes
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 352;
constexpr int kProdWarp0 = 8;
constexpr int kNumProducers = 64;
constexpr int kMmaWarp = 10;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by more than 2^8

template <int D>
struct Cfg {
    static constexpr int SW = D >= 64 ? 128 : 64;         // swizzle span == bytes per box row
    static constexpr int NBOX = D * 2 / SW;               // 64-/32-column boxes per row
    static constexpr int BOX_BYTES = kBM * SW;            // one 128-row box
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;   // 128 rows x D bf16
    static constexpr int KST = 2, VST = 2;                // K and V ring slots
    static constexpr uint32_t LAYOUT = SW == 128 ? 2u : 4u;  // descriptor swizzle code
    static constexpr int KSTEPS = D / 16;                 // MMA K-steps of Q*K^T
    static constexpr int KPB = (SW / 2) / 16;             // K-steps per box
    static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
    static constexpr uint32_t NCOLS = 512;
    static constexpr int OFF_Q = 0;                       // Q0, Q1
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    // barriers
    static constexpr int B_Q = 0;
    static constexpr int B_KFULL = 1;
    static constexpr int B_KEMPTY = B_KFULL + KST;
    static constexpr int B_VFULL = B_KEMPTY + KST;
    static constexpr int B_VEMPTY = B_VFULL + VST;
    static constexpr int B_SFULL = B_VEMPTY + VST;        // 2: one per query tile
    static constexpr int B_PFULL = B_SFULL + 2;           // 2
    static constexpr int B_OFULL = B_PFULL + 2;
    static constexpr int B_DRAIN = B_OFULL + 1;
    static constexpr int NBARS = B_DRAIN + 1;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + 8 * NBARS;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
    static constexpr int SMEM_USED = OFF_ABORT + 4;
    // + slack for 1024-byte alignment; at least 116 KB so that one CTA (and its 512 TMEM
    // columns) owns an SM even for small d
    static constexpr int SMEM_BYTES = SMEM_USED + 1024 > 118784 ? SMEM_USED + 1024 : 118784;
    static_assert(D == 32 || D == 64 || D == 128, "d must be 32, 64 or 128");
    static_assert(COL_O1 + D <= NCOLS, "TMEM overflow");
    static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
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

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Issues the cp.async copies of tile rows [first, first+128) of the class's real-token list
// (rows past n_c repeat row n_c-1; they are masked or never stored) into a 128-row tile laid
// out as the UMMA canonical K-major layout with 128-byte (64-byte for d = 32) swizzle.
// Producer warp pw (0/1) copies tile rows [64*pw, 64*pw+64); 16 consecutive lanes cover one
// 256-byte row so every warp instruction reads whole rows.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const uint16_t* __restrict__ g,
                                          const RowMap& rows, int first, int n_c, int pw, int lane) {
    using C = Cfg<D>;
    constexpr int CPR = D * 2 / 16;   // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;     // rows per warp instruction
    constexpr int NI = 64 / RPI;      // warp instructions per producer warp
    int ia = first + 64 * pw + lane, ib = ia + 32;
    ia = ia < n_c ? ia : n_c - 1;
    ib = ib < n_c ? ib : n_c - 1;
    const int ra = rows(ia), rb = rows(ib);
    const int c = lane % CPR;
    const int rsub = lane / CPR;
    const uint32_t box = static_cast<uint32_t>((c * 16) / C::SW);
    const uint32_t cb = static_cast<uint32_t>(((c * 16) % C::SW) / 16);
#pragma unroll
    for (int k = 0; k < NI; ++k) {
        const int rl = k * RPI + rsub;  // 0..63
        const int grow = __shfl_sync(0xffffffffu, (k * RPI < 32) ? ra : rb, rl & 31);
        const int r = 64 * pw + rl;     // tile row 0..127
        const uint32_t sw = C::SW == 128 ? (cb ^ static_cast<uint32_t>(r & 7))
                                         : (cb ^ static_cast<uint32_t>((r >> 1) & 3));
        const uint32_t d = dst + box * C::BOX_BYTES + static_cast<uint32_t>(r) * C::SW + sw * 16u;
        cp_async_16(d, g + static_cast<size_t>(grow) * D + c * 8);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) skiparse_attn_fwd_kernel(const AttnParams p) {
    using C = Cfg<D>;
    const int pair = blockIdx.x;
    const int head = blockIdx.y;
    const int seq = blockIdx.z;
    const int q2 = p.P * p.P;
    const int b = seq / q2, c = seq % q2, ci = c / p.P, cj = c % p.P;
    const int Rc = p.Rc[ci], Sc = p.Sc[cj];
    const int n_c = p.T * Rc * Sc;
    const int q_first = pair * 2 * kBM;
    if (q_first >= n_c) return;  // uniform over the CTA, before any shared state
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
        ptx::mbar_init(bar(C::B_Q), kNumProducers);
        for (int s = 0; s < C::KST; ++s) {
            ptx::mbar_init(bar(C::B_KFULL + s), kNumProducers);
            ptx::mbar_init(bar(C::B_KEMPTY + s), 1);
        }
        for (int s = 0; s < C::VST; ++s) {
            ptx::mbar_init(bar(C::B_VFULL + s), kNumProducers);
            ptx::mbar_init(bar(C::B_VEMPTY + s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(bar(C::B_SFULL + i), 1);
            ptx::mbar_init(bar(C::B_PFULL + i), kBM);
        }
        ptx::mbar_init(bar(C::B_OFULL), 1);
        ptx::mbar_init(bar(C::B_DRAIN), 1);
        *abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::NCOLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProdWarp0 || warp == kProdWarp0 + 1) {
        // ------------------------------------------------------------------ producers
        // Load order Q, K0, V0, K1, V1, ... Each load is one cp.async group; a load's full
        // barrier is signalled (after this thread's copies completed and a proxy fence) once
        // the next load has been issued, so two loads are in flight per thread.
        const int pw = warp - kProdWarp0;
        const int fault_skip = (p.fault == 1 && pw == 0 && lane == 0);
        load_tile<D>(sbase + C::OFF_Q, p.q, rows, q_first, n_c, pw, lane);
        load_tile<D>(sbase + C::OFF_Q + C::TILE_BYTES, p.q, rows, q_first + kBM, n_c, pw, lane);
        cp_async_commit();
        uint32_t prev_bar = bar(C::B_Q);
        bool ok = true;
        for (int L = 0; L < 2 * nkv; ++L) {
            const int j = L >> 1;
            const bool is_v = L & 1;
            const int nst = is_v ? C::VST : C::KST;
            const int s = j % nst;
            if (j >= nst) {
                const int empty = (is_v ? C::B_VEMPTY : C::B_KEMPTY) + s;
                int w_ok = 1;
                if (lane == 0) w_ok = ptx::mbar_wait(bar(empty), ((j / nst) - 1) & 1, abort, lim);
                w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
                if (!w_ok) {
                    ok = false;
                    break;
                }
            }
            const uint32_t dst = sbase + (is_v ? C::OFF_V : C::OFF_K) + s * C::TILE_BYTES;
            load_tile<D>(dst, is_v ? p.v : p.k, rows, j * kBN, n_c, pw, lane);
            cp_async_commit();
            cp_async_wait<1>();   // the previous load has landed
            fence_proxy_async();  // make it visible to the tensor core (async proxy)
            if (!(fault_skip && L == 1)) ptx::mbar_arrive(prev_bar);
            prev_bar = bar((is_v ? C::B_VFULL : C::B_KFULL) + s);
        }
        cp_async_wait<0>();
        if (ok) {
            fence_proxy_async();
            ptx::mbar_arrive(prev_bar);
        } else {
            record_abort(abort, p.status);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, kBN, false);
            const uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, D, true);
            const uint32_t q0 = sbase + C::OFF_Q, q1 = q0 + C::TILE_BYTES;
            auto issue_s = [&](uint32_t qs, uint32_t ks, uint32_t d_tmem) {
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk) {
                    const uint32_t off = (kk / C::KPB) * C::BOX_BYTES + (kk % C::KPB) * 32;
                    const uint64_t ad = ptx::smem_desc(qs + off, 16, 8 * C::SW, C::LAYOUT);
                    const uint64_t bd = ptx::smem_desc(ks + off, 16, 8 * C::SW, C::LAYOUT);
                    ptx::mma_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_o = [&](uint32_t p_tmem, uint32_t vs, uint32_t d_tmem, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t bd = ptx::smem_desc(vs + kk * 16 * C::SW, C::BOX_BYTES, 8 * C::SW, C::LAYOUT);
                    ptx::mma_ts(d_tmem, p_tmem + kk * 8, bd, idesc_o, (acc || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = ptx::mbar_wait(bar(C::B_Q), 0, abort, lim) &&
                      ptx::mbar_wait(bar(C::B_KFULL + 0), 0, abort, lim);
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t k0 = sbase + C::OFF_K;
                issue_s(q0, k0, tmem + C::COL_S0);
                ptx::mma_commit(bar(C::B_SFULL + 0));
                issue_s(q1, k0, tmem + C::COL_S1);
                ptx::mma_commit(bar(C::B_SFULL + 1));
                ptx::mma_commit(bar(C::B_KEMPTY + 0));
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const int vs = j % C::VST;
                const uint32_t v_smem = sbase + C::OFF_V + vs * C::TILE_BYTES;
                if (!ptx::mbar_wait(bar(C::B_VFULL + vs), (j / C::VST) & 1, abort, lim) ||
                    !ptx::mbar_wait(bar(C::B_PFULL + 0), j & 1, abort, lim)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                issue_o(tmem + C::COL_S0, v_smem, tmem + C::COL_O0, j > 0);
                const bool more = j + 1 < nkv;
                const int ks = (j + 1) % C::KST;
                const uint32_t k_smem = sbase + C::OFF_K + ks * C::TILE_BYTES;
                if (more) {
                    if (!ptx::mbar_wait(bar(C::B_KFULL + ks), ((j + 1) / C::KST) & 1, abort, lim)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    issue_s(q0, k_smem, tmem + C::COL_S0);
                    ptx::mma_commit(bar(C::B_SFULL + 0));
                }
                if (!ptx::mbar_wait(bar(C::B_PFULL + 1), j & 1, abort, lim)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                issue_o(tmem + C::COL_S1, v_smem, tmem + C::COL_O1, j > 0);
                ptx::mma_commit(bar(C::B_VEMPTY + vs));
                if (more) {
                    issue_s(q1, k_smem, tmem + C::COL_S1);
                    ptx::mma_commit(bar(C::B_SFULL + 1));
                    ptx::mma_commit(bar(C::B_KEMPTY + ks));
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
        // ------------------------------------------------------------------ softmax (WG 0/1)
        const int qt = warp >> 2;                       // query tile 0 or 1
        const int row = threadIdx.x & 127;              // TMEM lane == row in the tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_col = qt ? C::COL_S1 : C::COL_S0;
        const uint32_t o_col = qt ? C::COL_O1 : C::COL_O0;
        const uint32_t sfull = bar(C::B_SFULL + qt), pfull = bar(C::B_PFULL + qt);
        const float sl2 = p.scale_log2;
        const float thresh = kRescaleLog2 / sl2;       // in raw score units
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            if (!ptx::mbar_wait(sfull, j & 1, abort, lim)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            float sc[kBN];
            {
                uint32_t sv[32];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    ptx::tmem_ld32(tmem + lane_base + s_col + 32 * g, sv);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sc[32 * g + e] = __uint_as_float(sv[e]);
                }
            }
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
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            // lazy rescale: keep the running max unless this tile exceeds it by > 2^8
            const bool grow = (j == 0) || (mx > m_run + thresh);
            float alpha = 1.f;
            if (grow) {
                alpha = (j == 0) ? 0.f : ptx::ex2_approx((m_run - mx) * sl2);
                m_run = mx;
            }
            const float neg = -m_run * sl2;
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ptx::ex2_approx(fmaf(sc[32 * g + 2 * e], sl2, neg));
                    const float p1 = ptx::ex2_approx(fmaf(sc[32 * g + 2 * e + 1], sl2, neg));
                    sum0 += p0;
                    sum1 += p1;
                    pk[e] = ptx::pack_bf16x2(p0, p1);
                }
                ptx::tmem_st16(tmem + lane_base + s_col + 16 * g, pk);
            }
            l_run = l_run * alpha + (sum0 + sum1);
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
                // O_qt was completed by the previous P*V (the commit behind this tile's S covers it)
#pragma unroll
                for (int g = 0; g < D / 32; ++g) {
                    uint32_t ov[32];
                    const uint32_t o_addr = tmem + lane_base + o_col + 32 * g;
                    ptx::tmem_ld32(o_addr, ov);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    ptx::tmem_st32(o_addr, ov);
                }
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(pfull);
        }
        if (ok && ptx::mbar_wait(bar(C::B_OFULL), 0, abort, lim)) {
            ptx::tc_fence_after();
            const int qi = q_first + qt * kBM + row;
            const float inv_l = 1.f / l_run;
            uint4* dst = nullptr;
            if (qi < n_c) dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(rows(qi)) * D);
#pragma unroll
            for (int g = 0; g < D / 32; ++g) {
                uint32_t ov[32];
                ptx::tmem_ld32(tmem + lane_base + o_col + 32 * g, ov);
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

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::NCOLS);
    }
}

template <int D>
int launch_d(const AttnParams& p, const Geometry& g, cudaStream_t stream) {
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
    dim3 grid((n_max + 2 * kBM - 1) / (2 * kBM), g.heads, g.B * g.P * g.P);
    skiparse_attn_fwd_kernel<D><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
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

int launch_attn_fwd(const AttnParams& p, const Geometry& g, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (g.d) {
        case 32: return launch_d<32>(p, g, st);
        case 64: return launch_d<64>(p, g, st);
        case 128: return launch_d<128>(p, g, st);
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
}

}  // namespace skiparse
