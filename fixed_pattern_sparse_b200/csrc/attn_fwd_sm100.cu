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
// so the softmax of one query tile overlaps the tensor-core work of the other. The softmax
// releases P in two halves of the key tile, and O += P V on the first half starts while the
// exponentials of the second half run.
// Softmax rescales O lazily: only when a row maximum grows by more than 2^8 (FlashAttention-4's
// lazy rescaling); the stale maximum keeps every p <= 256, exact after the final division.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "attn_common.cuh"

namespace skiparse {
namespace {

constexpr int kBM = 128;   // queries per tile == TMEM lanes
constexpr int kBN = 128;   // keys per tile
constexpr int kThreads = 352;
constexpr int kProdWarp0 = 8;
constexpr int kNumProducers = 64;
constexpr int kMmaWarp = 10;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by more than 2^8
constexpr int kPParts = 2;            // P is released to the tensor core in two halves of the key tile

template <int D>
struct Cfg : TileGeom<D> {
    using G = TileGeom<D>;
    using G::SW;
    using G::NBOX;
    using G::BOX_BYTES;
    using G::TILE_BYTES;
    using G::LAYOUT;
    using G::KSTEPS;
    using G::KPB;
    static constexpr int KST = 2, VST = 2;                // K and V ring slots
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
    static constexpr int B_PFULL = B_SFULL + 2;           // 2 x kPParts: (query tile, part of the key tile)
    static constexpr int B_OFULL = B_PFULL + 2 * kPParts;
    static constexpr int B_DRAIN = B_OFULL + 1;
    static constexpr int NBARS = B_DRAIN + 1;
    static constexpr int OFF_TMEM_SLOT = OFF_BAR + 8 * NBARS;
    static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
    static constexpr int SMEM_USED = OFF_ABORT + 4;
    // + slack for 1024-byte alignment; at least 116 KB so that one CTA (and its 512 TMEM
    // columns) owns an SM even for small d
    static constexpr int SMEM_BYTES = SMEM_USED + 1024 > 118784 ? SMEM_USED + 1024 : 118784;
    static_assert(COL_O1 + D <= NCOLS, "TMEM overflow");
    static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) skiparse_attn_fwd_kernel(const AttnParams p) {
    using C = Cfg<D>;
    const int pair = blockIdx.x;
    const int head = blockIdx.y;
    const int seq = blockIdx.z;
    const int q2 = p.Ph * p.Pw;
    const int b = seq / q2, c = seq % q2, ci = c / p.Pw, cj = c % p.Pw;
    const int Rc = p.Rc[ci], Sc = p.Sc[cj];
    const int n_c = p.T * Rc * Sc;
    const int q_first = pair * 2 * kBM;
    if (q_first >= n_c) return;  // uniform over the CTA, before any shared state
    const int nkv = (n_c + kBN - 1) / kBN;
    RowMap rows;
    rows.init(p.T, p.H, p.W, p.heads, p.Ph, p.Pw, p.mode, ci, cj, Rc, Sc, b, head);

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
            for (int h = 0; h < kPParts; ++h) ptx::mbar_init(bar(C::B_PFULL + kPParts * i + h), kBM);
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

    if (warp >= kProdWarp0) {
      if (warp == kProdWarp0 || warp == kProdWarp0 + 1) {
        // ------------------------------------------------------------------ producers
        // Load order Q, K0, V0, K1, V1, ... Every thread arrives on a load's full barrier with
        // cp.async.mbarrier.arrive.noinc right after issuing its copies; the arrival fires when
        // they have landed, so a tile is released as soon as it is in shared memory.
        const int pw = warp - kProdWarp0;
        const int fault_skip = (p.fault == 1 && pw == 0 && lane == 0);
        load_tile<D>(sbase + C::OFF_Q, p.q, rows, q_first, n_c, pw, lane, p.nrows, p.status);
        load_tile<D>(sbase + C::OFF_Q + C::TILE_BYTES, p.q, rows, q_first + kBM, n_c, pw, lane, p.nrows,
                     p.status);
        cp_async_arrive_noinc(bar(C::B_Q));
        bool ok = true;
        TileRows kv{0, 0};  // token rows of key step j, shared by its K and V tiles
        for (int L = 0; L < 2 * nkv; ++L) {
            const int j = L >> 1;
            const bool is_v = L & 1;
            const int nst = is_v ? C::VST : C::KST;
            const int s = j % nst;
            if (!is_v) kv = tile_rows(rows, j * kBN, n_c, pw, lane, p.nrows, p.status);
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
            load_tile_rows<D>(dst, is_v ? p.v : p.k, kv, pw, lane);
            // test hook: one thread never signals the first K tile
            if (!(fault_skip && L == 0)) cp_async_arrive_noinc(bar((is_v ? C::B_VFULL : C::B_KFULL) + s));
        }
        cp_async_commit();
        cp_async_wait<0>();  // no copy of this thread outlives it
        if (!ok) record_abort(abort, p.status);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, kBN, false);
            const uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, D, true);
            const uint32_t q0 = sbase + C::OFF_Q, q1 = q0 + C::TILE_BYTES;
            // Descriptors are built once; a K-step only advances the 14-bit start-address field.
            const uint64_t qd0 = ptx::smem_desc(q0, 16, 8 * C::SW, C::LAYOUT);
            const uint64_t qd1 = ptx::smem_desc(q1, 16, 8 * C::SW, C::LAYOUT);
            const uint64_t kd0 = ptx::smem_desc(sbase + C::OFF_K, 16, 8 * C::SW, C::LAYOUT);
            const uint64_t vd0 = ptx::smem_desc(sbase + C::OFF_V, C::BOX_BYTES, 8 * C::SW, C::LAYOUT);
            auto issue_s = [&](uint64_t qd, int kslot, uint32_t d_tmem) {
                const uint64_t kd = kd0 + ((kslot * C::TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::KSTEPS; ++kk) {
                    const uint32_t off = ((kk / C::KPB) * C::BOX_BYTES + (kk % C::KPB) * 32) >> 4;
                    ptx::mma_ss(d_tmem, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // O += P V over one part of the key tile (keys [h, h+1) * kBN / kPParts), as soon as
            // the softmax has released that part of P
            auto issue_o_half = [&](uint32_t p_tmem, int vslot, uint32_t d_tmem, bool acc, int h) {
                const uint64_t vd = vd0 + ((vslot * C::TILE_BYTES) >> 4);
                constexpr int KPP = kBN / 16 / kPParts;  // K-steps per part
#pragma unroll
                for (int k4 = 0; k4 < KPP; ++k4) {
                    const int kk = h * KPP + k4;
                    ptx::mma_ts(d_tmem, p_tmem + kk * 8, vd + ((kk * 16 * C::SW) >> 4), idesc_o,
                                (acc || kk > 0) ? 1u : 0u);
                }
            };
            auto issue_o = [&](int qt, int vslot, bool acc, int phase) -> bool {
                const uint32_t p_tmem = tmem + (qt ? C::COL_S1 : C::COL_S0);
                const uint32_t d_tmem = tmem + (qt ? C::COL_O1 : C::COL_O0);
                for (int h = 0; h < kPParts; ++h) {
                    if (!ptx::mbar_wait(bar(C::B_PFULL + kPParts * qt + h), phase, abort, lim)) return false;
                    ptx::tc_fence_after();
                    issue_o_half(p_tmem, vslot, d_tmem, acc, h);
                }
                return true;
            };
            bool ok = ptx::mbar_wait(bar(C::B_Q), 0, abort, lim) &&
                      ptx::mbar_wait(bar(C::B_KFULL + 0), 0, abort, lim);
            if (ok) {
                fence_proxy_async();  // cp.async data observed through the barriers, for the MMA
                ptx::tc_fence_after();
                issue_s(qd0, 0, tmem + C::COL_S0);
                ptx::mma_commit(bar(C::B_SFULL + 0));
                issue_s(qd1, 0, tmem + C::COL_S1);
                ptx::mma_commit(bar(C::B_SFULL + 1));
                ptx::mma_commit(bar(C::B_KEMPTY + 0));
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const int vs = j % C::VST;
                const bool v_ok = ptx::mbar_wait(bar(C::B_VFULL + vs), (j / C::VST) & 1, abort, lim);
                if (v_ok) fence_proxy_async();
                if (!v_ok || !issue_o(0, vs, j > 0, j & 1)) {
                    ok = false;
                    break;
                }
                const bool more = j + 1 < nkv;
                const int ks = (j + 1) % C::KST;
                if (more) {
                    if (!ptx::mbar_wait(bar(C::B_KFULL + ks), ((j + 1) / C::KST) & 1, abort, lim)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async();
                    ptx::tc_fence_after();
                    issue_s(qd0, ks, tmem + C::COL_S0);
                    ptx::mma_commit(bar(C::B_SFULL + 0));
                }
                if (!issue_o(1, vs, j > 0, j & 1)) {
                    ok = false;
                    break;
                }
                ptx::mma_commit(bar(C::B_VEMPTY + vs));
                if (more) {
                    issue_s(qd1, ks, tmem + C::COL_S1);
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
      }
    } else {
        // ------------------------------------------------------------------ softmax (WG 0/1)
        const int qt = warp >> 2;                       // query tile 0 or 1
        const int row = threadIdx.x & 127;              // TMEM lane == row in the tile
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_base + (qt ? C::COL_S1 : C::COL_S0);
        const uint32_t o_col = qt ? C::COL_O1 : C::COL_O0;
        const uint32_t sfull = bar(C::B_SFULL + qt);
        const float sl2 = p.scale_log2;
        const float thresh = kRescaleLog2 / sl2;       // in raw score units
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            // Every wait of a softmax warp is made uniform over the warp (a lane can see the abort
            // flag while another sees the phase complete): the tcgen05.ld/st below are
            // .sync.aligned and need all 32 lanes.
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(sfull, j & 1, abort, lim))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const bool last = (j == nkv - 1);
            // The row max is taken over the whole tile before any exponential (the first tile
            // sets the reference max; the ragged last tile has masked keys).
            float sc[kBN];
            {
                uint32_t sv[kBN];
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    ptx::tmem_ld32(s_addr + 32 * g, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * g]));
                ptx::tmem_wait_ld();  // one wait for the whole 128-column row
#pragma unroll
                for (int e = 0; e < kBN; ++e) sc[e] = __uint_as_float(sv[e]);
            }
            if (last) {
                const int valid = n_c - j * kBN;
#pragma unroll
                for (int e = 0; e < kBN; ++e)
                    if (e >= valid) sc[e] = -INFINITY;
            }
            // row max with 3-input max instructions, four independent chains
            float mx0 = ptx::max3f(sc[0], sc[1], sc[2]), mx1 = ptx::max3f(sc[3], sc[4], sc[5]);
            float mx2 = ptx::max3f(sc[6], sc[7], sc[8]), mx3 = ptx::max3f(sc[9], sc[10], sc[11]);
#pragma unroll
            for (int e = 12; e + 8 <= kBN; e += 8) {
                mx0 = ptx::max3f(mx0, sc[e], sc[e + 1]);
                mx1 = ptx::max3f(mx1, sc[e + 2], sc[e + 3]);
                mx2 = ptx::max3f(mx2, sc[e + 4], sc[e + 5]);
                mx3 = ptx::max3f(mx3, sc[e + 6], sc[e + 7]);
            }
            static_assert((kBN - 12) % 8 == 4, "tail of the max chains");
            mx0 = ptx::max3f(mx0, sc[kBN - 4], sc[kBN - 3]);
            mx1 = ptx::max3f(mx1, sc[kBN - 2], sc[kBN - 1]);
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
            float alpha = 1.f;
            if (j == 0 || mx > m_run + thresh) {
                alpha = (j == 0) ? 0.f : ptx::ex2_approx((m_run - mx) * sl2);
                m_run = mx;
            }
            // P = 2^(S*scale*log2(e) - m), written as bf16 pairs over the first 64 columns of S.
            // Each half of the key tile is released to the tensor core as soon as it is stored,
            // so O += P V on the first half overlaps the exponentials of the second.
            const float neg = -m_run * sl2;
            float sum0 = 0.f, sum1 = 0.f, sum2 = 0.f, sum3 = 0.f;  // four short addition chains
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = fmaf(sc[32 * g + 2 * e], sl2, neg);
                    const float x1 = fmaf(sc[32 * g + 2 * e + 1], sl2, neg);
                    const float p0 = ptx::ex2_approx(x0);
                    const float p1 = ptx::ex2_approx(x1);
                    if (e & 1) {
                        sum2 += p0;
                        sum3 += p1;
                    } else {
                        sum0 += p0;
                        sum1 += p1;
                    }
                    pk[e] = ptx::pack_bf16x2(p0, p1);
                }
                ptx::tmem_st16(s_addr + 16 * g, pk);
                if (g == 1 && j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // Rare: a row max grew by more than 2^8. This warp rescales its rows of O_qt
                    // before releasing the first half of P, i.e. before this tile's P*V
                    // accumulates into O_qt; O_qt was completed by the previous P*V (the commit
                    // behind this tile's S covers it). Half of the scores are consumed here,
                    // which leaves room in registers.
#pragma unroll
                    for (int go = 0; go < D / 16; ++go) {
                        uint32_t ov[16];
                        const uint32_t o_addr = tmem + lane_base + o_col + 16 * go;
                        ptx::tmem_ld16(o_addr, ov);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        ptx::tmem_st16(o_addr, ov);
                    }
                }
                if (g & 1) {
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(bar(C::B_PFULL + kPParts * qt + (g >> 1)));
                }
            }
            l_run = l_run * alpha + ((sum0 + sum1) + (sum2 + sum3));
        }
        if (ok && __all_sync(0xffffffffu, ptx::mbar_wait(bar(C::B_OFULL), 0, abort, lim))) {
            ptx::tc_fence_after();
            const int qi = q_first + qt * kBM + row;
            const float inv_l = 1.f / l_run;
            uint4* dst = nullptr;
            if (qi < n_c && row_ok(rows(qi), p.nrows, p.status)) {
                const int grow = rows(qi);
                dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(grow) * D);
                // log-sum-exp (natural log) of the scaled scores: m*log2(e)/sqrt(d) + log2(l), in ln
                if (p.lse) p.lse[grow] = (m_run * sl2 + ptx::lg2_approx(l_run)) * 0.6931471805599453f;
            }
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
    // per device: the kernel's shared-memory attribute is set (host threads may race here;
    // setting it twice is harmless, the flag only has to be a race-free read)
    static std::atomic<int> attr_done_dev[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return static_cast<int>(e);
    if (dev >= 0 && dev < 64 && !attr_done_dev[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(skiparse_attn_fwd_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return static_cast<int>(e);
        attr_done_dev[dev].store(1, std::memory_order_release);
    }
    int n_max = 0;
    for (int ci = 0; ci < g.Ph; ++ci)
        for (int cj = 0; cj < g.Pw; ++cj) {
            const int n_c = g.T * g.Rc[ci] * g.Sc[cj];
            n_max = n_c > n_max ? n_c : n_max;
        }
    dim3 grid((n_max + 2 * kBM - 1) / (2 * kBM), g.heads, g.B * g.Ph * g.Pw);
    skiparse_attn_fwd_kernel<D><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
    return static_cast<int>(cudaGetLastError());
}

// Diagnostic: y = 2^x by the MUFU instruction exactly as the softmax evaluates it, so its
// error can be tested against fp64.
__global__ void skiparse_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) y[i] = ptx::ex2_approx(x[i]);
}

}  // namespace

int launch_exp2(const float* x, float* y, long long n, void* stream) {
    if (n <= 0) return static_cast<int>(cudaSuccess);
    const int threads = 256;
    const long long blocks = (n + threads - 1) / threads;
    skiparse_exp2_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    return static_cast<int>(cudaGetLastError());
}

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
