// attn_common.cuh -- pieces shared by the Skiparse attention kernels (forward and backward):
// tile geometry of the UMMA canonical K-major layout, the class-local-token -> global-row map,
// and the producers' 16-byte cp.async gather of class rows into that layout.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"
#include "skiparse_internal.cuh"

namespace skiparse {

constexpr int kTileRows = 128;  // rows of a Q/K/V tile == TMEM lanes

// A 128-row tile of d bf16 columns in shared memory: boxes of 128 rows x (swizzle span) bytes,
// 128-byte swizzle (64-byte for d = 32), 1024-byte aligned -- the canonical K-major layout
// that tcgen05 shared-memory descriptors describe (and, read the other way, MN-major).
template <int D>
struct TileGeom {
    static constexpr int SW = D >= 64 ? 128 : 64;         // swizzle span == bytes per box row
    static constexpr int NBOX = D * 2 / SW;               // 64-/32-column boxes per row
    static constexpr int BOX_BYTES = kTileRows * SW;      // one 128-row box
    static constexpr int TILE_BYTES = BOX_BYTES * NBOX;   // 128 rows x D bf16
    static constexpr uint32_t LAYOUT = SW == 128 ? 2u : 4u;  // descriptor swizzle code
    static constexpr int KSTEPS = D / 16;                 // MMA K-steps over d
    static constexpr int KPB = (SW / 2) / 16;             // K-steps per box
    static_assert(D == 32 || D == 64 || D == 128, "d must be 32, 64 or 128");
    // byte offset of K-step kk (16 columns) inside a K-major tile
    static constexpr uint32_t kstep_off(int kk) { return (kk / KPB) * BOX_BYTES + (kk % KPB) * 32; }
};

// Division by a divisor that is fixed for a whole CTA, as one multiply-high, an add and a shift
// (T. Granlund and P. Montgomery, "Division by invariant integers using multiplication",
// PLDI 1994): for d >= 1 and 0 <= n < 2^31, n div d = (umulhi(n, m) + n) >> l with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1 (umulhi(n, m) < n, so the sum fits
// 32 bits). The producers evaluate the class-local -> token row map for every row they load;
// with runtime divisions it cost them more issue slots than the copies themselves.
struct FastDiv {
    uint32_t m;
    uint32_t l;
    __host__ __device__ void init(int d) {
        const uint32_t dd = d < 1 ? 1u : static_cast<uint32_t>(d);
        l = 0;
        while ((1ull << l) < dd) ++l;
        m = static_cast<uint32_t>((((1ull << 32) * ((1ull << l) - dd)) / dd) + 1);
    }
    __device__ __forceinline__ int div(int n) const {
        return static_cast<int>((__umulhi(static_cast<uint32_t>(n), m) + static_cast<uint32_t>(n)) >> l);
    }
};

// Global row (token*heads + head) of the class-local real token i of (b, ci, cj).
struct RowMap {
    int T, H, W, heads, Ph, Pw, mode;
    int ci, cj, Rc, Sc, b, head;
    FastDiv dSc, dRc, dPh, dPw;
    __device__ __forceinline__ void init(int T_, int H_, int W_, int heads_, int Ph_, int Pw_,
                                         int mode_, int ci_, int cj_, int Rc_, int Sc_, int b_,
                                         int head_) {
        T = T_; H = H_; W = W_; heads = heads_; Ph = Ph_; Pw = Pw_; mode = mode_;
        ci = ci_; cj = cj_; Rc = Rc_; Sc = Sc_; b = b_; head = head_;
        dSc.init(Sc);
        dRc.init(Rc);
        dPh.init(Ph);
        dPw.init(Pw);
    }
    // axis_coord (skiparse_internal.cuh) with the group-wise division by P done as above
    __device__ __forceinline__ int coord(int sub, int cls, int P, const FastDiv& dP) const {
        if (mode == 0) return cls + P * sub;
        const int blk = dP.div(sub);
        return blk * P * P + cls * P + (sub - blk * P);
    }
    __device__ __forceinline__ int operator()(int i) const {
        const int tr = dSc.div(i);
        const int s = i - tr * Sc;
        const int t = dRc.div(tr);
        const int r = tr - t * Rc;
        const int h = coord(r, ci, Ph, dPh);
        const int w = coord(s, cj, Pw, dPw);
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
// Arrives on `bar` when all cp.async copies this thread has issued so far have landed (the
// arrival counts against the barrier's expected count: no pending-count increment), so a
// tile's full barrier completes as soon as its data is in shared memory, independently of what
// the producer issues next.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The two token rows a producer lane copies for tile rows [first, first+128) of the class's
// real-token list: tile rows 64*pw + lane and 64*pw + lane + 32 (rows past n_c repeat row
// n_c-1; they are masked or never stored). K and V tiles of one key step share them. nrows and
// status serve the debug build's bounds check (the tensor's row count, the error word).
struct TileRows {
    int ra, rb;
};
__device__ __forceinline__ TileRows tile_rows(const RowMap& rows, int first, int n_c, int pw, int lane,
                                              long long nrows, int* status) {
    int ia = first + 64 * pw + lane, ib = ia + 32;
    ia = ia < n_c ? ia : n_c - 1;
    ib = ib < n_c ? ib : n_c - 1;
    return TileRows{static_cast<int>(load_row(rows(ia), nrows, status)),
                    static_cast<int>(load_row(rows(ib), nrows, status))};
}

// Issues the cp.async copies of a 128-row tile whose token rows tile_rows() gave into the
// UMMA canonical K-major layout with 128-byte (64-byte for d = 32) swizzle. Producer warp pw
// (0/1) copies tile rows [64*pw, 64*pw+64); 16 consecutive lanes cover one 256-byte row so
// every warp instruction reads whole rows.
template <int D>
__device__ __forceinline__ void load_tile_rows(uint32_t dst, const uint16_t* __restrict__ g,
                                               const TileRows& tr, int pw, int lane) {
    using C = TileGeom<D>;
    constexpr int CPR = D * 2 / 16;   // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;     // rows per warp instruction
    constexpr int NI = 64 / RPI;      // warp instructions per producer warp
    const int c = lane % CPR;
    const int rsub = lane / CPR;
    const uint32_t box = static_cast<uint32_t>((c * 16) / C::SW);
    const uint32_t cb = static_cast<uint32_t>(((c * 16) % C::SW) / 16);
#pragma unroll
    for (int k = 0; k < NI; ++k) {
        const int rl = k * RPI + rsub;  // 0..63
        const int grow = __shfl_sync(0xffffffffu, (k * RPI < 32) ? tr.ra : tr.rb, rl & 31);
        const int r = 64 * pw + rl;     // tile row 0..127
        const uint32_t sw = C::SW == 128 ? (cb ^ static_cast<uint32_t>(r & 7))
                                         : (cb ^ static_cast<uint32_t>((r >> 1) & 3));
        const uint32_t d = dst + box * C::BOX_BYTES + static_cast<uint32_t>(r) * C::SW + sw * 16u;
        cp_async_16(d, g + static_cast<size_t>(grow) * D + c * 8);
    }
}

// tile_rows + load_tile_rows for a tile loaded from one tensor only.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const uint16_t* __restrict__ g,
                                          const RowMap& rows, int first, int n_c, int pw, int lane,
                                          long long nrows, int* status) {
    load_tile_rows<D>(dst, g, tile_rows(rows, first, n_c, pw, lane, nrows, status), pw, lane);
}


}  // namespace skiparse
