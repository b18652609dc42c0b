// skiparse_internal.cuh -- geometry and launch parameters shared by the C-ABI host code and the
// sm_100a kernels of libskiparse.so.
//
// Geometry of Skiparse-2D (summary page of OSP-Next, sections 核心方法 and 方法步骤详情):
//   class of a spatial coordinate x along one axis:
//     token-wise  : x mod P                 (pixel-unshuffle-like)
//     group-wise  : (x div P) mod P         (patch-unshuffle-like)
//   position inside the class's sub-grid along that axis:
//     token-wise  : x div P
//     group-wise  : (x div P^2)*P + x mod P (each P-wide block stays together)
//   H and W are padded at the end to the next multiple of P^2 (any-resolution rule).
// Because the coordinate map is increasing in the sub-grid position, the real (unpadded)
// tokens of a class occupy a prefix [0, Rc) x [0, Sc) of its sub-grid; the kernels enumerate
// only those, so the pad-key mask reduces to the ragged tail of the last key tile.
//
// Skiparse-1D (the flattened-sequence variant the summary page's 技术新颖性 and 实验结果
// sections compare with) is the same one-axis rule on the in-frame index x = h*W + w with
// ratio P^2. The kernels therefore take the class count of each axis separately: Skiparse-2D
// runs on the (H, W) frame with (P, P) classes, Skiparse-1D on a (1, H*W) frame with
// (1, P^2) classes; the rearranged layouts, the row maps and the launch grids are the same.
#pragma once

#include <cstdint>

namespace skiparse {

// Debug build (SKIPARSE_DEBUG=1, libskiparse_debug.so): every token row index a kernel computes
// for a global load or store is checked against the row count of its tensor. An index outside
// is recorded as kErrBounds in the device status word and never used: a load reads row 0
// instead, a store is dropped. No access leaves its tensor, so the check cannot itself fault.
// Release builds compile the checks out.
#ifndef SKIPARSE_DEBUG
#define SKIPARSE_DEBUG 0
#endif

constexpr int kMaxP = 8;
constexpr int kMaxAxisClasses = kMaxP * kMaxP;  // Skiparse-1D: P^2 classes on one axis

// Spatial coordinate of sub-grid position `sub` of class `cls` along one axis.
__host__ __device__ __forceinline__ int axis_coord(int sub, int cls, int P, int mode) {
    return mode == 0 ? cls + P * sub : (sub / P) * P * P + cls * P + (sub % P);
}

// Class and sub-grid position of spatial coordinate x along one axis.
__host__ __device__ __forceinline__ void axis_class(int x, int P, int mode, int& cls, int& sub) {
    if (mode == 0) {
        cls = x % P;
        sub = x / P;
    } else {
        cls = (x / P) % P;
        sub = (x / (P * P)) * P + x % P;
    }
}

struct Geometry {
    int B, T, heads, d, P, mode;
    int H, W;          // frame axes the class rule runs on: (H, W), or (1, H*W) for Skiparse-1D
    int Ph, Pw;        // classes along each axis: (P, P), or (1, P^2) for Skiparse-1D
    int Hp, Wp;        // padded extents (multiples of Ph^2 and Pw^2)
    int R, S;          // padded sub-grid extents Hp/Ph, Wp/Pw
    long long n;       // padded subsequence length T*R*S
    int Rc[kMaxAxisClasses];  // real sub-grid rows of class row ci
    int Sc[kMaxAxisClasses];  // real sub-grid columns of class column cj
};

// Parameters of the fused attention kernel.
struct AttnParams {
    const uint16_t* q;             // bf16 bits, (B,T,H,W,heads,d)
    const uint16_t* k;
    const uint16_t* v;
    uint16_t* out;
    float* lse;                    // optional (nullptr): log-sum-exp of q.k/sqrt(d) per (token, head)
    int* status;                   // device error word
    int T, H, W, heads, Ph, Pw, mode;  // H, W, Ph, Pw as in Geometry
    int Rc[kMaxAxisClasses], Sc[kMaxAxisClasses];
    float scale_log2;              // log2(e)/sqrt(d)
    unsigned long long wait_limit_ns;
    int fault;                     // test hook: 1 = one producer never signals the first K tile
    long long nrows;               // (token, head) rows of q, k, v, out, lse: the debug bound
};

// Parameters of the backward kernels.
struct BwdParams {
    const uint16_t* q;             // bf16 bits, (B,T,H,W,heads,d)
    const uint16_t* k;
    const uint16_t* v;
    const uint16_t* out;           // the forward output O
    const uint16_t* dout;          // upstream gradient dO
    const float* lse;              // (B,T,H,W,heads) natural-log log-sum-exp from the forward
    float* delta;                  // (B,T,H,W,heads) D = rowsum(dO o O), written by the first launch
    uint16_t* dq;
    uint16_t* dk;
    uint16_t* dv;
    int* status;
    int T, H, W, heads, Ph, Pw, mode;  // H, W, Ph, Pw as in Geometry
    int Rc[kMaxAxisClasses], Sc[kMaxAxisClasses];
    float scale_log2;              // log2(e)/sqrt(d)
    float scale;                   // 1/sqrt(d)
    unsigned long long wait_limit_ns;
    long long nrows;               // (token, head) rows of every tensor above: the debug bound
    int fault;                     // test hook: 1 = one producer never signals the key-major
                                   // kernel's first streamed tile
};

struct RearrangeParams {
    const void* src;
    void* dst;
    int B, T, H, W, Ph, Pw, mode, R, S;  // H, W, Ph, Pw as in Geometry
    long long n;          // padded subsequence length
    int row_chunks;       // 16-byte chunks per token row (heads*d*2/16)
    long long nrows;      // rows to write: B*P*P*n (rearrange, switch) or B*T*H*W (unrearrange)
    long long src_rows;   // token rows of the source tensor: the debug bound
    int* status;          // device error word
};

// Status codes (mirror include/skiparse.h).
enum : int { kOk = 0, kErrLaunch = 4, kErrTimeout = 5, kErrBounds = 6 };

// The row index a global load may use: `row` itself, or (debug builds, row outside
// [0, nrows)) row 0 after recording kErrBounds.
__device__ __forceinline__ long long load_row(long long row, long long nrows, int* status) {
#if SKIPARSE_DEBUG
    if (row < 0 || row >= nrows) {
        atomicExch(status, kErrBounds);
        return 0;
    }
#endif
    return row;
}

// Whether a global access may use row index `row` (debug builds: false, after recording
// kErrBounds, when it lies outside [0, nrows)); the caller then skips the access.
__device__ __forceinline__ bool row_ok(long long row, long long nrows, int* status) {
#if SKIPARSE_DEBUG
    if (row < 0 || row >= nrows) {
        atomicExch(status, kErrBounds);
        return false;
    }
#endif
    return true;
}

// Launchers (defined in the kernel translation units). They return the cudaError_t as int.
int launch_attn_fwd(const AttnParams& p, const Geometry& g, void* stream);
int launch_attn_bwd(const BwdParams& p, const Geometry& g, void* stream);
int launch_rearrange(const RearrangeParams& p, int kind, void* stream);  // 0 fwd, 1 inverse, 2 switch
int attn_smem_bytes(int d);
int launch_exp2(const float* x, float* y, long long n, void* stream);
int launch_mma_rate(long long* clocks, int ctas, int pattern, int groups, unsigned long long wait_ns,
                    void* stream);
int launch_softmax_rate(long long* clocks, int ctas, int warps_per_subpartition, int reps, void* stream);

}  // namespace skiparse
