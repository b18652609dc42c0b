/*
 * skiparse_oracle.h -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU oracle for Skiparse-2D (and Skiparse-1D) sparse attention (OSP-Next). Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may call it. It
 * shares no code, header or constant with the CUDA library in fixed_pattern_sparse_b200/.
 *
 * Source of the method: the paper.rainbus.top summary of "OSP-Next: Efficient
 * High-Quality Video Generation with Sparse Sequence Parallelism, HiF8 Quantization,
 * and Reinforcement Learning" (arXiv 2605.28691), sections 核心方法 (core method) and
 * 方法步骤详情 (method step details); the chatpaper.ai page's English abstract.
 *
 * bf16 values are passed as their raw 16-bit patterns (uint16_t) and widened exactly.
 * Every function returns 0 on success and a negative number on a bad argument.
 */
#ifndef SKIPARSE_ORACLE_H
#define SKIPARSE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_TOKEN_WISE 0
#define ORACLE_GROUP_WISE 1

/* H or W padded up to the next multiple of P*P (the any-resolution rule). */
int oracle_padded_extent(int X, int P);

/* Class coordinate and sub-grid coordinate of one spatial index (a row h or column w). */
int oracle_axis_map(int x, int P, int mode, int* cls, int* sub);

/* Padded subsequence length n = T * (Hp/P) * (Wp/P). */
long long oracle_subseq_len(int T, int H, int W, int P);

/* x (B,T,H,W,heads,d) -> y (B*P*P, n, heads, d); pad slots are 0.
 * valid (B*P*P*n bytes, may be NULL) receives 1 for a real token and 0 for a pad slot. */
int oracle_rearrange(const uint16_t* x, uint16_t* y, uint8_t* valid,
                     int B, int T, int H, int W, int heads, int d, int P, int mode);

/* Inverse: y (B*P*P, n, heads, d) -> x (B,T,H,W,heads,d); pad slots are dropped. */
int oracle_unrearrange(const uint16_t* y, uint16_t* x,
                       int B, int T, int H, int W, int heads, int d, int P, int mode);
int oracle_unrearrange_f64(const double* y, double* x,
                           int B, int T, int H, int W, int heads, int d, int P, int mode);

/* Pattern switch: ysrc in src_mode's rearranged layout -> ydst in the other mode's rearranged
 * layout (both (B*P*P, n, heads, d)); pad slots of ydst are 0. */
int oracle_switch_mode(const uint16_t* ysrc, uint16_t* ydst,
                       int B, int T, int H, int W, int heads, int d, int P, int src_mode);

/* Dense softmax attention inside every subsequence, with the pad-key mask, in fp64.
 * yq/yk/yv (nseq, n, heads, d) bf16 bits, valid (nseq*n), yo (nseq, n, heads, d) fp64.
 * Pad-query rows of yo are left untouched. */
int oracle_masked_attention(const uint16_t* yq, const uint16_t* yk, const uint16_t* yv,
                            const uint8_t* valid, double* yo, long long nseq, long long n,
                            int heads, int d, int nthreads);

/* The whole forward pass: rearrange, masked attention, rearrange back.
 * q/k/v (B,T,H,W,heads,d) bf16 bits; out (B,T,H,W,heads,d) fp64. */
int oracle_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out,
                    int B, int T, int H, int W, int heads, int d, int P, int mode,
                    int nthreads);

/* The forward pass for selected output rows only. rows[i] = token * heads + head, where
 * token = ((b*T + t)*H + h)*W + w indexes the original layout; out_rows (nrows, d) fp64. */
int oracle_attn_fwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const long long* rows, long long nrows, double* out_rows,
                         int B, int T, int H, int W, int heads, int d, int P, int mode,
                         int nthreads);

/* Backward pass for an upstream gradient dout (all (B,T,H,W,heads,d) bf16 bits): dq, dk, dv
 * (B,T,H,W,heads,d) fp64; lse (B,T,H,W,heads) fp64, natural-log log-sum-exp of q.k/sqrt(d)
 * over each token's class (may be NULL). */
int oracle_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                    double* dq, double* dk, double* dv, double* lse,
                    int B, int T, int H, int W, int heads, int d, int P, int mode, int nthreads);

/* Backward for selected rows (token*heads + head): dq of the token as a query, dk and dv of
 * the token as a key; each output (nrows, d) fp64. */
int oracle_attn_bwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                         const long long* rows, long long nrows, double* dq_rows, double* dk_rows,
                         double* dv_rows, int B, int T, int H, int W, int heads, int d, int P,
                         int mode, int nthreads);

/* ---- Skiparse-1D (the 1D skip pattern on the flattened sequence; summary page sections
 * 技术新颖性 and 实验结果 compare it with Skiparse-2D but give no formula). Reading: the one-axis
 * rule above applied to the in-frame index x = h*W + w with ratio P^2 -- token-wise class
 * x mod P^2, group-wise class (x div P^2) mod P^2 -- and each frame's H*W positions padded at
 * the end to a multiple of P^4. The rearranged layout is (B*P*P, n, heads, d) with
 * n = T * Lp / P^2, subsequence b*P^2 + class, tokens in (t, position-in-class) order.
 * Arguments and return values as for the Skiparse-2D functions of the same name. */
int oracle1d_padded_length(int L, int P);
int oracle1d_index_map(int x, int P, int mode, int* cls, int* pos);
long long oracle1d_subseq_len(int T, int H, int W, int P);
int oracle1d_rearrange(const uint16_t* x, uint16_t* y, uint8_t* valid,
                       int B, int T, int H, int W, int heads, int d, int P, int mode);
int oracle1d_unrearrange(const uint16_t* y, uint16_t* x,
                         int B, int T, int H, int W, int heads, int d, int P, int mode);
int oracle1d_unrearrange_f64(const double* y, double* x,
                             int B, int T, int H, int W, int heads, int d, int P, int mode);
int oracle1d_switch_mode(const uint16_t* ysrc, uint16_t* ydst,
                         int B, int T, int H, int W, int heads, int d, int P, int src_mode);
int oracle1d_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out,
                      int B, int T, int H, int W, int heads, int d, int P, int mode,
                      int nthreads);
int oracle1d_attn_fwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const long long* rows, long long nrows, double* out_rows,
                           int B, int T, int H, int W, int heads, int d, int P, int mode,
                           int nthreads);
int oracle1d_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                      double* dq, double* dk, double* dv, double* lse,
                      int B, int T, int H, int W, int heads, int d, int P, int mode, int nthreads);
int oracle1d_attn_bwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* dout, const long long* rows, long long nrows,
                           double* dq_rows, double* dk_rows, double* dv_rows, int B, int T, int H,
                           int W, int heads, int d, int P, int mode, int nthreads);

#ifdef __cplusplus
}
#endif

#endif
