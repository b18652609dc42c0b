/*
 * skiparse_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow and deliberately obvious fp64 CPU restatement of Skiparse-2D sparse
 * attention. Only tests/, the smoke check and the benchmark's CPU-baseline leg use it;
 * it shares nothing with the CUDA library.
 *
 * Method source (cited per function below): the paper.rainbus.top summary of
 * "OSP-Next: Efficient High-Quality Video Generation with Sparse Sequence Parallelism,
 * HiF8 Quantization, and Reinforcement Learning", sections 核心方法 (core method) and
 * 方法步骤详情 (method step details), and the English abstract on the chatpaper.ai page.
 *
 * The pages' steps, in their order:
 *   1. rearrange the (B,T,H,W,C) tokens into P^2 subsequences of length N/P^2
 *      (token-wise: pixel-unshuffle-like; group-wise: patch-unshuffle-like),
 *      padding H and W up to the next multiple of P^2 and building an attention mask;
 *   2. run dense softmax attention inside each subsequence;
 *   3. rearrange the result back to the original layout.
 * Readings taken where the pages are silent (each is listed with its reason in the
 * design notes): group-wise class = ((h div P) mod P, (w div P) mod P); padding goes at
 * the bottom/right; rearranged layout (B*P^2, n, heads, d) with subsequence index
 * b*P^2 + ci*P + cj and tokens in (t, r, s) raster order; pad slots hold 0;
 * softmax scale 1/sqrt(d); no causal mask.
 * Skiparse-1D, the variant the pages compare against (技术新颖性, 实验结果), follows the same
 * three steps with the class rule on the flattened in-frame index (reading stated at
 * oracle1d_padded_length below).
 */
#include "skiparse_oracle.h"

/* Mutation hooks for the oracle's own tests (tests/test_oracle_mutants.py). A build with
 * ORACLE_MUTANT = k (1..8) plants plausible mistake k, one at a time, so that the test can
 * check that the pins catch every one of them; the normal build (0) plants none:
 *   1 group-wise sub-grid position x div P (blocks not kept together)
 *   2 group-wise class (x div P^2) mod P
 *   3 softmax scale 1 instead of 1/sqrt(d)
 *   4 exponent sign flipped, exp(m - s)
 *   5 padding to a multiple of P instead of P^2
 *   6 pad keys not masked (they take part in the softmax with zero vectors)
 *   7 Skiparse-1D frame flattened column-major (x = w*H + h instead of h*W + w)
 *   8 backward dS = P * dP (the D term dropped)                                          */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int check_shape(int B, int T, int H, int W, int heads, int d, int P, int mode) {
    if (B < 1 || T < 1 || H < 1 || W < 1 || heads < 1 || d < 1 || P < 1) return -1;
    if (mode != ORACLE_TOKEN_WISE && mode != ORACLE_GROUP_WISE) return -1;
    return 0;
}

/* Any-resolution rule (方法步骤详情): when H or W is not a multiple of P^2, pad it to
 * the nearest larger multiple. */
int oracle_padded_extent(int X, int P) {
    if (X < 1 || P < 1) return -1;
    int q = ORACLE_MUTANT == 5 ? P : P * P;
    return ((X + q - 1) / q) * q;
}

/* Class of one spatial coordinate and its position inside its class's sub-grid.
 * Token-wise (核心方法: like pixel unshuffle, the H x W map is cut into k x k sub-images,
 * each sub-image being one sequence): class = x mod P, sub-grid position = x div P.
 * Group-wise (核心方法: like patch unshuffle, tokens grouped by k x k blocks): the
 * block index x div P is distributed the token-wise way, so class = (x div P) mod P,
 * and each block keeps its P tokens together: sub-grid position = (x div P^2)*P + x mod P. */
int oracle_axis_map(int x, int P, int mode, int* cls, int* sub) {
    if (x < 0 || P < 1) return -1;
    if (mode == ORACLE_TOKEN_WISE) {
        *cls = x % P;
        *sub = x / P;
    } else if (mode == ORACLE_GROUP_WISE) {
        *cls = ORACLE_MUTANT == 2 ? (x / (P * P)) % P : (x / P) % P;
        *sub = ORACLE_MUTANT == 1 ? x / P : (x / (P * P)) * P + (x % P);
    } else {
        return -1;
    }
    return 0;
}

/* 方法步骤详情: each subsequence is 1/P^2 of the (padded) sequence. */
long long oracle_subseq_len(int T, int H, int W, int P) {
    int Hp = oracle_padded_extent(H, P), Wp = oracle_padded_extent(W, P);
    if (T < 1 || Hp < 0 || Wp < 0) return -1;
    return (long long)T * (Hp / P) * (Wp / P);
}

/* Skiparse-1D (技术新颖性 and 实验结果 on the summary page: the 1D skip pattern on the flattened
 * sequence, which Skiparse-2D applies to each spatial axis instead). The pages give no formula;
 * the reading taken here is the one-axis rule above on the flattened in-frame index
 * x = h*W + w with ratio P^2, so that there are P^2 subsequences as in Skiparse-2D:
 * token-wise class x mod P^2, group-wise class (x div P^2) mod P^2. Each frame's H*W
 * positions are padded at the end to the next multiple of P^4 (the one-axis any-resolution
 * rule with ratio P^2). */
int oracle1d_padded_length(int L, int P) {
    if (L < 1 || P < 1) return -1;
    return oracle_padded_extent(L, P * P);
}

int oracle1d_index_map(int x, int P, int mode, int* cls, int* pos) {
    if (P < 1) return -1;
    return oracle_axis_map(x, P * P, mode, cls, pos);
}

long long oracle1d_subseq_len(int T, int H, int W, int P) {
    if (T < 1 || H < 1 || W < 1 || P < 1) return -1;
    const int Lp = oracle1d_padded_length(H * W, P);
    return (long long)T * (Lp / (P * P));
}

/* ---- where every padded position goes ------------------------------------------
 * Both patterns cut each frame's padded positions f in [0, F) into P^2 classes. The
 * rearranged layout is (B*P^2, n, heads, d): subsequence b*P^2 + class, and inside it the
 * tokens of the class in frame order t, then in the order of their position in the class. */
typedef struct {
    int dims;             /* 2: Skiparse-2D; 1: Skiparse-1D */
    int B, T, H, W, heads, d, P, mode;
    long long F;          /* padded positions per frame */
    long long n;          /* subsequence length */
    int Hp, Wp, R, S;     /* Skiparse-2D: padded extents and sub-grid extents Hp/P, Wp/P */
} pattern;

static int pattern_init(pattern* pt, int dims, int B, int T, int H, int W, int heads, int d,
                        int P, int mode) {
    if (check_shape(B, T, H, W, heads, d, P, mode)) return -1;
    if (dims != 1 && dims != 2) return -1;
    memset(pt, 0, sizeof *pt);
    pt->dims = dims;
    pt->B = B; pt->T = T; pt->H = H; pt->W = W; pt->heads = heads; pt->d = d;
    pt->P = P; pt->mode = mode;
    if (dims == 2) {
        pt->Hp = oracle_padded_extent(H, P);
        pt->Wp = oracle_padded_extent(W, P);
        pt->R = pt->Hp / P;
        pt->S = pt->Wp / P;
        pt->F = (long long)pt->Hp * pt->Wp;
        pt->n = oracle_subseq_len(T, H, W, P);
    } else {
        pt->F = oracle1d_padded_length(H * W, P);
        pt->n = oracle1d_subseq_len(T, H, W, P);
    }
    return 0;
}

/* Slot of padded position f of frame t of batch element b: subsequence *seq, position *pos.
 * Returns 1 for a real token (then *tok is its index ((b*T + t)*H + h)*W + w in the original
 * layout), 0 for a pad slot, and -1 if the slot falls outside the rearranged tensor (never
 * for this oracle; it keeps the builds with a planted mistake from writing out of bounds). Skiparse-2D: f = h*Wp + w, class (ci, cj) from the two axis
 * maps, subsequence b*P^2 + ci*P + cj, position (t, r, s) in raster order. Skiparse-1D:
 * f = x = h*W + w, class c from the flattened-index map, subsequence b*P^2 + c, position
 * t*(F/P^2) + the position inside the class. */
static int pattern_slot(const pattern* pt, int b, int t, long long f, long long* seq,
                        long long* pos, long long* tok) {
    const long long q2 = (long long)pt->P * pt->P;
    if (pt->dims == 2) {
        const int h = (int)(f / pt->Wp), w = (int)(f % pt->Wp);
        int ci, r, cj, s;
        oracle_axis_map(h, pt->P, pt->mode, &ci, &r);
        oracle_axis_map(w, pt->P, pt->mode, &cj, &s);
        *seq = (long long)b * q2 + ci * pt->P + cj;
        *pos = ((long long)t * pt->R + r) * pt->S + s;
        if (*seq < 0 || *seq >= (long long)pt->B * q2 || *pos < 0 || *pos >= pt->n) return -1;
        if (h >= pt->H || w >= pt->W) return 0;
        *tok = (((long long)b * pt->T + t) * pt->H + h) * pt->W + w;
        return 1;
    }
    int c, s;
    oracle1d_index_map((int)f, pt->P, pt->mode, &c, &s);
    *seq = (long long)b * q2 + c;
    *pos = (long long)t * (pt->F / q2) + s;
    if (*seq < 0 || *seq >= (long long)pt->B * q2 || *pos < 0 || *pos >= pt->n) return -1;
    if (f >= (long long)pt->H * pt->W) return 0;
    const long long x = ORACLE_MUTANT == 7 ? (f % pt->H) * pt->W + f / pt->H : f;
    *tok = ((long long)b * pt->T + t) * ((long long)pt->H * pt->W) + x;
    return 1;
}

/* Batch element, frame and padded position of token `tok` of the original layout. */
static void pattern_locate(const pattern* pt, long long tok, int* b, int* t, long long* f) {
    const long long hw = (long long)pt->H * pt->W;
    const long long x = tok % hw;
    *t = (int)((tok / hw) % pt->T);
    *b = (int)(tok / (hw * pt->T));
    *f = pt->dims == 2 ? (x / pt->W) * pt->Wp + x % pt->W : x;
}

/* Step 1 (方法步骤详情): rearrange into P^2 subsequences, pad, and record the mask. */
static void rearrange_impl(const pattern* pt, const uint16_t* x, uint16_t* y, uint8_t* valid) {
    const long long row = (long long)pt->heads * pt->d;
    for (int b = 0; b < pt->B; ++b)
        for (int t = 0; t < pt->T; ++t)
            for (long long f = 0; f < pt->F; ++f) {
                long long seq, pos, tok = 0;
                const int real = pattern_slot(pt, b, t, f, &seq, &pos, &tok);
                if (real < 0) continue;
                uint16_t* dst = y + (seq * pt->n + pos) * row;
                for (long long e = 0; e < row; ++e) dst[e] = real ? x[tok * row + e] : 0;
                if (valid) valid[seq * pt->n + pos] = (uint8_t)real;
            }
}

/* Step 3 (方法步骤详情: rearrange back to the original layout), real tokens only. */
static void unrearrange_impl(const pattern* pt, const void* y, void* x, int elem_bytes,
                             long long row) {
    for (int b = 0; b < pt->B; ++b)
        for (int t = 0; t < pt->T; ++t)
            for (long long f = 0; f < pt->F; ++f) {
                long long seq, pos, tok = 0;
                if (pattern_slot(pt, b, t, f, &seq, &pos, &tok) != 1) continue;
                memcpy((char*)x + tok * row * elem_bytes,
                       (const char*)y + (seq * pt->n + pos) * row * elem_bytes,
                       (size_t)(row * elem_bytes));
            }
}

/* Pattern switch between layers (核心方法: token-wise and group-wise alternate between layers;
 * 方法步骤详情: under SSP a switch is a local rearrange plus one exchange). The local step: a
 * tensor in the source mode's rearranged layout goes straight to the other mode's rearranged
 * layout; every real token row moves from its source slot to its destination slot, pad slots
 * of the result are 0. */
static void switch_impl(const pattern* src, const pattern* dst, const uint16_t* ysrc,
                        uint16_t* ydst) {
    const long long row = (long long)src->heads * src->d;
    for (int b = 0; b < dst->B; ++b)
        for (int t = 0; t < dst->T; ++t)
            for (long long f = 0; f < dst->F; ++f) {
                long long dseq, dpos, sseq, spos, tok = 0;
                const int real = pattern_slot(dst, b, t, f, &dseq, &dpos, &tok);
                if (real < 0) continue;
                uint16_t* out = ydst + (dseq * dst->n + dpos) * row;
                if (real && pattern_slot(src, b, t, f, &sseq, &spos, &tok) == 1) {
                    for (long long e = 0; e < row; ++e) out[e] = ysrc[(sseq * src->n + spos) * row + e];
                } else {
                    for (long long e = 0; e < row; ++e) out[e] = 0;
                }
            }
}

int oracle_rearrange(const uint16_t* x, uint16_t* y, uint8_t* valid,
                     int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    rearrange_impl(&pt, x, y, valid);
    return 0;
}

int oracle1d_rearrange(const uint16_t* x, uint16_t* y, uint8_t* valid,
                       int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    rearrange_impl(&pt, x, y, valid);
    return 0;
}

int oracle_unrearrange(const uint16_t* y, uint16_t* x,
                       int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    unrearrange_impl(&pt, y, x, 2, (long long)heads * d);
    return 0;
}

int oracle1d_unrearrange(const uint16_t* y, uint16_t* x,
                         int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    unrearrange_impl(&pt, y, x, 2, (long long)heads * d);
    return 0;
}

int oracle_unrearrange_f64(const double* y, double* x,
                           int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    unrearrange_impl(&pt, y, x, 8, (long long)heads * d);
    return 0;
}

int oracle1d_unrearrange_f64(const double* y, double* x,
                             int B, int T, int H, int W, int heads, int d, int P, int mode) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    unrearrange_impl(&pt, y, x, 8, (long long)heads * d);
    return 0;
}

static int switch_dims(int dims, const uint16_t* ysrc, uint16_t* ydst, int B, int T, int H,
                       int W, int heads, int d, int P, int src_mode) {
    pattern src, dst;
    if (pattern_init(&src, dims, B, T, H, W, heads, d, P, src_mode)) return -1;
    if (pattern_init(&dst, dims, B, T, H, W, heads, d, P, 1 - src_mode)) return -1;
    switch_impl(&src, &dst, ysrc, ydst);
    return 0;
}

int oracle_switch_mode(const uint16_t* ysrc, uint16_t* ydst,
                       int B, int T, int H, int W, int heads, int d, int P, int src_mode) {
    return switch_dims(2, ysrc, ydst, B, T, H, W, heads, d, P, src_mode);
}

int oracle1d_switch_mode(const uint16_t* ysrc, uint16_t* ydst,
                         int B, int T, int H, int W, int heads, int d, int P, int src_mode) {
    return switch_dims(1, ysrc, ydst, B, T, H, W, heads, d, P, src_mode);
}

/* Step 2: dense softmax attention of one query row over the real keys of its own
 * subsequence (核心方法: each subsequence attends densely, which is why FlashAttention
 * runs natively; 方法步骤详情: padded keys are removed by the attention mask).
 * o = sum_j exp(s_j - m) v_j / sum_j exp(s_j - m), s_j = q.k_j / sqrt(d), m = max_j s_j. */
static void attend_one(const uint16_t* yq, const uint16_t* yk, const uint16_t* yv,
                       const uint8_t* valid, long long n, int heads, int d,
                       long long seq, long long i, int head, double* o, double* score) {
    const long long row = (long long)heads * d;
    const uint16_t* q = yq + ((seq * n + i) * heads + head) * d;
    const double scale = ORACLE_MUTANT == 3 ? 1.0 : 1.0 / sqrt((double)d);
    double m = -INFINITY;
    for (long long j = 0; j < n; ++j) {
        if (!valid[seq * n + j] && ORACLE_MUTANT != 6) continue;
        const uint16_t* kj = yk + (seq * n + j) * row + (long long)head * d;
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += bf16_bits_to_double(q[e]) * bf16_bits_to_double(kj[e]);
        score[j] = acc * scale;
        if (score[j] > m) m = score[j];
    }
    double denom = 0.0;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (long long j = 0; j < n; ++j) {
        if (!valid[seq * n + j] && ORACLE_MUTANT != 6) continue;
        const double p = ORACLE_MUTANT == 4 ? exp(m - score[j]) : exp(score[j] - m);
        denom += p;
        const uint16_t* vj = yv + (seq * n + j) * row + (long long)head * d;
        for (int e = 0; e < d; ++e) o[e] += p * bf16_bits_to_double(vj[e]);
    }
    for (int e = 0; e < d; ++e) o[e] /= denom;
}

/* ---- thread fan-out over independent query rows ------------------------------- */

typedef struct {
    const uint16_t *yq, *yk, *yv;
    const uint8_t* valid;
    long long n;
    int heads, d;
    /* work list: either all (seq, i, head) units, or an explicit unit list */
    long long nunits;
    const long long* units;  /* (seq*n + i)*heads + head, or NULL for "unit = index" */
    double* out;             /* indexed by unit (units == NULL) or by list position */
    int tid, nthreads;
} attn_job;

static void* attn_worker(void* arg) {
    attn_job* jb = (attn_job*)arg;
    double* score = (double*)malloc(sizeof(double) * (size_t)(jb->n > 0 ? jb->n : 1));
    if (!score) return (void*)1;
    for (long long u = jb->tid; u < jb->nunits; u += jb->nthreads) {
        const long long unit = jb->units ? jb->units[u] : u;
        const int head = (int)(unit % jb->heads);
        const long long tokslot = unit / jb->heads;
        const long long seq = tokslot / jb->n, i = tokslot % jb->n;
        if (!jb->valid[seq * jb->n + i]) continue;  /* pad queries produce no output */
        double* o = jb->out + (jb->units ? u : unit) * (long long)jb->d;
        attend_one(jb->yq, jb->yk, jb->yv, jb->valid, jb->n, jb->heads, jb->d, seq, i, head,
                   o, score);
    }
    free(score);
    return NULL;
}

static int run_attention(attn_job proto, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    attn_job* jobs = (attn_job*)malloc(sizeof(attn_job) * (size_t)nthreads);
    if (!th || !jobs) { free(th); free(jobs); return -2; }
    int rc = 0, started = 0;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].tid = t;
        jobs[t].nthreads = nthreads;
        if (pthread_create(&th[t], NULL, attn_worker, &jobs[t]) != 0) { rc = -3; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = -2;
    }
    free(th);
    free(jobs);
    return rc;
}

int oracle_masked_attention(const uint16_t* yq, const uint16_t* yk, const uint16_t* yv,
                            const uint8_t* valid, double* yo, long long nseq, long long n,
                            int heads, int d, int nthreads) {
    if (nseq < 1 || n < 1 || heads < 1 || d < 1) return -1;
    attn_job jb;
    memset(&jb, 0, sizeof jb);
    jb.yq = yq; jb.yk = yk; jb.yv = yv; jb.valid = valid;
    jb.n = n; jb.heads = heads; jb.d = d;
    jb.nunits = nseq * n * heads;
    jb.units = NULL;
    jb.out = yo;
    return run_attention(jb, nthreads);
}

typedef struct {
    uint16_t *yq, *yk, *yv;
    uint8_t* valid;
} rearranged;

static void free_rearranged(rearranged* r) {
    free(r->yq); free(r->yk); free(r->yv); free(r->valid);
}

static int rearrange_all(const pattern* pt, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, rearranged* r) {
    const long long nseq = (long long)pt->B * pt->P * pt->P;
    const size_t elems = (size_t)(nseq * pt->n * pt->heads * pt->d);
    memset(r, 0, sizeof *r);
    r->yq = (uint16_t*)malloc(elems * 2);
    r->yk = (uint16_t*)malloc(elems * 2);
    r->yv = (uint16_t*)malloc(elems * 2);
    r->valid = (uint8_t*)malloc((size_t)(nseq * pt->n));
    if (!r->yq || !r->yk || !r->yv || !r->valid) { free_rearranged(r); return -2; }
    rearrange_impl(pt, q, r->yq, r->valid);
    rearrange_impl(pt, k, r->yk, NULL);
    rearrange_impl(pt, v, r->yv, NULL);
    return 0;
}

static int attn_fwd_impl(const pattern* pt, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, double* out, int nthreads) {
    rearranged r;
    int rc = rearrange_all(pt, q, k, v, &r);
    if (rc) return rc;
    const long long nseq = (long long)pt->B * pt->P * pt->P;
    double* yo = (double*)calloc((size_t)(nseq * pt->n * pt->heads * pt->d), sizeof(double));
    if (!yo) { free_rearranged(&r); return -2; }
    rc = oracle_masked_attention(r.yq, r.yk, r.yv, r.valid, yo, nseq, pt->n, pt->heads, pt->d,
                                 nthreads);
    if (!rc) unrearrange_impl(pt, yo, out, 8, (long long)pt->heads * pt->d);
    free(yo);
    free_rearranged(&r);
    return rc;
}

int oracle_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out,
                    int B, int T, int H, int W, int heads, int d, int P, int mode,
                    int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_fwd_impl(&pt, q, k, v, out, nthreads);
}

int oracle1d_attn_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* out,
                      int B, int T, int H, int W, int heads, int d, int P, int mode,
                      int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_fwd_impl(&pt, q, k, v, out, nthreads);
}

/* The forward pass for selected output rows. The pages' three steps restricted to what
 * those rows need: for every (subsequence, head) that holds a requested query, the rearrange
 * of step 1 is run for that one subsequence and head (same index loops and pad mask as
 * oracle_rearrange), step 2 attends each requested query over it, and step 3 writes the
 * result to the requested row's slot of out_rows. */
typedef struct {
    const uint16_t *sq, *sk, *sv;   /* one subsequence, one head: (n, d) */
    const uint8_t* valid;
    long long n;
    int d;
    const long long* pos;           /* query positions inside the subsequence */
    const long long* slot;          /* where each result goes in out_rows */
    long long count;
    double* out;
    int tid, nthreads;
} rows_job;

static void* rows_worker(void* arg) {
    rows_job* jb = (rows_job*)arg;
    double* score = (double*)malloc(sizeof(double) * (size_t)jb->n);
    if (!score) return (void*)1;
    for (long long u = jb->tid; u < jb->count; u += jb->nthreads) {
        /* heads = 1 view: the gathered buffers hold only this head */
        attend_one(jb->sq, jb->sk, jb->sv, jb->valid, jb->n, 1, jb->d, 0, jb->pos[u], 0,
                   jb->out + jb->slot[u] * (long long)jb->d, score);
    }
    free(score);
    return NULL;
}

static int cmp_ll(const void* a, const void* b) {
    const long long x = *(const long long*)a, y = *(const long long*)b;
    return x < y ? -1 : x > y;
}

/* Sort key of each requested row: ((subsequence*heads + head) * n + position), with the
 * request's index beside it, so that the requests of one (subsequence, head) are adjacent. */
static long long* request_keys(const pattern* pt, const long long* rows, long long nrows) {
    long long* key = (long long*)malloc(sizeof(long long) * (size_t)nrows * 2);
    if (!key) return NULL;
    for (long long i = 0; i < nrows; ++i) {
        const int head = (int)(rows[i] % pt->heads);
        int b, t;
        long long f, seq, pos, tok;
        pattern_locate(pt, rows[i] / pt->heads, &b, &t, &f);
        if (pattern_slot(pt, b, t, f, &seq, &pos, &tok) < 0) seq = pos = 0;
        key[2 * i] = (seq * pt->heads + head) * pt->n + pos;
        key[2 * i + 1] = i;
    }
    qsort(key, (size_t)nrows, 2 * sizeof(long long), cmp_ll);
    return key;
}

/* Step 1 for one subsequence and one head: the same slot rule as rearrange_impl, keeping only
 * the slots of subsequence `seq`. Any of the destination buffers may be NULL. */
static void gather_subseq(const pattern* pt, long long seq, int head, const uint16_t* const* src,
                          uint16_t* const* dst, int nbuf, uint8_t* valid) {
    const long long q2 = (long long)pt->P * pt->P;
    const int b = (int)(seq / q2);
    const int d = pt->d;
    for (int t = 0; t < pt->T; ++t)
        for (long long f = 0; f < pt->F; ++f) {
            long long s, p, tok = 0;
            const int real = pattern_slot(pt, b, t, f, &s, &p, &tok);
            if (real < 0 || s != seq) continue;
            valid[p] = (uint8_t)real;
            const long long srow = tok * pt->heads + head;
            for (int i = 0; i < nbuf; ++i)
                for (int e = 0; e < d; ++e) dst[i][p * d + e] = real ? src[i][srow * d + e] : 0;
        }
}

static int check_rows(const pattern* pt, const long long* rows, long long nrows) {
    const long long ntok = (long long)pt->B * pt->T * pt->H * pt->W;
    if (nrows < 0) return -1;
    for (long long i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= ntok * pt->heads) return -1;
    return 0;
}

static int attn_fwd_rows_impl(const pattern* pt, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const long long* rows, long long nrows,
                              double* out_rows, int nthreads) {
    if (check_rows(pt, rows, nrows)) return -1;
    if (nrows == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    const long long n = pt->n;
    const int heads = pt->heads, d = pt->d;
    long long* key = request_keys(pt, rows, nrows);
    if (!key) return -2;
    uint16_t* sq = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint16_t* sk = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint16_t* sv = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint8_t* valid = (uint8_t*)malloc((size_t)n);
    long long* pos = (long long*)malloc(sizeof(long long) * (size_t)nrows);
    long long* slot = (long long*)malloc(sizeof(long long) * (size_t)nrows);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    rows_job* jobs = (rows_job*)malloc(sizeof(rows_job) * (size_t)nthreads);
    int rc = 0;
    if (!sq || !sk || !sv || !valid || !pos || !slot || !th || !jobs) rc = -2;
    for (long long g0 = 0; rc == 0 && g0 < nrows;) {
        const long long group = key[2 * g0] / n;  /* seq*heads + head */
        long long g1 = g0;
        while (g1 < nrows && key[2 * g1] / n == group) {
            pos[g1 - g0] = key[2 * g1] % n;
            slot[g1 - g0] = key[2 * g1 + 1];
            ++g1;
        }
        const uint16_t* src[3] = {q, k, v};
        uint16_t* dst[3] = {sq, sk, sv};
        gather_subseq(pt, group / heads, (int)(group % heads), src, dst, 3, valid);
        /* step 2 for the requested queries, step 3 by writing to their slots */
        int started = 0;
        for (int t = 0; t < nthreads; ++t) {
            rows_job* jb = &jobs[t];
            jb->sq = sq; jb->sk = sk; jb->sv = sv; jb->valid = valid;
            jb->n = n; jb->d = d; jb->pos = pos; jb->slot = slot; jb->count = g1 - g0;
            jb->out = out_rows; jb->tid = t; jb->nthreads = nthreads;
            if (pthread_create(&th[t], NULL, rows_worker, jb) != 0) { rc = -3; break; }
            ++started;
        }
        for (int t = 0; t < started; ++t) {
            void* ret = NULL;
            pthread_join(th[t], &ret);
            if (ret) rc = -2;
        }
        g0 = g1;
    }
    free(key); free(sq); free(sk); free(sv); free(valid); free(pos); free(slot); free(th); free(jobs);
    return rc;
}

int oracle_attn_fwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const long long* rows, long long nrows, double* out_rows,
                         int B, int T, int H, int W, int heads, int d, int P, int mode,
                         int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_fwd_rows_impl(&pt, q, k, v, rows, nrows, out_rows, nthreads);
}

int oracle1d_attn_fwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const long long* rows, long long nrows, double* out_rows,
                           int B, int T, int H, int W, int heads, int d, int P, int mode,
                           int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_fwd_rows_impl(&pt, q, k, v, rows, nrows, out_rows, nthreads);
}


/* ------------------------------------------------------------------ backward pass
 * Gradients of the Skiparse-2D forward for an upstream gradient dO, by the definition of
 * softmax attention inside each subsequence (the same three steps as the forward: rearrange
 * with the pad mask, per-subsequence dense attention -- here its derivative -- and rearrange
 * back). With s_ij = q_i.k_j, L_i = log sum_j exp(s_ij/sqrt(d)), P_ij = exp(s_ij/sqrt(d) - L_i),
 * O_i = sum_j P_ij v_j, D_i = dO_i.O_i:
 *   dV_j = sum_i P_ij dO_i,  dP_ij = dO_i.v_j,  dS_ij = P_ij (dP_ij - D_i),
 *   dQ_i = sum_j dS_ij k_j / sqrt(d),  dK_j = sum_i dS_ij q_i / sqrt(d).               */

typedef struct {
    const uint16_t *yq, *yk, *yv, *ydo;
    const uint8_t* valid;
    double *ydq, *ydk, *ydv, *ylse;   /* (nseq, n, heads, d) / (nseq, n, heads) */
    long long nseq, n;
    int heads, d;
    int tid, nthreads;
} bwd_job;

static void* bwd_worker(void* arg) {
    bwd_job* jb = (bwd_job*)arg;
    const long long n = jb->n;
    const int d = jb->d, heads = jb->heads;
    const long long row = (long long)heads * d;
    const double scale = 1.0 / sqrt((double)d);
    double* p = (double*)malloc(sizeof(double) * (size_t)n);
    double* dp = (double*)malloc(sizeof(double) * (size_t)n);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    if (!p || !dp || !o) { free(p); free(dp); free(o); return (void*)1; }
    for (long long unit = jb->tid; unit < jb->nseq * heads; unit += jb->nthreads) {
        const long long seq = unit / heads;
        const int head = (int)(unit % heads);
        #define AT(buf, j) ((buf) + (seq * n + (j)) * row + (long long)head * d)
        for (long long i = 0; i < n; ++i) {
            if (!jb->valid[seq * n + i]) continue;
            const uint16_t* qi = AT(jb->yq, i);
            const uint16_t* doi = AT(jb->ydo, i);
            double m = -INFINITY;
            for (long long j = 0; j < n; ++j) {
                if (!jb->valid[seq * n + j]) continue;
                const uint16_t* kj = AT(jb->yk, j);
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += bf16_bits_to_double(qi[e]) * bf16_bits_to_double(kj[e]);
                p[j] = acc * scale;
                if (p[j] > m) m = p[j];
            }
            double sum = 0.0;
            for (long long j = 0; j < n; ++j)
                if (jb->valid[seq * n + j]) sum += exp(p[j] - m);
            const double lse = m + log(sum);
            if (jb->ylse) jb->ylse[(seq * n + i) * heads + head] = lse;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (long long j = 0; j < n; ++j) {
                if (!jb->valid[seq * n + j]) continue;
                p[j] = exp(p[j] - lse);
                const uint16_t* vj = AT(jb->yv, j);
                for (int e = 0; e < d; ++e) o[e] += p[j] * bf16_bits_to_double(vj[e]);
            }
            double D = 0.0;
            for (int e = 0; e < d; ++e) D += bf16_bits_to_double(doi[e]) * o[e];
            double* dqi = jb->ydq + (seq * n + i) * row + (long long)head * d;
            for (long long j = 0; j < n; ++j) {
                if (!jb->valid[seq * n + j]) continue;
                const uint16_t* vj = AT(jb->yv, j);
                const uint16_t* kj = AT(jb->yk, j);
                double dpv = 0.0;
                for (int e = 0; e < d; ++e) dpv += bf16_bits_to_double(doi[e]) * bf16_bits_to_double(vj[e]);
                const double ds = ORACLE_MUTANT == 8 ? p[j] * dpv : p[j] * (dpv - D);
                double* dvj = jb->ydv + (seq * n + j) * row + (long long)head * d;
                double* dkj = jb->ydk + (seq * n + j) * row + (long long)head * d;
                for (int e = 0; e < d; ++e) {
                    dvj[e] += p[j] * bf16_bits_to_double(doi[e]);
                    dkj[e] += ds * bf16_bits_to_double(qi[e]) * scale;
                    dqi[e] += ds * bf16_bits_to_double(kj[e]) * scale;
                }
            }
        }
        #undef AT
    }
    free(p); free(dp); free(o);
    return NULL;
}

static int attn_bwd_impl(const pattern* pt, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const uint16_t* dout, double* dq, double* dk,
                         double* dv, double* lse, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    rearranged r;
    int rc = rearrange_all(pt, q, k, v, &r);
    if (rc) return rc;
    const long long n = pt->n;
    const int heads = pt->heads, d = pt->d;
    const long long nseq = (long long)pt->B * pt->P * pt->P;
    const size_t elems = (size_t)(nseq * n * heads * d);
    uint16_t* ydo = (uint16_t*)malloc(elems * 2);
    double* ydq = (double*)calloc(elems, sizeof(double));
    double* ydk = (double*)calloc(elems, sizeof(double));
    double* ydv = (double*)calloc(elems, sizeof(double));
    double* ylse = lse ? (double*)calloc((size_t)(nseq * n * heads), sizeof(double)) : NULL;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    bwd_job* jobs = (bwd_job*)malloc(sizeof(bwd_job) * (size_t)nthreads);
    if (!ydo || !ydq || !ydk || !ydv || (lse && !ylse) || !th || !jobs) rc = -2;
    if (!rc) {
        rearrange_impl(pt, dout, ydo, NULL);
        int started = 0;
        for (int t = 0; t < nthreads; ++t) {
            bwd_job* jb = &jobs[t];
            jb->yq = r.yq; jb->yk = r.yk; jb->yv = r.yv; jb->ydo = ydo; jb->valid = r.valid;
            jb->ydq = ydq; jb->ydk = ydk; jb->ydv = ydv; jb->ylse = ylse;
            jb->nseq = nseq; jb->n = n; jb->heads = heads; jb->d = d;
            jb->tid = t; jb->nthreads = nthreads;
            if (pthread_create(&th[t], NULL, bwd_worker, jb) != 0) { rc = -3; break; }
            ++started;
        }
        for (int t = 0; t < started; ++t) {
            void* ret = NULL;
            pthread_join(th[t], &ret);
            if (ret) rc = -2;
        }
    }
    if (!rc) {
        const long long row = (long long)heads * d;
        unrearrange_impl(pt, ydq, dq, 8, row);
        unrearrange_impl(pt, ydk, dk, 8, row);
        unrearrange_impl(pt, ydv, dv, 8, row);
        if (lse) unrearrange_impl(pt, ylse, lse, 8, heads);
    }
    free(ydo); free(ydq); free(ydk); free(ydv); free(ylse); free(th); free(jobs);
    free_rearranged(&r);
    return rc;
}

int oracle_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                    double* dq, double* dk, double* dv, double* lse,
                    int B, int T, int H, int W, int heads, int d, int P, int mode, int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_bwd_impl(&pt, q, k, v, dout, dq, dk, dv, lse, nthreads);
}

int oracle1d_attn_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                      double* dq, double* dk, double* dv, double* lse,
                      int B, int T, int H, int W, int heads, int d, int P, int mode, int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_bwd_impl(&pt, q, k, v, dout, dq, dk, dv, lse, nthreads);
}

/* Gradients for selected rows (token*heads + head of the original layout): dq of the token as
 * a query, dk and dv of the token as a key. Per (subsequence, head) holding a requested row:
 * the subsequence is gathered as in oracle_attn_fwd_rows, L_i and D_i are computed for all of
 * its queries, then each requested row's gradients follow from the formulas above. */
typedef struct {
    const uint16_t *sq, *sk, *sv, *sdo;   /* one subsequence, one head: (n, d) */
    const uint8_t* valid;
    long long n;
    int d;
    double *L, *Dl;                       /* (n) */
    const long long* pos; const long long* slot; long long count;
    double *dq, *dk, *dv;                 /* requested rows (nrows, d) */
    int phase;                            /* 0: L and D for every query; 1: requested rows */
    int tid, nthreads;
} bwdrows_job;

static double dotbf(const uint16_t* a, const uint16_t* b, int d) {
    double acc = 0.0;
    for (int e = 0; e < d; ++e) acc += bf16_bits_to_double(a[e]) * bf16_bits_to_double(b[e]);
    return acc;
}

static void* bwdrows_worker(void* arg) {
    bwdrows_job* jb = (bwdrows_job*)arg;
    const long long n = jb->n;
    const int d = jb->d;
    const double scale = 1.0 / sqrt((double)d);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    double* sc = (double*)malloc(sizeof(double) * (size_t)n);
    if (!o || !sc) { free(o); free(sc); return (void*)1; }
    if (jb->phase == 0) {
        for (long long i = jb->tid; i < n; i += jb->nthreads) {
            if (!jb->valid[i]) continue;
            double m = -INFINITY;
            for (long long j = 0; j < n; ++j) {
                if (!jb->valid[j]) continue;
                sc[j] = dotbf(jb->sq + i * d, jb->sk + j * d, d) * scale;
                if (sc[j] > m) m = sc[j];
            }
            double sum = 0.0;
            for (long long j = 0; j < n; ++j) if (jb->valid[j]) sum += exp(sc[j] - m);
            const double L = m + log(sum);
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (long long j = 0; j < n; ++j) {
                if (!jb->valid[j]) continue;
                const double pij = exp(sc[j] - L);
                for (int e = 0; e < d; ++e) o[e] += pij * bf16_bits_to_double(jb->sv[j * d + e]);
            }
            double D = 0.0;
            for (int e = 0; e < d; ++e) D += bf16_bits_to_double(jb->sdo[i * d + e]) * o[e];
            jb->L[i] = L;
            jb->Dl[i] = D;
        }
    } else {
        for (long long u = jb->tid; u < jb->count; u += jb->nthreads) {
            const long long x = jb->pos[u];
            double* dq = jb->dq + jb->slot[u] * (long long)d;
            double* dk = jb->dk + jb->slot[u] * (long long)d;
            double* dv = jb->dv + jb->slot[u] * (long long)d;
            for (int e = 0; e < d; ++e) { dq[e] = 0.0; dk[e] = 0.0; dv[e] = 0.0; }
            if (!jb->valid[x]) continue;
            for (long long j = 0; j < n; ++j) {          /* x as the query */
                if (!jb->valid[j]) continue;
                const double pxj = exp(dotbf(jb->sq + x * d, jb->sk + j * d, d) * scale - jb->L[x]);
                const double ds = pxj * (dotbf(jb->sdo + x * d, jb->sv + j * d, d) - jb->Dl[x]);
                for (int e = 0; e < d; ++e) dq[e] += ds * bf16_bits_to_double(jb->sk[j * d + e]) * scale;
            }
            for (long long i = 0; i < n; ++i) {          /* x as the key */
                if (!jb->valid[i]) continue;
                const double pix = exp(dotbf(jb->sq + i * d, jb->sk + x * d, d) * scale - jb->L[i]);
                const double ds = pix * (dotbf(jb->sdo + i * d, jb->sv + x * d, d) - jb->Dl[i]);
                for (int e = 0; e < d; ++e) {
                    dk[e] += ds * bf16_bits_to_double(jb->sq[i * d + e]) * scale;
                    dv[e] += pix * bf16_bits_to_double(jb->sdo[i * d + e]);
                }
            }
        }
    }
    free(o); free(sc);
    return NULL;
}

static int run_bwdrows(bwdrows_job proto, int nthreads, int phase) {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    bwdrows_job* jobs = (bwdrows_job*)malloc(sizeof(bwdrows_job) * (size_t)nthreads);
    int rc = 0, started = 0;
    if (!th || !jobs) { free(th); free(jobs); return -2; }
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].phase = phase; jobs[t].tid = t; jobs[t].nthreads = nthreads;
        if (pthread_create(&th[t], NULL, bwdrows_worker, &jobs[t]) != 0) { rc = -3; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = -2;
    }
    free(th); free(jobs);
    return rc;
}

static int attn_bwd_rows_impl(const pattern* pt, const uint16_t* q, const uint16_t* k,
                              const uint16_t* v, const uint16_t* dout, const long long* rows,
                              long long nrows, double* dq_rows, double* dk_rows, double* dv_rows,
                              int nthreads) {
    if (check_rows(pt, rows, nrows)) return -1;
    if (nrows == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    const long long n = pt->n;
    const int heads = pt->heads, d = pt->d;
    long long* key = request_keys(pt, rows, nrows);
    if (!key) return -2;
    uint16_t* sq = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint16_t* sk = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint16_t* sv = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint16_t* sdo = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(n * d));
    uint8_t* valid = (uint8_t*)malloc((size_t)n);
    double* L = (double*)malloc(sizeof(double) * (size_t)n);
    double* Dl = (double*)malloc(sizeof(double) * (size_t)n);
    long long* pos = (long long*)malloc(sizeof(long long) * (size_t)nrows);
    long long* slot = (long long*)malloc(sizeof(long long) * (size_t)nrows);
    int rc = 0;
    if (!sq || !sk || !sv || !sdo || !valid || !L || !Dl || !pos || !slot) rc = -2;
    for (long long g0 = 0; rc == 0 && g0 < nrows;) {
        const long long group = key[2 * g0] / n;
        long long g1 = g0;
        while (g1 < nrows && key[2 * g1] / n == group) {
            pos[g1 - g0] = key[2 * g1] % n;
            slot[g1 - g0] = key[2 * g1 + 1];
            ++g1;
        }
        const uint16_t* src[4] = {q, k, v, dout};
        uint16_t* dst[4] = {sq, sk, sv, sdo};
        gather_subseq(pt, group / heads, (int)(group % heads), src, dst, 4, valid);
        bwdrows_job jb;
        memset(&jb, 0, sizeof jb);
        jb.sq = sq; jb.sk = sk; jb.sv = sv; jb.sdo = sdo; jb.valid = valid;
        jb.n = n; jb.d = d; jb.L = L; jb.Dl = Dl;
        jb.pos = pos; jb.slot = slot; jb.count = g1 - g0;
        jb.dq = dq_rows; jb.dk = dk_rows; jb.dv = dv_rows;
        rc = run_bwdrows(jb, nthreads, 0);
        if (!rc) rc = run_bwdrows(jb, nthreads, 1);
        g0 = g1;
    }
    free(key); free(sq); free(sk); free(sv); free(sdo); free(valid); free(L); free(Dl); free(pos); free(slot);
    return rc;
}

int oracle_attn_bwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                         const long long* rows, long long nrows, double* dq_rows, double* dk_rows,
                         double* dv_rows, int B, int T, int H, int W, int heads, int d, int P,
                         int mode, int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 2, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_bwd_rows_impl(&pt, q, k, v, dout, rows, nrows, dq_rows, dk_rows, dv_rows, nthreads);
}

int oracle1d_attn_bwd_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* dout, const long long* rows, long long nrows,
                           double* dq_rows, double* dk_rows, double* dv_rows, int B, int T, int H,
                           int W, int heads, int d, int P, int mode, int nthreads) {
    pattern pt;
    if (pattern_init(&pt, 1, B, T, H, W, heads, d, P, mode)) return -1;
    return attn_bwd_rows_impl(&pt, q, k, v, dout, rows, nrows, dq_rows, dk_rows, dv_rows, nthreads);
}
