/*
 * oracle.c -- float64 CPU oracle for pair-bias multi-query attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  The
 * product path (the CUDA library) never calls it and shares no code, header,
 * table or helper with it.
 *
 * What it computes (page "Making Full-Context AlphaGenome Fit on an RTX 3090",
 * section "Why stock FlashAttention was not a drop-in replacement", Eq. L_ij):
 *
 *   s_ij  = (sum_d q[b,h,i,d] * k[b,j,d]) / sqrt(D)
 *           + bias[h, floor(i/block), floor(j/block)]
 *   L_ij  = cap * tanh(s_ij / cap)          (cap = +inf: L_ij = s_ij)
 *   lse_i = log(sum_j exp(L_ij))            (natural log)
 *   out_i = sum_j exp(L_ij - lse_i) * v[b,j,:]
 *
 * Multi-query layout: eight (in general H) query heads read one K head and
 * one V head that all of them share (same section, tensor shapes Q, K, V).
 * The compact bias holds one cell per block x block square of (query, key)
 * positions and the dense model repeats each cell over its square; the
 * oracle builds that repeated row literally, one query row at a time.
 * Lengths that are not a multiple of the block end in a partial block whose
 * compact cell applies as it does to the others (P = ceil(L/block)); the page
 * lists tails among what is not yet supported (section "What has not yet
 * been demonstrated") and tail handling as next work (section "Where I would
 * take it next"), and floor(i/block) is the plain reading for them.  The bias
 * may also be one per batch item, [B,H,P,P], since each sequence has its own
 * pair representation (section "Profiling pointed at one very large object").
 * No mask: every key is attended (section "What this does -- and does not --
 * mean" lists masks among the unsupported features).  The softmax is written as the plain
 * two-pass definition (max, then sum), not the tiled online recurrence of
 * section "Online softmax, one block at a time"; the page states that the
 * recurrence reaches this same result up to floating-point reordering.
 *
 * Pair-bias projection (section "Profiling pointed at one very large
 * object": the dense path projects a compact pair representation to the
 * per-head bias before repeating it):
 *   bias[h,p,q] = sum_c pair[p,q,c] * W[c,h]
 * read as a plain linear map without bias term or activation (the page names
 * no other term).
 *
 * Backward (agref_attn_bwd_ex, agref_attn_bwd_sample): the gradients of out
 * with respect to q, k, v and the compact bias by the chain rule through the
 * softmax and the soft cap, written out at the end of this file.  The page
 * lists a backward pass only as later work for fine-tuning (section "Where I
 * would take it next").
 *
 * Everything is float64.  Callers widen the exact bf16 / fp32 bit patterns
 * that the GPU receives to float64 before calling.
 *
 * AGREF_MUTANT (compile-time, default 0) plants one deliberate mistake so
 * that the tests can show each pin catches a plausible error.  A mutant
 * library is only ever built into the test's temporary folder.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef AGREF_MUTANT
#define AGREF_MUTANT 0
#endif

#define AGREF_OK 0
#define AGREF_EINVAL 1
#define AGREF_ENOMEM 2

int agref_mutant_id(void) { return AGREF_MUTANT; }

static int set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

int agref_max_threads(int nthreads) { return set_threads(nthreads); }

/* ---- pair-bias projection --------------------------------------------- */

int agref_pair_bias_project(const double *pair, const double *W, double *bias,
                            long P, long Cp, long H, int nthreads) {
    if (P < 0 || Cp <= 0 || H <= 0) return AGREF_EINVAL;
    if (P == 0) return AGREF_OK;
    if (!pair || !W || !bias) return AGREF_EINVAL;
    set_threads(nthreads);
    long p;
#pragma omp parallel for schedule(static)
    for (p = 0; p < P; ++p) {
        for (long q = 0; q < P; ++q) {
            const double *cell = pair + (p * P + q) * Cp;
            for (long h = 0; h < H; ++h) {
                double acc = 0.0;
                for (long c = 0; c < Cp; ++c) {
#if AGREF_MUTANT == 9
                    acc += cell[c] * W[h * Cp + c]; /* W read as [H,Cp] */
#else
                    acc += cell[c] * W[c * H + h];
#endif
                }
#if AGREF_MUTANT == 8
                bias[(h * P + q) * P + p] = acc; /* p and q swapped */
#else
                bias[(h * P + p) * P + q] = acc;
#endif
            }
        }
    }
    return AGREF_OK;
}

/* ---- attention ----------------------------------------------------------- */

typedef struct {
    const double *q, *k, *v, *bias;
    long B, H, L, D, Dv, block, P;
    double cap;
    long bias_bstride; /* doubles between batch items' bias; 0 = one shared bias */
} attn_args;

/* The soft cap of Eq. L_ij; cap = +inf means no cap. */
static double soft_cap(double s, double cap) {
#if AGREF_MUTANT == 12
    (void)cap;
    return s; /* cap dropped */
#else
    if (isinf(cap)) return s;
    return cap * tanh(s / cap);
#endif
}

/*
 * One query row (b, h, i).  `logit` and `brow` are caller-owned scratch of
 * length L.  Writes Dv outputs to out_row and the row's lse; if prob_row is
 * not NULL it also receives the L softmax weights.
 */
static void attn_row(const attn_args *a, long b, long h, long i, double *logit,
                     double *brow, double *out_row, double *lse_out,
                     double *prob_row) {
    const long L = a->L, D = a->D, Dv = a->Dv, blk = a->block, P = a->P;
#if AGREF_MUTANT == 11
    const double *qi = a->q + ((b * a->H + 0) * L + i) * D; /* head 0 for all */
#else
    const double *qi = a->q + ((b * a->H + h) * L + i) * D;
#endif
    const double *kb = a->k + b * L * D;
#if AGREF_MUTANT == 10
    const double *vb = a->k + b * L * D; /* values read from K */
#else
    const double *vb = a->v + b * L * Dv;
#endif

    /* The compact bias row for query block floor(i/block), repeated over each
       key block: brow[j] = bias[b, h, floor(i/block), floor(j/block)].  A
       length that is not a multiple of the block ends in a partial block,
       which uses its compact cell like any other (P = ceil(L / block)). */
#if AGREF_MUTANT == 13
    const double *bias_b = a->bias; /* every item reads item 0's bias */
#else
    const double *bias_b = a->bias + b * a->bias_bstride;
#endif
#if AGREF_MUTANT == 5
    const long I = (i / blk + 1) % P; /* query block off by one */
#else
    const long I = i / blk;
#endif
    for (long j = 0; j < L; ++j) {
        const long J = j / blk;
#if AGREF_MUTANT == 1
        brow[j] = bias_b[(h * P + J) * P + I]; /* bias transposed */
#else
        brow[j] = bias_b[(h * P + I) * P + J];
#endif
    }

    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double M = -INFINITY;
    for (long j = 0; j < L; ++j) {
        const double *kj = kb + j * D;
        double dot = 0.0;
        for (long d = 0; d < D; ++d) dot += qi[d] * kj[d];
#if AGREF_MUTANT == 3
        double s = dot + brow[j]; /* 1/sqrt(D) dropped */
#elif AGREF_MUTANT == 4
        double s = (dot + brow[j]) * inv_sqrt_d; /* bias scaled too */
#else
        double s = dot * inv_sqrt_d + brow[j];
#endif
#if AGREF_MUTANT == 2
        double l = soft_cap(dot * inv_sqrt_d, a->cap) + brow[j]; /* cap before bias */
        (void)s;
#else
        double l = soft_cap(s, a->cap);
#endif
        logit[j] = l;
        if (l > M) M = l;
    }
    double Z = 0.0;
    for (long j = 0; j < L; ++j) Z += exp(logit[j] - M);
#if AGREF_MUTANT == 6
    const double lse = log(Z); /* max term dropped */
#else
    const double lse = M + log(Z);
#endif
    for (long c = 0; c < Dv; ++c) out_row[c] = 0.0;
    for (long j = 0; j < L; ++j) {
#if AGREF_MUTANT == 7
        const double w = exp(logit[j] - M); /* not normalised */
#else
        const double w = exp(logit[j] - lse);
#endif
        if (prob_row) prob_row[j] = w;
        const double *vj = vb + j * Dv;
        for (long c = 0; c < Dv; ++c) out_row[c] += w * vj[c];
    }
    *lse_out = lse;
}

static int check_args(const attn_args *a) {
    if (a->B < 0 || a->H <= 0 || a->L < 0 || a->D <= 0 || a->Dv <= 0 ||
        a->block <= 0)
        return AGREF_EINVAL;
    if (isnan(a->cap) || a->cap <= 0.0) return AGREF_EINVAL;
    if (a->B == 0 || a->L == 0) return AGREF_OK;
    if (!a->q || !a->k || !a->v || !a->bias) return AGREF_EINVAL;
    return AGREF_OK;
}

/*
 * Full attention.  q [B,H,L,D], k [B,L,D], v [B,L,Dv], bias [H,P,P] (or, with
 * bias_bstride = H*P*P, [B,H,P,P]: one bias per batch item, as each sequence
 * has its own pair representation) with P = ceil(L/block), all row-major
 * float64.  Any L >= 0: a last partial block uses its compact cell.  Writes
 * out [B,H,L,Dv] and lse [B,H,L].  If probs is not NULL it must hold B*H*L*L
 * doubles and receives the softmax weights (tiny inputs only).
 */
/* Compact cells per side for a length: ceil(L / block). */
static long cells(long L, long block) {
#if AGREF_MUTANT == 14
    return L / block; /* partial last block dropped */
#else
    return (L + block - 1) / block;
#endif
}

int agref_attn_fwd_ex(const double *q, const double *k, const double *v,
                      const double *bias, long bias_bstride, long B, long H,
                      long L, long D, long Dv, long block, double cap,
                      double *out, double *lse, double *probs, int nthreads) {
    attn_args a = {q, k, v, bias, B, H, L, D, Dv, block, 0, cap, bias_bstride};
    int rc = check_args(&a);
    if (rc != AGREF_OK || B == 0 || L == 0) return rc;
    if (!out || !lse || bias_bstride < 0) return AGREF_EINVAL;
    a.P = cells(L, block);
    set_threads(nthreads);
    const long rows = B * H * L;
    int failed = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)L);
        double *brow = (double *)malloc(sizeof(double) * (size_t)L);
        if (!logit || !brow) {
#pragma omp atomic write
            failed = 1;
        } else {
            long r;
#pragma omp for schedule(dynamic, 16)
            for (r = 0; r < rows; ++r) {
                const long i = r % L;
                const long h = (r / L) % H;
                const long b = r / (L * H);
                attn_row(&a, b, h, i, logit, brow, out + r * Dv, lse + r,
                         probs ? probs + r * L : NULL);
            }
        }
        free(logit);
        free(brow);
    }
    return failed ? AGREF_ENOMEM : AGREF_OK;
}

/*
 * Selected rows only: rows holds n triples (b, h, i).  out_rows [n, Dv],
 * lse_rows [n].  Used to check full-size outputs on a sample of rows.
 */
int agref_attn_rows_ex(const double *q, const double *k, const double *v,
                       const double *bias, long bias_bstride, long B, long H,
                       long L, long D, long Dv, long block, double cap,
                       const int64_t *rows, long n, double *out_rows,
                       double *lse_rows, int nthreads) {
    attn_args a = {q, k, v, bias, B, H, L, D, Dv, block, 0, cap, bias_bstride};
    int rc = check_args(&a);
    if (rc != AGREF_OK) return rc;
    if (n == 0) return AGREF_OK;
    if (!rows || !out_rows || !lse_rows || B == 0 || L == 0) return AGREF_EINVAL;
    for (long t = 0; t < n; ++t) {
        const int64_t b = rows[3 * t], h = rows[3 * t + 1], i = rows[3 * t + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= L) return AGREF_EINVAL;
    }
    if (bias_bstride < 0) return AGREF_EINVAL;
    a.P = cells(L, block);
    set_threads(nthreads);
    int failed = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)L);
        double *brow = (double *)malloc(sizeof(double) * (size_t)L);
        if (!logit || !brow) {
#pragma omp atomic write
            failed = 1;
        } else {
            long t;
#pragma omp for schedule(dynamic, 1)
            for (t = 0; t < n; ++t) {
                attn_row(&a, rows[3 * t], rows[3 * t + 1], rows[3 * t + 2], logit,
                         brow, out_rows + t * Dv, lse_rows + t, NULL);
            }
        }
        free(logit);
        free(brow);
    }
    return failed ? AGREF_ENOMEM : AGREF_OK;
}

/* The entry points with one bias shared by every batch item. */
int agref_attn_fwd(const double *q, const double *k, const double *v,
                   const double *bias, long B, long H, long L, long D, long Dv,
                   long block, double cap, double *out, double *lse,
                   double *probs, int nthreads) {
    return agref_attn_fwd_ex(q, k, v, bias, 0, B, H, L, D, Dv, block, cap, out,
                             lse, probs, nthreads);
}

int agref_attn_rows(const double *q, const double *k, const double *v,
                    const double *bias, long B, long H, long L, long D, long Dv,
                    long block, double cap, const int64_t *rows, long n,
                    double *out_rows, double *lse_rows, int nthreads) {
    return agref_attn_rows_ex(q, k, v, bias, 0, B, H, L, D, Dv, block, cap, rows,
                              n, out_rows, lse_rows, nthreads);
}

/* ---- attention backward ------------------------------------------------ */
/*
 * Gradients of the attention map above with respect to q, k, v and the
 * compact bias, for an upstream gradient dout [B,H,L,Dv] of out.  The page
 * names a backward pass only as later work for fine-tuning (section "Where I
 * would take it next"); what it must compute is the chain rule applied to
 * Eq. L_ij and the softmax.  With
 *   p_ij    = exp(L_ij - lse_i)                        softmax weight
 *   dp_ij   = sum_c dout[i,c] * v[j,c]
 *   delta_i = sum_j p_ij * dp_ij
 *   dL_ij   = p_ij * (dp_ij - delta_i)                 softmax Jacobian
 *   ds_ij   = dL_ij * (1 - tanh^2(s_ij / cap))         cap = +inf: ds = dL
 *           = dL_ij * (1 - (L_ij / cap)^2)
 * the gradients are
 *   dq[b,h,i,:]  = sum_j ds_ij * k[b,j,:] / sqrt(D)
 *   dk[b,j,:]    = sum_{h,i} ds_ij * q[b,h,i,:] / sqrt(D)   (K shared by the heads)
 *   dv[b,j,:]    = sum_{h,i} p_ij * dout[b,h,i,:]          (V shared by the heads)
 *   dbias cell (h, I, J) = sum_{i in block I, j in block J} ds_ij, summed over
 *                  the batch items that share the bias (bias_bstride = 0) or
 *                  kept per item (bias_bstride > 0, same layout as bias).
 * Three passes, each parallel over what it writes, so that no two threads
 * add into one value: rows (lse, delta, dq), keys (dk, dv), bias cells.
 */

/* lse_i and delta_i of row (b, h, i), from the forward row and its weights.
   logit, brow, prob are caller scratch of length L; orow of length Dv. */
static void bwd_row_stats(const attn_args *a, const double *dout, long b, long h,
                          long i, double *logit, double *brow, double *prob,
                          double *orow, double *lse_out, double *delta_out) {
    double lse = 0.0;
    attn_row(a, b, h, i, logit, brow, orow, &lse, prob);
    const long L = a->L, Dv = a->Dv;
    const double *gi = dout + ((b * a->H + h) * L + i) * Dv;
    const double *vb = a->v + b * L * Dv;
    double delta = 0.0;
    for (long j = 0; j < L; ++j) {
        double dp = 0.0;
        for (long c = 0; c < Dv; ++c) dp += gi[c] * vb[j * Dv + c];
        delta += prob[j] * dp;
    }
    *lse_out = lse;
    *delta_out = delta;
}

/* p_ij and ds_ij of one (query, key) pair, given the row's lse and delta. */
static void bwd_pair(const attn_args *a, const double *dout, long b, long h,
                     long i, long j, double lse, double delta, double *p_out,
                     double *ds_out) {
    const long L = a->L, D = a->D, Dv = a->Dv, blk = a->block, P = a->P;
    const double *qi = a->q + ((b * a->H + h) * L + i) * D;
    const double *kj = a->k + (b * L + j) * D;
    const double *vj = a->v + (b * L + j) * Dv;
    const double *gi = dout + ((b * a->H + h) * L + i) * Dv;
    const double *bias_b = a->bias + b * a->bias_bstride;
    double dot = 0.0;
    for (long d = 0; d < D; ++d) dot += qi[d] * kj[d];
    const double s = dot / sqrt((double)D) + bias_b[(h * P + i / blk) * P + j / blk];
    const double l = soft_cap(s, a->cap);
    const double p = exp(l - lse);
    double dp = 0.0;
    for (long c = 0; c < Dv; ++c) dp += gi[c] * vj[c];
#if AGREF_MUTANT == 16
    const double dl = p * dp; /* softmax Jacobian without the delta term */
    (void)delta;
#else
    const double dl = p * (dp - delta);
#endif
#if AGREF_MUTANT == 15
    const double g = 1.0; /* derivative of the soft cap dropped */
#else
    const double g = isinf(a->cap) ? 1.0 : 1.0 - (l / a->cap) * (l / a->cap);
#endif
    *p_out = p;
    *ds_out = dl * g;
}

/* dk and dv of key (b, j): sums over every head and query row. */
static void bwd_key(const attn_args *a, const double *dout, const double *lse,
                    const double *delta, long b, long j, double *dk_row,
                    double *dv_row) {
    const long L = a->L, D = a->D, Dv = a->Dv, H = a->H;
    for (long d = 0; d < D; ++d) dk_row[d] = 0.0;
    for (long c = 0; c < Dv; ++c) dv_row[c] = 0.0;
#if AGREF_MUTANT == 17
    const double scale = 1.0; /* 1/sqrt(D) missing from dk */
#else
    const double scale = 1.0 / sqrt((double)D);
#endif
    for (long h = 0; h < H; ++h) {
        for (long i = 0; i < L; ++i) {
            const long r = (b * H + h) * L + i;
            double p, ds;
            bwd_pair(a, dout, b, h, i, j, lse[r], delta[r], &p, &ds);
            const double *qi = a->q + r * D;
            const double *gi = dout + r * Dv;
            for (long d = 0; d < D; ++d) dk_row[d] += ds * qi[d] * scale;
            for (long c = 0; c < Dv; ++c) dv_row[c] += p * gi[c];
        }
    }
}

/* One compact bias cell (h, I, J) of item b's bias; with a shared bias
   (bias_bstride = 0) the sum runs over every item and b is ignored. */
static double bwd_cell(const attn_args *a, const double *dout, const double *lse,
                       const double *delta, long b, long h, long I, long J) {
    const long L = a->L, blk = a->block, H = a->H;
#if AGREF_MUTANT == 18
    const long b0 = a->bias_bstride ? b : 0, b1 = b0 + 1; /* shared: item 0 only */
#else
    const long b0 = a->bias_bstride ? b : 0, b1 = a->bias_bstride ? b + 1 : a->B;
#endif
    double acc = 0.0;
    for (long bb = b0; bb < b1; ++bb) {
        for (long i = I * blk; i < (I + 1) * blk && i < L; ++i) {
            const long r = (bb * H + h) * L + i;
            for (long j = J * blk; j < (J + 1) * blk && j < L; ++j) {
                double p, ds;
                bwd_pair(a, dout, bb, h, i, j, lse[r], delta[r], &p, &ds);
                acc += ds;
            }
        }
    }
    return acc;
}

/* lse and delta for every row (b, h, i). */
static int bwd_all_row_stats(const attn_args *a, const double *dout, double *lse,
                             double *delta) {
    const long rows = a->B * a->H * a->L, L = a->L;
    int failed = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)L);
        double *brow = (double *)malloc(sizeof(double) * (size_t)L);
        double *prob = (double *)malloc(sizeof(double) * (size_t)L);
        double *orow = (double *)malloc(sizeof(double) * (size_t)a->Dv);
        if (!logit || !brow || !prob || !orow) {
#pragma omp atomic write
            failed = 1;
        } else {
            long r;
#pragma omp for schedule(dynamic, 16)
            for (r = 0; r < rows; ++r) {
                bwd_row_stats(a, dout, r / (L * a->H), (r / L) % a->H, r % L, logit,
                              brow, prob, orow, lse + r, delta + r);
            }
        }
        free(logit);
        free(brow);
        free(prob);
        free(orow);
    }
    return failed ? AGREF_ENOMEM : AGREF_OK;
}

/*
 * Full backward.  Inputs as agref_attn_fwd_ex plus dout [B,H,L,Dv].  Writes
 * dq [B,H,L,D], dk [B,L,D], dv [B,L,Dv] and dbias in the layout of bias
 * ([H,P,P] when bias_bstride = 0, else item b at dbias + b*bias_bstride);
 * lse_out and delta_out [B,H,L] are optional.
 */
int agref_attn_bwd_ex(const double *q, const double *k, const double *v,
                      const double *bias, long bias_bstride, const double *dout,
                      long B, long H, long L, long D, long Dv, long block,
                      double cap, double *dq, double *dk, double *dv,
                      double *dbias, double *lse_out, double *delta_out,
                      int nthreads) {
    attn_args a = {q, k, v, bias, B, H, L, D, Dv, block, 0, cap, bias_bstride};
    int rc = check_args(&a);
    if (rc != AGREF_OK || B == 0 || L == 0) return rc;
    if (!dout || !dq || !dk || !dv || !dbias || bias_bstride < 0) return AGREF_EINVAL;
    a.P = cells(L, block);
    set_threads(nthreads);
    const long rows = B * H * L, P = a.P;
    double *lse = (double *)malloc(sizeof(double) * (size_t)rows);
    double *delta = (double *)malloc(sizeof(double) * (size_t)rows);
    if (!lse || !delta) {
        free(lse);
        free(delta);
        return AGREF_ENOMEM;
    }
    rc = bwd_all_row_stats(&a, dout, lse, delta);
    if (rc == AGREF_OK) {
        const double scale = 1.0 / sqrt((double)D);
        long r;
#pragma omp parallel for schedule(dynamic, 16)
        for (r = 0; r < rows; ++r) {
            const long i = r % L, h = (r / L) % H, b = r / (L * H);
            double *dqi = dq + r * D;
            for (long d = 0; d < D; ++d) dqi[d] = 0.0;
            for (long j = 0; j < L; ++j) {
                double p, ds;
                bwd_pair(&a, dout, b, h, i, j, lse[r], delta[r], &p, &ds);
                const double *kj = k + (b * L + j) * D;
                for (long d = 0; d < D; ++d) dqi[d] += ds * kj[d] * scale;
            }
        }
        long t;
#pragma omp parallel for schedule(dynamic, 4)
        for (t = 0; t < B * L; ++t)
            bwd_key(&a, dout, lse, delta, t / L, t % L, dk + t * D, dv + t * Dv);
        const long items = bias_bstride ? B : 1;
        long c;
#pragma omp parallel for schedule(dynamic, 4)
        for (c = 0; c < items * H * P * P; ++c) {
            const long J = c % P, I = (c / P) % P, h = (c / (P * P)) % H,
                       b = c / (P * P * H);
            dbias[b * bias_bstride + (h * P + I) * P + J] =
                bwd_cell(&a, dout, lse, delta, b, h, I, J);
        }
        if (lse_out) memcpy(lse_out, lse, sizeof(double) * (size_t)rows);
        if (delta_out) memcpy(delta_out, delta, sizeof(double) * (size_t)rows);
    }
    free(lse);
    free(delta);
    return rc;
}

/*
 * Selected gradients only, to check full-size results on a sample:
 * rows (b,h,i) x n_rows -> dq_rows [n_rows, D]; keys (b,j) x n_keys ->
 * dk_rows [n_keys, D], dv_rows [n_keys, Dv]; cells (b,h,I,J) x n_cells ->
 * dbias_cells [n_cells] (b ignored for a shared bias).  Row statistics are
 * computed for every row when keys or cells are asked for (they sum over all
 * rows), else only for the rows asked for.
 */
int agref_attn_bwd_sample(const double *q, const double *k, const double *v,
                          const double *bias, long bias_bstride, const double *dout,
                          long B, long H, long L, long D, long Dv, long block,
                          double cap, const int64_t *rows, long n_rows,
                          double *dq_rows, const int64_t *keys, long n_keys,
                          double *dk_rows, double *dv_rows, const int64_t *cellv,
                          long n_cells, double *dbias_cells, int nthreads) {
    attn_args a = {q, k, v, bias, B, H, L, D, Dv, block, 0, cap, bias_bstride};
    int rc = check_args(&a);
    if (rc != AGREF_OK) return rc;
    if (B == 0 || L == 0 || !dout || bias_bstride < 0) return AGREF_EINVAL;
    a.P = cells(L, block);
    const long P = a.P;
    for (long t = 0; t < n_rows; ++t)
        if (rows[3 * t] < 0 || rows[3 * t] >= B || rows[3 * t + 1] < 0 ||
            rows[3 * t + 1] >= H || rows[3 * t + 2] < 0 || rows[3 * t + 2] >= L)
            return AGREF_EINVAL;
    for (long t = 0; t < n_keys; ++t)
        if (keys[2 * t] < 0 || keys[2 * t] >= B || keys[2 * t + 1] < 0 ||
            keys[2 * t + 1] >= L)
            return AGREF_EINVAL;
    for (long t = 0; t < n_cells; ++t)
        if (cellv[4 * t] < 0 || cellv[4 * t] >= B || cellv[4 * t + 1] < 0 ||
            cellv[4 * t + 1] >= H || cellv[4 * t + 2] < 0 || cellv[4 * t + 2] >= P ||
            cellv[4 * t + 3] < 0 || cellv[4 * t + 3] >= P)
            return AGREF_EINVAL;
    set_threads(nthreads);
    const long nr = B * H * L;
    double *lse = (double *)malloc(sizeof(double) * (size_t)nr);
    double *delta = (double *)malloc(sizeof(double) * (size_t)nr);
    if (!lse || !delta) {
        free(lse);
        free(delta);
        return AGREF_ENOMEM;
    }
    if (n_keys > 0 || n_cells > 0) {
        rc = bwd_all_row_stats(&a, dout, lse, delta);
    } else {
        int failed = 0;
#pragma omp parallel
        {
            double *logit = (double *)malloc(sizeof(double) * (size_t)L);
            double *brow = (double *)malloc(sizeof(double) * (size_t)L);
            double *prob = (double *)malloc(sizeof(double) * (size_t)L);
            double *orow = (double *)malloc(sizeof(double) * (size_t)Dv);
            if (!logit || !brow || !prob || !orow) {
#pragma omp atomic write
                failed = 1;
            } else {
                long t;
#pragma omp for schedule(dynamic, 1)
                for (t = 0; t < n_rows; ++t) {
                    const long b = rows[3 * t], h = rows[3 * t + 1], i = rows[3 * t + 2];
                    const long r = (b * H + h) * L + i;
                    bwd_row_stats(&a, dout, b, h, i, logit, brow, prob, orow, lse + r,
                                  delta + r);
                }
            }
            free(logit);
            free(brow);
            free(prob);
            free(orow);
        }
        rc = failed ? AGREF_ENOMEM : AGREF_OK;
    }
    if (rc == AGREF_OK) {
        const double scale = 1.0 / sqrt((double)D);
        long t;
#pragma omp parallel for schedule(dynamic, 1)
        for (t = 0; t < n_rows; ++t) {
            const long b = rows[3 * t], h = rows[3 * t + 1], i = rows[3 * t + 2];
            const long r = (b * H + h) * L + i;
            double *dqi = dq_rows + t * D;
            for (long d = 0; d < D; ++d) dqi[d] = 0.0;
            for (long j = 0; j < L; ++j) {
                double p, ds;
                bwd_pair(&a, dout, b, h, i, j, lse[r], delta[r], &p, &ds);
                for (long d = 0; d < D; ++d) dqi[d] += ds * k[(b * L + j) * D + d] * scale;
            }
        }
#pragma omp parallel for schedule(dynamic, 1)
        for (t = 0; t < n_keys; ++t)
            bwd_key(&a, dout, lse, delta, keys[2 * t], keys[2 * t + 1], dk_rows + t * D,
                    dv_rows + t * Dv);
#pragma omp parallel for schedule(dynamic, 1)
        for (t = 0; t < n_cells; ++t)
            dbias_cells[t] = bwd_cell(&a, dout, lse, delta, cellv[4 * t],
                                      cellv[4 * t + 1], cellv[4 * t + 2], cellv[4 * t + 3]);
    }
    free(lse);
    free(delta);
    return rc;
}
