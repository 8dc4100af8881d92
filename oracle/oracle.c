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
