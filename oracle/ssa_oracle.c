/*
 * ssa_oracle.c -- plain, slow fp64 CPU oracle for the SSA block-sparse attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * Source: "SSA: Sparse Sparse Attention by Aligning Full and Sparse Attention
 * Outputs in Feature Space" (arXiv 2511.20102), as summarised on the
 * paperlayer.ai page for v4.  The page prints no formulas; each function states
 * the reading it implements.
 *
 * Layout: every tensor is a contiguous fp64 array [BH, T, d] (batch and heads
 * flattened), block j covers tokens [j*s, (j+1)*s), nb = T/s, b(t) = t/s.
 * Selections are int32 [BH, T, k], ascending, padded with -1.
 * Parallelism: OpenMP over independent rows only; no blocking or reordering of
 * the arithmetic beyond the plain definitions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef int64_t i64;

int ora_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------------
 * Block pooling -- page section 3 ("scores preceding blocks using mean-pooled
 * keys"): Kbar[j] = (1/s) * sum of the s keys of block j, unweighted.
 * ------------------------------------------------------------------------- */
void ora_block_pool(i64 BH, i64 T, i64 d, i64 s, const double *K, double *Kbar) {
    i64 nb = T / s;
#pragma omp parallel for collapse(2) schedule(static)
    for (i64 bh = 0; bh < BH; ++bh) {
        for (i64 j = 0; j < nb; ++j) {
            for (i64 c = 0; c < d; ++c) {
                double acc = 0.0;
                for (i64 t = j * s; t < (j + 1) * s; ++t) acc += K[(bh * T + t) * d + c];
                Kbar[(bh * nb + j) * d + c] = acc / (double)s;
            }
        }
    }
}

/* ---------------------------------------------------------------------------
 * Block selection -- page section 3 ("scores preceding blocks ... selects the
 * top-k blocks for each query"; receptive field k*s tokens).
 * Reading: the query's own block b(t) is always kept and counted within k; the
 * other k-1 are the highest scores r_j = q_t . Kbar_j over strictly preceding
 * blocks j < b(t); ties go to the lower block index; the result is stored in
 * ascending block order and padded with -1 when fewer than k-1 blocks precede.
 * r_km1 / r_k receive the (k-1)-th and k-th best candidate scores (NaN when
 * that rank does not exist) so that callers can spot near-ties.
 * ------------------------------------------------------------------------- */
typedef struct {
    double score;
    int32_t j;
} ora_cand;

static int ora_cand_order(const void *pa, const void *pb) {
    const ora_cand *a = (const ora_cand *)pa, *b = (const ora_cand *)pb;
    if (a->score > b->score) return -1; /* higher score first */
    if (a->score < b->score) return 1;
    return (a->j > b->j) - (a->j < b->j); /* equal scores: lower index first */
}

static int ora_int_order(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void ora_block_select(i64 BH, i64 G, i64 T, i64 d, i64 s, i64 k, const double *Q, const double *Kbar,
                      int32_t *idx, double *r_km1, double *r_k) {
    /* BH key/value heads, each shared by the G consecutive query heads of its group (G = 1: one query head
     * per key head); the group's score of block j is the sum of its query heads' scores. */
    i64 nb = T / s;
#pragma omp parallel
    {
        ora_cand *cand = (ora_cand *)malloc(sizeof(ora_cand) * (size_t)(nb > 0 ? nb : 1));
        int32_t *chosen = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
#pragma omp for collapse(2) schedule(dynamic, 64)
        for (i64 bh = 0; bh < BH; ++bh) {
            for (i64 t = 0; t < T; ++t) {
                i64 bt = t / s;
                for (i64 j = 0; j < bt; ++j) {
                    const double *kb = Kbar + (bh * nb + j) * d;
                    double r = 0.0;
                    for (i64 g = 0; g < G; ++g) {
                        const double *q = Q + ((bh * G + g) * T + t) * d;
                        for (i64 c = 0; c < d; ++c) r += q[c] * kb[c];
                    }
                    cand[j].score = r;
                    cand[j].j = (int32_t)j;
                }
                qsort(cand, (size_t)bt, sizeof(ora_cand), ora_cand_order);
                i64 take = (k - 1 < bt) ? k - 1 : bt;
                for (i64 i = 0; i < take; ++i) chosen[i] = cand[i].j;
                chosen[take] = (int32_t)bt;
                qsort(chosen, (size_t)(take + 1), sizeof(int32_t), ora_int_order);
                int32_t *row = idx + (bh * T + t) * k;
                for (i64 i = 0; i < k; ++i) row[i] = (i <= take) ? chosen[i] : -1;
                if (r_km1) r_km1[bh * T + t] = (take >= 1 && bt > take) ? cand[take - 1].score : NAN;
                if (r_k) r_k[bh * T + t] = (bt > take) ? cand[take].score : NAN;
            }
        }
        free(cand);
        free(chosen);
    }
}

/* Candidate scores of listed rows -- page section 3: every strictly preceding
 * block j < b(t) is scored r_j = q_t . Kbar_j.  For the n (head, query) pairs
 * (bh_list[i], t_list[i]), out[i * nb + j] = r_j for j < b(t) and NaN for the
 * blocks that are not candidates (bh_list names key/value heads; with G > 1 the
 * score is the group's sum, as in block_select).  Used to check that a selection
 * which differs from block_select's on a near-tie row is still a valid top set. */
void ora_block_scores(i64 BH, i64 G, i64 T, i64 d, i64 s, i64 n, const i64 *bh_list, const i64 *t_list,
                      const double *Q, const double *Kbar, double *out) {
    i64 nb = T / s;
    (void)BH;
#pragma omp parallel for schedule(static)
    for (i64 i = 0; i < n; ++i) {
        i64 bh = bh_list[i], t = t_list[i], bt = t / s;
        for (i64 j = 0; j < nb; ++j) {
            if (j >= bt) {
                out[i * nb + j] = NAN;
                continue;
            }
            const double *kb = Kbar + (bh * nb + j) * d;
            double r = 0.0;
            for (i64 g = 0; g < G; ++g) {
                const double *q = Q + ((bh * G + g) * T + t) * d;
                for (i64 c = 0; c < d; ++c) r += q[c] * kb[c];
            }
            out[i * nb + j] = r;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Attended set S(t).
 * Full attention (paper section 3: every preceding token takes part): S(t) = {0..t}.
 * Sparse attention (page section 3: the selected blocks' tokens form the
 * reduced key/value matrices): S(t) = union over the selected blocks of their
 * tokens, restricted to positions <= t (causal inside the query's own block).
 * attended_set() writes the positions of S(t) in ascending order (the selection
 * row is ascending and duplicate-free) and returns |S(t)|.
 * ------------------------------------------------------------------------- */
static i64 attended_set(const int32_t *sel_row, i64 k, i64 s, i64 t, i64 *pos) {
    i64 n = 0;
    if (!sel_row) {
        for (i64 u = 0; u <= t; ++u) pos[n++] = u;
        return n;
    }
    for (i64 i = 0; i < k; ++i) {
        if (sel_row[i] < 0) continue;
        for (i64 u = (i64)sel_row[i] * s; u < ((i64)sel_row[i] + 1) * s && u <= t; ++u) pos[n++] = u;
    }
    return n;
}

/* 1 when every row of idx is ascending, duplicate-free, within [0, b(t)], holds
 * b(t), and has its -1 padding only at the end; 0 otherwise. */
int ora_check_selection(i64 BH, i64 T, i64 s, i64 k, const int32_t *idx) {
    for (i64 r = 0; r < BH * T; ++r) {
        i64 t = r % T, bt = t / s, last = -1, seen_current = 0, padded = 0;
        for (i64 i = 0; i < k; ++i) {
            int32_t j = idx[r * k + i];
            if (j < 0) {
                if (j != -1) return 0;
                padded = 1;
                continue;
            }
            if (padded || j <= last || j > bt) return 0;
            if (j == bt) seen_current = 1;
            last = j;
        }
        if (!seen_current) return 0;
    }
    return 1;
}

/* Softmax attention for one query row over S(t): fills o[d] and returns LSE.
 * logits x_u = scale * q_t . k_u ; lse = log sum_{u in S(t)} exp(x_u);
 * o = sum_{u in S(t)} exp(x_u - lse) v_u.  pos is scratch of T entries. */
static double attend_row(i64 d, i64 s, i64 k, double scale, const double *Qh, const double *Kh, const double *Vh,
                         const int32_t *sel_row, i64 t, double *o, i64 *pos) {
    const double *q = Qh + t * d;
    i64 n = attended_set(sel_row, k, s, t, pos);
    double m = -INFINITY;
    for (i64 a = 0; a < n; ++a) {
        double x = 0.0;
        for (i64 c = 0; c < d; ++c) x += q[c] * Kh[pos[a] * d + c];
        x *= scale;
        if (x > m) m = x;
    }
    double l = 0.0;
    for (i64 c = 0; c < d; ++c) o[c] = 0.0;
    for (i64 a = 0; a < n; ++a) {
        double x = 0.0;
        for (i64 c = 0; c < d; ++c) x += q[c] * Kh[pos[a] * d + c];
        double p = exp(x * scale - m);
        l += p;
        for (i64 c = 0; c < d; ++c) o[c] += p * Vh[pos[a] * d + c];
    }
    for (i64 c = 0; c < d; ++c) o[c] /= l;
    return m + log(l);
}

/* Forward for the query rows listed in rows[0..nrows) of every head (rows == NULL:
 * all T rows).  O is [BH, nrows, d], lse is [BH, nrows].  idx == NULL selects full
 * causal attention, otherwise the sparse stream over the given selection.  Query
 * head bh reads key/value head bh / G (grouped-query attention; G = 1 for one key
 * head per query head) and, in the sparse stream, that key head's selection:
 * K, V are [BH / G, T, d], idx is [BH / G, T, k]. */
void ora_attn_fwd(i64 BH, i64 G, i64 T, i64 d, i64 s, i64 k, double scale, const double *Q, const double *K,
                  const double *V, const int32_t *idx, i64 nrows, const i64 *rows, double *O, double *lse) {
    i64 n = rows ? nrows : T;
#pragma omp parallel
    {
        i64 *pos = (i64 *)malloc(sizeof(i64) * (size_t)T);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (i64 bh = 0; bh < BH; ++bh) {
            for (i64 r = 0; r < n; ++r) {
                i64 t = rows ? rows[r] : r;
                const i64 kh = bh / G; /* key/value head (and selection) of query head bh */
                const int32_t *sel_row = idx ? idx + (kh * T + t) * k : NULL;
                lse[bh * n + r] = attend_row(d, s, k, scale, Q + bh * T * d, K + kh * T * d, V + kh * T * d,
                                             sel_row, t, O + (bh * n + r) * d, pos);
            }
        }
        free(pos);
    }
}

/* ---------------------------------------------------------------------------
 * Backward of o_t = softmax_{u in S(t)}(scale q_t.k_u) v_u with upstream dO.
 * Page section 4.2: in the sparse stream, keys outside S(t) take no part in the
 * normalisation and receive zero gradient; no gradient flows through the
 * selection (idx is a constant).  With P_tu the softmax weight, D_t = dO_t . o_t
 * and dP_tu = dO_t . v_u:
 *   dQ_t = scale * sum_{u in S(t)} P_tu (dP_tu - D_t) k_u
 *   dK_u = scale * sum_{t : u in S(t)} P_tu (dP_tu - D_t) q_t
 *   dV_u = sum_{t : u in S(t)} P_tu dO_t
 * Computes dQ for query rows qrows[0..nq) and dK, dV for key rows krows[0..nk)
 * (NULL: all rows); outputs are [BH, nq, d] and [BH / G, nk, d]: with grouped
 * query heads (G > 1) a key head's gradients sum over the G query heads reading it.
 * ------------------------------------------------------------------------- */
/* x rounded to the nearest bfloat16 value (8 significant bits, ties to even), as a forward output
 * stored in bfloat16 holds it. */
static double round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    const double m = frexp(x, &e);            /* x = m * 2^e, 0.5 <= |m| < 1 */
    return ldexp(nearbyint(ldexp(m, 8)), e - 8); /* default rounding mode: to nearest, ties to even */
}

/* round_o != 0: D_t = dO_t . o_t uses o_t rounded to bfloat16 -- the value a backward pass receives
 * when the forward stores its output in bfloat16 (the backward takes the stored output as input). */
void ora_attn_bwd(i64 BH, i64 G, i64 T, i64 d, i64 s, i64 k, double scale, const double *Q, const double *K,
                  const double *V, const double *dO, const int32_t *idx, i64 nq, const i64 *qrows, i64 nk,
                  const i64 *krows, double *dQ, double *dK, double *dV, int round_o) {
    i64 nQ = qrows ? nq : T, nK = krows ? nk : T, BHk = BH / G;
    double *lse = (double *)malloc(sizeof(double) * (size_t)(BH * T));
    double *Dt = (double *)malloc(sizeof(double) * (size_t)(BH * T));
    i64 *kslot = (i64 *)malloc(sizeof(i64) * (size_t)T); /* key position -> output row, or -1 */
    for (i64 u = 0; u < T; ++u) kslot[u] = krows ? -1 : u;
    if (krows)
        for (i64 r = 0; r < nK; ++r) kslot[krows[r]] = r;
    memset(dK, 0, sizeof(double) * (size_t)(BHk * nK * d));
    memset(dV, 0, sizeof(double) * (size_t)(BHk * nK * d));

    /* Forward over every row: LSE_t and D_t = dO_t . o_t. */
#pragma omp parallel
    {
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        i64 *pos = (i64 *)malloc(sizeof(i64) * (size_t)T);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (i64 bh = 0; bh < BH; ++bh) {
            for (i64 t = 0; t < T; ++t) {
                const i64 kh = bh / G;
                const int32_t *sel_row = idx ? idx + (kh * T + t) * k : NULL;
                lse[bh * T + t] =
                    attend_row(d, s, k, scale, Q + bh * T * d, K + kh * T * d, V + kh * T * d, sel_row, t, o, pos);
                double acc = 0.0;
                for (i64 c = 0; c < d; ++c) acc += dO[(bh * T + t) * d + c] * (round_o ? round_bf16(o[c]) : o[c]);
                Dt[bh * T + t] = acc;
            }
        }
        free(o);
        free(pos);
    }

    /* dQ rows. */
#pragma omp parallel
    {
        i64 *pos = (i64 *)malloc(sizeof(i64) * (size_t)T);
#pragma omp for collapse(2) schedule(dynamic, 16)
        for (i64 bh = 0; bh < BH; ++bh) {
            for (i64 r = 0; r < nQ; ++r) {
                i64 t = qrows ? qrows[r] : r, kh = bh / G;
                const double *q = Q + (bh * T + t) * d, *g = dO + (bh * T + t) * d;
                const int32_t *sel_row = idx ? idx + (kh * T + t) * k : NULL;
                double *out = dQ + (bh * nQ + r) * d;
                for (i64 c = 0; c < d; ++c) out[c] = 0.0;
                i64 n = attended_set(sel_row, k, s, t, pos);
                for (i64 a = 0; a < n; ++a) {
                    const double *ku = K + (kh * T + pos[a]) * d, *vu = V + (kh * T + pos[a]) * d;
                    double x = 0.0, dp = 0.0;
                    for (i64 c = 0; c < d; ++c) {
                        x += q[c] * ku[c];
                        dp += g[c] * vu[c];
                    }
                    double p = exp(scale * x - lse[bh * T + t]);
                    double ds = p * (dp - Dt[bh * T + t]);
                    for (i64 c = 0; c < d; ++c) out[c] += scale * ds * ku[c];
                }
            }
        }
        free(pos);
    }

    /* dK, dV rows: every query of every head of a key head's group scatters into the keys of
     * S(t); each thread keeps its own accumulators, summed at the end. */
    for (i64 kh = 0; kh < BHk; ++kh) {
#pragma omp parallel
        {
            i64 *pos = (i64 *)malloc(sizeof(i64) * (size_t)T);
            double *ak = (double *)calloc((size_t)(nK * d), sizeof(double));
            double *av = (double *)calloc((size_t)(nK * d), sizeof(double));
#pragma omp for schedule(dynamic, 16)
            for (i64 gt = 0; gt < G * T; ++gt) {
                const i64 bh = kh * G + gt / T, t = gt % T;
                const int32_t *sel_row = idx ? idx + (kh * T + t) * k : NULL;
                const double *q = Q + (bh * T + t) * d, *g = dO + (bh * T + t) * d;
                i64 n = attended_set(sel_row, k, s, t, pos);
                for (i64 a = 0; a < n; ++a) {
                    i64 r = kslot[pos[a]];
                    if (r < 0) continue;
                    const double *ku = K + (kh * T + pos[a]) * d, *vu = V + (kh * T + pos[a]) * d;
                    double x = 0.0, dp = 0.0;
                    for (i64 c = 0; c < d; ++c) {
                        x += q[c] * ku[c];
                        dp += g[c] * vu[c];
                    }
                    double p = exp(scale * x - lse[bh * T + t]);
                    double ds = p * (dp - Dt[bh * T + t]);
                    for (i64 c = 0; c < d; ++c) {
                        ak[r * d + c] += scale * ds * q[c];
                        av[r * d + c] += p * g[c];
                    }
                }
            }
#pragma omp critical
            {
                for (i64 e = 0; e < nK * d; ++e) {
                    dK[kh * nK * d + e] += ak[e];
                    dV[kh * nK * d + e] += av[e];
                }
            }
            free(pos);
            free(ak);
            free(av);
        }
    }
    free(lse);
    free(Dt);
    free(kslot);
}

/* ---------------------------------------------------------------------------
 * Rotary position embedding -- page section 6 and Appendix K: the model's
 * queries and keys carry rotary positions, and continued training at 32k uses
 * "RoPE scaling factor 4", which stretches the rotation periods.  The pages
 * print neither the rotation nor the base.  Reading: the rotate-half form, pairs
 * (x_i, x_{i+d/2}) for i < d/2 turned by the angle
 *   a(t, i) = (pos0 + t) * base^(-2i/d) / factor
 * (factor 4 divides every frequency by 4, i.e. positions are interpolated);
 * inverse != 0 turns by -a (the transpose, which carries gradients back).
 * X is [rows, d] with rows = heads * T (row r is position r % T); out may be X.
 * ------------------------------------------------------------------------- */
void ora_rope(i64 rows, i64 T, i64 d, const double *X, i64 pos0, double base, double factor, int inverse,
              double *out) {
    i64 h = d / 2;
#pragma omp parallel for schedule(static)
    for (i64 r = 0; r < rows; ++r) {
        double t = (double)(pos0 + r % T);
        for (i64 i = 0; i < h; ++i) {
            double a = t * pow(base, -2.0 * (double)i / (double)d) / factor;
            if (inverse) a = -a;
            double c = cos(a), sn = sin(a);
            double x0 = X[r * d + i], x1 = X[r * d + i + h];
            out[r * d + i] = x0 * c - x1 * sn;
            out[r * d + i + h] = x0 * sn + x1 * c;
        }
    }
}

/* ---------------------------------------------------------------------------
 * Bidirectional alignment -- page section 5: full-attention outputs are pulled
 * toward the sparse ones (sparsity term, stop-gradient on o_s), a commitment
 * term keeps the sparse outputs near the full ones (stop-gradient on o_f), both
 * SmoothL1, weighted.  Reading: beta-SmoothL1, mean over all n elements.
 *   huber(x) = 0.5 x^2 / beta  if |x| < beta,  |x| - 0.5 beta  otherwise
 *   L = w_s * mean huber(o_f - o_s) + w_c * mean huber(o_s - o_f)
 * ------------------------------------------------------------------------- */
static double huber(double x, double beta) {
    double a = fabs(x);
    return a < beta ? 0.5 * x * x / beta : a - 0.5 * beta;
}

static double huber_slope(double x, double beta) {
    if (fabs(x) < beta) return x / beta;
    return x > 0 ? 1.0 : -1.0;
}

/* Adjusted L2 variant -- page section 7.5 (ablation, Table 3: an "adjusted L2"
 * alignment in place of SmoothL1; the pages do not print it).  Reading: the
 * quadratic branch of the SmoothL1 above kept for every x,
 *   l2adj(x) = 0.5 x^2 / beta,
 * which equals SmoothL1 wherever |x| < beta, so the weights need no retuning. */
static double l2adj(double x, double beta) { return 0.5 * x * x / beta; }

static double l2adj_slope(double x, double beta) { return x / beta; }

/* kind 0: SmoothL1 (the default of section 5); kind 1: adjusted L2. */
static double align_elem(int kind, double x, double beta) { return kind ? l2adj(x, beta) : huber(x, beta); }

static double align_slope(int kind, double x, double beta) {
    return kind ? l2adj_slope(x, beta) : huber_slope(x, beta);
}

double ora_align_fwd(i64 n, const double *of, const double *os, double beta, double w_s, double w_c, int kind) {
    double a = 0.0, b = 0.0;
    for (i64 i = 0; i < n; ++i) {
        a += align_elem(kind, of[i] - os[i], beta);
        b += align_elem(kind, os[i] - of[i], beta);
    }
    return w_s * a / (double)n + w_c * b / (double)n;
}

/* dL/do_f = g * w_s * loss'(o_f - o_s) / n   (o_s is a constant in the sparsity term)
 * dL/do_s = g * w_c * loss'(o_s - o_f) / n   (o_f is a constant in the commitment term) */
void ora_align_bwd(i64 n, const double *of, const double *os, double beta, double w_s, double w_c, double g,
                   double *dof, double *dos, int kind) {
    for (i64 i = 0; i < n; ++i) {
        dof[i] = g * w_s * align_slope(kind, of[i] - os[i], beta) / (double)n;
        dos[i] = g * w_c * align_slope(kind, os[i] - of[i], beta) / (double)n;
    }
}
