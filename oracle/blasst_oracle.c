/*
 * CPU oracle for the BLASST attention forward -- TEST INFRASTRUCTURE ONLY.
 * See blasst_oracle.h for what is computed, the passages followed and the
 * readings taken where the pages are silent.
 *
 * Plain loops in float64: no blocking, fusion or reordering beyond the
 * blockwise order the algorithm itself prescribes.  OpenMP only distributes
 * independent query tiles (prefill) or (sequence, KV head) pairs (decode)
 * over threads; it does not change any arithmetic.
 */
#include "blasst_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double oracle_bf16_to_double(uint16_t h) {
    /* A bfloat16 is the upper half of an IEEE binary32 value. */
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_split_begin(int nk, int S, int s) {
    return (int)(((int64_t)s * nk) / S);
}

/*
 * One query tile against KV blocks [j0, j1) of one KV head.
 *
 * The tile's rows are the query vectors qrows[r] (already converted to
 * float64); row r may attend to keys first[r]..limit[r] (inclusive; first
 * may be NULL, meaning 0).  State m, l, acc is the blockwise online-softmax
 * state, initialised here.
 *
 * Block j (keys c in [j*Bc, min((j+1)*Bc, Lkv))):
 *   S[r][c]  = scale * q_r . k_c, or -inf when c > limit[r] or c < first[r]
 *   visited  = some S[r][c] is finite
 *   mt[r]    = max_c S[r][c]                         (block-local row max)
 *   skip     = ln_lambda > -inf and for every row:  mt[r] == -inf  or
 *              mt[r] - m[r] < ln_lambda              (criterion, per tile)
 *   kept     : m_new = max(m, mt); alpha = exp(m - m_new);
 *              p = exp(S - m_new); l = alpha*l + sum p;
 *              acc = alpha*acc + sum_c p_c v_c;  m = m_new
 *   skipped  : no exp, no V, no P.V; m, l, acc unchanged
 */
static void run_tile(int nrows, const double *qrows, const int *first,
                     const int *limit, const uint16_t *kh, const uint16_t *vh, int Lkv, int d,
                     double scale, double ln_lambda, int Bc, int j0, int j1,
                     double *m, double *l, double *acc, uint8_t *mask,
                     double *margin, int64_t *n_visited, int64_t *n_skipped) {
    double *S = (double *)malloc(sizeof(double) * (size_t)nrows * Bc);
    double *mt = (double *)malloc(sizeof(double) * (size_t)nrows);
    double *kd = (double *)malloc(sizeof(double) * (size_t)Bc * d);
    double *vd = (double *)malloc(sizeof(double) * (size_t)Bc * d);

    for (int r = 0; r < nrows; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.0;
        for (int x = 0; x < d; ++x) acc[(size_t)r * d + x] = 0.0;
    }

    for (int j = j0; j < j1; ++j) {
        int c0 = j * Bc;
        int c1 = c0 + Bc < Lkv ? c0 + Bc : Lkv;
        int nc = c1 - c0;

        /* Is any entry of this (tile, block) pair unmasked? */
        int visited = 0;
        for (int r = 0; r < nrows; ++r) {
            int lo = first ? first[r] : 0;
            if (lo < c0) lo = c0;
            int hi = limit[r] < c1 - 1 ? limit[r] : c1 - 1;
            if (lo <= hi) visited = 1;
        }
        if (!visited) {
            if (mask) mask[j] = ORACLE_NOT_VISITED;
            if (margin) margin[j] = NAN;
            continue;
        }
        *n_visited += 1;

        /* K block, then scores and block-local row max. */
        for (int c = 0; c < nc; ++c)
            for (int x = 0; x < d; ++x)
                kd[(size_t)c * d + x] =
                    oracle_bf16_to_double(kh[(size_t)(c0 + c) * d + x]);
        for (int r = 0; r < nrows; ++r) {
            mt[r] = -INFINITY;
            for (int c = 0; c < nc; ++c) {
                double s;
                if (c0 + c > limit[r] || (first && c0 + c < first[r])) {
                    s = -INFINITY;
                } else {
                    double dot = 0.0;
                    for (int x = 0; x < d; ++x)
                        dot += qrows[(size_t)r * d + x] * kd[(size_t)c * d + x];
                    s = scale * dot;
                }
                S[(size_t)r * Bc + c] = s;
                if (s > mt[r]) mt[r] = s;
            }
        }

        /* Skip criterion: every row's block max lies more than |ln lambda|
         * below its running max. */
        int skip = ln_lambda > -INFINITY;
        double mu = -INFINITY;
        for (int r = 0; r < nrows; ++r) {
            if (mt[r] == -INFINITY) continue; /* fully masked row: no vote */
            double diff = mt[r] - m[r];       /* +inf while m = -inf */
            if (!(diff < ln_lambda)) skip = 0;
            if (diff > mu) mu = diff;
        }
        if (margin) margin[j] = mu - ln_lambda;
        if (skip) {
            *n_skipped += 1;
            if (mask) mask[j] = ORACLE_SKIPPED;
            continue;
        }
        if (mask) mask[j] = ORACLE_KEPT;

        /* Kept block: exp, V load and P.V product. */
        for (int c = 0; c < nc; ++c)
            for (int x = 0; x < d; ++x)
                vd[(size_t)c * d + x] =
                    oracle_bf16_to_double(vh[(size_t)(c0 + c) * d + x]);
        for (int r = 0; r < nrows; ++r) {
            if (mt[r] == -INFINITY) continue; /* p = 0, alpha = 1 */
            double m_new = m[r] > mt[r] ? m[r] : mt[r];
            double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - m_new);
            double psum = 0.0;
            double *a = acc + (size_t)r * d;
            for (int x = 0; x < d; ++x) a[x] *= alpha;
            for (int c = 0; c < nc; ++c) {
                double s = S[(size_t)r * Bc + c];
                if (s == -INFINITY) continue;
                double p = exp(s - m_new);
                psum += p;
                for (int x = 0; x < d; ++x) a[x] += p * vd[(size_t)c * d + x];
            }
            l[r] = alpha * l[r] + psum;
            m[r] = m_new;
        }
    }
    free(S);
    free(mt);
    free(kd);
    free(vd);
}

static int set_threads(int n_threads);

/*
 * One decode tile (the G heads of a KV head, every key visible) against
 * blocks [j0, j1) with the batched decision rule ("batched load
 * scheduling": the Q.K products of a batch of `batch` consecutive blocks are
 * formed before any of their V loads is decided).  Per batch
 * [jb, min(jb + batch, j1)):
 *   mt[r](j)  block-local row maxima of every block of the batch
 *   Mb[r]     = max(M[r], max over the batch of mt[r](j)), M[r] the max over
 *               all blocks before the batch (-inf at the start)
 *   skip(j)   = ln_lambda > -inf and for every row mt[r](j) - Mb[r] < ln_lambda
 *   kept j    : the online-softmax update of run_tile (m is the max over
 *               kept blocks, the reference of l and acc)
 *   M[r]      = Mb[r] after the batch.
 * With batch = 1, Mb = max(M, mt(j)) and the decisions are run_tile's.
 * margin[j] = max_r(mt[r](j) - Mb[r]) - ln_lambda.
 */
static void run_tile_batched(int nrows, const double *qrows,
                             const uint16_t *kh, const uint16_t *vh, int Lkv,
                             int d, double scale, double ln_lambda, int Bc,
                             int j0, int j1, int batch, double *m, double *l,
                             double *acc, uint8_t *mask, double *margin,
                             int64_t *n_visited, int64_t *n_skipped) {
    double *S = (double *)malloc(sizeof(double) * (size_t)batch * nrows * Bc);
    double *mt = (double *)malloc(sizeof(double) * (size_t)batch * nrows);
    double *M = (double *)malloc(sizeof(double) * (size_t)nrows);
    double *Mb = (double *)malloc(sizeof(double) * (size_t)nrows);
    double *vd = (double *)malloc(sizeof(double) * (size_t)Bc * d);

    for (int r = 0; r < nrows; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.0;
        M[r] = -INFINITY;
        for (int x = 0; x < d; ++x) acc[(size_t)r * d + x] = 0.0;
    }
    for (int jb = j0; jb < j1; jb += batch) {
        int je = jb + batch < j1 ? jb + batch : j1;
        /* 1. scores and block maxima of the whole batch */
        for (int j = jb; j < je; ++j) {
            int c0 = j * Bc;
            int nc = (c0 + Bc < Lkv ? c0 + Bc : Lkv) - c0;
            double *Sj = S + (size_t)(j - jb) * nrows * Bc;
            double *mj = mt + (size_t)(j - jb) * nrows;
            for (int r = 0; r < nrows; ++r) {
                mj[r] = -INFINITY;
                for (int c = 0; c < nc; ++c) {
                    double dot = 0.0;
                    for (int x = 0; x < d; ++x)
                        dot += qrows[(size_t)r * d + x] *
                               oracle_bf16_to_double(kh[(size_t)(c0 + c) * d + x]);
                    double sc = scale * dot;
                    Sj[(size_t)r * Bc + c] = sc;
                    if (sc > mj[r]) mj[r] = sc;
                }
            }
        }
        /* 2. the batch's criterion max */
        for (int r = 0; r < nrows; ++r) {
            Mb[r] = M[r];
            for (int j = jb; j < je; ++j) {
                double v = mt[(size_t)(j - jb) * nrows + r];
                if (v > Mb[r]) Mb[r] = v;
            }
        }
        /* 3. decisions in block order; kept blocks update the state */
        for (int j = jb; j < je; ++j) {
            int c0 = j * Bc;
            int nc = (c0 + Bc < Lkv ? c0 + Bc : Lkv) - c0;
            const double *Sj = S + (size_t)(j - jb) * nrows * Bc;
            const double *mj = mt + (size_t)(j - jb) * nrows;
            *n_visited += 1;
            int skip = ln_lambda > -INFINITY;
            double mu = -INFINITY;
            for (int r = 0; r < nrows; ++r) {
                double diff = mj[r] - Mb[r];
                if (!(diff < ln_lambda)) skip = 0;
                if (diff > mu) mu = diff;
            }
            if (margin) margin[j] = mu - ln_lambda;
            if (skip) {
                *n_skipped += 1;
                if (mask) mask[j] = ORACLE_SKIPPED;
                continue;
            }
            if (mask) mask[j] = ORACLE_KEPT;
            for (int c = 0; c < nc; ++c)
                for (int x = 0; x < d; ++x)
                    vd[(size_t)c * d + x] =
                        oracle_bf16_to_double(vh[(size_t)(c0 + c) * d + x]);
            for (int r = 0; r < nrows; ++r) {
                double m_new = m[r] > mj[r] ? m[r] : mj[r];
                double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - m_new);
                double psum = 0.0;
                double *a = acc + (size_t)r * d;
                for (int x = 0; x < d; ++x) a[x] *= alpha;
                for (int c = 0; c < nc; ++c) {
                    double p = exp(Sj[(size_t)r * Bc + c] - m_new);
                    psum += p;
                    for (int x = 0; x < d; ++x) a[x] += p * vd[(size_t)c * d + x];
                }
                l[r] = alpha * l[r] + psum;
                m[r] = m_new;
            }
        }
        for (int r = 0; r < nrows; ++r) M[r] = Mb[r];
    }
    free(S);
    free(mt);
    free(M);
    free(Mb);
    free(vd);
}

int oracle_decode_batched(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int Hq, int Hkv, int Lkv,
                          int d, double scale, double ln_lambda, int Bc,
                          int num_splits, int batch, double *o, double *lse,
                          double *o_part, double *lse_part, uint8_t *mask,
                          double *margin, int64_t *counts, int n_threads) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || Lkv < 1 || d < 1 ||
        Bc < 1 || num_splits < 1 || batch < 1 || !(ln_lambda <= 0.0))
        return -1;
    int nk = (Lkv + Bc - 1) / Bc;
    int G = Hq / Hkv;
    int S = num_splits;
    double *op = (double *)malloc(sizeof(double) * (size_t)B * Hq * S * d);
    double *lp = (double *)malloc(sizeof(double) * (size_t)B * Hq * S);
    set_threads(n_threads);
    int64_t vis = 0, skp = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : vis, skp)
    for (int bh = 0; bh < B * Hkv; ++bh) {
        int b = bh / Hkv, hkv = bh % Hkv;
        double *qrows = (double *)malloc(sizeof(double) * (size_t)G * d);
        double *m = (double *)malloc(sizeof(double) * (size_t)G);
        double *l = (double *)malloc(sizeof(double) * (size_t)G);
        double *acc = (double *)malloc(sizeof(double) * (size_t)G * d);
        for (int g = 0; g < G; ++g) {
            const uint16_t *qg = q + ((size_t)b * Hq + hkv * G + g) * d;
            for (int x = 0; x < d; ++x)
                qrows[(size_t)g * d + x] = oracle_bf16_to_double(qg[x]);
        }
        const uint16_t *kh = k + (size_t)bh * Lkv * d;
        const uint16_t *vh = v + (size_t)bh * Lkv * d;
        uint8_t *mk = mask ? mask + (size_t)bh * nk : NULL;
        double *mg = margin ? margin + (size_t)bh * nk : NULL;
        for (int s = 0; s < S; ++s) {
            int j0 = oracle_split_begin(nk, S, s);
            int j1 = oracle_split_begin(nk, S, s + 1);
            int64_t uv = 0, us = 0;
            run_tile_batched(G, qrows, kh, vh, Lkv, d, scale, ln_lambda, Bc,
                             j0, j1, batch, m, l, acc, mk, mg, &uv, &us);
            vis += uv;
            skp += us;
            for (int g = 0; g < G; ++g) {
                size_t row = ((size_t)b * Hq + hkv * G + g) * S + s;
                if (l[g] > 0.0) {
                    for (int x = 0; x < d; ++x)
                        op[row * d + x] = acc[(size_t)g * d + x] / l[g];
                    lp[row] = m[g] + log(l[g]);
                } else { /* empty split */
                    for (int x = 0; x < d; ++x) op[row * d + x] = 0.0;
                    lp[row] = -INFINITY;
                }
            }
        }
        free(qrows);
        free(m);
        free(l);
        free(acc);
    }
    oracle_combine(op, lp, B * Hq, S, d, o, lse);
    if (o_part) memcpy(o_part, op, sizeof(double) * (size_t)B * Hq * S * d);
    if (lse_part) memcpy(lse_part, lp, sizeof(double) * (size_t)B * Hq * S);
    free(op);
    free(lp);
    counts[0] = vis;
    counts[1] = skp;
    return 0;
}

static int set_threads(int n_threads) {
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
    return omp_get_max_threads();
#else
    (void)n_threads;
    return 1;
#endif
}

int oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   int B, int Hq, int Hkv, int Lq, int Lkv, int d,
                   double scale, int causal, double ln_lambda, int Br, int Bc,
                   int n_units, const int32_t *units,
                   double *o, double *lse, uint8_t *mask, double *margin,
                   int64_t *counts, int n_threads) {
    return oracle_prefill_window(q, k, v, B, Hq, Hkv, Lq, Lkv, d, scale,
                                 causal, 0, ln_lambda, Br, Bc, n_units, units,
                                 o, lse, mask, margin, counts, n_threads);
}

int oracle_prefill_window(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int B, int Hq, int Hkv, int Lq,
                          int Lkv, int d, double scale, int causal,
                          int window, double ln_lambda, int Br, int Bc,
                          int n_units, const int32_t *units, double *o,
                          double *lse, uint8_t *mask, double *margin,
                          int64_t *counts, int n_threads) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || Lq < 1 || Lkv < 1 ||
        d < 1 || Br < 1 || Bc < 1 || n_units < 0 || !(ln_lambda <= 0.0) ||
        window < 0 || (window > 0 && !causal))
        return -1;
    int nq = (Lq + Br - 1) / Br;
    int nk = (Lkv + Bc - 1) / Bc;
    int G = Hq / Hkv;
    for (int u = 0; u < n_units; ++u) {
        int b = units[3 * u], hq = units[3 * u + 1], i = units[3 * u + 2];
        if (b < 0 || b >= B || hq < 0 || hq >= Hq || i < 0 || i >= nq)
            return -1;
    }
    set_threads(n_threads);
    int64_t vis = 0, skp = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : vis, skp)
    for (int u = 0; u < n_units; ++u) {
        int b = units[3 * u], hq = units[3 * u + 1], i = units[3 * u + 2];
        int hkv = hq / G;
        int r0 = i * Br;
        int r1 = r0 + Br < Lq ? r0 + Br : Lq;
        int nrows = r1 - r0;
        double *qrows = (double *)malloc(sizeof(double) * (size_t)nrows * d);
        int *limit = (int *)malloc(sizeof(int) * (size_t)nrows);
        int *first = (int *)malloc(sizeof(int) * (size_t)nrows);
        double *m = (double *)malloc(sizeof(double) * (size_t)nrows);
        double *l = (double *)malloc(sizeof(double) * (size_t)nrows);
        double *acc = (double *)malloc(sizeof(double) * (size_t)nrows * d);
        const uint16_t *qh = q + ((size_t)b * Hq + hq) * (size_t)Lq * d;
        const uint16_t *kh = k + ((size_t)b * Hkv + hkv) * (size_t)Lkv * d;
        const uint16_t *vh = v + ((size_t)b * Hkv + hkv) * (size_t)Lkv * d;
        for (int r = 0; r < nrows; ++r) {
            for (int x = 0; x < d; ++x)
                qrows[(size_t)r * d + x] =
                    oracle_bf16_to_double(qh[(size_t)(r0 + r) * d + x]);
            int lim = Lkv - 1;
            int lo = 0;
            if (causal) {
                int diag = r0 + r + (Lkv - Lq); /* bottom-right alignment */
                if (diag < lim) lim = diag;
                /* sliding window: the `window` keys ending at the diagonal */
                if (window > 0 && diag - window + 1 > 0) lo = diag - window + 1;
            }
            limit[r] = lim;
            first[r] = lo;
        }
        int64_t uv = 0, us = 0;
        run_tile(nrows, qrows, first, limit, kh, vh, Lkv, d, scale, ln_lambda, Bc, 0,
                 nk, m, l, acc, mask ? mask + (size_t)u * nk : NULL,
                 margin ? margin + (size_t)u * nk : NULL, &uv, &us);
        vis += uv;
        skp += us;
        double *ou = o + (size_t)u * Br * d;
        double *lu = lse + (size_t)u * Br;
        for (int r = 0; r < Br; ++r) {
            if (r < nrows && l[r] > 0.0) {
                for (int x = 0; x < d; ++x)
                    ou[(size_t)r * d + x] = acc[(size_t)r * d + x] / l[r];
                lu[r] = m[r] + log(l[r]);
            } else {
                for (int x = 0; x < d; ++x) ou[(size_t)r * d + x] = 0.0;
                lu[r] = -INFINITY;
            }
        }
        free(qrows);
        free(limit);
        free(first);
        free(m);
        free(l);
        free(acc);
    }
    counts[0] = vis;
    counts[1] = skp;
    return 0;
}

void oracle_combine(const double *o_part, const double *lse_part, int n,
                    int S, int d, double *o, double *lse) {
    for (int i = 0; i < n; ++i) {
        const double *ls = lse_part + (size_t)i * S;
        const double *os = o_part + (size_t)i * S * d;
        double mx = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (ls[s] > mx) mx = ls[s];
        double *oi = o + (size_t)i * d;
        for (int x = 0; x < d; ++x) oi[x] = 0.0;
        if (mx == -INFINITY) {
            lse[i] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int s = 0; s < S; ++s) sum += exp(ls[s] - mx);
        double L = mx + log(sum);
        lse[i] = L;
        for (int s = 0; s < S; ++s) {
            if (ls[s] == -INFINITY) continue;
            double w = exp(ls[s] - L);
            for (int x = 0; x < d; ++x) oi[x] += w * os[(size_t)s * d + x];
        }
    }
}

int oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  int B, int Hq, int Hkv, int Lkv, int d, double scale,
                  double ln_lambda, int Bc, int num_splits,
                  double *o, double *lse, double *o_part, double *lse_part,
                  uint8_t *mask, double *margin, int64_t *counts,
                  int n_threads) {
    return oracle_decode_window(q, k, v, B, Hq, Hkv, Lkv, d, scale, 0,
                                ln_lambda, Bc, num_splits, o, lse, o_part,
                                lse_part, mask, margin, counts, n_threads);
}

int oracle_decode_window(const uint16_t *q, const uint16_t *k,
                         const uint16_t *v, int B, int Hq, int Hkv, int Lkv,
                         int d, double scale, int window, double ln_lambda,
                         int Bc, int num_splits, double *o, double *lse,
                         double *o_part, double *lse_part, uint8_t *mask,
                         double *margin, int64_t *counts, int n_threads) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || Lkv < 1 || d < 1 ||
        Bc < 1 || num_splits < 1 || !(ln_lambda <= 0.0) || window < 0)
        return -1;
    int nk = (Lkv + Bc - 1) / Bc;
    /* sliding window: the decode token (position Lkv - 1) sees the last
     * `window` keys; the splits divide the blocks that hold them */
    int key_lo = (window > 0 && Lkv - window > 0) ? Lkv - window : 0;
    int jlo = key_lo / Bc;
    int G = Hq / Hkv;
    int S = num_splits;
    double *op = (double *)malloc(sizeof(double) * (size_t)B * Hq * S * d);
    double *lp = (double *)malloc(sizeof(double) * (size_t)B * Hq * S);
    set_threads(n_threads);
    int64_t vis = 0, skp = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : vis, skp)
    for (int bh = 0; bh < B * Hkv; ++bh) {
        int b = bh / Hkv, hkv = bh % Hkv;
        double *qrows = (double *)malloc(sizeof(double) * (size_t)G * d);
        int *limit = (int *)malloc(sizeof(int) * (size_t)G);
        int *first = (int *)malloc(sizeof(int) * (size_t)G);
        double *m = (double *)malloc(sizeof(double) * (size_t)G);
        double *l = (double *)malloc(sizeof(double) * (size_t)G);
        double *acc = (double *)malloc(sizeof(double) * (size_t)G * d);
        for (int g = 0; g < G; ++g) {
            const uint16_t *qg = q + ((size_t)b * Hq + hkv * G + g) * d;
            for (int x = 0; x < d; ++x)
                qrows[(size_t)g * d + x] = oracle_bf16_to_double(qg[x]);
            limit[g] = Lkv - 1; /* the decode token sees the whole cache */
            first[g] = key_lo;  /* ... or its last `window` keys */
        }
        if (mask)
            for (int j = 0; j < jlo; ++j)
                mask[(size_t)bh * nk + j] = ORACLE_NOT_VISITED;
        if (margin)
            for (int j = 0; j < jlo; ++j) margin[(size_t)bh * nk + j] = NAN;
        const uint16_t *kh = k + (size_t)bh * Lkv * d;
        const uint16_t *vh = v + (size_t)bh * Lkv * d;
        uint8_t *mk = mask ? mask + (size_t)bh * nk : NULL;
        double *mg = margin ? margin + (size_t)bh * nk : NULL;
        for (int s = 0; s < S; ++s) {
            int j0 = jlo + oracle_split_begin(nk - jlo, S, s);
            int j1 = jlo + oracle_split_begin(nk - jlo, S, s + 1);
            int64_t uv = 0, us = 0;
            run_tile(G, qrows, first, limit, kh, vh, Lkv, d, scale, ln_lambda,
                     Bc, j0, j1, m, l, acc, mk, mg, &uv, &us);
            vis += uv;
            skp += us;
            for (int g = 0; g < G; ++g) {
                size_t row = ((size_t)b * Hq + hkv * G + g) * S + s;
                if (l[g] > 0.0) {
                    for (int x = 0; x < d; ++x)
                        op[row * d + x] = acc[(size_t)g * d + x] / l[g];
                    lp[row] = m[g] + log(l[g]);
                } else { /* empty split */
                    for (int x = 0; x < d; ++x) op[row * d + x] = 0.0;
                    lp[row] = -INFINITY;
                }
            }
        }
        free(qrows);
        free(limit);
        free(first);
        free(m);
        free(l);
        free(acc);
    }
    oracle_combine(op, lp, B * Hq, S, d, o, lse);
    if (o_part) memcpy(o_part, op, sizeof(double) * (size_t)B * Hq * S * d);
    if (lse_part) memcpy(lse_part, lp, sizeof(double) * (size_t)B * Hq * S);
    free(op);
    free(lp);
    counts[0] = vis;
    counts[1] = skp;
    return 0;
}

/*
 * Paged, variable-length decode.  The logical cache of (sequence b, KV head
 * h) is gathered from the page pool token by token -- token t of sequence b
 * is row (h * page_size + t % page_size) of page
 * block_table[b * max_pages + t / page_size] -- and then decoded exactly as
 * oracle_decode decodes a contiguous cache of length seq_lens[b].
 */
int oracle_decode_paged(const uint16_t *q, const uint16_t *k_pool,
                        const uint16_t *v_pool, int64_t page_stride,
                        int num_pages, int page_size,
                        const int32_t *block_table, int max_pages,
                        const int32_t *seq_lens, int B, int Hq, int Hkv, int d,
                        double scale, double ln_lambda, int per_length, int Bc,
                        int num_splits, int nk_max, double *o, double *lse,
                        double *o_part, double *lse_part, uint8_t *mask,
                        double *margin, int64_t *counts, int n_threads) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || Bc < 1 ||
        num_splits < 1 || page_size < 1 || num_pages < 0 || max_pages < 0 ||
        nk_max < 0 || isnan(ln_lambda) || ln_lambda == INFINITY ||
        (!per_length && ln_lambda > 0.0) ||
        page_stride < (int64_t)Hkv * page_size * d)
        return -1;
    /* Every length and every page id the lengths reach must be valid. */
    for (int b = 0; b < B; ++b) {
        int L = seq_lens[b];
        if (L < 0 || (int64_t)L > (int64_t)max_pages * page_size ||
            (L + Bc - 1) / Bc > nk_max)
            return -1;
        for (int p = 0; p < (L + page_size - 1) / page_size; ++p) {
            int id = block_table[(size_t)b * max_pages + p];
            if (id < 0 || id >= num_pages) return -1;
        }
    }
    int G = Hq / Hkv;
    int S = num_splits;
    double *op = (double *)malloc(sizeof(double) * (size_t)B * Hq * S * d);
    double *lp = (double *)malloc(sizeof(double) * (size_t)B * Hq * S);
    if (mask) memset(mask, ORACLE_NOT_VISITED, (size_t)B * Hkv * nk_max);
    if (margin)
        for (size_t i = 0; i < (size_t)B * Hkv * nk_max; ++i) margin[i] = NAN;
    set_threads(n_threads);
    int64_t vis = 0, skp = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(+ : vis, skp)
    for (int bh = 0; bh < B * Hkv; ++bh) {
        int b = bh / Hkv, hkv = bh % Hkv;
        int L = seq_lens[b];
        int nk = (L + Bc - 1) / Bc;
        /* lambda = a / L with L this sequence's own context length */
        double lnl = ln_lambda;
        if (per_length && L > 0 && ln_lambda > -INFINITY) {
            lnl = ln_lambda - log((double)L);
            if (lnl > 0.0) lnl = 0.0;
        }
        /* gather the logical K and V rows of (b, hkv) */
        uint16_t *kh = (uint16_t *)malloc(sizeof(uint16_t) * ((size_t)L * d + 1));
        uint16_t *vh = (uint16_t *)malloc(sizeof(uint16_t) * ((size_t)L * d + 1));
        for (int t = 0; t < L; ++t) {
            int id = block_table[(size_t)b * max_pages + t / page_size];
            size_t src = (size_t)id * page_stride +
                         ((size_t)hkv * page_size + t % page_size) * d;
            memcpy(kh + (size_t)t * d, k_pool + src, sizeof(uint16_t) * d);
            memcpy(vh + (size_t)t * d, v_pool + src, sizeof(uint16_t) * d);
        }
        double *qrows = (double *)malloc(sizeof(double) * (size_t)G * d);
        int *limit = (int *)malloc(sizeof(int) * (size_t)G);
        double *m = (double *)malloc(sizeof(double) * (size_t)G);
        double *l = (double *)malloc(sizeof(double) * (size_t)G);
        double *acc = (double *)malloc(sizeof(double) * (size_t)G * d);
        for (int g = 0; g < G; ++g) {
            const uint16_t *qg = q + ((size_t)b * Hq + hkv * G + g) * d;
            for (int x = 0; x < d; ++x)
                qrows[(size_t)g * d + x] = oracle_bf16_to_double(qg[x]);
            limit[g] = L - 1;
        }
        uint8_t *mk = mask ? mask + (size_t)bh * nk_max : NULL;
        double *mg = margin ? margin + (size_t)bh * nk_max : NULL;
        for (int s = 0; s < S; ++s) {
            int j0 = oracle_split_begin(nk, S, s);
            int j1 = oracle_split_begin(nk, S, s + 1);
            int64_t uv = 0, us = 0;
            run_tile(G, qrows, NULL, limit, kh, vh, L, d, scale, lnl, Bc, j0, j1, m,
                     l, acc, mk, mg, &uv, &us);
            vis += uv;
            skp += us;
            for (int g = 0; g < G; ++g) {
                size_t row = ((size_t)b * Hq + hkv * G + g) * S + s;
                if (l[g] > 0.0) {
                    for (int x = 0; x < d; ++x)
                        op[row * d + x] = acc[(size_t)g * d + x] / l[g];
                    lp[row] = m[g] + log(l[g]);
                } else { /* empty split */
                    for (int x = 0; x < d; ++x) op[row * d + x] = 0.0;
                    lp[row] = -INFINITY;
                }
            }
        }
        free(kh);
        free(vh);
        free(qrows);
        free(limit);
        free(m);
        free(l);
        free(acc);
    }
    oracle_combine(op, lp, B * Hq, S, d, o, lse);
    if (o_part) memcpy(o_part, op, sizeof(double) * (size_t)B * Hq * S * d);
    if (lse_part) memcpy(lse_part, lp, sizeof(double) * (size_t)B * Hq * S);
    free(op);
    free(lp);
    counts[0] = vis;
    counts[1] = skp;
    return 0;
}
