/*
 * dash_oracle.c -- plain, slow, fp64 CPU oracle for the DashAttention forward pass and
 * its backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this
 * file: only the tests, the smoke check and the CPU-baseline leg of the benchmark do.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *   [P1] "DashAttention: Making Sparse Attention Fully Differentiable with Adaptive
 *        Block Selection" (alanhou.org), section "Core Mechanism" (the two-stage
 *        diagram: keys and values cut into fixed blocks; coarse scores Q * block_summary; alpha-entmax
 *        gives sparse block weights p; fine logits Q * K_block plus log(p); softmax;
 *        weighted sum of V) and section "Key Concepts" (alpha-entmax; alpha=1 is
 *        softmax, alpha=2 is sparsemax; higher alpha is sparser; hierarchical prior).
 *   [P3] "DashAttention and the year sparse attention became a field", section
 *        "What alpha-entmax changes" (Stage 0 summary head initialised at zero, i.e.
 *        mean pooling; Stage 1 alpha-entmax over chunk scores; Stage 2 softmax over
 *        the routed chunks' tokens with the routing weights as a log prior;
 *        alpha = 1.5 at inference).
 *   The entmax formula p_j = [(alpha-1) s_j - tau]_+^(1/(alpha-1)) with tau such that
 *   sum_j p_j = 1 is the standard definition of alpha-entmax that [P1] and [P3] name.
 *
 * Readings where the pages are silent (stated once here, used everywhere below):
 *   - block summary = arithmetic mean of the block's keys (the zero-initialised head);
 *     with a learned head ([P3] "What alpha-entmax changes": Stage 0 is a small attention
 *     head initialised at zero), an attention pooling of the block's keys with one query
 *     vector w_g per KV head: kbar_j = sum_i softmax_i(w_g . k_i / sqrt(d)) k_i, which is
 *     the mean when w_g = 0;
 *   - only complete blocks strictly before the query's own block are scored;
 *   - coarse score s_j = coarse_scale * (q . kbar_j) / sqrt(d); fine logits use 1/sqrt(d);
 *   - the query's own block is always attended causally with prior weight 1 (log 0 prior);
 *   - query head h reads KV head floor(h / (Hq/Hkv));
 *   - a block whose x_j equals tau exactly gets weight 0 (strict ">");
 *   - head aggregation (the optional variant): the heads of a KV group average their block
 *     distributions and share the result as their prior (oracle_forward_rows_agg);
 *   - backward (oracle_backward, oracle_backward_dq_rows): the exact gradient of the
 *     forward above ([P1] "Core Mechanism" / "Key Concepts": the selection is
 *     differentiable) through the fine softmax, log p, the alpha-entmax Jacobian on the
 *     support, the coarse scores and the mean summaries; the own block has no coarse term.
 *
 * Parity pins (tests/test_oracle_pins.py): exact tau is checked against 200-step
 * bisection, brute force over supports and scipy's constrained optimiser on the
 * variational definition; alpha=2 against sparsemax; alpha->1 against softmax;
 * equal prior and T <= 2 blocks against dense causal attention (torch SDPA);
 * non-dispersiveness; a hand-derived worked example; the backward against central finite
 * differences of the fp64 forward, against torch autograd of dense attention, and through
 * two exact identities (dv rows sum to the group's dout, dk rows to zero).
 *
 * Inputs: element arrays are float32 (dtype 0), bf16 bit patterns (dtype 1, uint16) or
 * float64 (dtype 2); all are widened exactly to double.  Every routine is fp64.
 * Threads: OpenMP over independent rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG -1
#define ORC_ERR_NOMEM -2

/* ---------------------------------------------------------------- element access */

static double elem(const void* base, int dtype, long long i) {
    if (dtype == 0) return (double)((const float*)base)[i];
    if (dtype == 2) return ((const double*)base)[i];
    uint32_t u = ((uint32_t)((const uint16_t*)base)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- alpha-entmax */

/* f(tau) = sum_i [x_i - tau]_+^e, e = 1/(alpha-1).  Strictly decreasing for tau < max x. */
static double entmax_f(const double* x, long long n, double e, double tau) {
    double s = 0.0;
    for (long long i = 0; i < n; ++i) {
        double z = x[i] - tau;
        if (z > 0.0) s += pow(z, e);
    }
    return s;
}

static int cmp_desc(const void* a, const void* b) {
    double u = *(const double*)a, v = *(const double*)b;
    return (u < v) - (u > v);
}

/* Root of g(tau) = sum_{i<k} (y_i - tau)^e - 1 on [lo, hi], where g(lo) >= 0 > g(hi)
 * and all y_i >= hi, by plain bisection to the last representable digit. */
static double bisect_topk(const double* y, long long k, double e, double lo, double hi) {
    for (int it = 0; it < 400; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        double g = -1.0;
        for (long long i = 0; i < k; ++i) g += pow(y[i] - mid, e);
        if (g >= 0.0) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/*
 * Exact, sort-based threshold (x already multiplied by alpha-1).
 * With y = x sorted descending, f is a fixed polynomial-like function of tau on each
 * interval [y_(k+1), y_(k)), namely g_k(tau) = sum_{i<=k} (y_(i) - tau)^e.  The support
 * size k* is the largest k with f(y_(k)) < 1 (f(y_(k)) is non-decreasing in k), and
 * tau lies in [y_(k*+1), y_(k*)).  On that interval tau is the root of g_k*:
 *   alpha = 2   : tau = (sum_{i<=k} y_i - 1) / k                      (sparsemax)
 *   alpha = 1.5 : tau = mu - sqrt(mu^2 - (S2 - 1)/k), mu = S1/k         (smaller root)
 *   otherwise   : bisection of g_k* on the bracket.
 */
static double tau_sort(const double* x, long long n, double alpha) {
    double e = 1.0 / (alpha - 1.0);
    double* y = (double*)malloc((size_t)n * sizeof(double));
    if (!y) return NAN;
    memcpy(y, x, (size_t)n * sizeof(double));
    qsort(y, (size_t)n, sizeof(double), cmp_desc);
    /* binary search for k* over k in [1, n]; f(y_(k)) = sum_{i<k} (y_i - y_k)^e */
    long long lo = 1, hi = n;
    while (lo < hi) {
        long long mid = (lo + hi + 1) / 2;
        double fk = 0.0;
        for (long long i = 0; i < mid - 1; ++i) fk += pow(y[i] - y[mid - 1], e);
        if (fk < 1.0) lo = mid; else hi = mid - 1;
    }
    long long k = lo;
    double upper = y[k - 1];
    double lower = (k < n) ? y[k] : -INFINITY;
    if (lower < y[0] - 1.0) lower = y[0] - 1.0;
    double tau;
    if (alpha == 2.0) {
        double s1 = 0.0;
        for (long long i = 0; i < k; ++i) s1 += y[i];
        tau = (s1 - 1.0) / (double)k;
    } else if (alpha == 1.5) {
        double s1 = 0.0, s2 = 0.0;
        for (long long i = 0; i < k; ++i) { s1 += y[i]; s2 += y[i] * y[i]; }
        double mu = s1 / (double)k;
        double disc = mu * mu - (s2 - 1.0) / (double)k;
        if (disc < 0.0) disc = 0.0;
        tau = mu - sqrt(disc);
    } else {
        tau = bisect_topk(y, k, e, lower, upper);
    }
    /* the closed forms are exact up to rounding; keep tau inside its bracket */
    if (tau > upper) tau = upper;
    if (tau < lower) tau = lower;
    free(y);
    return tau;
}

/* 200-step bisection of f(tau) - 1 on [max x - 1, max x]. */
static double tau_bisect(const double* x, long long n, double alpha, int iters) {
    double e = 1.0 / (alpha - 1.0);
    double m = -INFINITY;
    for (long long i = 0; i < n; ++i) if (x[i] > m) m = x[i];
    double lo = m - 1.0, hi = m;
    for (int it = 0; it < iters; ++it) {
        double mid = 0.5 * (lo + hi);
        if (entmax_f(x, n, e, mid) >= 1.0) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Brute force over every nonempty support S (n <= 20): tau_S solves
 * sum_{i in S} (x_i - tau)^e = 1 with tau below min_S x; keep the S whose own
 * support {i : x_i > tau_S} equals S.  Returns NAN if none or more than one qualifies. */
static double tau_brute(const double* x, long long n, double alpha) {
    if (n < 1 || n > 20) return NAN;
    double e = 1.0 / (alpha - 1.0);
    double found = NAN;
    int nfound = 0;
    double* ys = (double*)malloc((size_t)n * sizeof(double));
    if (!ys) return NAN;
    for (unsigned long mask = 1; mask < (1ul << n); ++mask) {
        long long k = 0;
        double mn = INFINITY, mx = -INFINITY;
        for (long long i = 0; i < n; ++i) if (mask & (1ul << i)) {
            ys[k++] = x[i];
            if (x[i] < mn) mn = x[i];
            if (x[i] > mx) mx = x[i];
        }
        /* need g(mn) < 1, i.e. the root lies strictly below min_S */
        double gmn = 0.0;
        for (long long i = 0; i < k; ++i) gmn += pow(ys[i] - mn, e);
        if (gmn >= 1.0) continue;
        double t = bisect_topk(ys, k, e, mx - 1.0, mn);
        int ok = 1;
        for (long long i = 0; i < n && ok; ++i) {
            int in = (mask & (1ul << i)) != 0;
            if (in != (x[i] > t)) ok = 0;
        }
        if (ok) { found = t; ++nfound; }
    }
    free(ys);
    return nfound == 1 ? found : NAN;
}

/* Public: tau for scores s (x = (alpha-1) s).  method 0 sort, 1 bisection, 2 brute force. */
int oracle_entmax_tau(const double* s, long long n, double alpha, int method, double* tau_out) {
    if (!s || !tau_out || n < 1 || !(alpha > 1.0)) return ORC_ERR_ARG;
    double* x = (double*)malloc((size_t)n * sizeof(double));
    if (!x) return ORC_ERR_NOMEM;
    for (long long i = 0; i < n; ++i) x[i] = (alpha - 1.0) * s[i];
    double t;
    if (method == 0) t = tau_sort(x, n, alpha);
    else if (method == 1) t = tau_bisect(x, n, alpha, 200);
    else if (method == 2) t = tau_brute(x, n, alpha);
    else { free(x); return ORC_ERR_ARG; }
    free(x);
    *tau_out = t;
    return ORC_OK;
}

/* Public: p = alpha-entmax(s), p_j = [(alpha-1) s_j - tau]_+^(1/(alpha-1)). */
int oracle_entmax(const double* s, long long n, double alpha, double* p, double* tau_out) {
    double tau;
    int rc = oracle_entmax_tau(s, n, alpha, 0, &tau);
    if (rc) return rc;
    double e = 1.0 / (alpha - 1.0);
    for (long long i = 0; i < n; ++i) {
        double z = (alpha - 1.0) * s[i] - tau;
        p[i] = z > 0.0 ? pow(z, e) : 0.0;
    }
    if (tau_out) *tau_out = tau;
    return ORC_OK;
}

/* ---------------------------------------------------------------- block summaries */

/* kbar[b,g,j,:] = mean of the blk keys of complete block j (j < floor(Tk/blk)). */
int oracle_block_summary(const void* k, int kdtype, long long B, long long Hkv, long long Tk,
                         long long d, long long blk, double* kbar) {
    if (!k || !kbar || B < 1 || Hkv < 1 || Tk < 0 || d < 1 || blk < 1) return ORC_ERR_ARG;
    long long nbs = Tk / blk;
    #pragma omp parallel for collapse(2) schedule(static)
    for (long long bg = 0; bg < B * Hkv; ++bg)
        for (long long j = 0; j < nbs; ++j) {
            double* o = kbar + (bg * nbs + j) * d;
            for (long long c = 0; c < d; ++c) o[c] = 0.0;
            for (long long i = 0; i < blk; ++i) {
                long long base = (bg * Tk + j * blk + i) * d;
                for (long long c = 0; c < d; ++c) o[c] += elem(k, kdtype, base + c);
            }
            for (long long c = 0; c < d; ++c) o[c] /= (double)blk;
        }
    return ORC_OK;
}

/* Learned summary head: kbar[b,g,j,:] = sum_i a_i k_i over the blk keys of complete block j,
 * a = softmax(w[g,:] . k_i / sqrt(d)).  w is fp64 [Hkv, d]; w = NULL gives the mean. */
int oracle_block_summary_w(const void* k, int kdtype, const double* w, long long B, long long Hkv,
                           long long Tk, long long d, long long blk, double* kbar) {
    if (!w) return oracle_block_summary(k, kdtype, B, Hkv, Tk, d, blk, kbar);
    if (!k || !kbar || B < 1 || Hkv < 1 || Tk < 0 || d < 1 || blk < 1) return ORC_ERR_ARG;
    long long nbs = Tk / blk;
    double isd = 1.0 / sqrt((double)d);
    int fail = 0;
    #pragma omp parallel
    {
        double* a = (double*)malloc((size_t)blk * sizeof(double));
        if (!a) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for collapse(2) schedule(static)
        for (long long bg = 0; bg < B * Hkv; ++bg)
            for (long long j = 0; j < nbs; ++j) {
                if (!a) continue;
                const double* wg = w + (bg % Hkv) * d;
                double m = -INFINITY;
                for (long long i = 0; i < blk; ++i) {
                    long long base = (bg * Tk + j * blk + i) * d;
                    double s = 0.0;
                    for (long long c = 0; c < d; ++c) s += wg[c] * elem(k, kdtype, base + c);
                    a[i] = s * isd;
                    if (a[i] > m) m = a[i];
                }
                double den = 0.0;
                for (long long i = 0; i < blk; ++i) { a[i] = exp(a[i] - m); den += a[i]; }
                double* o = kbar + (bg * nbs + j) * d;
                for (long long c = 0; c < d; ++c) o[c] = 0.0;
                for (long long i = 0; i < blk; ++i) {
                    long long base = (bg * Tk + j * blk + i) * d;
                    for (long long c = 0; c < d; ++c) o[c] += (a[i] / den) * elem(k, kdtype, base + c);
                }
            }
        free(a);
    }
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

/* ---------------------------------------------------------------- one row */

typedef struct {
    const void* q; int qdt;      /* gathered query rows [nrows, d] */
    const void* k; int kdt;      /* [B, Hkv, Tk, d] */
    const void* v; int vdt;      /* [B, Hkv, Tk, d] */
    long long B, Hq, Hkv, Tk, d, blk;
    double alpha, cs;
    const double* wsum;          /* learned summary head [Hkv, d], or NULL for the mean */
} orc_problem;

/* Coarse stage for one row: x_j = (alpha-1) * cs * (q . kbar_j) / sqrt(d) for j < bt,
 * then tau and p.  kbar for (b, g) is passed in (fp64).  Returns bt. */
static long long row_select(const orc_problem* P, long long r, long long t, const double* kbar_bg,
                            double* x, double* p, double* tau_out) {
    long long bt = t / P->blk;
    double e = 1.0 / (P->alpha - 1.0);
    double isd = 1.0 / sqrt((double)P->d);
    for (long long j = 0; j < bt; ++j) {
        double dot = 0.0;
        for (long long c = 0; c < P->d; ++c)
            dot += elem(P->q, P->qdt, r * P->d + c) * kbar_bg[j * P->d + c];
        x[j] = (P->alpha - 1.0) * P->cs * dot * isd;
    }
    if (bt == 0) { *tau_out = NAN; return 0; }
    double tau = tau_sort(x, bt, P->alpha);
    for (long long j = 0; j < bt; ++j) {
        double z = x[j] - tau;
        p[j] = z > 0.0 ? pow(z, e) : 0.0;
    }
    *tau_out = tau;
    return bt;
}

/* Fine stage for one row with given past-block weights w[0..bt) and diagonal weight wd.
 * Logits over the tokens of every block with w > 0 and the causal part of the own block:
 * l_i = (q . k_i)/sqrt(d) + log w_block(i); o = sum softmax(l)_i v_i.
 * logw[j] (if non-NULL) overrides log(w[j]) to avoid underflow of tiny weights. */
static void row_fine(const orc_problem* P, long long r, long long b, long long g, long long t,
                     const double* w, const double* logw, double wd, double* lbuf, double* out) {
    long long bt = t / P->blk, d = P->d;
    double isd = 1.0 / sqrt((double)d);
    long long base_bg = (b * P->Hkv + g) * P->Tk;
    double m = -INFINITY;
    /* first pass: logits (stored per token 0..t; -inf where excluded) */
    for (long long i = 0; i <= t; ++i) {
        long long j = i / P->blk;
        double lw;
        if (j == bt) lw = log(wd);
        else if (w[j] > 0.0) lw = logw ? logw[j] : log(w[j]);
        else { lbuf[i] = -INFINITY; continue; }
        double dot = 0.0;
        for (long long c = 0; c < d; ++c)
            dot += elem(P->q, P->qdt, r * d + c) * elem(P->k, P->kdt, (base_bg + i) * d + c);
        lbuf[i] = dot * isd + lw;
        if (lbuf[i] > m) m = lbuf[i];
    }
    double den = 0.0;
    for (long long c = 0; c < d; ++c) out[c] = 0.0;
    for (long long i = 0; i <= t; ++i) {
        if (lbuf[i] == -INFINITY) continue;
        double a = exp(lbuf[i] - m);
        den += a;
        for (long long c = 0; c < d; ++c) out[c] += a * elem(P->v, P->vdt, (base_bg + i) * d + c);
    }
    for (long long c = 0; c < d; ++c) out[c] /= den;
}

/* kbar for every (b, g), computed once per call from the keys themselves. */
static double* all_kbar(const orc_problem* P) {
    long long nbs = P->Tk / P->blk;
    size_t cnt = (size_t)(P->B * P->Hkv * (nbs > 0 ? nbs : 1) * P->d);
    double* kb = (double*)malloc(cnt * sizeof(double));
    if (!kb) return NULL;
    if (nbs > 0 && oracle_block_summary_w(P->k, P->kdt, P->wsum, P->B, P->Hkv, P->Tk, P->d, P->blk, kb)) {
        free(kb);
        return NULL;
    }
    return kb;
}

static int check_problem(const orc_problem* P, const long long* rows, long long nrows) {
    if (!P->q || !P->k || nrows < 0 || !rows) return ORC_ERR_ARG;
    if (P->B < 1 || P->Hq < 1 || P->Hkv < 1 || P->Hq % P->Hkv || P->d < 1 || P->blk < 1) return ORC_ERR_ARG;
    if (!(P->alpha > 1.0)) return ORC_ERR_ARG;
    for (long long r = 0; r < nrows; ++r) {
        long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        if (b < 0 || b >= P->B || h < 0 || h >= P->Hq || t < 0 || t >= P->Tk) return ORC_ERR_ARG;
    }
    return ORC_OK;
}

/*
 * Block selection for listed rows (b, h, t).  q_rows holds the rows' query vectors.
 * Outputs (row-major, nbmax = floor(Tk/blk) columns, zero beyond bt):
 *   x_out[r, j] = (alpha-1) s_j,  p_out[r, j] = entmax weight,  tau_out[r] (NaN if bt=0),
 *   bt_out[r] = number of scored past blocks, nsel_out[r] = #{j : p_j > 0}.
 * Any output pointer may be NULL.
 */
int oracle_select_rows_w(const void* q_rows, int qdt, const void* k, int kdt, const double* w_summary,
                         long long B, long long Hq, long long Hkv, long long Tk, long long d,
                         long long blk, double alpha, double coarse_scale,
                         const long long* rows, long long nrows,
                         double* x_out, double* p_out, double* tau_out,
                         long long* bt_out, long long* nsel_out, int nthreads) {
    orc_problem P = {q_rows, qdt, k, kdt, NULL, 0, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale, w_summary};
    int rc = check_problem(&P, rows, nrows);
    if (rc) return rc;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    double* kb = all_kbar(&P);
    if (!kb) return ORC_ERR_NOMEM;
    long long nbs = Tk / blk, G = Hq / Hkv;
    int fail = 0;
    #pragma omp parallel
    {
        double* x = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* p = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        if (!x || !p) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < nrows; ++r) {
            if (!x || !p) continue;
            long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            long long g = h / G;
            double tau;
            long long bt = row_select(&P, r, t, kb + (b * Hkv + g) * nbs * d, x, p, &tau);
            long long ns = 0;
            for (long long j = 0; j < bt; ++j) ns += p[j] > 0.0;
            if (x_out) for (long long j = 0; j < nbs; ++j) x_out[r * nbs + j] = j < bt ? x[j] : 0.0;
            if (p_out) for (long long j = 0; j < nbs; ++j) p_out[r * nbs + j] = j < bt ? p[j] : 0.0;
            if (tau_out) tau_out[r] = tau;
            if (bt_out) bt_out[r] = bt;
            if (nsel_out) nsel_out[r] = ns;
        }
        free(x);
        free(p);
    }
    free(kb);
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

/*
 * Full forward for listed rows: coarse selection, then the prior-weighted fine softmax.
 * out[r, :] (fp64), and optionally tau_out[r], nsel_out[r] (past blocks with p > 0).
 * For decode, pass the cache as k/v with Tk = Tmax and t = kv_len - 1.
 */
int oracle_forward_rows_w(const void* q_rows, int qdt, const void* k, int kdt, const void* v, int vdt,
                          const double* w_summary, long long B, long long Hq, long long Hkv, long long Tk,
                          long long d, long long blk, double alpha, double coarse_scale,
                          const long long* rows, long long nrows,
                          double* out, double* tau_out, long long* nsel_out, int nthreads) {
    orc_problem P = {q_rows, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale, w_summary};
    int rc = check_problem(&P, rows, nrows);
    if (rc || !v || !out) return rc ? rc : ORC_ERR_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    double* kb = all_kbar(&P);
    if (!kb) return ORC_ERR_NOMEM;
    long long nbs = Tk / blk, G = Hq / Hkv;
    int fail = 0;
    #pragma omp parallel
    {
        double* x = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* p = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* lp = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* lbuf = (double*)malloc((size_t)Tk * sizeof(double));
        if (!x || !p || !lp || !lbuf) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < nrows; ++r) {
            if (!x || !p || !lp || !lbuf) continue;
            long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            long long g = h / G;
            double tau;
            long long bt = row_select(&P, r, t, kb + (b * Hkv + g) * nbs * d, x, p, &tau);
            long long ns = 0;
            /* log p_j = log(x_j - tau) / (alpha - 1): no underflow for tiny weights */
            for (long long j = 0; j < bt; ++j) {
                ns += p[j] > 0.0;
                lp[j] = p[j] > 0.0 ? log(x[j] - tau) / (alpha - 1.0) : -INFINITY;
            }
            row_fine(&P, r, b, g, t, p, lp, 1.0, lbuf, out + r * d);
            if (tau_out) tau_out[r] = tau;
            if (nsel_out) nsel_out[r] = ns;
        }
        free(x); free(p); free(lp); free(lbuf);
    }
    free(kb);
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

/*
 * Head-aggregated selection ("DashAttention and the year sparse attention became a field",
 * section "Non-dispersive attention at long context": entmax head aggregation).  Reading:
 * the G query heads of a KV group share one block distribution at each position,
 *   pbar_j = (1/G) sum_{h in group} p_{h,j}
 * (support: the union of the heads' supports), and every head of the group uses log pbar_j
 * as its prior in the fine stage; the own block keeps prior 1.
 * q_group [nrows, G, d]: the query vectors of all G heads of row r's KV group at the row's
 * position, in head order; row (b, h, t) uses its own head h % G for the fine logits.
 * nsel_out[r] = #{j : pbar_j > 0}.
 */
int oracle_forward_rows_agg(const void* q_group, int qdt, const void* k, int kdt, const void* v, int vdt,
                            const double* w_summary, long long B, long long Hq, long long Hkv, long long Tk,
                            long long d, long long blk, double alpha, double coarse_scale,
                            const long long* rows, long long nrows,
                            double* out, long long* nsel_out, int nthreads) {
    orc_problem P = {q_group, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale, w_summary};
    int rc = check_problem(&P, rows, nrows);
    if (rc || !v || !out) return rc ? rc : ORC_ERR_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    double* kb = all_kbar(&P);
    if (!kb) return ORC_ERR_NOMEM;
    long long nbs = Tk / blk, G = Hq / Hkv;
    int fail = 0;
    #pragma omp parallel
    {
        double* x = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* p = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* pbar = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
        double* lbuf = (double*)malloc((size_t)Tk * sizeof(double));
        if (!x || !p || !pbar || !lbuf) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < nrows; ++r) {
            if (!x || !p || !pbar || !lbuf) continue;
            long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            long long g = h / G, bt = t / blk;
            for (long long j = 0; j < bt; ++j) pbar[j] = 0.0;
            for (long long hh = 0; hh < G; ++hh) {
                double tau;
                /* row index r * G + hh addresses query vector hh of row r's group */
                row_select(&P, r * G + hh, t, kb + (b * Hkv + g) * nbs * d, x, p, &tau);
                for (long long j = 0; j < bt; ++j) pbar[j] += p[j] / (double)G;
            }
            long long ns = 0;
            for (long long j = 0; j < bt; ++j) ns += pbar[j] > 0.0;
            row_fine(&P, r * G + h % G, b, g, t, pbar, NULL, 1.0, lbuf, out + r * d);
            if (nsel_out) nsel_out[r] = ns;
        }
        free(x); free(p); free(pbar); free(lbuf);
    }
    free(kb);
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

/*
 * Backward of the full causal forward (mean summaries), for every row (b, h, t):
 * given dout [B, Hq, T, d] (the gradient of a scalar loss with respect to out), returns
 * dq [B, Hq, T, d], dk, dv [B, Hkv, T, d] in fp64 (zeroed here).  The chain, per row:
 *   fine stage  l_i = q . k_i / sqrt(d) + log p_j(i) over the row's tokens, P = softmax(l),
 *               o = sum P_i v_i:  dP_i = dout . v_i, dl_i = P_i (dP_i - dout . o),
 *               dv_i += P_i dout, dq += dl_i k_i / sqrt(d), dk_i += dl_i q / sqrt(d),
 *               d log p_j = sum of dl_i over the tokens of past block j;
 *   entmax      p = alpha-entmax(s) has the Jacobian diag(g) - g g^T / sum(g) with
 *               g_j = p_j^(2 - alpha) on the support (0 elsewhere), so with dp_j = d log p_j / p_j:
 *               ds_j = g_j dp_j - g_j (sum_k g_k dp_k) / sum_k g_k;
 *   scores      s_j = cs (q . kbar_j) / sqrt(d):  dq += ds_j cs kbar_j / sqrt(d),
 *               dkbar_j += ds_j cs q / sqrt(d);
 *   summaries   kbar_j = mean of block j's keys:  dk_i += dkbar_j / blk.
 * The own block has prior 1 (no gradient into the coarse stage).  Serial over rows.
 */
/* Scratch of one row's backward: x, p, log p, d log p over the past blocks, the logits over
 * the row's tokens, and d-vectors o, q, dout. */
typedef struct {
    double *x, *p, *lp, *dlp, *lbuf, *o, *qv, *gv;
} bwd_scratch;

static int bwd_scratch_alloc(bwd_scratch* S, long long nbs, long long Tk, long long d) {
    S->x = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
    S->p = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
    S->lp = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
    S->dlp = (double*)malloc((size_t)(nbs + 1) * sizeof(double));
    S->lbuf = (double*)malloc((size_t)Tk * sizeof(double));
    S->o = (double*)malloc((size_t)d * sizeof(double));
    S->qv = (double*)malloc((size_t)d * sizeof(double));
    S->gv = (double*)malloc((size_t)d * sizeof(double));
    return S->x && S->p && S->lp && S->dlp && S->lbuf && S->o && S->qv && S->gv;
}

static void bwd_scratch_free(bwd_scratch* S) {
    free(S->x); free(S->p); free(S->lp); free(S->dlp); free(S->lbuf); free(S->o); free(S->qv); free(S->gv);
}

/* The chain above for row (b, h, t): adds the row's dq into dq_row; when dk is not NULL also
 * its shares of dk, dv and dkbar (the summary term reaches dk later, from dkbar). */
static void backward_row(const orc_problem* P, const double* kb, const void* dout, int ddt,
                         long long b, long long h, long long t, bwd_scratch* S,
                         double* dq_row, double* dk, double* dv, double* dkbar) {
    const void* k = P->k; const void* v = P->v;
    const int kdt = P->kdt, vdt = P->vdt;
    const long long G = P->Hq / P->Hkv, d = P->d, blk = P->blk, nbs = P->Tk / P->blk;
    const long long g = h / G, bt = t / blk, row = (b * P->Hq + h) * P->Tk + t;
    const long long kvbase = (b * P->Hkv + g) * P->Tk;
    const double isd = 1.0 / sqrt((double)d), alpha = P->alpha;
    const double* kbg = kb + (b * P->Hkv + g) * nbs * d;
    for (long long c = 0; c < d; ++c) {
        S->qv[c] = elem(P->q, P->qdt, row * d + c);
        S->gv[c] = elem(dout, ddt, row * d + c);
    }
    /* coarse stage (row_select reads q row r = row) */
    double tau = NAN;
    row_select(P, row, t, kbg, S->x, S->p, &tau);
    for (long long j = 0; j < bt; ++j) S->lp[j] = S->p[j] > 0.0 ? log(S->x[j] - tau) / (alpha - 1.0) : -INFINITY;
    /* fine forward: logits, max, softmax, output */
    double m = -INFINITY;
    for (long long i = 0; i <= t; ++i) {
        const long long j = i / blk;
        const double lw = j == bt ? 0.0 : S->lp[j];
        if (lw == -INFINITY) { S->lbuf[i] = -INFINITY; continue; }
        double dot = 0.0;
        for (long long c = 0; c < d; ++c) dot += S->qv[c] * elem(k, kdt, (kvbase + i) * d + c);
        S->lbuf[i] = dot * isd + lw;
        if (S->lbuf[i] > m) m = S->lbuf[i];
    }
    double den = 0.0;
    for (long long c = 0; c < d; ++c) S->o[c] = 0.0;
    for (long long i = 0; i <= t; ++i) {
        if (S->lbuf[i] == -INFINITY) continue;
        const double a = exp(S->lbuf[i] - m);
        den += a;
        for (long long c = 0; c < d; ++c) S->o[c] += a * elem(v, vdt, (kvbase + i) * d + c);
    }
    for (long long c = 0; c < d; ++c) S->o[c] /= den;
    double Drow = 0.0;
    for (long long c = 0; c < d; ++c) Drow += S->gv[c] * S->o[c];
    /* fine backward */
    for (long long j = 0; j < bt; ++j) S->dlp[j] = 0.0;
    for (long long i = 0; i <= t; ++i) {
        if (S->lbuf[i] == -INFINITY) continue;
        const double Pi = exp(S->lbuf[i] - m) / den;
        double dPi = 0.0;
        for (long long c = 0; c < d; ++c) dPi += S->gv[c] * elem(v, vdt, (kvbase + i) * d + c);
        const double dl = Pi * (dPi - Drow);
        for (long long c = 0; c < d; ++c) {
            dq_row[c] += dl * elem(k, kdt, (kvbase + i) * d + c) * isd;
            if (dk) {
                dv[(kvbase + i) * d + c] += Pi * S->gv[c];
                dk[(kvbase + i) * d + c] += dl * S->qv[c] * isd;
            }
        }
        const long long j = i / blk;
        if (j < bt) S->dlp[j] += dl;
    }
    /* entmax backward on the support, then the coarse scores */
    double sg = 0.0, sgdp = 0.0;
    for (long long j = 0; j < bt; ++j) {
        if (!(S->p[j] > 0.0)) continue;
        const double gj = pow(S->p[j], 2.0 - alpha);
        sg += gj;
        sgdp += gj * (S->dlp[j] / S->p[j]);
    }
    for (long long j = 0; j < bt; ++j) {
        if (!(S->p[j] > 0.0)) continue;
        const double gj = pow(S->p[j], 2.0 - alpha);
        const double ds = gj * (S->dlp[j] / S->p[j]) - gj * sgdp / sg;
        const double f = ds * P->cs * isd;
        for (long long c = 0; c < d; ++c) {
            dq_row[c] += f * kbg[j * d + c];
            if (dkbar) dkbar[((b * P->Hkv + g) * nbs + j) * d + c] += f * S->qv[c];
        }
    }
}

int oracle_backward(const void* q, int qdt, const void* k, int kdt, const void* v, int vdt,
                    const void* dout, int ddt, long long B, long long Hq, long long Hkv, long long Tk,
                    long long d, long long blk, double alpha, double coarse_scale,
                    double* dq, double* dk, double* dv) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORC_ERR_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || blk < 1 || Tk < 1 || !(alpha > 1.0)) return ORC_ERR_ARG;
    orc_problem P = {q, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale, NULL};
    double* kb = all_kbar(&P);
    if (!kb) return ORC_ERR_NOMEM;
    const long long nbs = Tk / blk;
    memset(dq, 0, (size_t)(B * Hq * Tk * d) * sizeof(double));
    memset(dk, 0, (size_t)(B * Hkv * Tk * d) * sizeof(double));
    memset(dv, 0, (size_t)(B * Hkv * Tk * d) * sizeof(double));
    double* dkbar = (double*)calloc((size_t)(B * Hkv * (nbs > 0 ? nbs : 1) * d), sizeof(double));
    bwd_scratch S = {NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL};
    int rc = ORC_OK;
    if (!dkbar || !bwd_scratch_alloc(&S, nbs, Tk, d)) rc = ORC_ERR_NOMEM;
    for (long long b = 0; rc == ORC_OK && b < B; ++b)
        for (long long h = 0; h < Hq; ++h)
            for (long long t = 0; t < Tk; ++t)
                backward_row(&P, kb, dout, ddt, b, h, t, &S, dq + ((b * Hq + h) * Tk + t) * d, dk, dv, dkbar);
    /* summaries: every key of complete block j receives dkbar_j / blk */
    for (long long bg = 0; rc == ORC_OK && bg < B * Hkv; ++bg)
        for (long long j = 0; j < nbs; ++j)
            for (long long i = 0; i < blk; ++i)
                for (long long c = 0; c < d; ++c)
                    dk[(bg * Tk + j * blk + i) * d + c] += dkbar[(bg * nbs + j) * d + c] / (double)blk;
    bwd_scratch_free(&S);
    free(dkbar); free(kb);
    return rc;
}

/*
 * dq of the listed rows (b, h, t) only -- the same per-row chain as oracle_backward, whose dq
 * rows do not depend on any other row.  q and dout are the full [B, Hq, T, d] tensors;
 * dq_out [nrows, d].  OpenMP over rows when nthreads != 1.
 */
int oracle_backward_dq_rows(const void* q, int qdt, const void* k, int kdt, const void* v, int vdt,
                            const void* dout, int ddt, long long B, long long Hq, long long Hkv,
                            long long Tk, long long d, long long blk, double alpha, double coarse_scale,
                            const long long* rows, long long nrows, double* dq_out, int nthreads) {
    if (!q || !k || !v || !dout || (nrows > 0 && (!rows || !dq_out))) return ORC_ERR_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || blk < 1 || Tk < 1 || !(alpha > 1.0)) return ORC_ERR_ARG;
    orc_problem P = {q, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale, NULL};
    if (check_problem(&P, rows, nrows) != ORC_OK) return ORC_ERR_ARG;
    double* kb = all_kbar(&P);
    if (!kb) return ORC_ERR_NOMEM;
    const long long nbs = Tk / blk;
    int fail = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads()) if (nthreads != 1)
    {
        bwd_scratch S;
        if (!bwd_scratch_alloc(&S, nbs, Tk, d)) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long long r = 0; r < nrows; ++r) {
                double* out = dq_out + r * d;
                for (long long c = 0; c < d; ++c) out[c] = 0.0;
                backward_row(&P, kb, dout, ddt, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2], &S, out, NULL, NULL, NULL);
            }
        }
        bwd_scratch_free(&S);
    }
    free(kb);
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

int oracle_select_rows(const void* q_rows, int qdt, const void* k, int kdt,
                       long long B, long long Hq, long long Hkv, long long Tk, long long d,
                       long long blk, double alpha, double coarse_scale,
                       const long long* rows, long long nrows,
                       double* x_out, double* p_out, double* tau_out,
                       long long* bt_out, long long* nsel_out, int nthreads) {
    return oracle_select_rows_w(q_rows, qdt, k, kdt, NULL, B, Hq, Hkv, Tk, d, blk, alpha, coarse_scale,
                                rows, nrows, x_out, p_out, tau_out, bt_out, nsel_out, nthreads);
}

int oracle_forward_rows(const void* q_rows, int qdt, const void* k, int kdt, const void* v, int vdt,
                        long long B, long long Hq, long long Hkv, long long Tk, long long d,
                        long long blk, double alpha, double coarse_scale,
                        const long long* rows, long long nrows,
                        double* out, double* tau_out, long long* nsel_out, int nthreads) {
    return oracle_forward_rows_w(q_rows, qdt, k, kdt, v, vdt, NULL, B, Hq, Hkv, Tk, d, blk, alpha,
                                 coarse_scale, rows, nrows, out, tau_out, nsel_out, nthreads);
}

/*
 * Fine stage alone with caller-given weights: w_rows[r, j] for past blocks j < bt
 * (row-major with floor(Tk/blk) columns) and diagonal weight w_diag[r].
 * Used to check that equal weights on every block reproduce dense causal attention.
 */
int oracle_fine_rows_given_p(const void* q_rows, int qdt, const void* k, int kdt, const void* v, int vdt,
                             long long B, long long Hq, long long Hkv, long long Tk, long long d,
                             long long blk, const long long* rows, long long nrows,
                             const double* w_rows, const double* w_diag, double* out, int nthreads) {
    orc_problem P = {q_rows, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, blk, 1.5, 1.0, NULL};
    int rc = check_problem(&P, rows, nrows);
    if (rc || !v || !out || !w_rows || !w_diag) return rc ? rc : ORC_ERR_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long long nbs = Tk / blk, G = Hq / Hkv;
    int fail = 0;
    #pragma omp parallel
    {
        double* lbuf = (double*)malloc((size_t)Tk * sizeof(double));
        if (!lbuf) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(dynamic, 1)
        for (long long r = 0; r < nrows; ++r) {
            if (!lbuf) continue;
            long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
            row_fine(&P, r, b, h / G, t, w_rows + r * nbs, NULL, w_diag[r], lbuf, out + r * d);
        }
        free(lbuf);
    }
    return fail ? ORC_ERR_NOMEM : ORC_OK;
}

/* Dense causal softmax attention over tokens 0..t (separate code, no blocks, no prior). */
int oracle_dense_causal_rows(const void* q_rows, int qdt, const void* k, int kdt, const void* v, int vdt,
                             long long B, long long Hq, long long Hkv, long long Tk, long long d,
                             const long long* rows, long long nrows, double* out, int nthreads) {
    orc_problem P = {q_rows, qdt, k, kdt, v, vdt, B, Hq, Hkv, Tk, d, 1, 1.5, 1.0, NULL};
    int rc = check_problem(&P, rows, nrows);
    if (rc || !v || !out) return rc ? rc : ORC_ERR_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    long long G = Hq / Hkv;
    #pragma omp parallel for schedule(dynamic, 1)
    for (long long r = 0; r < nrows; ++r) {
        long long b = rows[3 * r], h = rows[3 * r + 1], t = rows[3 * r + 2];
        long long base = (b * Hkv + h / G) * Tk;
        double isd = 1.0 / sqrt((double)d), m = -INFINITY, den = 0.0;
        double* o = out + r * d;
        for (long long i = 0; i <= t; ++i) {
            double dot = 0.0;
            for (long long c = 0; c < d; ++c)
                dot += elem(q_rows, qdt, r * d + c) * elem(k, kdt, (base + i) * d + c);
            dot *= isd;
            if (dot > m) m = dot;
        }
        for (long long c = 0; c < d; ++c) o[c] = 0.0;
        for (long long i = 0; i <= t; ++i) {
            double dot = 0.0;
            for (long long c = 0; c < d; ++c)
                dot += elem(q_rows, qdt, r * d + c) * elem(k, kdt, (base + i) * d + c);
            double a = exp(dot * isd - m);
            den += a;
            for (long long c = 0; c < d; ++c) o[c] += a * elem(v, vdt, (base + i) * d + c);
        }
        for (long long c = 0; c < d; ++c) o[c] /= den;
    }
    return ORC_OK;
}
