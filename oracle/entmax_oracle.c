/*
 * entmax_oracle.c -- plain, slow, fp64 CPU reference for 1.5-entmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg load
 * it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (page "svd-sst2-roberta-adasplash", sections 2.1-2.4, and
 * the AdaSplash model cards "roberta-base-adasplash" / "distilbert-sst2-
 * adasplash", section "Mathematical Formulation"):
 *
 *   S_ij = scale * <Q_i, K_j>                        (section 3, affinity step)
 *   allowed(i,j) = key_mask[b,j] && (!causal || j <= i)
 *                  && (window == 0 || j >= i - window + 1)
 *   p_ij = max(0, (S_ij - tau_i)/2)^2,  sum_j p_ij = 1  (Theorem 1)
 *   O_i  = sum_j p_ij V_j                              (context aggregation)
 *   backward: closed-form Jacobian of section 2.4,
 *     dL/dS_j = 1[j in S] sqrt(p_j) (g_j - sum_k sqrt(p_k) g_k / sum_k sqrt(p_k))
 *
 * alpha = 1 is softmax (the pages' branch for |alpha - 1| < 1e-4 in the same
 * routine): p_ij = exp(S_ij - tau_i), tau_i = log sum_j exp(S_ij).
 *
 * General alpha in (1, 2] (the pages' alpha-entmax by bisection, page
 * "svd-sst2-roberta-adasplash", section 4, the entmax_bisect routine): with
 * a = alpha - 1, p_ij = max(0, a (S_ij - tau_i))^(1/a), sum_j p_ij = 1 (tau in
 * score units; alpha = 1.5 gives the formula above), and the Jacobian
 * dp_i/ds_j = w_i (delta_ij - w_j / sum_k w_k) with w = p^(2 - alpha).
 *
 * tau (alpha = 1.5) is obtained two ways:
 *   - eo_tau_sort:   exact, from the closed form on a sorted row (on a support
 *                    of size k, sum (z_i - tau)^2 = 4 is a quadratic in tau);
 *   - eo_tau_bisect: the pages' bisection (Theorem 2), 25 halvings of a
 *                    bracket, final midpoint.
 *
 * Every input is fp64 holding values already rounded to bf16 (eo_round_bf16
 * does that rounding from the IEEE-754 definition, round-to-nearest-even).
 *
 * Empty rows (no allowed key) follow the library's documented convention:
 * O_i = 0, tau_i = +inf, zero gradients.
 *
 * Parallelism: OpenMP over rows or heads only; the arithmetic of one row is
 * sequential and in textbook order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* bf16 rounding: keep the top 16 bits of the IEEE-754 binary32 pattern,     */
/* rounding the dropped 16 bits to nearest, ties to the even kept pattern.   */
/* ------------------------------------------------------------------------ */
double eo_round_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
        return (double)x; /* NaN stays NaN */
    }
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) {
        kept += 1u; /* carries into the exponent when the mantissa overflows */
    }
    uint32_t r = kept << 16;
    float f;
    memcpy(&f, &r, sizeof f);
    return (double)f;
}

void eo_round_bf16_array(const float* x, double* out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = eo_round_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* g(tau) = sum_i [ (s_i - tau)/2 ]_+^2   (Theorem 1 constraint function)   */
/* ------------------------------------------------------------------------ */
double eo_g(const double* s, int n, double tau)
{
    double acc = 0.0;
    for (int i = 0; i < n; ++i) {
        double t = (s[i] - tau) / 2.0;
        if (t > 0.0) acc += t * t;
    }
    return acc;
}

static int cmp_desc(const void* a, const void* b)
{
    double x = *(const double*)a, y = *(const double*)b;
    return (x < y) - (x > y);
}

/* ------------------------------------------------------------------------ */
/* Exact tau by sorting.  For the k largest scores z_1 >= ... >= z_k taken  */
/* as the support, sum_{i<=k} (z_i - tau)^2 = 4 gives (smaller root)         */
/*   tau_k = mu_k - sqrt(4/k - (q_k - mu_k^2)),                              */
/* mu_k = mean of z_1..z_k, q_k = mean of squares.  The support size is the */
/* largest k for which that root exists and lies at or below z_k (then every */
/* kept score is above tau, every dropped one at or below it: the KKT       */
/* conditions of Theorem 1).  Returns the support size, writes tau.         */
/* n == 0 gives tau = +inf and support 0.                                    */
/* ------------------------------------------------------------------------ */
int eo_tau_sort(const double* s, int n, double* tau_out)
{
    if (n <= 0) {
        *tau_out = INFINITY;
        return 0;
    }
    double* z = (double*)malloc(sizeof(double) * (size_t)n);
    memcpy(z, s, sizeof(double) * (size_t)n);
    qsort(z, (size_t)n, sizeof(double), cmp_desc);
    double sum = 0.0, sumsq = 0.0;
    int kstar = 1;
    double tau = z[0] - 2.0; /* k = 1: (z_1 - tau)^2 = 4 */
    for (int k = 1; k <= n; ++k) {
        sum += z[k - 1];
        sumsq += z[k - 1] * z[k - 1];
        double mu = sum / k;
        double var = sumsq / k - mu * mu;
        double delta = 4.0 / k - var;
        if (delta < 0.0) continue;
        double tk = mu - sqrt(delta);
        if (tk <= z[k - 1]) {
            kstar = k;
            tau = tk;
        }
    }
    free(z);
    *tau_out = tau;
    return kstar;
}

/* ------------------------------------------------------------------------ */
/* tau by bisection on [lo, hi] (Theorem 2): n_iter halvings, each keeping  */
/* the half that still brackets the root (g(mid) > 1 means the root lies    */
/* right of mid), then the midpoint of the final bracket.                   */
/* ------------------------------------------------------------------------ */
double eo_tau_bisect_bracket(const double* s, int n, double lo, double hi, int n_iter)
{
    for (int it = 0; it < n_iter; ++it) {
        double mid = 0.5 * (lo + hi);
        if (eo_g(s, n, mid) > 1.0) lo = mid;
        else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* The bracket the model cards state: [max - 2, max - 2/sqrt(n)], n = number */
/* of scores in the row (the allowed keys).  n == 0 gives +inf.              */
double eo_tau_bisect(const double* s, int n, int n_iter)
{
    if (n <= 0) return INFINITY;
    double m = s[0];
    for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    return eo_tau_bisect_bracket(s, n, m - 2.0, m - 2.0 / sqrt((double)n), n_iter);
}

/* The wider bracket of Theorem 2: [min - 2, max]. */
double eo_tau_bisect_wide(const double* s, int n, int n_iter)
{
    if (n <= 0) return INFINITY;
    double mx = s[0], mn = s[0];
    for (int i = 1; i < n; ++i) {
        if (s[i] > mx) mx = s[i];
        if (s[i] < mn) mn = s[i];
    }
    return eo_tau_bisect_bracket(s, n, mn - 2.0, mx, n_iter);
}

/* p_i = [ (s_i - tau)/2 ]_+^2 (Theorem 1).  No renormalisation. */
void eo_entmax15(const double* s, int n, double tau, double* p)
{
    for (int i = 0; i < n; ++i) {
        double t = (s[i] - tau) / 2.0;
        p[i] = t > 0.0 ? t * t : 0.0;
    }
}

/* Jacobian-vector product of section 2.4 for one row:                     */
/*   ds_j = sqrt(p_j) (g_j - sum_k sqrt(p_k) g_k / sum_k sqrt(p_k)),        */
/* zero where p_j == 0.                                                     */
void eo_entmax15_jvp(const double* p, const double* g, int n, double* ds)
{
    double r = 0.0, w = 0.0;
    for (int k = 0; k < n; ++k) {
        double sp = sqrt(p[k]);
        r += sp;
        w += sp * g[k];
    }
    double u = r > 0.0 ? w / r : 0.0;
    for (int j = 0; j < n; ++j) ds[j] = p[j] > 0.0 ? sqrt(p[j]) * (g[j] - u) : 0.0;
}

/* ------------------------------------------------------------------------ */
/* alpha-entmax, alpha in (1, 2].  a = alpha - 1.                            */
/*   g_alpha(tau) = sum_i max(0, a (s_i - tau))^(1/a)                         */
/* is continuous and strictly decreasing where positive, so g_alpha = 1 has  */
/* one root.  The max alone gives g_alpha(max - 1/a) >= 1; n equal terms of  */
/* 1/n give g_alpha(max - n^(-a)/a) <= 1 (every term is at most 1/n there).  */
/* The root is found by halving that bracket until the midpoint no longer    */
/* changes in fp64 (at most 2000 halvings): the exact root to rounding.      */
/* ------------------------------------------------------------------------ */
double eo_g_alpha(const double* s, int n, double tau, double alpha)
{
    const double a = alpha - 1.0;
    double acc = 0.0;
    for (int i = 0; i < n; ++i) {
        double t = a * (s[i] - tau);
        if (t > 0.0) acc += pow(t, 1.0 / a);
    }
    return acc;
}

double eo_tau_alpha(const double* s, int n, double alpha)
{
    if (n <= 0) return INFINITY;
    const double a = alpha - 1.0;
    double m = s[0];
    for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    double lo = m - 1.0 / a, hi = m - pow((double)n, -a) / a;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (eo_g_alpha(s, n, mid, alpha) > 1.0) lo = mid;
        else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* The pages' procedure for general alpha on the same bracket: n_iter halvings, final midpoint. */
double eo_tau_alpha_bisect(const double* s, int n, double alpha, int n_iter)
{
    if (n <= 0) return INFINITY;
    const double a = alpha - 1.0;
    double m = s[0];
    for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    double lo = m - 1.0 / a, hi = m - pow((double)n, -a) / a;
    for (int it = 0; it < n_iter; ++it) {
        double mid = 0.5 * (lo + hi);
        if (eo_g_alpha(s, n, mid, alpha) > 1.0) lo = mid;
        else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* p_i = max(0, a (s_i - tau))^(1/a). */
void eo_entmax_alpha(const double* s, int n, double tau, double alpha, double* p)
{
    const double a = alpha - 1.0;
    for (int i = 0; i < n; ++i) {
        double t = a * (s[i] - tau);
        p[i] = t > 0.0 ? pow(t, 1.0 / a) : 0.0;
    }
}

/* Jacobian-vector product of alpha-entmax: w_j = p_j^(2 - alpha) on the    */
/* support, ds_j = w_j (g_j - sum_k w_k g_k / sum_k w_k).                   */
void eo_entmax_alpha_jvp(const double* p, const double* g, int n, double alpha, double* ds)
{
    double r = 0.0, acc = 0.0;
    for (int k = 0; k < n; ++k) {
        if (p[k] <= 0.0) continue;
        double w = pow(p[k], 2.0 - alpha);
        r += w;
        acc += w * g[k];
    }
    double u = r > 0.0 ? acc / r : 0.0;
    for (int j = 0; j < n; ++j) ds[j] = p[j] > 0.0 ? pow(p[j], 2.0 - alpha) * (g[j] - u) : 0.0;
}

/* ------------------------------------------------------------------------ */
/* alpha = 1: softmax.  The pages' alpha-entmax routine takes this branch     */
/* when |alpha - 1| < 1e-4 (page "svd-sst2-roberta-adasplash", section 4,     */
/* entmax_bisect), and it is the alpha -> 1 limit of alpha-entmax.           */
/*   p_i = exp(s_i - tau),  tau = log sum_k exp(s_k),                        */
/* so tau plays the threshold's role (p = exp(s - tau) sums to 1).  tau is   */
/* written as m + log sum_k exp(s_k - m), m = max_k s_k, so that no term     */
/* overflows.  The Jacobian is the alpha-entmax one with w = p^(2-1) = p:    */
/* ds_j = p_j (g_j - sum_k p_k g_k), which eo_entmax_alpha_jvp computes at   */
/* alpha = 1 (there sum_k w_k = 1).                                          */
/* ------------------------------------------------------------------------ */
double eo_tau_softmax(const double* s, int n)
{
    if (n <= 0) return INFINITY;
    double m = s[0];
    for (int i = 1; i < n; ++i) if (s[i] > m) m = s[i];
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += exp(s[i] - m);
    return m + log(acc);
}

void eo_softmax(const double* s, int n, double tau, double* p)
{
    for (int i = 0; i < n; ++i) p[i] = exp(s[i] - tau);
}

/* tau and p of one row for any alpha: softmax (alpha = 1), the closed form */
/* (alpha = 1.5, sort) or the converged bisection; tau_method 1 = the pages' */
/* n_iter halvings (alpha > 1).                                             */
static double row_tau(const double* s, int n, double alpha, int tau_method, int n_iter)
{
    if (alpha == 1.0) return eo_tau_softmax(s, n);
    if (alpha == 1.5) {
        double tau;
        if (tau_method == 0) eo_tau_sort(s, n, &tau);
        else tau = eo_tau_bisect(s, n, n_iter > 0 ? n_iter : 25);
        return tau;
    }
    if (tau_method == 0) return eo_tau_alpha(s, n, alpha);
    return eo_tau_alpha_bisect(s, n, alpha, n_iter > 0 ? n_iter : 25);
}

static void row_probs(const double* s, int n, double tau, double alpha, double* p)
{
    if (alpha == 1.0) eo_softmax(s, n, tau, p);
    else if (alpha == 1.5) eo_entmax15(s, n, tau, p);
    else eo_entmax_alpha(s, n, tau, alpha, p);
}

/* ------------------------------------------------------------------------ */
/* Attention.  Tensors are [B,H,L,D] row-major fp64; key_mask is [B,L]      */
/* (1 = valid) or NULL for all valid.                                       */
/* ------------------------------------------------------------------------ */
static int allowed(const unsigned char* key_mask, int b, int L, int causal, int window, int i, int j)
{
    if (key_mask && !key_mask[(size_t)b * L + j]) return 0;
    if (causal && j > i) return 0;
    if (window > 0 && j < i - window + 1) return 0;
    return 1;
}

/* One query row: fills O_i (D values), returns tau.  tau_method 0 = sort,  */
/* 1 = bisection (25 iterations unless n_iter > 0 given).  Scratch s, idx   */
/* and p hold L entries each.                                               */
static double row_forward(const double* Q, const double* K, const double* V,
                          const unsigned char* key_mask, int causal, int window, double scale, double alpha,
                          int H, int L, int D, int b, int h, int i, int tau_method, int n_iter,
                          double* s, int* idx, double* p, double* O_row)
{
    const size_t head = ((size_t)b * H + h) * (size_t)L * D;
    const double* q = Q + head + (size_t)i * D;
    int n = 0;
    for (int j = 0; j < L; ++j) {
        if (!allowed(key_mask, b, L, causal, window, i, j)) continue;
        const double* k = K + head + (size_t)j * D;
        double acc = 0.0;
        for (int t = 0; t < D; ++t) acc += q[t] * k[t];
        s[n] = scale * acc;
        idx[n] = j;
        ++n;
    }
    for (int t = 0; t < D; ++t) O_row[t] = 0.0;
    if (n == 0) return INFINITY;
    const double tau = row_tau(s, n, alpha, tau_method, n_iter);
    row_probs(s, n, tau, alpha, p);
    for (int e = 0; e < n; ++e) {
        if (p[e] == 0.0) continue;
        const double* v = V + head + (size_t)idx[e] * D;
        for (int t = 0; t < D; ++t) O_row[t] += p[e] * v[t];
    }
    return tau;
}

/* Forward for a list of rows, row id = (b*H + h)*L + i.  O_rows is         */
/* [nrows, D], tau_rows [nrows].                                            */
void eo_attn_fwd_rows(const double* Q, const double* K, const double* V,
                      const unsigned char* key_mask, int causal, int window, double scale, double alpha,
                      int B, int H, int L, int D, const long long* row_ids, long long nrows,
                      int tau_method, int n_iter, double* O_rows, double* tau_rows)
{
    (void)B;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* p = (double*)malloc(sizeof(double) * (size_t)L);
        int* idx = (int*)malloc(sizeof(int) * (size_t)L);
#pragma omp for schedule(dynamic, 16)
        for (long long r = 0; r < nrows; ++r) {
            long long id = row_ids[r];
            int i = (int)(id % L);
            long long bh = id / L;
            int h = (int)(bh % H);
            int b = (int)(bh / H);
            tau_rows[r] = row_forward(Q, K, V, key_mask, causal, window, scale, alpha, H, L, D, b, h, i,
                                      tau_method, n_iter, s, idx, p, O_rows + (size_t)r * D);
        }
        free(s);
        free(p);
        free(idx);
    }
}

/* Auxiliary rows of the backward's row scalar (page "svd-sst2-roberta-adasplash", section 2.4, the   */
/* closed-form Jacobian: u_i = sum_j sqrt(p_ij) dA_ij / sum_j sqrt(p_ij)), alpha = 1.5: for each listed   */
/* row, Otil_i = sum_j sqrt(p_ij) V_j and r_i = sum_j sqrt(p_ij), with p from the exact tau (sort).       */
/* Otil_rows is [nrows, D], r_rows [nrows]; a row with no allowed key gets zeros.                       */
void eo_attn_aux_rows(const double* Q, const double* K, const double* V,
                      const unsigned char* key_mask, int causal, int window, double scale,
                      int B, int H, int L, int D, const long long* row_ids, long long nrows,
                      double* Otil_rows, double* r_rows)
{
    (void)B;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)L);
        double* p = (double*)malloc(sizeof(double) * (size_t)L);
        int* idx = (int*)malloc(sizeof(int) * (size_t)L);
#pragma omp for schedule(dynamic, 16)
        for (long long r = 0; r < nrows; ++r) {
            long long id = row_ids[r];
            int i = (int)(id % L);
            long long bh = id / L;
            int h = (int)(bh % H);
            int b = (int)(bh / H);
            const size_t head = ((size_t)b * H + h) * (size_t)L * D;
            const double* q = Q + head + (size_t)i * D;
            double* out = Otil_rows + (size_t)r * D;
            int n = 0;
            for (int j = 0; j < L; ++j) {
                if (!allowed(key_mask, b, L, causal, window, i, j)) continue;
                const double* k = K + head + (size_t)j * D;
                double acc = 0.0;
                for (int t = 0; t < D; ++t) acc += q[t] * k[t];
                s[n] = scale * acc;
                idx[n] = j;
                ++n;
            }
            for (int t = 0; t < D; ++t) out[t] = 0.0;
            r_rows[r] = 0.0;
            if (n == 0) continue;
            double tau;
            eo_tau_sort(s, n, &tau);
            eo_entmax15(s, n, tau, p);
            for (int e = 0; e < n; ++e) {
                if (p[e] == 0.0) continue;
                const double w = sqrt(p[e]);
                const double* v = V + head + (size_t)idx[e] * D;
                for (int t = 0; t < D; ++t) out[t] += w * v[t];
                r_rows[r] += w;
            }
        }
        free(s);
        free(p);
        free(idx);
    }
}

/* Full forward: O [B,H,L,D], tau [B,H,L]. */
void eo_attn_fwd(const double* Q, const double* K, const double* V,
                 const unsigned char* key_mask, int causal, int window, double scale, double alpha,
                 int B, int H, int L, int D, int tau_method, double* O, double* tau)
{
    long long nrows = (long long)B * H * L;
    long long* ids = (long long*)malloc(sizeof(long long) * (size_t)nrows);
    for (long long r = 0; r < nrows; ++r) ids[r] = r;
    eo_attn_fwd_rows(Q, K, V, key_mask, causal, window, scale, alpha, B, H, L, D, ids, nrows,
                     tau_method, 25, O, tau);
    free(ids);
}

/* Backward for a list of heads bh = b*H + h (gradients of all rows and keys */
/* of each listed head).  tau is recomputed here (exact): the              */
/* oracle takes nothing from the code under test.  dQ, dK, dV are [nheads,  */
/* L, D] in the order of bh_ids.                                            */
void eo_attn_bwd_heads(const double* Q, const double* K, const double* V,
                       const unsigned char* key_mask, int causal, int window, double scale, double alpha,
                       int B, int H, int L, int D, const double* dO,
                       const long long* bh_ids, int nheads,
                       double* dQ, double* dK, double* dV)
{
    (void)B;
    size_t per_head = (size_t)L * D;
    memset(dQ, 0, sizeof(double) * per_head * (size_t)nheads);
    memset(dK, 0, sizeof(double) * per_head * (size_t)nheads);
    memset(dV, 0, sizeof(double) * per_head * (size_t)nheads);
    for (int hh = 0; hh < nheads; ++hh) {
        long long bh = bh_ids[hh];
        int b = (int)(bh / H);
        size_t head = (size_t)bh * per_head;
        double* dQh = dQ + (size_t)hh * per_head;
        double* dKh = dK + (size_t)hh * per_head;
        double* dVh = dV + (size_t)hh * per_head;
#pragma omp parallel
        {
            double* s = (double*)malloc(sizeof(double) * (size_t)L);
            double* p = (double*)malloc(sizeof(double) * (size_t)L);
            double* g = (double*)malloc(sizeof(double) * (size_t)L);
            double* ds = (double*)malloc(sizeof(double) * (size_t)L);
            int* idx = (int*)malloc(sizeof(int) * (size_t)L);
            double* dK_loc = (double*)calloc(per_head, sizeof(double));
            double* dV_loc = (double*)calloc(per_head, sizeof(double));
#pragma omp for schedule(dynamic, 8)
            for (int i = 0; i < L; ++i) {
                const double* q = Q + head + (size_t)i * D;
                const double* go = dO + head + (size_t)i * D;
                int n = 0;
                for (int j = 0; j < L; ++j) {
                    if (!allowed(key_mask, b, L, causal, window, i, j)) continue;
                    const double* k = K + head + (size_t)j * D;
                    double acc = 0.0;
                    for (int t = 0; t < D; ++t) acc += q[t] * k[t];
                    s[n] = scale * acc;
                    idx[n] = j;
                    ++n;
                }
                if (n == 0) continue;
                const double tau = row_tau(s, n, alpha, 0, 0);
                row_probs(s, n, tau, alpha, p);
                /* g_j = dL/dp_ij = <dO_i, V_j> (O_i = sum_j p_ij V_j) */
                for (int e = 0; e < n; ++e) {
                    const double* v = V + head + (size_t)idx[e] * D;
                    double acc = 0.0;
                    for (int t = 0; t < D; ++t) acc += go[t] * v[t];
                    g[e] = acc;
                }
                if (alpha == 1.5) eo_entmax15_jvp(p, g, n, ds);
                else eo_entmax_alpha_jvp(p, g, n, alpha, ds);
                for (int e = 0; e < n; ++e) {
                    if (p[e] == 0.0) continue;
                    int j = idx[e];
                    const double* k = K + head + (size_t)j * D;
                    for (int t = 0; t < D; ++t) {
                        dQh[(size_t)i * D + t] += scale * ds[e] * k[t];
                        dK_loc[(size_t)j * D + t] += scale * ds[e] * q[t];
                        dV_loc[(size_t)j * D + t] += p[e] * go[t];
                    }
                }
            }
#pragma omp critical
            {
                for (size_t t = 0; t < per_head; ++t) {
                    dKh[t] += dK_loc[t];
                    dVh[t] += dV_loc[t];
                }
            }
            free(s); free(p); free(g); free(ds); free(idx); free(dK_loc); free(dV_loc);
        }
    }
}

int eo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void eo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
