/*
 * laplex_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, sequential fp64 restatement of the LAPLEX operator, used only
 * by tests/, by __graft_entry__.smoke() and by the CPU-baseline leg of bench.py
 * to check the CUDA path.  It shares no code, header or constant with the CUDA
 * library and must never be called from the product path.
 *
 * Sources (web pages, cited by title and section):
 *   [IT] "Riepilogo Tecnico: LAPLEX - La FFT dei Nuclei di Laplace Apprendibili"
 *        (gist.science, Italian technical summary of arXiv 2605.24584)
 *   [FR] "Resume Technique : LAPLEX - La FFT des Kernels Laplaciens Apprenables"
 *        (gist.science, French technical summary; same content as [IT])
 *
 * Conventions: anchors s[] are sorted ascending by the caller; vectors are
 * row-major [len, B]; every sum is taken in fp64 in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/*
 * Symmetric case, [IT] §2.2 "Caso Simmetrico": with the anchors sorted, K splits
 * into a lower and an upper triangular part.  The lower part
 *     L_i = sum_{j<=i} exp(s_j - s_i) x_j
 * obeys the printed recurrence L_{i+1} = x_{i+1} + exp(s_i - s_{i+1}) L_i; the
 * upper part U_i = sum_{j>=i} exp(s_i - s_j) x_j is its mirror (the suffix scan
 * the same passage names).  Both include the diagonal, so y = L + U - x.
 */
void orc_sym_sorted(int64_t n, int64_t B, const double* s, const double* x, double* y)
{
    for (int64_t c = 0; c < B; ++c) {
        double L = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            double d = (i == 0) ? 0.0 : exp(s[i - 1] - s[i]);
            L = x[i * B + c] + d * L;
            y[i * B + c] = L;
        }
        double U = 0.0;
        for (int64_t i = n - 1; i >= 0; --i) {
            double d = (i == n - 1) ? 0.0 : exp(s[i] - s[i + 1]);
            U = x[i * B + c] + d * U;
            y[i * B + c] += U - x[i * B + c];
        }
    }
}

/* first index i in sorted sa[0..n) with sa[i] >= v (plain binary search) */
static int64_t lower_bound(const double* sa, int64_t n, double v)
{
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        if (sa[mid] < v) lo = mid + 1; else hi = mid;
    }
    return lo;
}

/*
 * General case a != b, [IT] §2.2 "Caso Generale": the contributions of the
 * b-anchors are gathered into the intervals cut by the sorted a-anchors, as two
 * summary vectors u and v, which the symmetric recurrences then propagate.
 * For b_j, lb = first a-index with a >= b_j:
 *     u_lb     += exp(b_j - a_lb)     x_j   (reaches every a_i >= b_j)
 *     v_{lb-1} += exp(a_{lb-1} - b_j) x_j   (reaches every a_i <  b_j)
 *     L_i = u_i + exp(a_{i-1} - a_i) L_{i-1},  U_i = v_i + exp(a_i - a_{i+1}) U_{i+1},
 *     y = L + U      (no diagonal: every pair (i, j) sits in exactly one part).
 * x is [k, B] in sorted-b order, y is [n, B] in sorted-a order.
 */
void orc_general_sorted(int64_t n, int64_t k, int64_t B, const double* sa, const double* sb,
                        const double* x, double* y)
{
    if (n <= 0) return;
    double* u = (double*)calloc((size_t)(n * B), sizeof(double));
    double* v = (double*)calloc((size_t)(n * B), sizeof(double));
    for (int64_t j = 0; j < k; ++j) {
        int64_t lb = lower_bound(sa, n, sb[j]);
        for (int64_t c = 0; c < B; ++c) {
            if (lb < n) u[lb * B + c] += exp(sb[j] - sa[lb]) * x[j * B + c];
            if (lb > 0) v[(lb - 1) * B + c] += exp(sa[lb - 1] - sb[j]) * x[j * B + c];
        }
    }
    for (int64_t c = 0; c < B; ++c) {
        double L = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            double d = (i == 0) ? 0.0 : exp(sa[i - 1] - sa[i]);
            L = u[i * B + c] + d * L;
            y[i * B + c] = L;
        }
        double U = 0.0;
        for (int64_t i = n - 1; i >= 0; --i) {
            double d = (i == n - 1) ? 0.0 : exp(sa[i] - sa[i + 1]);
            U = v[i * B + c] + d * U;
            y[i * B + c] += U;
        }
    }
    free(u);
    free(v);
}

/*
 * Signed sums for the anchor gradient of the backward pass ("LAPLEX - La FFT dei
 * Nuclei di Laplace Apprendibili", technical summary §2.3 and §4.1, name the
 * differentiability w.r.t. the anchors without a formula).
 * With |.|' = sign and sign(0) = 0,
 *     D_i = sum_j sign(s_i - s_j) exp(-|s_i - s_j|) v_j
 *         = (sum over s_j < s_i) - (sum over s_j > s_i).
 * Computed group by group over runs of equal anchors: every member of a run
 * sees the same strictly-lower sum exp(s_prev - s_run) * (all of v up to the
 * previous run), and the mirror for the strictly-upper sum.  Output D is [n, B].
 */
void orc_signed_sorted(int64_t n, int64_t B, const double* s, const double* v, double* D)
{
    for (int64_t c = 0; c < B; ++c) {
        double below = 0.0;       /* sum_{j < run start} exp(s_j - s_{run start - 1}) v_j */
        int64_t i = 0;
        while (i < n) {
            int64_t e = i;
            while (e < n && s[e] == s[i]) ++e;
            double lower = (i == 0) ? 0.0 : exp(s[i - 1] - s[i]) * below;
            double run = 0.0;
            for (int64_t m = i; m < e; ++m) {
                D[m * B + c] = lower;
                run += v[m * B + c];
            }
            below = lower + run;
            i = e;
        }
        double above = 0.0;
        i = n - 1;
        while (i >= 0) {
            int64_t b = i;
            while (b >= 0 && s[b] == s[i]) --b;
            double upper = (i == n - 1) ? 0.0 : exp(s[i] - s[i + 1]) * above;
            double run = 0.0;
            for (int64_t m = i; m > b; --m) {
                D[m * B + c] -= upper;
                run += v[m * B + c];
            }
            above = upper + run;
            i = b;
        }
    }
}

/*
 * Dense rows by the definition, [IT] §2.1 "L'Operatore":
 *     LAPLEX(a, phi; b, psi)_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j),
 * evaluated for m chosen rows i, summing over every j with |a_i - b_j| < cutoff
 * (found by binary search in the sorted b).  With cutoff >= 746 the skipped
 * terms are exactly 0.0 in fp64 (exp underflows), so each row equals the full
 * dense row.  phi/psi may be NULL (unphased).  For each row and column c:
 *     out[r, c]  = sum_j K_ij x_j
 *     sgn[r, c]  = sum_j sign(a_i - b_j) exp(-|a_i - b_j|) x_j   (if sgn != NULL)
 *     absn[r, c] = sum_j exp(-|a_i - b_j|) |x_j|                 (if absn != NULL)
 */
void orc_rows_window(int64_t m, const double* ra, const double* rphi,
                     int64_t k, int64_t B, const double* sb, const double* spsi,
                     const double* x, double cutoff,
                     double* out, double* sgn, double* absn)
{
    for (int64_t r = 0; r < m; ++r) {
        double ai = ra[r];
        int64_t lo = lower_bound(sb, k, ai - cutoff);
        int64_t hi = lower_bound(sb, k, ai + cutoff);
        while (hi < k && sb[hi] <= ai + cutoff) ++hi;
        for (int64_t c = 0; c < B; ++c) {
            double acc = 0.0, accs = 0.0, acca = 0.0;
            for (int64_t j = lo; j < hi; ++j) {
                double diff = ai - sb[j];
                double w = exp(-fabs(diff));
                double ph = (rphi && spsi) ? cos(rphi[r] - spsi[j]) : 1.0;
                double xv = x[j * B + c];
                acc += w * ph * xv;
                if (diff > 0) accs += w * xv;
                else if (diff < 0) accs -= w * xv;
                acca += w * fabs(xv);
            }
            out[r * B + c] = acc;
            if (sgn) sgn[r * B + c] = accs;
            if (absn) absn[r * B + c] = acca;
        }
    }
}

/*
 * One-sided decayed sums at query points (not a step of the method: the mass
 * of the terms below a threshold, used by the parity criterion of fp32
 * results).  For anchors sb (ascending, k of them) with values v [k, B] and
 * query points q (ascending, m of them):
 *     dir > 0:  out_i = sum_{j: sb_j < q_i} exp(sb_j - q_i) v_j
 *     dir < 0:  out_i = sum_{j: sb_j > q_i} exp(q_i - sb_j) v_j
 * by one sweep over the merged order: the running sum at the last anchor
 * passed, decayed to the query.
 */
void orc_onesided_sorted(int64_t k, int64_t m, int64_t B, const double* sb, const double* v,
                         const double* q, int dir, double* out)
{
    double* acc = (double*)calloc((size_t)B, sizeof(double));
    if (dir > 0) {
        int64_t j = 0;
        double last = 0.0;
        int any = 0;
        for (int64_t i = 0; i < m; ++i) {
            while (j < k && sb[j] < q[i]) {
                const double f = any ? exp(last - sb[j]) : 0.0;
                for (int64_t c = 0; c < B; ++c) acc[c] = v[j * B + c] + f * acc[c];
                last = sb[j];
                any = 1;
                ++j;
            }
            const double f = any ? exp(last - q[i]) : 0.0;
            for (int64_t c = 0; c < B; ++c) out[i * B + c] = f * acc[c];
        }
    } else {
        int64_t j = k - 1;
        double last = 0.0;
        int any = 0;
        for (int64_t i = m - 1; i >= 0; --i) {
            while (j >= 0 && sb[j] > q[i]) {
                const double f = any ? exp(sb[j] - last) : 0.0;
                for (int64_t c = 0; c < B; ++c) acc[c] = v[j * B + c] + f * acc[c];
                last = sb[j];
                any = 1;
                --j;
            }
            const double f = any ? exp(q[i] - last) : 0.0;
            for (int64_t c = 0; c < B; ++c) out[i * B + c] = f * acc[c];
        }
    }
    free(acc);
}
