/*
 * fp64 CPU oracle for the QK-RMSNorm sliding-window attention core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes, and where the pages define it:
 *   - norm(x): parameter-free RMSNorm over head_dim, applied to q and k right
 *     before the attention product ("autoresearch" README on gitee, section
 *     7.3 "CausalSelfAttention", item 3 "RMSNorm"; Russian code review on
 *     web3.okx.com, paragraph on QK norm).  No gain, no bias.  eps is an
 *     argument (the pages' call passes none; the caller fixes it).
 *   - causal softmax attention with a left window w, FlashAttention-3
 *     window_size=(w, 0) semantics: key j is visible to query i iff
 *     0 <= i - j <= w ("autoresearch" README, section 5.2.1 "Flash Attention 3"
 *     and section 5.2.2 "sliding window attention").  window < 0 means no
 *     left limit (full causal).
 *   - the analytic backward of both, with the RMSNorm gradient.
 *
 * Everything is the plain definition written out in fp64: two-pass softmax
 * (max, then sum), delta computed as sum_j P_ij dP_ij (not as dO.o), and the
 * key-side gradients computed column by column.  No tiling, no fusion, no
 * online softmax.
 *
 * Layouts: q, k, v, o, dO, dq, dk, dv are [B, T, H, D] row-major fp64;
 * lse and delta are [B, H, T].  Work is split over (head, row) with OpenMP.
 *
 * Parity status: every function here is pinned by the CPU tests
 * (library cross-check, finite differences, closed forms, invariants).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Visibility of key j to query i under window w (w < 0: unlimited). */
static int visible(long i, long j, long w) {
    if (j > i) return 0;
    if (w >= 0 && i - j > w) return 0;
    return 1;
}

/* First key visible to query i. */
static long first_key(long i, long w) {
    if (w < 0 || i - w < 0) return 0;
    return i - w;
}

/* Last query that sees key j. */
static long last_query(long j, long w, long T) {
    if (w < 0 || j + w > T - 1) return T - 1;
    return j + w;
}

/* RMSNorm of one row of length D: r = 1/sqrt(mean(x^2) + eps), xhat = r*x. */
static double rms_row(const double *x, long D, double eps, double *xhat) {
    double ss = 0.0;
    for (long d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = 1.0 / sqrt(ss / (double)D + eps);
    for (long d = 0; d < D; ++d) xhat[d] = r * x[d];
    return r;
}

/* Gradient of RMSNorm: given g = dL/dxhat, return dL/dx = r (g - xhat (g.xhat)/D). */
static void rms_row_bwd(const double *g, const double *xhat, double r, long D, double *dx) {
    double gx = 0.0;
    for (long d = 0; d < D; ++d) gx += g[d] * xhat[d];
    for (long d = 0; d < D; ++d) dx[d] = r * (g[d] - xhat[d] * gx / (double)D);
}

static double dot(const double *a, const double *b, long D) {
    double s = 0.0;
    for (long d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* Per-head views: row t of head (b, h) starts at ((b*T + t)*H + h)*D. */
#define ROW(ptr, b, t, h) ((ptr) + ((((long)(b) * T + (t)) * H + (h)) * D))

/* Normalise all rows of one head of x into xh (T x D contiguous), r into rr. */
static void norm_head(const double *x, long b, long h, long T, long H, long D, double eps,
                      double *xh, double *rr) {
    for (long t = 0; t < T; ++t) rr[t] = rms_row(ROW(x, b, t, h), D, eps, xh + t * D);
}

/* Softmax statistics of query row i: returns lse_i; s_ij over visible keys. */
static double row_lse(const double *qh, const double *kh, long i, long w, long D, double scale) {
    long j0 = first_key(i, w);
    double m = -INFINITY;
    for (long j = j0; j <= i; ++j) {
        double s = scale * dot(qh + i * D, kh + j * D, D);
        if (s > m) m = s;
    }
    double sum = 0.0;
    for (long j = j0; j <= i; ++j) {
        double s = scale * dot(qh + i * D, kh + j * D, D);
        sum += exp(s - m);
    }
    return m + log(sum);
}

/*
 * Forward for the heads listed in `heads` (flat b*H + h indices; NULL means
 * all B*H heads).  Writes o [B,T,H,D] and lse [B,H,T] for those heads only.
 */
void oracle_attn_fwd(const double *q, const double *k, const double *v,
                     long B, long T, long H, long D, long window, double eps, double scale,
                     double *o, double *lse, const long *heads, long n_heads) {
    long nh = heads ? n_heads : B * H;
    double *qh = (double *)malloc(sizeof(double) * T * D);
    double *kh = (double *)malloc(sizeof(double) * T * D);
    double *rq = (double *)malloc(sizeof(double) * T);
    double *rk = (double *)malloc(sizeof(double) * T);
    for (long n = 0; n < nh; ++n) {
        long bh = heads ? heads[n] : n;
        long b = bh / H, h = bh % H;
        norm_head(q, b, h, T, H, D, eps, qh, rq);
        norm_head(k, b, h, T, H, D, eps, kh, rk);
#pragma omp parallel for schedule(dynamic, 4)
        for (long i = 0; i < T; ++i) {
            double L = row_lse(qh, kh, i, window, D, scale);
            lse[(b * H + h) * T + i] = L;
            double *oi = ROW(o, b, i, h);
            for (long d = 0; d < D; ++d) oi[d] = 0.0;
            for (long j = first_key(i, window); j <= i; ++j) {
                double p = exp(scale * dot(qh + i * D, kh + j * D, D) - L);
                const double *vj = ROW(v, b, j, h);
                for (long d = 0; d < D; ++d) oi[d] += p * vj[d];
            }
        }
    }
    free(qh); free(kh); free(rq); free(rk);
}

/*
 * Backward for the listed heads.  Recomputes the forward statistics, then:
 *   dV_j = sum_i P_ij dO_i ; dP_ij = dO_i . v_j ; delta_i = sum_j P_ij dP_ij ;
 *   dS_ij = P_ij (dP_ij - delta_i) ;
 *   dqhat_i = scale sum_j dS_ij khat_j ; dkhat_j = scale sum_i dS_ij qhat_i ;
 *   dq, dk through the RMSNorm gradient.
 * Also returns lse and delta [B,H,T] (may be NULL).
 */
void oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                     long B, long T, long H, long D, long window, double eps, double scale,
                     double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
                     const long *heads, long n_heads) {
    long nh = heads ? n_heads : B * H;
    double *qh = (double *)malloc(sizeof(double) * T * D);
    double *kh = (double *)malloc(sizeof(double) * T * D);
    double *rq = (double *)malloc(sizeof(double) * T);
    double *rk = (double *)malloc(sizeof(double) * T);
    double *L = (double *)malloc(sizeof(double) * T);
    double *delta = (double *)malloc(sizeof(double) * T);
    for (long n = 0; n < nh; ++n) {
        long bh = heads ? heads[n] : n;
        long b = bh / H, h = bh % H;
        norm_head(q, b, h, T, H, D, eps, qh, rq);
        norm_head(k, b, h, T, H, D, eps, kh, rk);
        /* Row pass: lse_i, delta_i, dq_i. */
#pragma omp parallel for schedule(dynamic, 4)
        for (long i = 0; i < T; ++i) {
            const double *dOi = ROW(dO, b, i, h);
            long j0 = first_key(i, window);
            double Li = row_lse(qh, kh, i, window, D, scale);
            double di = 0.0;
            for (long j = j0; j <= i; ++j) {
                double p = exp(scale * dot(qh + i * D, kh + j * D, D) - Li);
                di += p * dot(dOi, ROW(v, b, j, h), D);
            }
            L[i] = Li;
            delta[i] = di;
            double *g = (double *)malloc(sizeof(double) * D);
            for (long d = 0; d < D; ++d) g[d] = 0.0;
            for (long j = j0; j <= i; ++j) {
                double p = exp(scale * dot(qh + i * D, kh + j * D, D) - Li);
                double ds = p * (dot(dOi, ROW(v, b, j, h), D) - di);
                for (long d = 0; d < D; ++d) g[d] += scale * ds * kh[j * D + d];
            }
            rms_row_bwd(g, qh + i * D, rq[i], D, ROW(dq, b, i, h));
            free(g);
        }
        /* Column pass: dv_j, dk_j (needs every lse_i and delta_i). */
#pragma omp parallel for schedule(dynamic, 4)
        for (long j = 0; j < T; ++j) {
            double *g = (double *)malloc(sizeof(double) * D);
            double *dvj = ROW(dv, b, j, h);
            const double *vj = ROW(v, b, j, h);
            for (long d = 0; d < D; ++d) { g[d] = 0.0; dvj[d] = 0.0; }
            long i1 = last_query(j, window, T);
            for (long i = j; i <= i1; ++i) {
                if (!visible(i, j, window)) continue;
                const double *dOi = ROW(dO, b, i, h);
                double p = exp(scale * dot(qh + i * D, kh + j * D, D) - L[i]);
                double ds = p * (dot(dOi, vj, D) - delta[i]);
                for (long d = 0; d < D; ++d) {
                    dvj[d] += p * dOi[d];
                    g[d] += scale * ds * qh[i * D + d];
                }
            }
            rms_row_bwd(g, kh + j * D, rk[j], D, ROW(dk, b, j, h));
            free(g);
        }
        for (long i = 0; i < T; ++i) {
            if (lse_out) lse_out[(b * H + h) * T + i] = L[i];
            if (delta_out) delta_out[(b * H + h) * T + i] = delta[i];
        }
    }
    free(qh); free(kh); free(rq); free(rk); free(L); free(delta);
}
