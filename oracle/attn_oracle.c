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
 *   - grouped K/V heads (n_kv_head < n_head: "autoresearch" README, section 7.3,
 *     where n_kv_head may be smaller than n_head, and section 10.2.1, item 4,
 *     n_kv_head = n_head / 2): query head h reads K/V head h / (H / Hkv), as in
 *     FlashAttention's grouped-query convention, and dk, dv of a K/V head sum
 *     the contributions of every query head of its group.  Hkv = H is plain
 *     multi-head attention.
 *
 * Everything is the plain definition written out in fp64: two-pass softmax
 * (max, then sum), delta computed as sum_j P_ij dP_ij (not as dO.o), and the
 * key-side gradients computed column by column.  No tiling, no fusion, no
 * online softmax.
 *
 * Layouts: q, o, dO, dq are [B, T, H, D] row-major fp64; k, v, dk, dv are
 * [B, T, Hkv, D]; lse and delta are [B, H, T].  Work is split over (head, row)
 * with OpenMP.
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

/* Per-head views: row t of head (b, h) of a tensor with NH heads starts at
 * ((b*T + t)*NH + h)*D.  ROW is a query-side tensor (H heads), KROW a K/V-side
 * tensor (Hkv heads). */
#define ROWN(ptr, b, t, h, NH) ((ptr) + ((((long)(b) * T + (t)) * (NH) + (h)) * D))
#define ROW(ptr, b, t, h) ROWN(ptr, b, t, h, H)
#define KROW(ptr, b, t, h) ROWN(ptr, b, t, h, Hkv)

/* Normalise all rows of one head of x (NH heads) into xh (T x D contiguous), r into rr. */
static void norm_head(const double *x, long b, long h, long T, long NH, long D, double eps,
                      double *xh, double *rr) {
    for (long t = 0; t < T; ++t) rr[t] = rms_row(ROWN(x, b, t, h, NH), D, eps, xh + t * D);
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
 * Forward for the query heads listed in `heads` (flat b*H + h indices; NULL
 * means all B*H heads).  Writes o [B,T,H,D] and lse [B,H,T] for those heads
 * only.  k and v have Hkv heads (H a multiple of Hkv).
 */
void oracle_attn_fwd_gqa(const double *q, const double *k, const double *v,
                         long B, long T, long H, long Hkv, long D, long window, double eps, double scale,
                         double *o, double *lse, const long *heads, long n_heads) {
    long nh = heads ? n_heads : B * H;
    long grp = H / Hkv;
    double *qh = (double *)malloc(sizeof(double) * T * D);
    double *kh = (double *)malloc(sizeof(double) * T * D);
    double *rq = (double *)malloc(sizeof(double) * T);
    double *rk = (double *)malloc(sizeof(double) * T);
    for (long n = 0; n < nh; ++n) {
        long bh = heads ? heads[n] : n;
        long b = bh / H, h = bh % H, hk = h / grp;
        norm_head(q, b, h, T, H, D, eps, qh, rq);
        norm_head(k, b, hk, T, Hkv, D, eps, kh, rk);
#pragma omp parallel for schedule(dynamic, 4)
        for (long i = 0; i < T; ++i) {
            double L = row_lse(qh, kh, i, window, D, scale);
            lse[(b * H + h) * T + i] = L;
            double *oi = ROW(o, b, i, h);
            for (long d = 0; d < D; ++d) oi[d] = 0.0;
            for (long j = first_key(i, window); j <= i; ++j) {
                double p = exp(scale * dot(qh + i * D, kh + j * D, D) - L);
                const double *vj = KROW(v, b, j, hk);
                for (long d = 0; d < D; ++d) oi[d] += p * vj[d];
            }
        }
    }
    free(qh); free(kh); free(rq); free(rk);
}

void oracle_attn_fwd(const double *q, const double *k, const double *v,
                     long B, long T, long H, long D, long window, double eps, double scale,
                     double *o, double *lse, const long *heads, long n_heads) {
    oracle_attn_fwd_gqa(q, k, v, B, T, H, H, D, window, eps, scale, o, lse, heads, n_heads);
}

/*
 * Backward for the K/V heads listed in `heads` (flat b*Hkv + hk indices; NULL
 * means all B*Hkv heads), and for every query head of their groups.
 * Recomputes the forward statistics of each query head h, then:
 *   dV_j = sum_h sum_i P_ij dO_i ; dP_ij = dO_i . v_j ; delta_i = sum_j P_ij dP_ij ;
 *   dS_ij = P_ij (dP_ij - delta_i) ;
 *   dqhat_i = scale sum_j dS_ij khat_j ; dkhat_j = scale sum_h sum_i dS_ij qhat_i ;
 *   dq, dk through the RMSNorm gradient (sum_h over the query heads of the
 *   K/V head's group; a single head when Hkv = H).
 * Also returns lse and delta [B,H,T] of those query heads (may be NULL).
 */
void oracle_attn_bwd_gqa(const double *q, const double *k, const double *v, const double *dO,
                         long B, long T, long H, long Hkv, long D, long window, double eps, double scale,
                         double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
                         const long *heads, long n_heads) {
    long nh = heads ? n_heads : B * Hkv;
    long grp = H / Hkv;
    double *qh = (double *)malloc(sizeof(double) * T * D);
    double *kh = (double *)malloc(sizeof(double) * T * D);
    double *rq = (double *)malloc(sizeof(double) * T);
    double *rk = (double *)malloc(sizeof(double) * T);
    double *L = (double *)malloc(sizeof(double) * T);
    double *delta = (double *)malloc(sizeof(double) * T);
    double *gk = (double *)malloc(sizeof(double) * T * D);  /* dkhat_j, summed over the group */
    for (long n = 0; n < nh; ++n) {
        long bhk = heads ? heads[n] : n;
        long b = bhk / Hkv, hk = bhk % Hkv;
        norm_head(k, b, hk, T, Hkv, D, eps, kh, rk);
        for (long t = 0; t < T * D; ++t) gk[t] = 0.0;
        for (long j = 0; j < T; ++j) {
            double *dvj = KROW(dv, b, j, hk);
            for (long d = 0; d < D; ++d) dvj[d] = 0.0;
        }
        for (long h = hk * grp; h < (hk + 1) * grp; ++h) {
            norm_head(q, b, h, T, H, D, eps, qh, rq);
            /* Row pass: lse_i, delta_i, dq_i. */
#pragma omp parallel for schedule(dynamic, 4)
            for (long i = 0; i < T; ++i) {
                const double *dOi = ROW(dO, b, i, h);
                long j0 = first_key(i, window);
                double Li = row_lse(qh, kh, i, window, D, scale);
                double di = 0.0;
                for (long j = j0; j <= i; ++j) {
                    double p = exp(scale * dot(qh + i * D, kh + j * D, D) - Li);
                    di += p * dot(dOi, KROW(v, b, j, hk), D);
                }
                L[i] = Li;
                delta[i] = di;
                double *g = (double *)malloc(sizeof(double) * D);
                for (long d = 0; d < D; ++d) g[d] = 0.0;
                for (long j = j0; j <= i; ++j) {
                    double p = exp(scale * dot(qh + i * D, kh + j * D, D) - Li);
                    double ds = p * (dot(dOi, KROW(v, b, j, hk), D) - di);
                    for (long d = 0; d < D; ++d) g[d] += scale * ds * kh[j * D + d];
                }
                rms_row_bwd(g, qh + i * D, rq[i], D, ROW(dq, b, i, h));
                free(g);
            }
            /* Column pass: this query head's share of dv_j and dkhat_j (needs
             * every lse_i and delta_i of the head). */
#pragma omp parallel for schedule(dynamic, 4)
            for (long j = 0; j < T; ++j) {
                double *g = gk + j * D;
                double *dvj = KROW(dv, b, j, hk);
                const double *vj = KROW(v, b, j, hk);
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
            }
            for (long i = 0; i < T; ++i) {
                if (lse_out) lse_out[(b * H + h) * T + i] = L[i];
                if (delta_out) delta_out[(b * H + h) * T + i] = delta[i];
            }
        }
        /* dk through the RMSNorm gradient of the summed dkhat. */
#pragma omp parallel for schedule(static)
        for (long j = 0; j < T; ++j) rms_row_bwd(gk + j * D, kh + j * D, rk[j], D, KROW(dk, b, j, hk));
    }
    free(qh); free(kh); free(rq); free(rk); free(L); free(delta); free(gk);
}

void oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                     long B, long T, long H, long D, long window, double eps, double scale,
                     double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
                     const long *heads, long n_heads) {
    oracle_attn_bwd_gqa(q, k, v, dO, B, T, H, H, D, window, eps, scale, dq, dk, dv, lse_out, delta_out,
                        heads, n_heads);
}
