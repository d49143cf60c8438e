/*
 * Float64 CPU oracle of the JetBlock token mixer (Jet-Nemotron).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain definition that the
 * CUDA library is checked against. It shares no code with the CUDA library
 * and must never be linked into, or called from, the product path.
 *
 * Sources (Jet-Nemotron paper, Chinese translation on adg.csdn.net, and the
 * explainer on xugj520.cn):
 *   - kernel generator: paper section 2.4 ("new attention block design"):
 *     the generator shares the Q/K/V projections' input, starts with a linear
 *     reduction, applies SiLU, then a final linear layer that outputs the conv
 *     kernel weights. Explainer section 2.2 fixes hidden width 32, kernel 4.
 *   - dynamic causal conv, applied to V only: paper section 2.4; news page
 *     (ai.valimart.net) "design new attention module".
 *   - Gated DeltaNet time mixing: paper section 2.3 (data-dependent gate plus
 *     delta rule), in the form
 *       S_t = a_t (S_{t-1} - b_t (S_{t-1} k_t) k_t^T) + b_t v_t k_t^T,
 *       o_t = S_t q_t,  a_t = exp(g_t),  S in R^{dv x dk},
 *     on L2-normalised q and k, with no 1/sqrt(dk) scale.
 *
 * Readings where the pages are silent: no biases in the generator, no
 * normalisation or activation of the conv taps or the conv output, tap 0 is
 * the current token, one kernel per head shared by its dv channels, the conv
 * acts on raw V and the decode history keeps raw V, L2-norm eps 1e-6 inside
 * the square root.
 *
 * Layouts (row-major): x[B,T,D], W1[D,R], W2[R,H*W], conv weights w[B,T,H,W]
 * (column h*W+j of W2 is tap j of head h), v and o [B,T,H,dv], q and k
 * [B,T,H,dk], g and beta [B,T,H], S[B,H,dv,dk], history hist[B,W-1,H,dv]
 * holding v_{-(W-1)} .. v_{-1} (oldest first).
 *
 * All functions take and return float64. Parallelism (OpenMP) is only over
 * independent items (tokens, or (batch, head) chains); the arithmetic order
 * inside each item is the plain sequential order of the definition.
 */
#include <math.h>
#include <stddef.h>
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

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Kernel generator: h = SiLU(x W1) (D -> R), w = h W2 (R -> H*W). No bias. */
void oracle_kernel_gen(const double* x, const double* W1, const double* W2, double* w,
                       long N, int D, int R, int HW) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        double* z = (double*)calloc((size_t)R, sizeof(double));
        const double* xn = x + n * (long)D;
        for (int d = 0; d < D; ++d) {
            const double xd = xn[d];
            const double* w1 = W1 + (long)d * R;
            for (int r = 0; r < R; ++r) z[r] += xd * w1[r];
        }
        for (int r = 0; r < R; ++r) z[r] = silu(z[r]);
        double* wn = w + n * (long)HW;
        for (int c = 0; c < HW; ++c) {
            double acc = 0.0;
            for (int r = 0; r < R; ++r) acc += z[r] * W2[(long)r * HW + c];
            wn[c] = acc;
        }
        free(z);
    }
}

/* V at sequence position tau (tau may be negative: then it comes from the
 * history, or is zero when there is none). */
static double v_at(const double* v, const double* hist, int b, long tau, int h, int c,
                   long T, int H, int dv, int W) {
    if (tau >= 0) return v[((b * T + tau) * H + h) * (long)dv + c];
    if (!hist) return 0.0;
    const long m = tau + (W - 1);            /* 0 .. W-2 */
    if (m < 0) return 0.0;
    return hist[(((long)b * (W - 1) + m) * H + h) * (long)dv + c];
}

/* Dynamic causal conv on V: v'_t[h,c] = sum_j w_t[h,j] v_{t-j}[h,c].
 * hist may be NULL (zeros). hist_out may be NULL; else it receives the last
 * W-1 raw V tokens of [hist, v], oldest first. */
void oracle_dyn_conv(const double* v, const double* w, const double* hist, double* out,
                     double* hist_out, int B, long T, int H, int dv, int W) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (long t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const double* wt = w + ((b * T + t) * H + h) * (long)W;
                for (int c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < W; ++j)
                        acc += wt[j] * v_at(v, hist, b, t - j, h, c, T, H, dv, W);
                    out[((b * T + t) * H + h) * (long)dv + c] = acc;
                }
            }
    if (hist_out) {
        for (int b = 0; b < B; ++b)
            for (int m = 0; m < W - 1; ++m)
                for (int h = 0; h < H; ++h)
                    for (int c = 0; c < dv; ++c)
                        hist_out[(((long)b * (W - 1) + m) * H + h) * (long)dv + c] =
                            v_at(v, hist, b, T - (W - 1) + m, h, c, T, H, dv, W);
    }
}

/* y = x / sqrt(sum x^2 + eps) */
static void l2norm(const double* x, double* y, int n, double eps) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    const double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] * inv;
}

/* Gated DeltaNet, token by token (the definition). S0 may be NULL (zeros). */
void oracle_gdn_sequential(const double* q, const double* k, const double* v,
                           const double* g, const double* beta, const double* S0,
                           double* o, double* S_out, int B, long T, int H, int dk, int dv,
                           double eps) {
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
            double* qh = (double*)malloc(sizeof(double) * (size_t)dk);
            double* kh = (double*)malloc(sizeof(double) * (size_t)dk);
            const long sbase = ((long)b * H + h) * (long)dv * dk;
            for (long i = 0; i < (long)dv * dk; ++i) S[i] = S0 ? S0[sbase + i] : 0.0;
            for (long t = 0; t < T; ++t) {
                const long bth = (b * T + t) * H + h;
                l2norm(q + bth * dk, qh, dk, eps);
                l2norm(k + bth * dk, kh, dk, eps);
                const double a = exp(g[bth]), bt = beta[bth];
                for (int i = 0; i < dv; ++i) {
                    double* Si = S + (long)i * dk;
                    double u = 0.0;                      /* (S_{t-1} k_t)_i */
                    for (int j = 0; j < dk; ++j) u += Si[j] * kh[j];
                    const double vi = v[bth * dv + i];
                    for (int j = 0; j < dk; ++j)
                        Si[j] = a * (Si[j] - bt * u * kh[j]) + bt * vi * kh[j];
                    double oi = 0.0;                     /* (S_t q_t)_i */
                    for (int j = 0; j < dk; ++j) oi += Si[j] * qh[j];
                    o[bth * dv + i] = oi;
                }
            }
            for (long i = 0; i < (long)dv * dk; ++i) S_out[sbase + i] = S[i];
            free(S); free(qh); free(kh);
        }
}

/* One decode step per sequence, in the single-token update form:
 *   u = S k,  S' = a S + (b v - a b u) k^T,  o = S' q.
 * S is updated in place. q,k [B,H,dk], v and o [B,H,dv], g and beta [B,H]. */
void oracle_gdn_decode_step(const double* q, const double* k, const double* v,
                            const double* g, const double* beta, double* S, double* o,
                            int B, int H, int dk, int dv, double eps) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const long bh = (long)b * H + h;
            double* qh = (double*)malloc(sizeof(double) * (size_t)dk);
            double* kh = (double*)malloc(sizeof(double) * (size_t)dk);
            l2norm(q + bh * dk, qh, dk, eps);
            l2norm(k + bh * dk, kh, dk, eps);
            const double a = exp(g[bh]), bt = beta[bh];
            for (int i = 0; i < dv; ++i) {
                double* Si = S + (bh * dv + i) * (long)dk;
                double u = 0.0;
                for (int j = 0; j < dk; ++j) u += Si[j] * kh[j];
                const double c = bt * v[bh * dv + i] - a * bt * u;
                double oi = 0.0;
                for (int j = 0; j < dk; ++j) {
                    Si[j] = a * Si[j] + c * kh[j];
                    oi += Si[j] * qh[j];
                }
                o[bh * dv + i] = oi;
            }
            free(qh); free(kh);
        }
}

/* Gated DeltaNet in chunked (WY / UT-transform) form, written out from the
 * token recurrence. Within a chunk of L tokens with local index r:
 *   G_r = sum_{s<=r} g_s,  gam_r = exp(G_r)
 *   A_ri = beta_r exp(G_r - G_i) (k_r . k_i)  for i < r  (strictly lower)
 *   (I + A) U = diag(beta) V,  (I + A) W = diag(beta gam) K   (forward substitution)
 *   Wt = U - W S0^T                      (the per-token residual values)
 *   O_r = gam_r S0 q_r + sum_{i<=r} exp(G_r - G_i) (q_r . k_i) Wt_i
 *   S_L = gam_L S0 + sum_i exp(G_L - G_i) Wt_i k_i^T
 * It is an identity check of the token form, not a separate definition. */
void oracle_gdn_chunked(const double* q, const double* k, const double* v,
                        const double* g, const double* beta, const double* S0,
                        double* o, double* S_out, int B, long T, int H, int dk, int dv,
                        int C, double eps) {
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double* S  = (double*)malloc(sizeof(double) * (size_t)dv * dk);
            double* Kh = (double*)malloc(sizeof(double) * (size_t)C * dk);
            double* Qh = (double*)malloc(sizeof(double) * (size_t)C * dk);
            double* G  = (double*)malloc(sizeof(double) * (size_t)C);
            double* A  = (double*)malloc(sizeof(double) * (size_t)C * C);
            double* U  = (double*)malloc(sizeof(double) * (size_t)C * dv);
            double* Wm = (double*)malloc(sizeof(double) * (size_t)C * dk);
            double* Wt = (double*)malloc(sizeof(double) * (size_t)C * dv);
            const long sbase = ((long)b * H + h) * (long)dv * dk;
            for (long i = 0; i < (long)dv * dk; ++i) S[i] = S0 ? S0[sbase + i] : 0.0;
            for (long t0 = 0; t0 < T; t0 += C) {
                const int L = (int)((T - t0) < C ? (T - t0) : C);
                double acc = 0.0;
                for (int r = 0; r < L; ++r) {
                    const long bth = (b * T + t0 + r) * H + h;
                    l2norm(q + bth * dk, Qh + (long)r * dk, dk, eps);
                    l2norm(k + bth * dk, Kh + (long)r * dk, dk, eps);
                    acc += g[bth];
                    G[r] = acc;
                }
                for (int r = 0; r < L; ++r) {
                    const double br = beta[(b * T + t0 + r) * H + h];
                    for (int i = 0; i < L; ++i) {
                        double a = 0.0;
                        if (i < r) {
                            double kk = 0.0;
                            for (int j = 0; j < dk; ++j) kk += Kh[(long)r * dk + j] * Kh[(long)i * dk + j];
                            a = br * exp(G[r] - G[i]) * kk;
                        }
                        A[(long)r * C + i] = a;
                    }
                }
                /* forward substitution: row r of X = rhs_r - sum_{i<r} A_ri X_i */
                for (int r = 0; r < L; ++r) {
                    const long bth = (b * T + t0 + r) * H + h;
                    const double br = beta[bth], gr = exp(G[r]);
                    for (int c = 0; c < dv; ++c) {
                        double x = br * v[bth * dv + c];
                        for (int i = 0; i < r; ++i) x -= A[(long)r * C + i] * U[(long)i * dv + c];
                        U[(long)r * dv + c] = x;
                    }
                    for (int c = 0; c < dk; ++c) {
                        double x = br * gr * Kh[(long)r * dk + c];
                        for (int i = 0; i < r; ++i) x -= A[(long)r * C + i] * Wm[(long)i * dk + c];
                        Wm[(long)r * dk + c] = x;
                    }
                }
                for (int r = 0; r < L; ++r)
                    for (int c = 0; c < dv; ++c) {
                        double ws = 0.0;
                        for (int j = 0; j < dk; ++j) ws += Wm[(long)r * dk + j] * S[(long)c * dk + j];
                        Wt[(long)r * dv + c] = U[(long)r * dv + c] - ws;
                    }
                for (int r = 0; r < L; ++r) {
                    const long bth = (b * T + t0 + r) * H + h;
                    const double gr = exp(G[r]);
                    for (int c = 0; c < dv; ++c) {
                        double qs = 0.0;
                        for (int j = 0; j < dk; ++j) qs += Qh[(long)r * dk + j] * S[(long)c * dk + j];
                        double inter = 0.0;
                        for (int i = 0; i <= r; ++i) {
                            double qk = 0.0;
                            for (int j = 0; j < dk; ++j) qk += Qh[(long)r * dk + j] * Kh[(long)i * dk + j];
                            inter += exp(G[r] - G[i]) * qk * Wt[(long)i * dv + c];
                        }
                        o[bth * dv + c] = gr * qs + inter;
                    }
                }
                const double gL = exp(G[L - 1]);
                for (int c = 0; c < dv; ++c)
                    for (int j = 0; j < dk; ++j) {
                        double s = gL * S[(long)c * dk + j];
                        for (int i = 0; i < L; ++i)
                            s += exp(G[L - 1] - G[i]) * Wt[(long)i * dv + c] * Kh[(long)i * dk + j];
                        S[(long)c * dk + j] = s;
                    }
            }
            for (long i = 0; i < (long)dv * dk; ++i) S_out[sbase + i] = S[i];
            free(S); free(Kh); free(Qh); free(G); free(A); free(U); free(Wm); free(Wt);
        }
}
