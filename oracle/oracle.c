/*
 * oracle.c -- plain, slow, sequential fp64 CPU reference of the HGRN2 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference legs use it.  It shares no code, header, helper or constant with
 * the CUDA library under linear_attention_hgrn2_b200/csrc.
 *
 * What it computes (source: "HGRN2: Gated Linear RNNs with State Expansion",
 * Qin et al. 2024, arXiv 2404.07904, as summarised on the paperlayer.ai page):
 *
 *   §2.1  the input gate is tied to the forget gate: input gate = 1 - f_t.
 *   §3.2  the input gate's element-wise product becomes an outer product, the
 *         hidden state is a d_k x d_v matrix, the forget gate is diagonal and
 *         the output is a matrix-vector product with the state.
 *   §3.2  multi-head: heads are independent, each with its own state.
 *   §5    one decay rate per key dimension (not one per head).
 *
 * Written out per head, with f_t = exp(log_f_t) and k_t = 1 - f_t:
 *
 *   S_t = Diag(f_t) S_{t-1} + k_t i_t^T          (d_k x d_v, row j = key dim)
 *   o_t = S_t^T q_t                              (reads the UPDATED state)
 *
 * k_t is computed as -expm1(log_f_t) so that it keeps full relative precision
 * when f_t is close to 1.
 *
 * Layouts: token tensors [B][T][H][D] (D fastest), states [B][H][d_k][d_v].
 * All arithmetic is double precision.  OpenMP (when enabled) only splits the
 * independent (batch, head) pairs; each pair runs the plain sequential loop.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define TOK(b, t, h, j, T, H, D) ((((size_t)(b) * (T) + (t)) * (H) + (h)) * (D) + (j))
#define ST(b, h, B, H, dk, dv) (((size_t)(b) * (H) + (h)) * (size_t)(dk) * (dv))

/* Forward: o and (optionally) hT from q, log_f, i and an optional h0.
 * Pointers h0 and hT may be NULL (h0 = NULL means a zero initial state). */
void oracle_fwd(const double *q, const double *log_f, const double *x,
                const double *h0, double *o, double *hT,
                int B, int T, int H, int dk, int dv)
{
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
            if (h0) memcpy(S, h0 + ST(b, h, B, H, dk, dv), sizeof(double) * dk * dv);
            for (int t = 0; t < T; ++t) {
                /* state update S_t = Diag(f_t) S_{t-1} + k_t i_t^T */
                for (int j = 0; j < dk; ++j) {
                    double a = log_f[TOK(b, t, h, j, T, H, dk)];
                    double f = exp(a);
                    double k = -expm1(a);
                    for (int v = 0; v < dv; ++v)
                        S[j * dv + v] = f * S[j * dv + v] + k * x[TOK(b, t, h, v, T, H, dv)];
                }
                /* output o_t = S_t^T q_t */
                for (int v = 0; v < dv; ++v) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j)
                        acc += q[TOK(b, t, h, j, T, H, dk)] * S[j * dv + v];
                    o[TOK(b, t, h, v, T, H, dv)] = acc;
                }
            }
            if (hT) memcpy(hT + ST(b, h, B, H, dk, dv), S, sizeof(double) * dk * dv);
            free(S);
        }
    }
}

/* One recurrent decode step, in place on S [B][H][dk][dv]:
 * S <- Diag(f) S + k i^T, then o = S^T q (updated state).  Token tensors are
 * [B][H][D].  This is the forward body above for a single t. */
void oracle_step(const double *q, const double *log_f, const double *x,
                 double *S, double *o, int B, int H, int dk, int dv)
{
#pragma omp parallel for collapse(2)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *s = S + ST(b, h, B, H, dk, dv);
            size_t tk = ((size_t)b * H + h) * dk, tv = ((size_t)b * H + h) * dv;
            for (int j = 0; j < dk; ++j) {
                double a = log_f[tk + j];
                double f = exp(a), k = -expm1(a);
                for (int v = 0; v < dv; ++v) s[j * dv + v] = f * s[j * dv + v] + k * x[tv + v];
            }
            for (int v = 0; v < dv; ++v) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += q[tk + j] * s[j * dv + v];
                o[tv + v] = acc;
            }
        }
    }
}

/* Backward by plain back-propagation through time of the forward above.
 *
 * Given dO = dL/do (same layout as o) and an optional dhT = dL/dhT, returns
 * dq, dlog_f, di and (optionally) dh0.  Going backwards over t, with dS the
 * gradient of the loss w.r.t. S_t:
 *
 *   dS      += q_t dO_t^T                  (o_t = S_t^T q_t)
 *   dq_t     = S_t dO_t
 *   dk_t     = dS i_t                      (S_t contains k_t i_t^T)
 *   di_t     = dS^T k_t
 *   df_t[j]  = sum_v dS[j,v] S_{t-1}[j,v]  (S_t contains Diag(f_t) S_{t-1})
 *   dlog_f_t = f_t * (df_t - dk_t)         (f = exp(a), k = 1 - exp(a))
 *   dS       = Diag(f_t) dS                (gradient w.r.t. S_{t-1})
 *
 * and finally dh0 = dS.  S_{t-1} is needed at every step; it is recomputed
 * from checkpoints stored every CKPT steps of a forward pass (a memory scheme
 * only: the arithmetic is the forward loop above, repeated).
 *
 * dk_out, when non-NULL, receives dL/dk_t (layout [B][T][H][dk]); it is not a
 * gradient of any input, it is exposed so that tests can check an alternative
 * closed-form expression of dlog_f against this one. */
#define CKPT 64
void oracle_bwd(const double *q, const double *log_f, const double *x,
                const double *h0, const double *dO, const double *dhT,
                double *dq, double *dlog_f, double *dx, double *dh0, double *dk_out,
                int B, int T, int H, int dk, int dv)
{
    int nck = (T + CKPT - 1) / CKPT;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            size_t sd = (size_t)dk * dv;
            /* ck[c] = state before step c*CKPT (i.e. S_{c*CKPT - 1}) */
            double *ck = (double *)calloc((size_t)(nck + 1) * sd, sizeof(double));
            double *seg = (double *)malloc((size_t)(CKPT + 1) * sd * sizeof(double));
            double *dS = (double *)calloc(sd, sizeof(double));
            double *S = (double *)calloc(sd, sizeof(double));
            if (h0) memcpy(S, h0 + ST(b, h, B, H, dk, dv), sizeof(double) * sd);
            /* forward pass storing checkpoints */
            for (int t = 0; t < T; ++t) {
                if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * sd, S, sizeof(double) * sd);
                for (int j = 0; j < dk; ++j) {
                    double a = log_f[TOK(b, t, h, j, T, H, dk)];
                    double f = exp(a), k = -expm1(a);
                    for (int v = 0; v < dv; ++v)
                        S[j * dv + v] = f * S[j * dv + v] + k * x[TOK(b, t, h, v, T, H, dv)];
                }
            }
            if (dhT) memcpy(dS, dhT + ST(b, h, B, H, dk, dv), sizeof(double) * sd);
            /* backward over checkpoint segments, last segment first */
            for (int c = nck - 1; c >= 0; --c) {
                int t0 = c * CKPT, t1 = t0 + CKPT < T ? t0 + CKPT : T;
                /* seg[m] = S_{t0 + m - 1}, m = 0 .. t1 - t0 */
                memcpy(seg, ck + (size_t)c * sd, sizeof(double) * sd);
                for (int t = t0; t < t1; ++t) {
                    double *prev = seg + (size_t)(t - t0) * sd, *cur = prev + sd;
                    for (int j = 0; j < dk; ++j) {
                        double a = log_f[TOK(b, t, h, j, T, H, dk)];
                        double f = exp(a), k = -expm1(a);
                        for (int v = 0; v < dv; ++v)
                            cur[j * dv + v] = f * prev[j * dv + v] + k * x[TOK(b, t, h, v, T, H, dv)];
                    }
                }
                for (int t = t1 - 1; t >= t0; --t) {
                    const double *Sp = seg + (size_t)(t - t0) * sd; /* S_{t-1} */
                    const double *St = Sp + sd;                     /* S_t */
                    const double *qt = q + TOK(b, t, h, 0, T, H, dk);
                    const double *gt = dO + TOK(b, t, h, 0, T, H, dv);
                    const double *xt = x + TOK(b, t, h, 0, T, H, dv);
                    for (int j = 0; j < dk; ++j)
                        for (int v = 0; v < dv; ++v) dS[j * dv + v] += qt[j] * gt[v];
                    for (int j = 0; j < dk; ++j) {
                        double acc = 0.0;
                        for (int v = 0; v < dv; ++v) acc += St[j * dv + v] * gt[v];
                        dq[TOK(b, t, h, j, T, H, dk)] = acc;
                    }
                    for (int v = 0; v < dv; ++v) {
                        double acc = 0.0;
                        for (int j = 0; j < dk; ++j) {
                            double k = -expm1(log_f[TOK(b, t, h, j, T, H, dk)]);
                            acc += dS[j * dv + v] * k;
                        }
                        dx[TOK(b, t, h, v, T, H, dv)] = acc;
                    }
                    for (int j = 0; j < dk; ++j) {
                        double a = log_f[TOK(b, t, h, j, T, H, dk)];
                        double f = exp(a);
                        double dkj = 0.0, dfj = 0.0;
                        for (int v = 0; v < dv; ++v) {
                            dkj += dS[j * dv + v] * xt[v];
                            dfj += dS[j * dv + v] * Sp[j * dv + v];
                        }
                        if (dk_out) dk_out[TOK(b, t, h, j, T, H, dk)] = dkj;
                        dlog_f[TOK(b, t, h, j, T, H, dk)] = f * (dfj - dkj);
                        for (int v = 0; v < dv; ++v) dS[j * dv + v] *= f;
                    }
                }
            }
            if (dh0) memcpy(dh0 + ST(b, h, B, H, dk, dv), dS, sizeof(double) * sd);
            free(ck); free(seg); free(dS); free(S);
        }
    }
}

/* ------------------------------------------------------------------------
 * Scalar-decay variant (the contrast of §5: models such as Mamba2 or RetNet
 * keep ONE decay per head and token, and a key of their own):
 *
 *   S_t = g_t S_{t-1} + k_t v_t^T,      o_t = S_t^T q_t,      g_t = exp(log_g_t)
 *
 * q, k: [B][T][H][dk]; v, o: [B][T][H][dv]; log_g: [B][T][H]; states as above.
 * ------------------------------------------------------------------------ */
#define GATE(b, t, h, T, H) (((size_t)(b) * (T) + (t)) * (H) + (h))

void oracle_sd_fwd(const double *q, const double *k, const double *v, const double *log_g,
                   const double *h0, double *o, double *hT, int B, int T, int H, int dk, int dv)
{
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
            if (h0) memcpy(S, h0 + ST(b, h, B, H, dk, dv), sizeof(double) * dk * dv);
            for (int t = 0; t < T; ++t) {
                double g = exp(log_g[GATE(b, t, h, T, H)]);
                for (int j = 0; j < dk; ++j) {
                    double kj = k[TOK(b, t, h, j, T, H, dk)];
                    for (int c = 0; c < dv; ++c)
                        S[j * dv + c] = g * S[j * dv + c] + kj * v[TOK(b, t, h, c, T, H, dv)];
                }
                for (int c = 0; c < dv; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += q[TOK(b, t, h, j, T, H, dk)] * S[j * dv + c];
                    o[TOK(b, t, h, c, T, H, dv)] = acc;
                }
            }
            if (hT) memcpy(hT + ST(b, h, B, H, dk, dv), S, sizeof(double) * dk * dv);
            free(S);
        }
    }
}

/* Backward of oracle_sd_fwd by back-propagation through time.  Going backwards
 * over t, with dS the gradient w.r.t. S_t:
 *
 *   dS      += q_t dO_t^T
 *   dq_t     = S_t dO_t
 *   dk_t     = dS v_t
 *   dv_t     = dS^T k_t
 *   dlog_g_t = g_t * sum_{j,c} dS[j,c] S_{t-1}[j,c]
 *   dS       = g_t dS
 *
 * and dh0 = dS; S_{t-1} is recomputed from checkpoints as in oracle_bwd. */
void oracle_sd_bwd(const double *q, const double *k, const double *v, const double *log_g,
                   const double *h0, const double *dO, const double *dhT,
                   double *dq, double *dk_, double *dv_, double *dlog_g, double *dh0,
                   int B, int T, int H, int dk, int dv)
{
    int nck = (T + CKPT - 1) / CKPT;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            size_t sd = (size_t)dk * dv;
            double *ck = (double *)calloc((size_t)(nck + 1) * sd, sizeof(double));
            double *seg = (double *)malloc((size_t)(CKPT + 1) * sd * sizeof(double));
            double *dS = (double *)calloc(sd, sizeof(double));
            double *S = (double *)calloc(sd, sizeof(double));
            if (h0) memcpy(S, h0 + ST(b, h, B, H, dk, dv), sizeof(double) * sd);
            for (int t = 0; t < T; ++t) {
                if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * sd, S, sizeof(double) * sd);
                double g = exp(log_g[GATE(b, t, h, T, H)]);
                for (int j = 0; j < dk; ++j) {
                    double kj = k[TOK(b, t, h, j, T, H, dk)];
                    for (int c = 0; c < dv; ++c)
                        S[j * dv + c] = g * S[j * dv + c] + kj * v[TOK(b, t, h, c, T, H, dv)];
                }
            }
            if (dhT) memcpy(dS, dhT + ST(b, h, B, H, dk, dv), sizeof(double) * sd);
            for (int c0 = nck - 1; c0 >= 0; --c0) {
                int t0 = c0 * CKPT, t1 = t0 + CKPT < T ? t0 + CKPT : T;
                memcpy(seg, ck + (size_t)c0 * sd, sizeof(double) * sd);
                for (int t = t0; t < t1; ++t) {
                    double *prev = seg + (size_t)(t - t0) * sd, *cur = prev + sd;
                    double g = exp(log_g[GATE(b, t, h, T, H)]);
                    for (int j = 0; j < dk; ++j) {
                        double kj = k[TOK(b, t, h, j, T, H, dk)];
                        for (int c = 0; c < dv; ++c)
                            cur[j * dv + c] = g * prev[j * dv + c] + kj * v[TOK(b, t, h, c, T, H, dv)];
                    }
                }
                for (int t = t1 - 1; t >= t0; --t) {
                    const double *Sp = seg + (size_t)(t - t0) * sd, *St = Sp + sd;
                    const double *qt = q + TOK(b, t, h, 0, T, H, dk), *kt = k + TOK(b, t, h, 0, T, H, dk);
                    const double *vt = v + TOK(b, t, h, 0, T, H, dv), *gt = dO + TOK(b, t, h, 0, T, H, dv);
                    double g = exp(log_g[GATE(b, t, h, T, H)]);
                    for (int j = 0; j < dk; ++j)
                        for (int c = 0; c < dv; ++c) dS[j * dv + c] += qt[j] * gt[c];
                    double dg = 0.0;
                    for (int j = 0; j < dk; ++j) {
                        double aq = 0.0, ak = 0.0;
                        for (int c = 0; c < dv; ++c) {
                            aq += St[j * dv + c] * gt[c];
                            ak += dS[j * dv + c] * vt[c];
                            dg += dS[j * dv + c] * Sp[j * dv + c];
                        }
                        dq[TOK(b, t, h, j, T, H, dk)] = aq;
                        dk_[TOK(b, t, h, j, T, H, dk)] = ak;
                    }
                    for (int c = 0; c < dv; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < dk; ++j) acc += dS[j * dv + c] * kt[j];
                        dv_[TOK(b, t, h, c, T, H, dv)] = acc;
                    }
                    dlog_g[GATE(b, t, h, T, H)] = g * dg;
                    for (size_t e = 0; e < sd; ++e) dS[e] *= g;
                }
            }
            if (dh0) memcpy(dh0 + ST(b, h, B, H, dk, dv), dS, sizeof(double) * sd);
            free(ck); free(seg); free(dS); free(S);
        }
    }
}

/* Number of threads OpenMP will use (1 when built without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif
