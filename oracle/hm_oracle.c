/*
 * hm_oracle.c -- plain, slow, fp64 CPU oracle for the HedgeMamba mixer scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) links, loads or calls this file.  Only the tests,
 * the smoke check and the benchmark's CPU-baseline leg use it.
 *
 * Every function below is the plain definition of one step, written out in
 * double precision with straightforward loops.  There is no chunking, no
 * blocking and no reordering of sums beyond what the definition states.  The
 * only parallelism is an OpenMP loop over independent (batch, head) pairs or
 * independent rows, which does not change any arithmetic.
 *
 * Sources (the pages this follows):
 *   [HM]  "HedgeMamba: fusing linear attention and state space models"
 *         (gsyq.cn news 1418924), sec. 2.1 (Hedgehog map), sec. 2.3 (mixer:
 *         value projection, doubled state, num/den normalisation, gate and
 *         conv kept), sec. 3.1 (stage-1 identity initialisation), sec. 5.2
 *         (walk-through of the mixer listing), sec. 5.3 (feature-map listing).
 *   [LA]  "Linear attention explained" (cnblogs ying-chease 22790249),
 *         sec. 2 (kernel form, associativity), sec. 3 (recurrent form),
 *         sec. 4.3 (RetNet constant decay), Q/K/V/S shape section.
 *   [SSM] "State space models: Mamba, S4" (quant67 56-ssm), sec. 3.2 (dt
 *         through softplus), sec. 4.2 (affine-map composition).
 *
 * Layouts (row-major, C order):
 *   token-major activations  [B, L, H, X]  (X = d, F or dv)
 *   state S                  [B, H, F, dv]  (row = feature, column = value)
 *   state z                  [B, H, F]
 *   dt                       [B, L, H]
 *   A_log                    [H]
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define HMO_EXPORT __attribute__((visibility("default")))

/* softplus(x) = log(1 + e^x), evaluated without overflow:
 * for x > 0 it is x + log1p(e^-x); otherwise log1p(e^x).  [SSM] sec. 3.2. */
HMO_EXPORT double hmo_softplus(double x) {
    if (x > 0.0) return x + log1p(exp(-x));
    return log1p(exp(x));
}

/* Log of the per-(token, head) decay:
 *   l[b,t,h] = -softplus(dt[b,t,h]) * exp(A_log[h]),   a = exp(l).
 * (Mamba-style discretisation; the stage-1 identity init of [HM] sec. 3.1
 * is the case exp(A_log) = 0, i.e. a = 1.)  BL = B*L. */
HMO_EXPORT void hmo_log_decay(const double *dt, int64_t BL, int H,
                              const double *A_log, double *log_a) {
    for (int64_t r = 0; r < BL; ++r)
        for (int h = 0; h < H; ++h) {
            double rate = exp(A_log[h]);
            double sp = hmo_softplus(dt[r * H + h]);
            log_a[r * H + h] = (rate == 0.0) ? 0.0 : -sp * rate;
        }
}

/* Per-feature log decay (the per-dimension decay variant, see
 * hmo_scan_recurrent_ext):  l[b,t,h,f] = -softplus(dt[b,t,h]) * exp(A_log_f[h,f]).
 * BL = B*L; A_log_f is [H, F]; log_a_f is [BL, H, F]. */
HMO_EXPORT void hmo_log_decay_f(const double *dt, int64_t BL, int H, int F,
                                const double *A_log_f, double *log_a_f) {
    for (int64_t r = 0; r < BL; ++r)
        for (int h = 0; h < H; ++h) {
            double sp = hmo_softplus(dt[r * H + h]);
            for (int f = 0; f < F; ++f) {
                double rate = exp(A_log_f[(int64_t)h * F + f]);
                log_a_f[(r * H + h) * F + f] = (rate == 0.0) ? 0.0 : -sp * rate;
            }
        }
}

/* Step size Delta = softplus(dt) ([SSM] sec. 3.2), the factor of the input
 * term in the step-scaled variant; n values. */
HMO_EXPORT void hmo_step_size(const double *dt, int64_t n, double *delta) {
    for (int64_t i = 0; i < n; ++i) delta[i] = hmo_softplus(dt[i]);
}

/* Hedgehog feature map, [HM] sec. 2.1 and sec. 5.3:
 *   u   = W x + b                      (one Linear layer, W is [p, d])
 *   phi = softmax([u, -u])             over the 2p feature axis
 * The "+" half is features 0..p-1, the "-" half is p..2p-1.
 * x is [rows, d]; row r belongs to head (r mod H).  W for head h starts at
 * W + h * w_head_stride (stride 0 = one W shared by all heads); bias likewise
 * (nullable).  phi is [rows, 2p]. */
HMO_EXPORT void hmo_featmap(const double *x, int64_t rows, int H, int d, int p,
                            const double *W, int64_t w_head_stride,
                            const double *bias, int64_t b_head_stride,
                            double *phi) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        int h = (int)(r % H);
        const double *Wh = W + (int64_t)h * w_head_stride;
        const double *bh = bias ? bias + (int64_t)h * b_head_stride : NULL;
        const double *xr = x + r * d;
        double *out = phi + r * 2 * p;
        double *u = (double *)malloc(sizeof(double) * (size_t)p);
        double m = -INFINITY;
        for (int j = 0; j < p; ++j) {
            double acc = bh ? bh[j] : 0.0;
            for (int i = 0; i < d; ++i) acc += Wh[(int64_t)j * d + i] * xr[i];
            u[j] = acc;
            /* max over the concatenation [u, -u] */
            if (acc > m) m = acc;
            if (-acc > m) m = -acc;
        }
        double Z = 0.0;
        for (int j = 0; j < p; ++j) {
            out[j] = exp(u[j] - m);
            out[p + j] = exp(-u[j] - m);
            Z += out[j] + out[p + j];
        }
        for (int f = 0; f < 2 * p; ++f) out[f] /= Z;
        free(u);
    }
}

/* Rotary position embedding on feature vectors ([HM] sec. 5.2: RoPE is
 * applied to phi(Q) and phi(K) in the mixer).  Reading: the "rotate half"
 * pairing of the GPT-NeoX / Pythia models the pages distil from -- feature i
 * pairs with feature i + F/2 -- with angle pos * base^(-2i/F), i < F/2:
 *   x_i'       = x_i cos(angle) - x_{i+F/2} sin(angle)
 *   x_{i+F/2}' = x_i sin(angle) + x_{i+F/2} cos(angle)
 * x, y: [rows, F] (F even; y may alias x); pos: [rows] absolute positions. */
HMO_EXPORT void hmo_rope(const double *x, int64_t rows, int F, const double *pos,
                         double base, double *y) {
    int half = F / 2;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int i = 0; i < half; ++i) {
            double theta = pow(base, -2.0 * (double)i / (double)F);
            double ang = pos[r] * theta;
            double c = cos(ang), s = sin(ang);
            double a = x[r * F + i], b = x[r * F + i + half];
            y[r * F + i] = a * c - b * s;
            y[r * F + i + half] = a * s + b * c;
        }
    }
}

/* Decayed normalised recurrence (spec definition; [HM] sec. 2.3 and
 * 5.2 doubled state; [LA] sec. 3 recurrent form, sec. 4.3 decayed form):
 *   S_t = a_t S_{t-1} + phik_t v_t^T
 *   z_t = a_t z_{t-1} + phik_t
 *   o_t = (phiq_t^T S_t) / (phiq_t^T z_t)
 * phq, phk: [B, L, H, F]; v: [B, L, H, dv]; log_a: [B, L, H] or NULL (a = 1);
 * S0 [B,H,F,dv], z0 [B,H,F] or NULL (zero); o [B, L, H, dv];
 * S_out, z_out nullable.  Returns the number of (t, head) rows whose
 * denominator was not strictly positive (0 when all are). */
HMO_EXPORT int64_t hmo_scan_recurrent(int64_t B, int64_t L, int H, int F, int dv,
                                      const double *phq, const double *phk,
                                      const double *v, const double *log_a,
                                      const double *S0, const double *z0,
                                      double *o, double *S_out, double *z_out) {
    int64_t bad = 0;
    #pragma omp parallel for schedule(dynamic) reduction(+ : bad)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        int64_t b = bh / H;
        int h = (int)(bh % H);
        double *S = (double *)calloc((size_t)F * dv, sizeof(double));
        double *z = (double *)calloc((size_t)F, sizeof(double));
        if (S0) memcpy(S, S0 + bh * F * dv, sizeof(double) * (size_t)F * dv);
        if (z0) memcpy(z, z0 + bh * F, sizeof(double) * (size_t)F);
        for (int64_t t = 0; t < L; ++t) {
            int64_t row = (b * L + t) * H + h;
            double a = log_a ? exp(log_a[row]) : 1.0;
            const double *qk = phq + row * F;
            const double *kk = phk + row * F;
            const double *vv = v + row * dv;
            for (int f = 0; f < F; ++f) {
                z[f] = a * z[f] + kk[f];
                for (int c = 0; c < dv; ++c)
                    S[(int64_t)f * dv + c] = a * S[(int64_t)f * dv + c] + kk[f] * vv[c];
            }
            double den = 0.0;
            for (int f = 0; f < F; ++f) den += qk[f] * z[f];
            if (!(den > 0.0)) bad += 1;
            double *oo = o + row * dv;
            for (int c = 0; c < dv; ++c) {
                double num = 0.0;
                for (int f = 0; f < F; ++f) num += qk[f] * S[(int64_t)f * dv + c];
                oo[c] = num / den;
            }
        }
        if (S_out) memcpy(S_out + bh * F * dv, S, sizeof(double) * (size_t)F * dv);
        if (z_out) memcpy(z_out + bh * F, z, sizeof(double) * (size_t)F);
        free(S);
        free(z);
    }
    return bad;
}

/* The O(L^2) masked form, an independent way to reach the same outputs
 * ([LA] sec. 2 kernel form, with the decay of the spec recurrence
 * unrolled):
 *   w_ij = exp( sum_{j < t <= i} l_t ) * (phiq_i . phik_j),   j <= i
 *   o_i  = sum_j w_ij v_j / sum_j w_ij
 * The decay sum is accumulated directly (never as a difference of prefix
 * sums) so that l = -inf (a = 0) gives an exact zero weight.  Zero initial
 * state only.  Tiny sizes only. */
HMO_EXPORT void hmo_scan_quadratic(int64_t B, int64_t L, int H, int F, int dv,
                                   const double *phq, const double *phk,
                                   const double *v, const double *log_a,
                                   double *o) {
    #pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        int64_t b = bh / H;
        int h = (int)(bh % H);
        for (int64_t i = 0; i < L; ++i) {
            int64_t ri = (b * L + i) * H + h;
            double *oo = o + ri * dv;
            for (int c = 0; c < dv; ++c) oo[c] = 0.0;
            double den = 0.0;
            double logw = 0.0; /* sum_{j < t <= i} l_t for the current j */
            for (int64_t j = i; j >= 0; --j) {
                int64_t rj = (b * L + j) * H + h;
                if (j < i && log_a) {
                    int64_t rt = (b * L + (j + 1)) * H + h;
                    logw += log_a[rt];
                }
                double dot = 0.0;
                for (int f = 0; f < F; ++f) dot += phq[ri * F + f] * phk[rj * F + f];
                double w = exp(logw) * dot;
                den += w;
                for (int c = 0; c < dv; ++c) oo[c] += w * v[rj * dv + c];
            }
            for (int c = 0; c < dv; ++c) oo[c] /= den;
        }
    }
}

/* The recurrence with the two variants of the pages that the plain form
 * leaves out (both off gives exactly hmo_scan_recurrent):
 *
 *  - input scaled by the step size ([HM] sec. 5.2: the mixer calls Mamba's
 *    selective scan, whose discretised input is B-bar = Delta B; [SSM] sec.
 *    3.2: Delta = softplus(dt)).  With in_scale[b,t,h] = Delta_t:
 *        S_t = a_t S_{t-1} + Delta_t phik_t v_t^T,  z_t = a_t z_{t-1} + Delta_t phik_t
 *  - a decay per feature ([LA] sec. 4.4, gated linear attention's
 *    S_i = diag(alpha_i) S_{i-1} + k_i v_i^T; Mamba-1 keeps one A per state
 *    dimension).  With log_a_f[b,t,h,f]:
 *        S_t[f,:] = a_{t,f} S_{t-1}[f,:] + ...,  z_t[f] = a_{t,f} z_{t-1}[f] + ...
 *    replacing the scalar log_a.
 * in_scale [B,L,H] or NULL (1); log_a [B,L,H] or NULL; log_a_f [B,L,H,F] or
 * NULL (when given, log_a is ignored).  Other arguments and the return value
 * as hmo_scan_recurrent. */
HMO_EXPORT int64_t hmo_scan_recurrent_ext(int64_t B, int64_t L, int H, int F, int dv,
                                          const double *phq, const double *phk,
                                          const double *v, const double *log_a,
                                          const double *log_a_f, const double *in_scale,
                                          const double *S0, const double *z0,
                                          double *o, double *S_out, double *z_out) {
    int64_t bad = 0;
    #pragma omp parallel for schedule(dynamic) reduction(+ : bad)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        int64_t b = bh / H;
        int h = (int)(bh % H);
        double *S = (double *)calloc((size_t)F * dv, sizeof(double));
        double *z = (double *)calloc((size_t)F, sizeof(double));
        if (S0) memcpy(S, S0 + bh * F * dv, sizeof(double) * (size_t)F * dv);
        if (z0) memcpy(z, z0 + bh * F, sizeof(double) * (size_t)F);
        for (int64_t t = 0; t < L; ++t) {
            int64_t row = (b * L + t) * H + h;
            double sc = in_scale ? in_scale[row] : 1.0;
            const double *qk = phq + row * F;
            const double *kk = phk + row * F;
            const double *vv = v + row * dv;
            for (int f = 0; f < F; ++f) {
                double a = log_a_f ? exp(log_a_f[row * F + f]) : (log_a ? exp(log_a[row]) : 1.0);
                double kf = sc * kk[f];
                z[f] = a * z[f] + kf;
                for (int c = 0; c < dv; ++c)
                    S[(int64_t)f * dv + c] = a * S[(int64_t)f * dv + c] + kf * vv[c];
            }
            double den = 0.0;
            for (int f = 0; f < F; ++f) den += qk[f] * z[f];
            if (!(den > 0.0)) bad += 1;
            double *oo = o + row * dv;
            for (int c = 0; c < dv; ++c) {
                double num = 0.0;
                for (int f = 0; f < F; ++f) num += qk[f] * S[(int64_t)f * dv + c];
                oo[c] = num / den;
            }
        }
        if (S_out) memcpy(S_out + bh * F * dv, S, sizeof(double) * (size_t)F * dv);
        if (z_out) memcpy(z_out + bh * F, z, sizeof(double) * (size_t)F);
        free(S);
        free(z);
    }
    return bad;
}

/* The O(L^2) masked form of hmo_scan_recurrent_ext (zero initial state):
 *   w_ij = Delta_j * sum_f phiq_if phik_jf exp( sum_{j < t <= i} l_{t,f} ),  j <= i
 *   o_i  = sum_j w_ij v_j / sum_j w_ij
 * with l_{t,f} = log_a_f[t,f] (or log_a[t] for every f, or 0) and Delta_j =
 * in_scale[j] (or 1).  Each feature's decay sum is accumulated directly, as in
 * hmo_scan_quadratic.  Tiny sizes only. */
HMO_EXPORT void hmo_scan_quadratic_ext(int64_t B, int64_t L, int H, int F, int dv,
                                       const double *phq, const double *phk,
                                       const double *v, const double *log_a,
                                       const double *log_a_f, const double *in_scale,
                                       double *o) {
    #pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        int64_t b = bh / H;
        int h = (int)(bh % H);
        double *logw = (double *)malloc(sizeof(double) * (size_t)F);
        for (int64_t i = 0; i < L; ++i) {
            int64_t ri = (b * L + i) * H + h;
            double *oo = o + ri * dv;
            for (int c = 0; c < dv; ++c) oo[c] = 0.0;
            for (int f = 0; f < F; ++f) logw[f] = 0.0;
            double den = 0.0;
            for (int64_t j = i; j >= 0; --j) {
                int64_t rj = (b * L + j) * H + h;
                if (j < i) {
                    int64_t rt = (b * L + (j + 1)) * H + h;
                    for (int f = 0; f < F; ++f)
                        logw[f] += log_a_f ? log_a_f[rt * F + f] : (log_a ? log_a[rt] : 0.0);
                }
                double w = 0.0;
                for (int f = 0; f < F; ++f) w += phq[ri * F + f] * phk[rj * F + f] * exp(logw[f]);
                if (in_scale) w *= in_scale[rj];
                den += w;
                for (int c = 0; c < dv; ++c) oo[c] += w * v[rj * dv + c];
            }
            for (int c = 0; c < dv; ++c) oo[c] /= den;
        }
        free(logw);
    }
}

/* One recurrent decode step ([LA] sec. 3 and sec. 5, recurrent mode):
 * the recurrence above for a single new token per (batch, head), with the
 * state updated in place.  phq, phk [B,H,F]; v, o [B,H,dv]; log_a [B,H] or
 * NULL; S [B,H,F,dv]; z [B,H,F]. */
HMO_EXPORT int64_t hmo_decode_step(int64_t B, int H, int F, int dv,
                                   const double *phq, const double *phk,
                                   const double *v, const double *log_a,
                                   double *S, double *z, double *o) {
    return hmo_scan_recurrent(B, 1, H, F, dv, phq, phk, v, log_a, S, z, o, S, z);
}

/* Depthwise causal convolution along the sequence ([HM] sec. 2.2, 2.3 and
 * 3.1: the Mamba short conv, kept in the mixer):
 *   y[b,t,c] = bias[c] + sum_{j=0}^{K-1} w[c, j] * x[b, t-(K-1)+j, c]
 * with x = 0 for t-(K-1)+j < 0; no activation.  x, y [B, L, C]; w [C, K];
 * bias [C] or NULL. */
HMO_EXPORT void hmo_causal_conv(int64_t B, int64_t L, int C, int K,
                                const double *x, const double *w,
                                const double *bias, double *y) {
    #pragma omp parallel for schedule(static)
    for (int64_t bt = 0; bt < B * L; ++bt) {
        int64_t b = bt / L, t = bt % L;
        for (int c = 0; c < C; ++c) {
            double acc = bias ? bias[c] : 0.0;
            for (int j = 0; j < K; ++j) {
                int64_t s = t - (K - 1) + j;
                if (s >= 0) acc += w[(int64_t)c * K + j] * x[(b * L + s) * C + c];
            }
            y[bt * C + c] = acc;
        }
    }
}
