/*
 * CPU oracle for the RWKV-4 WKV operator and the per-channel diagonal linear
 * scan.  TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark call it; the library under test never
 * does, and this file shares no code with it.
 *
 * Everything is plain float64 arithmetic, one channel at a time, in the order
 * the defining formulas are written.  OpenMP only spreads independent
 * channels (or independent sample points) over host threads.
 *
 * Sources (web pages this project is built from):
 *   [RWKV-LLM]  "RWKV：基于RNN的LLM", section 二.1 Time-mixing block,
 *               eq. (14): the WKV definition, 1-based in the page,
 *                 wkv_t = (sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u+k_t} v_t)
 *                       / (sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u+k_t})
 *               section 一.2, eq. (10): w is a non-negative per-channel
 *               decay vector.
 *   [RWKV-EVO]  RWKV evolution article (RWKV-V1 to V4), section RWKV-V4:
 *               the same mixing rewritten as a per-token state update
 *               (RNN mode) for inference.
 *   [LRU]       review of "Resurrecting Recurrent Neural Networks for Long
 *               Sequences", linear-RNN section: x_t = lambda x_{t-1} + u_t,
 *               unrolled to x_t = sum_k lambda^{t-k} u_k.
 *   [MINGRU]    "Were RNNs All We Needed?" article, model-architecture
 *               section: the scan form v_t = a_t (.) v_{t-1} + b_t.
 *
 * Layout: k, v, y, a, b, h are [B, T, C] row-major with C fastest; w, u are
 * [C]; h0 is [B, C] or NULL (zeros).  A WKV state is [B, 3, C]: planes a, b,
 * p per batch row, standing for the past sums (num, den) = (a, b) e^p; NULL
 * or a = b = 0 is the empty past.  Inputs and results are float64 (the
 * caller widens the float32 / bf16 values the GPU path reads, exactly).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <omp.h>
#include <stdlib.h>

static int pick_threads(int nthreads) {
    return nthreads > 0 ? nthreads : omp_get_max_threads();
}

int oracle_max_threads(void) { return omp_get_max_threads(); }

/* ------------------------------------------------------------------------
 * WKV, definition form ([RWKV-LLM] eq. 14), 0-based: output at step t of
 * channel c is the weighted average of v_0..v_t with logits
 *     l_i = -(t-1-i) w_c + k_i   for i < t,      l_t = u_c + k_t.
 * Each point is an O(t) direct sum; the common factor e^{-m}, m = max l,
 * is taken out of numerator and denominator so no term overflows.
 *
 * A state before step 0 (RNN mode, [RWKV-EVO] section RWKV-V4; sequential
 * decoding, [RWKV-LLM] section 三) is the pair of past sums (num_0, den_0).  Step t
 * sees it decayed t times, so it adds e^{-t w} (num_0, den_0) to the sums:
 * one more term with logit -t w + p and weights (a, b) in place of (v_i, 1).
 * ------------------------------------------------------------------------ */
static int state_empty(const double *s, int64_t C) {
    /* s points at (a, b, p) of one channel, planes C apart */
    return !s || (s[0] == 0.0 && s[C] == 0.0) || (isinf(s[2 * C]) && s[2 * C] < 0);
}

/* sums over i < t (and the state) of e^{l_i - m} (v_i, 1), with m the largest
 * logit among them and `extra` (a logit the caller adds itself) */
static void past_sums(int64_t C, double w, const double *k, const double *v,
                      const double *s, int64_t t, double extra,
                      double *m_out, double *num, double *den) {
    int has_s = !state_empty(s, C);
    double m = extra;
    for (int64_t i = 0; i < t; ++i) {
        double l = -(double)(t - 1 - i) * w + k[i * C];
        if (l > m) m = l;
    }
    double ls = has_s ? -(double)t * w + s[2 * C] : -INFINITY;
    if (ls > m) m = ls;
    double n = 0.0, d = 0.0;
    for (int64_t i = 0; i < t; ++i) {
        double e = exp(-(double)(t - 1 - i) * w + k[i * C] - m);
        n += e * v[i * C];
        d += e;
    }
    if (has_s) {
        double e = exp(ls - m);
        n += e * s[0];
        d += e * s[C];
    }
    *m_out = m;
    *num = n;
    *den = d;
}

static double wkv_direct_one(int64_t C, double w, double u, const double *k,
                             const double *v, const double *s, int64_t t) {
    /* k, v point at channel c of batch row b (stride C between steps);
     * s at that channel's state or NULL */
    double lt = u + k[t * C];
    double m, num, den;
    past_sums(C, w, k, v, s, t, lt, &m, &num, &den);
    double e_t = exp(lt - m);
    return (num + e_t * v[t * C]) / (den + e_t);
}

static const double *state_at(const double *s, int64_t b, int64_t c, int64_t C) {
    return s ? s + b * 3 * C + c : NULL;
}

/* points[j] is the flat index b*T*C + t*C + c of the j-th requested output */
void oracle_wkv_direct_points_s(int64_t B, int64_t T, int64_t C,
                                const double *w, const double *u,
                                const double *k, const double *v, const double *s_in,
                                int64_t n, const int64_t *points, double *out,
                                int nthreads) {
    (void)B;
#pragma omp parallel for schedule(dynamic, 16) num_threads(pick_threads(nthreads))
    for (int64_t j = 0; j < n; ++j) {
        int64_t f = points[j];
        int64_t b = f / (T * C);
        int64_t t = (f / C) % T;
        int64_t c = f % C;
        const double *kb = k + b * T * C + c;
        const double *vb = v + b * T * C + c;
        out[j] = wkv_direct_one(C, w[c], u[c], kb, vb, state_at(s_in, b, c, C), t);
    }
}

void oracle_wkv_direct_points(int64_t B, int64_t T, int64_t C,
                              const double *w, const double *u,
                              const double *k, const double *v,
                              int64_t n, const int64_t *points, double *out,
                              int nthreads) {
    oracle_wkv_direct_points_s(B, T, C, w, u, k, v, NULL, n, points, out, nthreads);
}

/* every output by the definition: O(T^2) per channel, small inputs only;
 * s_out (if not NULL) gets the past sums after the last step, the same
 * definition at t = T without a current token, as (a, b, p) with p the
 * largest logit */
void oracle_wkv_direct_s(int64_t B, int64_t T, int64_t C,
                         const double *w, const double *u,
                         const double *k, const double *v, const double *s_in,
                         double *y, double *s_out, int nthreads) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(pick_threads(nthreads))
    for (int64_t bc = 0; bc < B * C; ++bc) {
        int64_t b = bc / C, c = bc % C;
        const double *kb = k + b * T * C + c;
        const double *vb = v + b * T * C + c;
        const double *sb = state_at(s_in, b, c, C);
        for (int64_t t = 0; t < T; ++t)
            y[b * T * C + t * C + c] = wkv_direct_one(C, w[c], u[c], kb, vb, sb, t);
        if (s_out) {
            double m, num, den;
            past_sums(C, w[c], kb, vb, sb, T, -INFINITY, &m, &num, &den);
            double *so = s_out + b * 3 * C + c;
            so[0] = num;
            so[C] = den;
            so[2 * C] = m;
        }
    }
}

void oracle_wkv_direct(int64_t B, int64_t T, int64_t C,
                       const double *w, const double *u,
                       const double *k, const double *v, double *y, int nthreads) {
    oracle_wkv_direct_s(B, T, C, w, u, k, v, NULL, y, NULL, nthreads);
}

/* ------------------------------------------------------------------------
 * WKV, RNN mode ([RWKV-EVO] section RWKV-V4; [LRU] RWKV variant): the
 * state before step t is the pair of past sums
 *     num_t = sum_{i<t} e^{-(t-1-i)w + k_i} v_i,   den_t = sum_{i<t} e^{-(t-1-i)w + k_i}
 * which obeys num_{t+1} = e^{-w} num_t + e^{k_t} v_t (same for den with 1).
 * The output adds the current token with bonus u:
 *     y_t = (num_t + e^{u+k_t} v_t) / (den_t + e^{u+k_t}).
 * The pair is stored as (a, b) = (num, den) * e^{-p}; p is the largest
 * exponent seen so far, so every exp() below has a non-positive argument.
 * Starting state: s_in, or empty sums (a = b = 0, p = -inf) when it is NULL;
 * the state after the last step goes to s_out when it is not NULL.
 * ------------------------------------------------------------------------ */
void oracle_wkv_rnn_s(int64_t B, int64_t T, int64_t C,
                      const double *w, const double *u,
                      const double *k, const double *v, const double *s_in,
                      double *y, double *s_out, int nthreads) {
#pragma omp parallel for schedule(static) num_threads(pick_threads(nthreads))
    for (int64_t bc = 0; bc < B * C; ++bc) {
        int64_t b = bc / C, c = bc % C;
        double wc = w[c], uc = u[c];
        double a = 0.0, d = 0.0, p = -INFINITY;
        const double *sb = state_at(s_in, b, c, C);
        if (!state_empty(sb, C)) {
            a = sb[0];
            d = sb[C];
            p = sb[2 * C];
        }
        for (int64_t t = 0; t < T; ++t) {
            int64_t o = b * T * C + t * C + c;
            double kt = k[o], vt = v[o];
            /* output: past sums plus the current token with bonus u */
            double x = uc + kt;
            double q = p > x ? p : x;
            double ep = exp(p - q), ex = exp(x - q);
            y[o] = (ep * a + ex * vt) / (ep * d + ex);
            /* state update: decay the past by e^{-w}, add the current token */
            double pd = p - wc;
            double q2 = pd > kt ? pd : kt;
            double f_old = exp(pd - q2), f_new = exp(kt - q2);
            a = f_old * a + f_new * vt;
            d = f_old * d + f_new;
            p = q2;
        }
        if (s_out) {
            double *so = s_out + b * 3 * C + c;
            so[0] = a;
            so[C] = d;
            so[2 * C] = p;
        }
    }
}

void oracle_wkv_rnn(int64_t B, int64_t T, int64_t C,
                    const double *w, const double *u,
                    const double *k, const double *v, double *y, int nthreads) {
    oracle_wkv_rnn_s(B, T, C, w, u, k, v, NULL, y, NULL, nthreads);
}

/* ------------------------------------------------------------------------
 * WKV gradients.  The pages print no gradient formulas; eq. (14) is a
 * softmax-weighted mean
 *     y_t = sum_{j<=t} beta_{t,j} v_j,   beta_{t,j} = e^{l_{t,j}} / sum_i e^{l_{t,i}},
 *     l_{t,j} = -(t-1-j) w + k_j  (j < t),   l_{t,t} = u + k_t,
 * so with dL/dy_t = g_t, dy_t/dv_j = beta_{t,j} and dy_t/dl_{t,j} =
 * beta_{t,j} (v_j - y_t), and the logits depend on k_j (slope 1), on u (the
 * diagonal, slope 1) and on w (slope -(t-1-j) below the diagonal):
 *     gv_j = sum_{t>=j} g_t beta_{t,j}
 *     gk_j = sum_{t>=j} g_t beta_{t,j} (v_j - y_t)
 *     gu   = sum_t g_t beta_{t,t} (v_t - y_t)            (summed over b too)
 *     gw   = -sum_t sum_{j<t} (t-1-j) g_t beta_{t,j} (v_j - y_t)
 * Definition form: every beta by its own max-stabilised softmax, O(T^2) per
 * channel.  gw, gu are [C] sums over batch rows and steps.
 * ------------------------------------------------------------------------ */
void oracle_wkv_backward_direct(int64_t B, int64_t T, int64_t C,
                                const double *w, const double *u,
                                const double *k, const double *v, const double *gy,
                                double *gk, double *gv, double *gw, double *gu, int nthreads) {
    for (int64_t c = 0; c < C; ++c) { gw[c] = 0.0; gu[c] = 0.0; }
#pragma omp parallel for schedule(dynamic, 1) num_threads(pick_threads(nthreads))
    for (int64_t c = 0; c < C; ++c) {
        double gw_c = 0.0, gu_c = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            const double *kb = k + b * T * C + c, *vb = v + b * T * C + c, *gb = gy + b * T * C + c;
            double *gkb = gk + b * T * C + c, *gvb = gv + b * T * C + c;
            for (int64_t j = 0; j < T; ++j) { gkb[j * C] = 0.0; gvb[j * C] = 0.0; }
            for (int64_t t = 0; t < T; ++t) {
                /* logits of output t and their softmax */
                double m = u[c] + kb[t * C];
                for (int64_t j = 0; j < t; ++j) {
                    double l = -(double)(t - 1 - j) * w[c] + kb[j * C];
                    if (l > m) m = l;
                }
                double den = 0.0, num = 0.0;
                for (int64_t j = 0; j <= t; ++j) {
                    double l = j < t ? -(double)(t - 1 - j) * w[c] + kb[j * C] : u[c] + kb[t * C];
                    double e = exp(l - m);
                    den += e;
                    num += e * vb[j * C];
                }
                double y = num / den, g = gb[t * C];
                for (int64_t j = 0; j <= t; ++j) {
                    double l = j < t ? -(double)(t - 1 - j) * w[c] + kb[j * C] : u[c] + kb[t * C];
                    double beta = exp(l - m) / den;
                    double dl = g * beta * (vb[j * C] - y);   /* dL / d logit */
                    gvb[j * C] += g * beta;
                    gkb[j * C] += dl;
                    if (j == t) gu_c += dl;
                    else gw_c -= (double)(t - 1 - j) * dl;
                }
            }
        }
        gw[c] = gw_c;
        gu[c] = gu_c;
    }
}

/* ------------------------------------------------------------------------
 * The same gradients by recurrences, O(T) per channel: a forward sweep keeps
 * y_t and L_t = ln D_t (D_t the output's denominator, sum_i e^{l_{t,i}}); a
 * reverse sweep keeps, for the step j being visited, the sums over later
 * outputs t > j
 *     P_j  = sum_{t>j} e^{-(t-1-j) w} g_t / D_t,        Q_j  = the same with g_t y_t,
 *     R_j  = sum_{t>j} (t-1-j) e^{-(t-1-j) w} g_t / D_t, R2_j = the same with g_t y_t,
 * which obey  P_{j-1} = g_j / D_j + e^{-w} P_j  (Q likewise with g_j y_j) and
 * R_{j-1} = e^{-w} (R_j + P_j)  (R2 likewise with Q).  Then, since
 * beta_{t,j} = e^{k_j - (t-1-j) w} / D_t below the diagonal and
 * beta_{j,j} = e^{u + k_j} / D_j,
 *     gv_j = e^{u+k_j-L_j} g_j + e^{k_j} P_j
 *     gk_j = e^{u+k_j-L_j} g_j (v_j - y_j) + e^{k_j} (v_j P_j - Q_j)
 *     gu  += e^{u+k_j-L_j} g_j (v_j - y_j),   gw -= e^{k_j} (v_j R_j - R2_j).
 * The four sums share one scale e^{-rho}; rho_{j-1} = min(L_j, rho_j + w)
 * keeps every exponent <= 0, and rho_j >= k_j, so e^{k_j - rho_j} <= 1.
 * ------------------------------------------------------------------------ */
void oracle_wkv_backward_rnn(int64_t B, int64_t T, int64_t C,
                             const double *w, const double *u,
                             const double *k, const double *v, const double *gy,
                             double *gk, double *gv, double *gw, double *gu, int nthreads) {
    for (int64_t c = 0; c < C; ++c) { gw[c] = 0.0; gu[c] = 0.0; }
#pragma omp parallel num_threads(pick_threads(nthreads))
    {
        double *ys = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double *Ls = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t c = 0; c < C; ++c) {
            double gw_c = 0.0, gu_c = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                const double *kb = k + b * T * C + c, *vb = v + b * T * C + c;
                const double *gb = gy + b * T * C + c;
                double *gkb = gk + b * T * C + c, *gvb = gv + b * T * C + c;
                /* forward sweep (RNN mode, as oracle_wkv_rnn) keeping y_t, L_t */
                double a = 0.0, d = 0.0, p = -INFINITY;
                for (int64_t t = 0; t < T; ++t) {
                    double kt = kb[t * C], vt = vb[t * C];
                    double x = u[c] + kt, q = p > x ? p : x;
                    double e_past = exp(p - q), e_cur = exp(x - q);
                    double den = e_past * d + e_cur;
                    ys[t] = (e_past * a + e_cur * vt) / den;
                    Ls[t] = q + log(den);
                    double pd = p - w[c], q2 = pd > kt ? pd : kt;
                    double fo = exp(pd - q2), fn = exp(kt - q2);
                    a = fo * a + fn * vt;
                    d = fo * d + fn;
                    p = q2;
                }
                /* reverse sweep */
                double P = 0.0, Q = 0.0, R = 0.0, R2 = 0.0, rho = INFINITY;
                for (int64_t j = T - 1; j >= 0; --j) {
                    double kj = kb[j * C], vj = vb[j * C], gj = gb[j * C];
                    double diag = exp(u[c] + kj - Ls[j]) * gj;   /* g_j beta_{j,j} */
                    double sc = exp(kj - rho);                    /* e^{k_j} e^{-rho} */
                    gvb[j * C] = diag + sc * P;
                    gkb[j * C] = diag * (vj - ys[j]) + sc * (vj * P - Q);
                    gu_c += diag * (vj - ys[j]);
                    gw_c -= sc * (vj * R - R2);
                    /* sums for step j-1: add output j, decay the rest by e^{-w} */
                    double r2 = rho + w[c];
                    double nr = Ls[j] < r2 ? Ls[j] : r2;
                    double fnew = exp(nr - Ls[j]), fold = exp(nr - r2);
                    double Pn = fnew * gj + fold * P;
                    double Qn = fnew * gj * ys[j] + fold * Q;
                    R = fold * (R + P);
                    R2 = fold * (R2 + Q);
                    P = Pn;
                    Q = Qn;
                    rho = nr;
                }
            }
            gw[c] = gw_c;
            gu[c] = gu_c;
        }
        free(ys);
        free(Ls);
    }
}

/* ------------------------------------------------------------------------
 * Diagonal linear scan ([MINGRU] scan form, [LRU] x_t = lambda x_{t-1} + u_t
 * with a per-step, per-channel lambda):  h_t = a_t * h_{t-1} + b_t,
 * h_{-1} = h0 (zeros when h0 is NULL).
 * ------------------------------------------------------------------------ */
void oracle_scan_rnn(int64_t B, int64_t T, int64_t D,
                     const double *a, const double *b, const double *h0,
                     double *h, int nthreads) {
#pragma omp parallel for schedule(static) num_threads(pick_threads(nthreads))
    for (int64_t bd = 0; bd < B * D; ++bd) {
        int64_t bi = bd / D, d = bd % D;
        double s = h0 ? h0[bi * D + d] : 0.0;
        for (int64_t t = 0; t < T; ++t) {
            int64_t o = bi * T * D + t * D + d;
            s = a[o] * s + b[o];
            h[o] = s;
        }
    }
}

/* Unrolled form of the same scan at single points ([LRU] linear-RNN section,
 * x_t = sum_k lambda^{t-k} u_k, with lambda^{t-k} replaced by the product of
 * the per-step factors a_{k+1} ... a_t):
 *     h_t = sum_{k=0}^{t} (prod_{j=k+1}^{t} a_j) b_k + (prod_{j=0}^{t} a_j) h0.
 * The sum is accumulated from k = t down to 0 so each product is one multiply
 * longer than the last. */
void oracle_scan_direct_points(int64_t B, int64_t T, int64_t D,
                               const double *a, const double *b, const double *h0,
                               int64_t n, const int64_t *points, double *out,
                               int nthreads) {
    (void)B;
#pragma omp parallel for schedule(dynamic, 16) num_threads(pick_threads(nthreads))
    for (int64_t j = 0; j < n; ++j) {
        int64_t f = points[j];
        int64_t bi = f / (T * D);
        int64_t t = (f / D) % T;
        int64_t d = f % D;
        const double *ab = a + bi * T * D + d;
        const double *bb = b + bi * T * D + d;
        double prod = 1.0, acc = 0.0;
        for (int64_t kk = t; kk >= 0; --kk) {
            acc += prod * bb[kk * D];
            prod *= ab[kk * D];
        }
        if (h0) acc += prod * h0[bi * D + d];
        out[j] = acc;
    }
}
