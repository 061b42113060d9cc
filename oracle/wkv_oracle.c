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
 * [C]; h0 is [B, C] or NULL (zeros).  Inputs and results are float64 (the
 * caller widens the float32 / bf16 values the GPU path reads, exactly).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <omp.h>

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
 * ------------------------------------------------------------------------ */
static double wkv_direct_one(int64_t T, int64_t C, double w, double u,
                             const double *k, const double *v, int64_t t) {
    /* k, v point at channel c of batch row b (stride C between steps) */
    double m = u + k[t * C];
    for (int64_t i = 0; i < t; ++i) {
        double l = -(double)(t - 1 - i) * w + k[i * C];
        if (l > m) m = l;
    }
    double e_t = exp(u + k[t * C] - m);
    double num = e_t * v[t * C];
    double den = e_t;
    for (int64_t i = 0; i < t; ++i) {
        double e = exp(-(double)(t - 1 - i) * w + k[i * C] - m);
        num += e * v[i * C];
        den += e;
    }
    (void)T;
    return num / den;
}

/* points[j] is the flat index b*T*C + t*C + c of the j-th requested output */
void oracle_wkv_direct_points(int64_t B, int64_t T, int64_t C,
                              const double *w, const double *u,
                              const double *k, const double *v,
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
        out[j] = wkv_direct_one(T, C, w[c], u[c], kb, vb, t);
    }
}

/* every output by the definition: O(T^2) per channel, small inputs only */
void oracle_wkv_direct(int64_t B, int64_t T, int64_t C,
                       const double *w, const double *u,
                       const double *k, const double *v, double *y, int nthreads) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(pick_threads(nthreads))
    for (int64_t bc = 0; bc < B * C; ++bc) {
        int64_t b = bc / C, c = bc % C;
        const double *kb = k + b * T * C + c;
        const double *vb = v + b * T * C + c;
        for (int64_t t = 0; t < T; ++t)
            y[b * T * C + t * C + c] = wkv_direct_one(T, C, w[c], u[c], kb, vb, t);
    }
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
 * Starting state: empty sums (a = b = 0, p = -inf).
 * ------------------------------------------------------------------------ */
void oracle_wkv_rnn(int64_t B, int64_t T, int64_t C,
                    const double *w, const double *u,
                    const double *k, const double *v, double *y, int nthreads) {
#pragma omp parallel for schedule(static) num_threads(pick_threads(nthreads))
    for (int64_t bc = 0; bc < B * C; ++bc) {
        int64_t b = bc / C, c = bc % C;
        double wc = w[c], uc = u[c];
        double a = 0.0, d = 0.0, p = -INFINITY;
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
