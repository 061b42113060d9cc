// WKV gradients with respect to k, v, w and u.  The pages give no gradient
// formulas; eq. (14) of "RWKV：基于RNN的LLM" is a softmax-weighted mean,
//     y_t = sum_{j<=t} beta_{t,j} v_j,  beta_{t,j} = e^{l_{t,j}} / D_t,
//     l_{t,j} = -(t-1-j) w + k_j (j < t),  l_{t,t} = u + k_t,  D_t = sum_j e^{l_{t,j}},
// so with g_t = dL/dy_t:
//     gv_j = sum_{t>=j} g_t beta_{t,j},   gk_j = sum_{t>=j} g_t beta_{t,j} (v_j - y_t),
//     gu   = sum_t g_t beta_{t,t} (v_t - y_t),
//     gw   = -sum_t sum_{j<t} (t-1-j) g_t beta_{t,j} (v_j - y_t).
//
// One thread per (batch row, channel) makes two passes over time.  Forward:
// the RNN-mode state update, keeping y_t and L_t = ln D_t in a scratch
// buffer.  Reverse: the sums over later outputs t > j
//     P_j = sum_{t>j} e^{-(t-1-j) w} g_t / D_t,   Q_j = the same with g_t y_t,
//     R_j, R2_j = the same weighted by (t-1-j),
// stepped as P_{j-1} = g_j / D_j + e^{-w} P_j, R_{j-1} = e^{-w} (R_j + P_j),
// give  gv_j = e^{u+k_j-L_j} g_j + e^{k_j} P_j,
//       gk_j = e^{u+k_j-L_j} g_j (v_j - y_j) + e^{k_j} (v_j P_j - Q_j),
//       and the contributions to gu and gw.  The four sums share one scale
// e^{-rho} with rho_{j-1} = min(L_j, rho_j + w): every exponent evaluated is
// <= 0 (L_t >= k_j - (t-1-j) w for every j <= t), for any finite input.
// Per-row partial sums of gw and gu go to scratch; a second kernel adds them
// over the rows in a fixed order, so the result does not depend on timing.
#pragma once

#include "wkv_ops.cuh"

namespace wkvb {

constexpr int kBwdThreads = 128;

struct WkvBwdArgs {
    const float *w, *u;       // [C]
    const float *k, *v, *gy;  // [B, T, C]
    float *gk, *gv;           // [B, T, C]
    float *ys, *Ls;           // scratch [B, T, C]: y_t and ln D_t
    float *partial;           // scratch [B, 2, C]: per-row gw, gu
    float *gw, *gu;           // [C]
};

__global__ void __launch_bounds__(kBwdThreads)
    wkv_backward_serial_kernel(const WkvBwdArgs a, int B, int T, int C) {
    const long long i = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= static_cast<long long>(B) * C) return;
    const int b = static_cast<int>(i / C);
    const int c = static_cast<int>(i - static_cast<long long>(b) * C);
    const float w = a.w[c], u = a.u[c];
    const size_t base = static_cast<size_t>(b) * T * C + c;

    // forward: y_t and L_t = ln D_t, max-stabilised state (num, den) e^p
    {
        float sa = 0.f, sd = 0.f, p = kNoScale;
        for (int t = 0; t < T; ++t) {
            const size_t o = base + static_cast<size_t>(t) * C;
            const float kt = a.k[o], vt = a.v[o];
            const float x = u + kt;
            const float q = fmaxf(p, x);
            const float ep = fast_exp(p - q), ex = fast_exp(x - q);
            const float den = fmaf(ep, sd, ex);
            a.ys[o] = fmaf(ep, sa, ex * vt) / den;
            a.Ls[o] = q + logf(den);
            const float pd = p - w;
            const float q2 = fmaxf(pd, kt);
            const float fo = fast_exp(pd - q2), fn = fast_exp(kt - q2);
            sa = fmaf(fo, sa, fn * vt);
            sd = fmaf(fo, sd, fn);
            p = q2;
        }
    }

    // reverse
    float P = 0.f, Q = 0.f, R = 0.f, R2 = 0.f, rho = -kNoScale;  // rho = "+inf": no later output
    float gw = 0.f, gu = 0.f;
    for (int j = T - 1; j >= 0; --j) {
        const size_t o = base + static_cast<size_t>(j) * C;
        const float kj = a.k[o], vj = a.v[o], gj = a.gy[o], yj = a.ys[o], Lj = a.Ls[o];
        const float diag = fast_exp(u + kj - Lj) * gj;  // g_j beta_{j,j}
        const float sc = fast_exp(kj - rho);             // e^{k_j - rho}, <= 1
        const float dv = vj - yj;
        a.gv[o] = fmaf(sc, P, diag);
        a.gk[o] = fmaf(diag, dv, sc * fmaf(vj, P, -Q));
        gu = fmaf(diag, dv, gu);
        gw = fmaf(-sc, fmaf(vj, R, -R2), gw);
        // sums for step j-1: output j joins, the rest decay by e^{-w}
        const float r2 = rho + w;
        const float nr = fminf(Lj, r2);
        const float fnew = fast_exp(nr - Lj), fold = fast_exp(nr - r2);
        const float Pn = fmaf(fnew, gj, fold * P);
        const float Qn = fmaf(fnew * gj, yj, fold * Q);
        R = fold * (R + P);
        R2 = fold * (R2 + Q);
        P = Pn;
        Q = Qn;
        rho = nr;
    }
    a.partial[(static_cast<size_t>(b) * 2) * C + c] = gw;
    a.partial[(static_cast<size_t>(b) * 2 + 1) * C + c] = gu;
}

// gw[c], gu[c]: the rows' partial sums added in row order
__global__ void __launch_bounds__(kBwdThreads)
    wkv_backward_reduce_kernel(const WkvBwdArgs a, int B, int C) {
    const int c = blockIdx.x * kBwdThreads + threadIdx.x;
    if (c >= C) return;
    float gw = 0.f, gu = 0.f;
    for (int b = 0; b < B; ++b) {
        gw += a.partial[(static_cast<size_t>(b) * 2) * C + c];
        gu += a.partial[(static_cast<size_t>(b) * 2 + 1) * C + c];
    }
    a.gw[c] = gw;
    a.gu[c] = gu;
}

}  // namespace wkvb
