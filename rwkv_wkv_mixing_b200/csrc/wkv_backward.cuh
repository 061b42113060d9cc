// WKV gradients with respect to k, v, w and u.  The pages give no gradient
// formulas; eq. (14) of "RWKV：基于RNN的LLM" is a softmax-weighted mean,
//     y_t = sum_{j<=t} beta_{t,j} v_j,  beta_{t,j} = e^{l_{t,j}} / D_t,
//     l_{t,j} = -(t-1-j) w + k_j (j < t),  l_{t,t} = u + k_t,  D_t = sum_j e^{l_{t,j}},
// so with g_t = dL/dy_t:
//     gv_j = sum_{t>=j} g_t beta_{t,j},   gk_j = sum_{t>=j} g_t beta_{t,j} (v_j - y_t),
//     gu   = sum_t g_t beta_{t,t} (v_t - y_t),
//     gw   = -sum_t sum_{j<t} (t-1-j) g_t beta_{t,j} (v_j - y_t).
//
// Forward quantities: y_t and L_t = ln D_t from the RNN-mode state
// (num, den) before each step.  Reverse quantities: the sums over later
// outputs t > j
//     P_j = sum_{t>j} e^{-(t-1-j) w} g_t / D_t,   Q_j = the same with g_t y_t,
//     R_j, R2_j = the same weighted by (t-1-j),
// stepped as P_{j-1} = g_j / D_j + e^{-w} P_j, R_{j-1} = e^{-w} (R_j + P_j), give
//     gv_j = e^{u+k_j-L_j} g_j + e^{k_j} P_j,
//     gk_j = e^{u+k_j-L_j} g_j (v_j - y_j) + e^{k_j} (v_j P_j - Q_j),
// and the contributions to gu and gw.  The four sums share one scale e^{-rho}
// with rho_{j-1} = min(L_j, rho_j + w): every exponent evaluated is <= 0 for
// any finite input (L_t >= k_j - (t-1-j) w for all j <= t).
//
// Time-parallel: each channel's steps are cut into segments of kSeg steps,
// one thread per (row, segment, channel), consecutive threads on consecutive
// channels.  Both recurrences are linear, so a segment is summarised from
// the zero state and segments are chained by a short sequential pass per
// channel (Upper/Lower split, review of "Resurrecting Recurrent Neural
// Networks for Long Sequences", parallelisation section):
//   1. forward summary of each segment (the state its steps produce from empty);
//   2. per channel, forward carries: the state before each segment;
//   3. per segment, y_t and L_t from its carry (kept in scratch), then the
//      reverse summary of the segment from the zero state;
//   4. per channel, reverse carries: the sums over outputs after each segment;
//   5. per segment, the reverse pass from its carry: gk, gv and partial gw, gu;
//   6. gw, gu summed over rows and segments in a fixed order.
// A reverse state followed, backwards, by a segment of n steps whose summary
// is L is (P, Q, R, R2) -> L + e^{-n w} (P, Q, R + n P, R2 + n Q).
#pragma once

#include "wkv_ops.cuh"

namespace wkvb {

constexpr int kBwdThreads = 128;
constexpr int kSeg = 32;  // steps per segment (32: more threads in flight; 16 lengthens the carries)

struct WkvBwdArgs {
    const float *w, *u;       // [C]
    const float *k, *v, *gy;  // [B, T, C]
    float *gk, *gv;           // [B, T, C]
    float *ys, *Ls;           // scratch [B, T, C]: y_t and ln D_t
    float *fwd;               // scratch [B, S, 3, C]: forward summaries, then carries
    float *rev;               // scratch [B, S, 5, C]: reverse summaries, then carries
    float *partial;           // scratch [B, S, 2, C]: per-segment gw, gu
    float *gw, *gu;           // [C]
    int B, T, C, S;
};

// forward state: (num, den) = (a, d) e^p of the sums over the steps before
struct FwdState {
    float a, d, p;
};

// (P, Q, R, R2) e^{-rho}
struct RevState {
    float P, Q, R, R2, rho;
};

__device__ __forceinline__ void fwd_step(FwdState &s, float k, float v, float w) {
    const float pd = s.p - w;
    const float q = fmaxf(pd, k);
    const float fo = fast_exp(pd - q), fn = fast_exp(k - q);
    s.a = fmaf(fo, s.a, fn * v);
    s.d = fmaf(fo, s.d, fn);
    s.p = q;
}

// state l followed by a segment of n steps whose summary is r
__device__ __forceinline__ FwdState fwd_combine(const FwdState &l, const FwdState &r, float n,
                                                float w) {
    const float pd = fmaf(-n, w, l.p);
    const float m = fmaxf(pd, r.p);
    const float fl = fast_exp(pd - m), fr = fast_exp(r.p - m);
    return {fmaf(l.a, fl, r.a * fr), fmaf(l.d, fl, r.d * fr), m};
}

// the reverse state after (backwards over) a segment of n steps whose
// summary from zero is loc, starting from the state in
__device__ __forceinline__ RevState rev_combine(const RevState &loc, const RevState &in, float n,
                                               float w) {
    const float r_in = fmaf(n, w, in.rho);
    const float m = fminf(loc.rho, r_in);
    const float fl = fast_exp(m - loc.rho), fi = fast_exp(m - r_in);
    return {fmaf(loc.P, fl, fi * in.P), fmaf(loc.Q, fl, fi * in.Q),
            fmaf(loc.R, fl, fi * fmaf(n, in.P, in.R)), fmaf(loc.R2, fl, fi * fmaf(n, in.Q, in.R2)),
            m};
}

__device__ __forceinline__ bool seg_thread(const WkvBwdArgs &a, int &b, int &s, int &c, int &t0,
                                           int &t1) {
    const long long i = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= static_cast<long long>(a.B) * a.S * a.C) return false;
    c = static_cast<int>(i % a.C);
    const long long r = i / a.C;
    s = static_cast<int>(r % a.S);
    b = static_cast<int>(r / a.S);
    t0 = s * kSeg;
    t1 = min(a.T, t0 + kSeg);
    return true;
}

// 1. forward summary of each segment from the empty state
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_fwd_summary_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, t1;
    if (!seg_thread(a, b, s, c, t0, t1)) return;
    const float w = a.w[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    FwdState st{0.f, 0.f, kNoScale};
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        const size_t o = base + static_cast<size_t>(t) * a.C;
        fwd_step(st, a.k[o], a.v[o], w);
    }
    float *f = a.fwd + (static_cast<size_t>(b) * a.S + s) * 3 * a.C + c;
    f[0] = st.a;
    f[a.C] = st.d;
    f[2 * a.C] = st.p;
}

// 2. per (row, channel): the state before each segment, over its summaries
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_fwd_carry_kernel(const WkvBwdArgs a) {
    const long long i = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= static_cast<long long>(a.B) * a.C) return;
    const int c = static_cast<int>(i % a.C), b = static_cast<int>(i / a.C);
    const float w = a.w[c];
    FwdState x{0.f, 0.f, kNoScale};
    for (int s = 0; s < a.S; ++s) {
        float *f = a.fwd + (static_cast<size_t>(b) * a.S + s) * 3 * a.C + c;
        const FwdState loc{f[0], f[a.C], f[2 * a.C]};
        f[0] = x.a;
        f[a.C] = x.d;
        f[2 * a.C] = x.p;
        const int n = min(a.T, (s + 1) * kSeg) - s * kSeg;
        x = fwd_combine(x, loc, static_cast<float>(n), w);
    }
}

// 3. y_t, L_t of each segment from its carry; then the segment's reverse
//    summary from the zero state
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_outputs_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, t1;
    if (!seg_thread(a, b, s, c, t0, t1)) return;
    const float w = a.w[c], u = a.u[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    {
        const float *f = a.fwd + (static_cast<size_t>(b) * a.S + s) * 3 * a.C + c;
        FwdState st{f[0], f[a.C], f[2 * a.C]};
#pragma unroll 4
        for (int t = t0; t < t1; ++t) {
            const size_t o = base + static_cast<size_t>(t) * a.C;
            const float kt = a.k[o], vt = a.v[o];
            const float x = u + kt;
            const float q = fmaxf(st.p, x);
            const float ep = fast_exp(st.p - q), ex = fast_exp(x - q);
            const float den = fmaf(ep, st.d, ex);
            a.ys[o] = fmaf(ep, st.a, ex * vt) / den;
            a.Ls[o] = q + logf(den);
            fwd_step(st, kt, vt, w);
        }
    }
    RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
    for (int j = t1 - 1; j >= t0; --j) {
        const size_t o = base + static_cast<size_t>(j) * a.C;
        const float gj = a.gy[o], yj = a.ys[o], Lj = a.Ls[o];
        const float r2 = z.rho + w;
        const float nr = fminf(Lj, r2);
        const float fnew = fast_exp(nr - Lj), fold = fast_exp(nr - r2);
        const float Pn = fmaf(fnew, gj, fold * z.P);
        const float Qn = fmaf(fnew * gj, yj, fold * z.Q);
        z.R = fold * (z.R + z.P);
        z.R2 = fold * (z.R2 + z.Q);
        z.P = Pn;
        z.Q = Qn;
        z.rho = nr;
    }
    float *r = a.rev + (static_cast<size_t>(b) * a.S + s) * 5 * a.C + c;
    r[0] = z.P;
    r[a.C] = z.Q;
    r[2 * a.C] = z.R;
    r[3 * a.C] = z.R2;
    r[4 * a.C] = z.rho;
}

// 4. per (row, channel), backwards over segments: the sums over the outputs
//    after each segment
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_rev_carry_kernel(const WkvBwdArgs a) {
    const long long i = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= static_cast<long long>(a.B) * a.C) return;
    const int c = static_cast<int>(i % a.C), b = static_cast<int>(i / a.C);
    const float w = a.w[c];
    RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
    for (int s = a.S - 1; s >= 0; --s) {
        float *r = a.rev + (static_cast<size_t>(b) * a.S + s) * 5 * a.C + c;
        const RevState loc{r[0], r[a.C], r[2 * a.C], r[3 * a.C], r[4 * a.C]};
        r[0] = z.P;
        r[a.C] = z.Q;
        r[2 * a.C] = z.R;
        r[3 * a.C] = z.R2;
        r[4 * a.C] = z.rho;
        const int n = min(a.T, (s + 1) * kSeg) - s * kSeg;
        z = rev_combine(loc, z, static_cast<float>(n), w);
    }
}

// 5. per segment, the reverse pass from its carry: gk, gv, partial gw, gu
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_grads_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, t1;
    if (!seg_thread(a, b, s, c, t0, t1)) return;
    const float w = a.w[c], u = a.u[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    const float *r = a.rev + (static_cast<size_t>(b) * a.S + s) * 5 * a.C + c;
    RevState z{r[0], r[a.C], r[2 * a.C], r[3 * a.C], r[4 * a.C]};
    float gw = 0.f, gu = 0.f;
#pragma unroll 4
    for (int j = t1 - 1; j >= t0; --j) {
        const size_t o = base + static_cast<size_t>(j) * a.C;
        const float kj = a.k[o], vj = a.v[o], gj = a.gy[o], yj = a.ys[o], Lj = a.Ls[o];
        const float diag = fast_exp(u + kj - Lj) * gj;  // g_j beta_{j,j}
        const float sc = fast_exp(kj - z.rho);           // e^{k_j - rho}, <= 1
        const float dv = vj - yj;
        a.gv[o] = fmaf(sc, z.P, diag);
        a.gk[o] = fmaf(diag, dv, sc * fmaf(vj, z.P, -z.Q));
        gu = fmaf(diag, dv, gu);
        gw = fmaf(-sc, fmaf(vj, z.R, -z.R2), gw);
        const float r2 = z.rho + w;
        const float nr = fminf(Lj, r2);
        const float fnew = fast_exp(nr - Lj), fold = fast_exp(nr - r2);
        const float Pn = fmaf(fnew, gj, fold * z.P);
        const float Qn = fmaf(fnew * gj, yj, fold * z.Q);
        z.R = fold * (z.R + z.P);
        z.R2 = fold * (z.R2 + z.Q);
        z.P = Pn;
        z.Q = Qn;
        z.rho = nr;
    }
    float *pp = a.partial + (static_cast<size_t>(b) * a.S + s) * 2 * a.C + c;
    pp[0] = gw;
    pp[a.C] = gu;
}

// 6. gw[c], gu[c]: partial sums added over rows and segments in a fixed order
__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_reduce_kernel(const WkvBwdArgs a) {
    const int c = blockIdx.x * kBwdThreads + threadIdx.x;
    if (c >= a.C) return;
    float gw = 0.f, gu = 0.f;
    for (int bs = 0; bs < a.B * a.S; ++bs) {
        gw += a.partial[static_cast<size_t>(bs) * 2 * a.C + c];
        gu += a.partial[(static_cast<size_t>(bs) * 2 + 1) * a.C + c];
    }
    a.gw[c] = gw;
    a.gu[c] = gu;
}

}  // namespace wkvb
