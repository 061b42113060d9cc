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
// the zero state and segments are chained by a scan over the summaries of
// each channel (Upper/Lower split, review of "Resurrecting Recurrent Neural
// Networks for Long Sequences", parallelisation section).  y_t and L_t are
// recomputed per segment from the forward carry rather than stored; each
// kernel loads a segment's inputs into registers at once.  HBM traffic per
// element: k, v three times, gy twice, gk and gv once (40 B):
//   1. forward summary of each segment (the state its steps produce from empty);
//   2. per channel, forward carries: the state before each segment;
//   3. per segment, y_t and L_t from its carry (in registers), then the
//      reverse summary of the segment from the zero state;
//   4. per channel, reverse carries: the sums over outputs after each segment;
//   5. per segment, y_t and L_t again, then the reverse pass from its carry:
//      gk, gv and partial gw, gu;
//   6. gw, gu summed over rows and segments in a fixed order.
// A reverse state followed, backwards, by a segment of n steps whose summary
// is L is (P, Q, R, R2) -> L + e^{-n w} (P, Q, R + n P, R2 + n Q).
// (A single-pass form, segments chained by a decoupled look-back in each
// direction, measured slower at these segment lengths: the look-back's
// latency outweighs a 16- or 32-step segment's work.)
//
// These six kernels serve the shapes a TMA tensor map cannot describe.  The
// others take persistent_bwd.cuh: 32-step segments whose forward states and
// reverse summaries come from one pass over TMA-staged 128-step tiles, then
// the reverse carries and the reduction below (segment length a.L), then
// one TMA-staged gradient pass (k, v, gy read twice instead of three times).
#pragma once

#include "wkv_ops.cuh"

namespace wkvb {

constexpr int kBwdThreads = 128;
constexpr int kReduceWarps = 8;
constexpr int kReduceParts = 8;  // blocks per channel group in the gw, gu sum
constexpr int kSeg = 16;  // steps per segment: a segment's inputs and y_t, L_t sit in registers

struct WkvBwdArgs {
    const float *w, *u;       // [C]
    const float *k, *v, *gy;  // [B, T, C]
    float *gk, *gv;           // [B, T, C]
    float *fwd;               // scratch [B, S, 3, C]: forward summaries, then carries
    float *rev;               // scratch [B, S, 5, C]: reverse summaries, then carries
    float *partial;           // scratch [B, S, 2, C]: per-segment gw, gu
    float *gw, *gu;           // [C]
    float *red;               // scratch [kReduceParts, 2, C]: first-level sums of gw, gu
    unsigned *red_done;       // [ceil(C / 32)] counters, zero between launches
    int B, T, C, S;           // S = ceil(T / L) segments per row
    int L;                    // steps per segment: kSeg here, 32 on the tiled path
};

// forward state: (num, den) = (a, d) e^p of the sums over the steps before
struct FwdState {
    float a, d, p;
};

// (P, Q, R, R2) e^{-rho}
struct RevState {
    float P, Q, R, R2, rho;
};

// The factors of a max-stabilised sum e^{x-q}, e^{y-q} with q = max(x, y):
// one of the two is e^0 = 1, the other e^{-|x-y|}, so one exponential gives
// both (bit for bit what two would: e^{-(x-y)} and e^{y-x} round alike).
struct Pair {
    float fx, fy;  // e^{x-q}, e^{y-q}
    float q;       // max(x, y)
};
__device__ __forceinline__ Pair max_pair(float x, float y) {
    const float e = fast_exp(-fabsf(x - y));
    return x >= y ? Pair{1.f, e, x} : Pair{e, 1.f, y};
}
// the same about q = min(x, y): e^{q-x}, e^{q-y}
__device__ __forceinline__ Pair min_pair(float x, float y) {
    const float e = fast_exp(-fabsf(x - y));
    return x <= y ? Pair{1.f, e, x} : Pair{e, 1.f, y};
}

__device__ __forceinline__ void fwd_step(FwdState &s, float k, float v, float w) {
    const Pair f = max_pair(s.p - w, k);
    s.a = fmaf(f.fx, s.a, f.fy * v);
    s.d = fmaf(f.fx, s.d, f.fy);
    s.p = f.q;
}

// state l followed by a segment of n steps whose summary is r
__device__ __forceinline__ FwdState fwd_combine(const FwdState &l, const FwdState &r, float n,
                                                float w) {
    const Pair f = max_pair(fmaf(-n, w, l.p), r.p);
    return {fmaf(l.a, f.fx, r.a * f.fy), fmaf(l.d, f.fx, r.d * f.fy), f.q};
}

// the reverse state after (backwards over) a segment of n steps whose
// summary from zero is loc, starting from the state in
__device__ __forceinline__ RevState rev_combine(const RevState &loc, const RevState &in, float n,
                                               float w) {
    const Pair f = min_pair(loc.rho, fmaf(n, w, in.rho));
    const float fl = f.fx, fi = f.fy;
    return {fmaf(loc.P, fl, fi * in.P), fmaf(loc.Q, fl, fi * in.Q),
            fmaf(loc.R, fl, fi * fmaf(n, in.P, in.R)), fmaf(loc.R2, fl, fi * fmaf(n, in.Q, in.R2)),
            f.q};
}

__device__ __forceinline__ bool seg_thread(const WkvBwdArgs &a, int &b, int &s, int &c, int &t0,
                                           int &n) {
    const long long i = static_cast<long long>(blockIdx.x) * kBwdThreads + threadIdx.x;
    if (i >= static_cast<long long>(a.B) * a.S * a.C) return false;
    c = static_cast<int>(i % a.C);
    const long long r = i / a.C;
    s = static_cast<int>(r % a.S);
    b = static_cast<int>(r / a.S);
    t0 = s * kSeg;
    n = min(a.T - t0, kSeg);
    return true;
}

__device__ __forceinline__ int seg_len(const WkvBwdArgs &a, int s) {
    return min(a.T, (s + 1) * a.L) - s * a.L;
}

// one reverse step over output j: (P, Q) take g_j / D_j and g_j y_j / D_j,
// (R, R2) the previous (P, Q) once more; the common scale e^{-rho} moves to
// rho_{j-1} = min(L_j, rho_j + w)
__device__ __forceinline__ void rev_step(RevState &z, float gj, float yj, float Lj, float w) {
    const Pair f = min_pair(Lj, z.rho + w);
    const float fnew = f.fx, fold = f.fy;
    const float Pn = fmaf(fnew, gj, fold * z.P);
    const float Qn = fmaf(fnew * gj, yj, fold * z.Q);
    z.R = fold * (z.R + z.P);
    z.R2 = fold * (z.R2 + z.Q);
    z.P = Pn;
    z.Q = Qn;
    z.rho = f.q;
}

// one segment's values of a [B, T, C] input for one channel, all loads
// issued before any is used (steps past the segment's n <= kSeg are 0)
template <bool FULL>
__device__ __forceinline__ void seg_load(const float *x, size_t base, int t0, int n, int C,
                                         float (&r)[kSeg]) {
    const float *p = x + base + static_cast<size_t>(t0) * C;
#pragma unroll
    for (int i = 0; i < kSeg; ++i) r[i] = (FULL || i < n) ? p[static_cast<size_t>(i) * C] : 0.f;
}

// y_t, L_t = ln D_t and beta_{t,t} = e^{u+k_t} / D_t for the n <= kSeg steps
// of one segment, from the state st before it.  With q = max(p, u + k_t),
// D_t = (e^{p-q} d + e^{u+k_t-q}) e^q.
template <bool FULL>
__device__ __forceinline__ void seg_outputs(const float (&ks)[kSeg], const float (&vs)[kSeg],
                                            int n, FwdState st, float w, float u,
                                            float (&ys)[kSeg], float (&Ls)[kSeg],
                                            float (&bs)[kSeg]) {
#pragma unroll
    for (int i = 0; i < kSeg; ++i) {
        ys[i] = 0.f;
        Ls[i] = 0.f;
        bs[i] = 0.f;
        if (FULL || i < n) {
            const Pair f = max_pair(st.p, u + ks[i]);
            const float den = fmaf(f.fx, st.d, f.fy);  // in [1, T + 1]
            const float rden = __fdividef(1.f, den);
            ys[i] = fmaf(f.fx, st.a, f.fy * vs[i]) * rden;
            Ls[i] = f.q + __logf(den);
            bs[i] = f.fy * rden;
            fwd_step(st, ks[i], vs[i], w);
        }
    }
}

__device__ __forceinline__ FwdState load_fwd(const float *f, int C) {
    return {f[0], f[C], f[2 * C]};
}
__device__ __forceinline__ void store_fwd(float *f, int C, const FwdState &x) {
    f[0] = x.a;
    f[C] = x.d;
    f[2 * C] = x.p;
}

__device__ __forceinline__ RevState load_rev(const float *r, int C) {
    return {r[0], r[C], r[2 * C], r[3 * C], r[4 * C]};
}
__device__ __forceinline__ void store_rev(float *r, int C, const RevState &z) {
    r[0] = z.P;
    r[C] = z.Q;
    r[2 * C] = z.R;
    r[3 * C] = z.R2;
    r[4 * C] = z.rho;
}

// 1. forward summary of each segment from the empty state
template <bool FULL>
__device__ __forceinline__ void fwd_summary(const WkvBwdArgs &a, int b, int s, int c, int t0,
                                            int n) {
    const float w = a.w[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    float ks[kSeg], vs[kSeg];
    seg_load<FULL>(a.k, base, t0, n, a.C, ks);
    seg_load<FULL>(a.v, base, t0, n, a.C, vs);
    FwdState st{0.f, 0.f, kNoScale};
#pragma unroll
    for (int i = 0; i < kSeg; ++i)
        if (FULL || i < n) fwd_step(st, ks[i], vs[i], w);
    store_fwd(a.fwd + (static_cast<size_t>(b) * a.S + s) * 3 * a.C + c, a.C, st);
}

__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_fwd_summary_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, n;
    if (!seg_thread(a, b, s, c, t0, n)) return;
    if (n == kSeg)
        fwd_summary<true>(a, b, s, c, t0, n);
    else
        fwd_summary<false>(a, b, s, c, t0, n);
}

// Carries over segments, one block per (row, 32 channels): warp i of
// kCarryWarps takes a contiguous range of segments, folds it into one
// summary, takes the fold of the ranges before it (after it, in reverse)
// from shared memory, then writes the carry of every segment of its range.
// Lanes are consecutive channels, so every access is one 128-byte row.
constexpr int kCarryWarps = 8;

__device__ __forceinline__ void carry_range(const WkvBwdArgs &a, int &lo, int &hi, int &steps) {
    const int wi = threadIdx.x / 32;
    lo = static_cast<int>(static_cast<long long>(a.S) * wi / kCarryWarps);
    hi = static_cast<int>(static_cast<long long>(a.S) * (wi + 1) / kCarryWarps);
    steps = hi > lo ? min(a.T, hi * a.L) - lo * a.L : 0;
}

// 2. the forward state before each segment
__global__ void __launch_bounds__(32 * kCarryWarps) wkv_bwd_fwd_carry_kernel(const WkvBwdArgs a) {
    __shared__ FwdState part[kCarryWarps][32];
    __shared__ int part_n[kCarryWarps];
    const int cb = (a.C + 31) / 32;
    const int b = blockIdx.x / cb, lane = threadIdx.x % 32, wi = threadIdx.x / 32;
    const int c = (blockIdx.x % cb) * 32 + lane;
    const bool live = c < a.C;
    const float w = live ? a.w[c] : 0.f;
    int lo, hi, steps;
    carry_range(a, lo, hi, steps);
    float *f0 = a.fwd + static_cast<size_t>(b) * a.S * 3 * a.C + (live ? c : 0);
    FwdState x{0.f, 0.f, kNoScale};
    if (live) {
#pragma unroll 4
        for (int s = lo; s < hi; ++s)
            x = fwd_combine(x, load_fwd(f0 + static_cast<size_t>(s) * 3 * a.C, a.C),
                            static_cast<float>(seg_len(a, s)), w);
    }
    part[wi][lane] = x;
    if (lane == 0) part_n[wi] = steps;
    __syncthreads();
    if (!live) return;
    x = FwdState{0.f, 0.f, kNoScale};
    for (int v = 0; v < wi; ++v) x = fwd_combine(x, part[v][lane], static_cast<float>(part_n[v]), w);
    for (int s = lo; s < hi; s += 4) {
        FwdState loc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (s + i < hi) loc[i] = load_fwd(f0 + static_cast<size_t>(s + i) * 3 * a.C, a.C);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (s + i < hi) {
                store_fwd(f0 + static_cast<size_t>(s + i) * 3 * a.C, a.C, x);
                x = fwd_combine(x, loc[i], static_cast<float>(seg_len(a, s + i)), w);
            }
        }
    }
}

// 3. per segment: y_t, L_t from its carry (registers), then the segment's
//    reverse summary from the zero state
template <bool FULL>
__device__ __forceinline__ void rev_summary(const WkvBwdArgs &a, int b, int s, int c, int t0,
                                            int n) {
    const float w = a.w[c], u = a.u[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    const size_t bs_ = static_cast<size_t>(b) * a.S + s;
    float ks[kSeg], vs[kSeg], gs[kSeg], ys[kSeg], Ls[kSeg], bs[kSeg];
    seg_load<FULL>(a.k, base, t0, n, a.C, ks);
    seg_load<FULL>(a.v, base, t0, n, a.C, vs);
    seg_load<FULL>(a.gy, base, t0, n, a.C, gs);
    seg_outputs<FULL>(ks, vs, n, load_fwd(a.fwd + bs_ * 3 * a.C + c, a.C), w, u, ys, Ls, bs);
    RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
#pragma unroll
    for (int i = kSeg - 1; i >= 0; --i)
        if (FULL || i < n) rev_step(z, gs[i], ys[i], Ls[i], w);
    store_rev(a.rev + bs_ * 5 * a.C + c, a.C, z);
}

__global__ void __launch_bounds__(kBwdThreads) wkv_bwd_rev_summary_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, n;
    if (!seg_thread(a, b, s, c, t0, n)) return;
    if (n == kSeg)
        rev_summary<true>(a, b, s, c, t0, n);
    else
        rev_summary<false>(a, b, s, c, t0, n);
}

// 4. backwards over segments: the sums over the outputs after each segment
__global__ void __launch_bounds__(32 * kCarryWarps) wkv_bwd_rev_carry_kernel(const WkvBwdArgs a) {
    __shared__ RevState part[kCarryWarps][32];
    __shared__ int part_n[kCarryWarps];
    // launched as a programmatic dependent of the summaries' kernel on the
    // tiled path: the next kernel (the gradient tiles, whose producer starts
    // loading k, v, gy at once) may start launching as soon as every block
    // of this one runs; nothing global is read here before the summaries'
    // kernel has finished (both no-ops for an ordinary launch)
    allow_dependent_launch();
    grid_dependency_wait();
    const int cb = (a.C + 31) / 32;
    const int b = blockIdx.x / cb, lane = threadIdx.x % 32, wi = threadIdx.x / 32;
    const int c = (blockIdx.x % cb) * 32 + lane;
    const bool live = c < a.C;
    const float w = live ? a.w[c] : 0.f;
    int lo, hi, steps;
    carry_range(a, lo, hi, steps);
    float *r0 = a.rev + static_cast<size_t>(b) * a.S * 5 * a.C + (live ? c : 0);
    RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
    if (live) {
#pragma unroll 4
        for (int s = hi - 1; s >= lo; --s)
            z = rev_combine(load_rev(r0 + static_cast<size_t>(s) * 5 * a.C, a.C), z,
                            static_cast<float>(seg_len(a, s)), w);
    }
    part[wi][lane] = z;
    if (lane == 0) part_n[wi] = steps;
    __syncthreads();
    if (!live) return;
    z = RevState{0.f, 0.f, 0.f, 0.f, -kNoScale};
    for (int v = kCarryWarps - 1; v > wi; --v)
        z = rev_combine(part[v][lane], z, static_cast<float>(part_n[v]), w);
    for (int s = hi - 1; s >= lo; s -= 4) {
        RevState loc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (s - i >= lo) loc[i] = load_rev(r0 + static_cast<size_t>(s - i) * 5 * a.C, a.C);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (s - i >= lo) {
                store_rev(r0 + static_cast<size_t>(s - i) * 5 * a.C, a.C, z);
                z = rev_combine(loc[i], z, static_cast<float>(seg_len(a, s - i)), w);
            }
        }
    }
}

// 5. per segment: y_t, L_t again from the forward carry, then the reverse
//    pass from the reverse carry: gk, gv and the partial gw, gu
template <bool FULL>
__device__ __forceinline__ void seg_grads(const WkvBwdArgs &a, int b, int s, int c, int t0,
                                          int n) {
    const float w = a.w[c], u = a.u[c];
    const size_t base = static_cast<size_t>(b) * a.T * a.C + c;
    const size_t bs_ = static_cast<size_t>(b) * a.S + s;
    float ks[kSeg], vs[kSeg], gs[kSeg], ys[kSeg], Ls[kSeg], bs[kSeg];
    seg_load<FULL>(a.k, base, t0, n, a.C, ks);
    seg_load<FULL>(a.v, base, t0, n, a.C, vs);
    seg_load<FULL>(a.gy, base, t0, n, a.C, gs);
    seg_outputs<FULL>(ks, vs, n, load_fwd(a.fwd + bs_ * 3 * a.C + c, a.C), w, u, ys, Ls, bs);
    RevState z = load_rev(a.rev + bs_ * 5 * a.C + c, a.C);
    float gw = 0.f, gu = 0.f;
    // k_j, v_j are read again (from L1) rather than held across both sweeps
    const float *qk = a.k + base + static_cast<size_t>(t0) * a.C;
    const float *qv = a.v + base + static_cast<size_t>(t0) * a.C;
    float *pk = a.gk + base + static_cast<size_t>(t0) * a.C;
    float *pv = a.gv + base + static_cast<size_t>(t0) * a.C;
#pragma unroll
    for (int i = kSeg - 1; i >= 0; --i) {
        if (FULL || i < n) {
            const float kj = __ldg(qk + static_cast<size_t>(i) * a.C);
            const float vj = __ldg(qv + static_cast<size_t>(i) * a.C);
            const float diag = bs[i] * gs[i];       // g_j beta_{j,j}
            const float sc = fast_exp(kj - z.rho);  // e^{k_j - rho}, <= 1
            const float dv = vj - ys[i];
            pv[static_cast<size_t>(i) * a.C] = fmaf(sc, z.P, diag);
            pk[static_cast<size_t>(i) * a.C] = fmaf(diag, dv, sc * fmaf(vj, z.P, -z.Q));
            gu = fmaf(diag, dv, gu);
            gw = fmaf(-sc, fmaf(vj, z.R, -z.R2), gw);
            rev_step(z, gs[i], ys[i], Ls[i], w);
        }
    }
    float *pp = a.partial + bs_ * 2 * a.C + c;
    pp[0] = gw;
    pp[a.C] = gu;
}

__global__ void __launch_bounds__(kBwdThreads, 4) wkv_bwd_grads_kernel(const WkvBwdArgs a) {
    int b, s, c, t0, n;
    if (!seg_thread(a, b, s, c, t0, n)) return;
    if (n == kSeg)
        seg_grads<true>(a, b, s, c, t0, n);
    else
        seg_grads<false>(a, b, s, c, t0, n);
}

// 6. gw[c], gu[c]: the partials added over rows and segments in a fixed
//    order, in two levels within one launch.  Block (channel group, part)
//    adds part `part` of the (row, segment) range, warp by warp, and writes
//    that sum; the last of a channel group's kReduceParts blocks to finish
//    adds the parts in part order and resets the group's counter.
__global__ void __launch_bounds__(32 * kReduceWarps) wkv_bwd_reduce_kernel(const WkvBwdArgs a) {
    __shared__ float part[2][kReduceWarps][32];
    __shared__ bool last;
    // as in wkv_bwd_rev_carry_kernel: the next grid in the stream may start
    // launching at once (its own wait covers this one); the partials are read
    // only after their kernel has finished
    allow_dependent_launch();
    grid_dependency_wait();
    const int lane = threadIdx.x % 32, wi = threadIdx.x / 32;
    const int cg = blockIdx.x / kReduceParts, pi = blockIdx.x % kReduceParts;
    const int c = cg * 32 + lane;
    const long long nbs = static_cast<long long>(a.B) * a.S;
    const long long q = static_cast<long long>(pi) * kReduceWarps + wi;  // this warp's slice
    const long long lo = nbs * q / (kReduceParts * kReduceWarps);
    const long long hi = nbs * (q + 1) / (kReduceParts * kReduceWarps);
    float gw = 0.f, gu = 0.f;
    if (c < a.C) {
#pragma unroll 8
        for (long long bs = lo; bs < hi; ++bs) {
            gw += a.partial[static_cast<size_t>(bs) * 2 * a.C + c];
            gu += a.partial[(static_cast<size_t>(bs) * 2 + 1) * a.C + c];
        }
    }
    part[0][wi][lane] = gw;
    part[1][wi][lane] = gu;
    __syncthreads();
    if (wi == 0) {
        gw = 0.f;
        gu = 0.f;
        for (int i = 0; i < kReduceWarps; ++i) {
            gw += part[0][i][lane];
            gu += part[1][i][lane];
        }
        if (c < a.C) {
            a.red[static_cast<size_t>(pi) * 2 * a.C + c] = gw;
            a.red[(static_cast<size_t>(pi) * 2 + 1) * a.C + c] = gu;
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) last = atomicAdd(a.red_done + cg, 1u) == kReduceParts - 1u;
        __syncwarp();
        if (last) {
            __threadfence();
            gw = 0.f;
            gu = 0.f;
            if (c < a.C) {
                for (int i = 0; i < kReduceParts; ++i) {
                    gw += __ldcg(a.red + static_cast<size_t>(i) * 2 * a.C + c);
                    gu += __ldcg(a.red + (static_cast<size_t>(i) * 2 + 1) * a.C + c);
                }
                a.gw[c] = gw;
                a.gu[c] = gu;
            }
            if (lane == 0) a.red_done[cg] = 0u;
        }
    }
}

// The same sum in one level, for up to kReduceOneLevelRows (row, segment)s:
// block cg's warp wi adds rows wi, wi + kReduceOneWarps, ... of the channel
// group, and its first warp adds the warps' sums in warp order.  One pass
// over the partials and no cross-block counter.
constexpr int kReduceOneWarps = 32;
constexpr int kReduceOneLevelRows = 32 * kReduceOneWarps;
__global__ void __launch_bounds__(32 * kReduceOneWarps) wkv_bwd_reduce_one_kernel(const WkvBwdArgs a) {
    __shared__ float part[2][kReduceOneWarps][32];
    // as in wkv_bwd_rev_carry_kernel
    allow_dependent_launch();
    grid_dependency_wait();
    const int lane = threadIdx.x % 32, wi = threadIdx.x / 32;
    const int c = blockIdx.x * 32 + lane;
    const int nbs = a.B * a.S;
    float gw = 0.f, gu = 0.f;
    if (c < a.C) {
#pragma unroll 8
        for (int bs = wi; bs < nbs; bs += kReduceOneWarps) {
            gw += a.partial[static_cast<size_t>(bs) * 2 * a.C + c];
            gu += a.partial[(static_cast<size_t>(bs) * 2 + 1) * a.C + c];
        }
    }
    part[0][wi][lane] = gw;
    part[1][wi][lane] = gu;
    __syncthreads();
    if (wi == 0 && c < a.C) {
        gw = 0.f;
        gu = 0.f;
        for (int i = 0; i < kReduceOneWarps; ++i) {
            gw += part[0][i][lane];
            gu += part[1][i][lane];
        }
        a.gw[c] = gw;
        a.gu[c] = gu;
    }
}

}  // namespace wkvb
