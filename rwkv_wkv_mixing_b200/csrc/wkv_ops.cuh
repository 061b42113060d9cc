// Op policies for chunked_scan_kernel: the RWKV-4 WKV operator and the
// per-channel diagonal linear scan.
#pragma once

#include <cuda_bf16.h>

#include "chunked_scan.cuh"
#include "ptx.cuh"

namespace wkvb {

constexpr float kLog2e = 1.4426950408889634f;
// log2-scale of "no tokens yet"; finite so that differences of two sentinels
// stay finite, and 2^(sentinel - anything real) flushes to zero
constexpr float kNoScale = -1e30f;

// ---------------------------------------------------------------------------
// WKV, eq. (14) of "RWKV：基于RNN的LLM" (section 二.1, Time-mixing block).
//
// State before step t: the past sums
//   num_t = sum_{i<t} e^{-(t-1-i) w + k_i} v_i,  den_t = sum_{i<t} e^{-(t-1-i) w + k_i},
// kept as (a, b, p) with (num, den) = (a, b) * 2^p.  All exponents are in
// log2 units (k, u, w pre-multiplied by log2 e), and p is the largest exponent
// folded in so far, so every 2^x evaluated has x <= 0 and b >= 1 once a token
// has been added.  Outputs:
//   y_t = (num_t + e^{u + k_t} v_t) / (den_t + e^{u + k_t});
// state update:
//   (num, den)_{t+1} = e^{-w} (num, den)_t + e^{k_t} (v_t, 1).
// A chunk of L steps maps a state S to e^{-L w} S + (chunk summary), which is
// `combine`.
// ---------------------------------------------------------------------------
template <typename IO, int CPT_>
struct WkvOp {
    using io_t = IO;
    static constexpr int CPT = CPT_;
    static constexpr int NV = 3;
    static constexpr bool kExactDiv = sizeof(IO) == 4;
    struct Param {
        float uu;  // u * log2 e
        float ww;  // w * log2 e
    };
    struct State {
        float a, b, p;
    };
    struct Args {
        const IO *x0;  // k [B, T, C]
        const IO *x1;  // v [B, T, C]
        IO *y;         // y [B, T, C]
        const float *w, *u;  // [C]
    };

    __device__ __forceinline__ static Param param(const Args &args, int c, int C) {
        Param q{0.f, 0.f};
        if (c < C) {
            q.uu = args.u[c] * kLog2e;
            q.ww = args.w[c] * kLog2e;
        }
        return q;
    }
    __device__ __forceinline__ static State identity() { return {0.f, 0.f, kNoScale}; }
    __device__ __forceinline__ static State carry0(const Args &, int, int, int) {
        return identity();  // empty past before the first step
    }
    __device__ __forceinline__ static State nan_state() {
        const float n = __int_as_float(0x7fffffff);
        return {n, n, n};
    }
    __device__ __forceinline__ static float get(const State &s, int q) {
        return q == 0 ? s.a : (q == 1 ? s.b : s.p);
    }
    __device__ __forceinline__ static State make(const float (&v)[NV]) { return {v[0], v[1], v[2]}; }

    // state l, then a chunk whose summary is r and whose length is r_len steps
    __device__ __forceinline__ static State combine(const State &l, const State &r, float r_len,
                                                    const Param &q) {
        const float pd = l.p - r_len * q.ww;
        const float m = fmaxf(pd, r.p);
        const float fl = ex2_approx(pd - m), fr = ex2_approx(r.p - m);
        return {fmaf(l.a, fl, r.a * fr), fmaf(l.b, fl, r.b * fr), m};
    }

    // state update with token (k, v)
    __device__ __forceinline__ static void step1(State &s, float k, float v, const Param &q) {
        const float kk = k * kLog2e;
        const float pd = s.p - q.ww;
        const float d = pd - kk;
        const float e = ex2_approx(-fabsf(d));
        const bool old_wins = d >= 0.f;
        const float fo = old_wins ? 1.f : e, fn = old_wins ? e : 1.f;
        s.a = fmaf(s.a, fo, fn * v);
        s.b = fmaf(s.b, fo, fn);
        s.p = fmaxf(pd, kk);
    }

    // output at this step, then the state update
    __device__ __forceinline__ static float step2(State &s, float k, float v, const Param &q) {
        const float x = fmaf(k, kLog2e, q.uu);
        const float d = s.p - x;
        const float e = ex2_approx(-fabsf(d));
        const bool old_wins = d >= 0.f;
        const float fo = old_wins ? 1.f : e, fn = old_wins ? e : 1.f;
        const float num = fmaf(s.a, fo, fn * v);
        const float den = fmaf(s.b, fo, fn);
        // fp32 outputs use the correctly rounded quotient, so a constant
        // power-of-two v comes back exactly; bf16 outputs are rounded to 8
        // significant bits afterwards, where one ulp of fp32 cannot matter
        const float y = kExactDiv ? __fdiv_rn(num, den) : num * rcp_approx(den);
        step1(s, k, v, q);
        return y;
    }
};

// ---------------------------------------------------------------------------
// Diagonal linear scan h_t = a_t h_{t-1} + b_t ("Were RNNs All We Needed?",
// model-architecture section).  Chunk summary: (A, H) = (product of the a's,
// state produced from h = 0); state h followed by chunk (A, H) gives A h + H.
// ---------------------------------------------------------------------------
struct ScanOp {
    using io_t = float;
    static constexpr int CPT = 1;
    static constexpr int NV = 2;
    struct Param {};
    struct State {
        float A, H;
    };
    struct Args {
        const float *x0;  // a [B, T, D]
        const float *x1;  // b [B, T, D]
        float *y;         // h [B, T, D]
        const float *h0;  // [B, D] or nullptr
    };

    __device__ __forceinline__ static Param param(const Args &, int, int) { return {}; }
    __device__ __forceinline__ static State identity() { return {1.f, 0.f}; }
    __device__ __forceinline__ static State carry0(const Args &args, int b, int c, int C) {
        State s{1.f, 0.f};
        if (args.h0 != nullptr && c < C) s.H = args.h0[static_cast<size_t>(b) * C + c];
        return s;
    }
    __device__ __forceinline__ static State nan_state() {
        const float n = __int_as_float(0x7fffffff);
        return {n, n};
    }
    __device__ __forceinline__ static float get(const State &s, int q) { return q == 0 ? s.A : s.H; }
    __device__ __forceinline__ static State make(const float (&v)[NV]) { return {v[0], v[1]}; }
    __device__ __forceinline__ static State combine(const State &l, const State &r, float,
                                                    const Param &) {
        return {l.A * r.A, fmaf(r.A, l.H, r.H)};
    }
    __device__ __forceinline__ static void step1(State &s, float a, float b, const Param &) {
        s.H = fmaf(a, s.H, b);
        s.A *= a;
    }
    __device__ __forceinline__ static float step2(State &s, float a, float b, const Param &) {
        s.H = fmaf(a, s.H, b);
        return s.H;
    }
};

}  // namespace wkvb
