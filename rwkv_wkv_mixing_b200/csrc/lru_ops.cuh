// Op policy for the LRU's complex diagonal recurrence (review of
// "Resurrecting Recurrent Neural Networks for Long Sequences", linear-RNN
// section):
//
//     x_t = lambda x_{t-1} + gamma u_t,   lambda = r e^{i theta} = e^{-nu + i theta},
//     nu = e^{nu_log},  theta = e^{theta_log}   (the page's parameterisation),
//
// per complex channel, u and x stored as interleaved (re, im) float pairs.
// lambda does not change with t, so a chunk of n steps is summarised by its
// state from zero alone (its transition is lambda^n), and a state followed by
// a chunk of n steps is lambda^n x + H.  lambda^n = e^{-n nu} e^{i n theta}:
// the phase n theta reaches 10^6 radians for long sequences, far beyond what
// single precision can reduce, so n theta and its reduction to [-pi, pi]
// (subtracting the nearest multiple of 2 pi) are done in double precision and
// only the reduced phase and the magnitude go through single-precision
// functions.  Inside a sub-chunk the state steps with the single-precision
// lambda (at most a tile's worth of steps).  nu and theta themselves are kept
// in double: a phase n theta is only as exact as theta.
#pragma once

#include <cuda_runtime.h>

#include "wkv_ops.cuh"

namespace wkvb {

// unroll factor of the full-sub-chunk loops
#ifndef WKV_LRU_UNROLL
#define WKV_LRU_UNROLL 8
#endif

struct LruOp {
    using io_t = float2;
    static constexpr int CPT = 1;
    static constexpr int CG = 32;
    static constexpr int NV = 2;
    static constexpr int NIN = 1;            // u only
    static constexpr int kScalarsPerIo = 2;  // tensor maps see (re, im) as two floats
    static constexpr int kLruUnroll = WKV_LRU_UNROLL;
    static constexpr bool kGated = false;
    static constexpr bool kSerialForm = false;
    struct Param {
        float lr, li;      // lambda, rounded to single precision for the steps
        float g;           // gamma
        double nu, theta;  // e^{nu_log}, e^{theta_log} in double: lambda^n has
                           // phase n theta, which needs theta to ~1e-16
    };
    struct State {
        float r, i;
    };
    struct Args {
        const float2 *x0;  // u [B, T, D] complex
        const float2 *x1;  // unused (one input)
        float2 *y;         // x [B, T, D] complex
        const float *nu_log, *theta_log, *gamma;  // [D]; gamma may be nullptr (1)
        const float2 *h0;  // x_{-1} [B, D] complex, or nullptr (0)
    };
    struct Scratch {};

    // e^{i phase} for a phase given in double: reduced to [-pi, pi] in double
    __device__ __forceinline__ static void unit_phase(double phase, float &c, float &s) {
        constexpr double kTwoPi = 6.283185307179586, kInvTwoPi = 0.15915494309189535;
        const double red = fma(-kTwoPi, rint(phase * kInvTwoPi), phase);
        sincosf(static_cast<float>(red), &s, &c);
    }

    __device__ __forceinline__ static Param param(const Args &args, int c, int C) {
        Param q{0.f, 0.f, 1.f, 0.0, 0.0};
        if (c < C) {
            q.nu = exp(static_cast<double>(args.nu_log[c]));
            q.theta = exp(static_cast<double>(args.theta_log[c]));
            const float r = expf(-static_cast<float>(q.nu));
            float co, si;
            unit_phase(q.theta, co, si);
            q.lr = r * co;
            q.li = r * si;
            q.g = args.gamma != nullptr ? args.gamma[c] : 1.f;
        }
        return q;
    }
    __device__ __forceinline__ static State identity() { return {0.f, 0.f}; }
    __device__ __forceinline__ static State carry0(const Args &args, int b, int c, int C) {
        if (args.h0 == nullptr || c >= C) return identity();
        const float2 h = args.h0[static_cast<size_t>(b) * C + c];
        return {h.x, h.y};
    }
    __device__ __forceinline__ static void store_final(const Args &, int, int, int, const State &) {}
    __device__ __forceinline__ static State nan_state() {
        const float n = __int_as_float(0x7fffffff);
        return {n, n};
    }
    __device__ __forceinline__ static float get(const State &s, int q) { return q == 0 ? s.r : s.i; }
    __device__ __forceinline__ static State make(const float (&v)[NV]) { return {v[0], v[1]}; }
    __device__ __forceinline__ static void pack(const State &s, float &x, float &y,
                                                uint32_t &bits16) {
        x = s.r;
        y = s.i;
        bits16 = 0u;
    }
    __device__ __forceinline__ static State unpack(float x, float y, uint32_t) { return {x, y}; }

    // l followed by a chunk of n steps whose state from zero is r:
    // lambda^n l + r, lambda^n = e^{-n nu} e^{i n theta}
    __device__ __forceinline__ static State combine(const State &l, const State &r, float n,
                                                    const Param &q) {
        if (n == 0.f) return {l.r + r.r, l.i + r.i};
        const double nn = static_cast<double>(n);
        const float mag = expf(-static_cast<float>(nn * q.nu));
        float c, s;
        unit_phase(nn * q.theta, c, s);
        const float pr = mag * c, pi = mag * s;
        return {fmaf(pr, l.r, fmaf(-pi, l.i, r.r)), fmaf(pr, l.i, fmaf(pi, l.r, r.i))};
    }

    // one step x <- lambda x + gamma u
    __device__ __forceinline__ static void step(float &xr, float &xi, float2 u, const Param &q) {
        const float ur = q.g * u.x, ui = q.g * u.y;
        const float nr = fmaf(q.lr, xr, fmaf(-q.li, xi, ur));
        const float ni = fmaf(q.lr, xi, fmaf(q.li, xr, ui));
        xr = nr;
        xi = ni;
    }

    template <int LS>
    __device__ __forceinline__ static void summarize(const float2 *p0, const float2 *, int n,
                                                     const Param (&q)[1], State (&out)[1],
                                                     Scratch (&)[1]) {
        float xr = 0.f, xi = 0.f;
        if (n == LS) {
#pragma unroll(kLruUnroll)
            for (int i = 0; i < LS; ++i) step(xr, xi, p0[i * CG], q[0]);
        } else {
            for (int i = 0; i < n; ++i) step(xr, xi, p0[i * CG], q[0]);
        }
        out[0] = {xr, xi};
    }

    template <int LS>
    __device__ __forceinline__ static void sweep(const State (&carry)[1], const float2 *p0,
                                                 const float2 *, const float2 *, int n,
                                                 const Param (&q)[1], const Scratch (&)[1],
                                                 float2 *out, size_t ostride, bool valid) {
        float xr = carry[0].r, xi = carry[0].i;
        if (n == LS) {
#pragma unroll(kLruUnroll)
            for (int i = 0; i < LS; ++i) {
                step(xr, xi, p0[i * CG], q[0]);
                if (valid) out[i * ostride] = make_float2(xr, xi);
            }
        } else {
            for (int i = 0; i < n; ++i) {
                step(xr, xi, p0[i * CG], q[0]);
                if (valid) out[i * ostride] = make_float2(xr, xi);
            }
        }
    }
};

}  // namespace wkvb
