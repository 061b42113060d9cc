// Op policies for chunked_scan_kernel: the RWKV-4 WKV operator and the
// per-channel diagonal linear scan.
//
// An Op supplies, for the CPT channels one thread owns:
//   summarize(p0, p1, n, ...)  pass 1: the summary of an n-step sub-chunk
//                              (rows p0[i*CG], p1[i*CG]) from the empty state
//   sweep(carry, ...)          pass 2: outputs of the sub-chunk from the state
//                              before it, to out[i*ostride] (shared or global)
//   combine(l, r, r_len)       the state l followed by a chunk of r_len steps
//                              whose summary is r
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace wkvb {

constexpr float kLog2e = 1.4426950408889634f;

// unroll factor of the full-sub-chunk loops of the packed bf16 passes,
// without and with the gate (measured: 8 and 4; the gate's larger loop body
// runs faster with less code, the plain one with more)
#ifndef WKV_PACKED_UNROLL
#define WKV_PACKED_UNROLL 8
#endif
#ifndef WKV_PACKED_UNROLL_GATED
#define WKV_PACKED_UNROLL_GATED 4
#endif
// ... and of the scalar (fp32, one channel a thread) passes (32, the whole
// sub-chunk: wkv_long 298.7 against 306.8 us with 8)
#ifndef WKV_SCAN_UNROLL
#define WKV_SCAN_UNROLL 8
#endif
#ifndef WKV_SCAN_UNROLL_BF16
#define WKV_SCAN_UNROLL_BF16 8
#endif
#ifndef WKV_SCALAR_UNROLL
#define WKV_SCALAR_UNROLL 32
#endif
// log-scale of "no tokens yet": finite, so differences of two such values
// stay finite, and e^(kNoScale - anything real) is exactly zero
constexpr float kNoScale = -1e30f;

// ---- shared-memory access to CPT consecutive channels ---------------------
template <typename io_t, int CPT>
struct Vec;

template <>
struct Vec<float, 1> {
    __device__ __forceinline__ static void load(const float *p, float (&x)[1]) { x[0] = *p; }
    __device__ __forceinline__ static void store(float *p, const float (&x)[1]) { *p = x[0]; }
};

template <>
struct Vec<float, 2> {
    __device__ __forceinline__ static void load(const float *p, float (&x)[2]) {
        float2 t = *reinterpret_cast<const float2 *>(p);
        x[0] = t.x;
        x[1] = t.y;
    }
    __device__ __forceinline__ static void store(float *p, const float (&x)[2]) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    }
};

template <>
struct Vec<float, 4> {
    __device__ __forceinline__ static void load(const float *p, float (&x)[4]) {
        const float4 t = *reinterpret_cast<const float4 *>(p);
        x[0] = t.x;
        x[1] = t.y;
        x[2] = t.z;
        x[3] = t.w;
    }
    __device__ __forceinline__ static void store(float *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

template <>
struct Vec<__nv_bfloat16, 1> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[1]) {
        x[0] = __bfloat162float(*p);
    }
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, const float (&x)[1]) {
        *p = __float2bfloat16_rn(x[0]);  // round to nearest even
    }
};

template <>
struct Vec<__nv_bfloat16, 4> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[4]) {
        const uint2 t = *reinterpret_cast<const uint2 *>(p);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&t.y));
        x[0] = lo.x;
        x[1] = lo.y;
        x[2] = hi.x;
        x[3] = hi.y;
    }
    // round to nearest even
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, const float (&x)[4]) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
        uint2 t;
        t.x = *reinterpret_cast<const uint32_t *>(&lo);
        t.y = *reinterpret_cast<const uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(p) = t;
    }
};

template <>
struct Vec<__nv_bfloat16, 2> {
    __device__ __forceinline__ static void load(const __nv_bfloat16 *p, float (&x)[2]) {
        float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        x[0] = t.x;
        x[1] = t.y;
    }
    // round to nearest even
    __device__ __forceinline__ static void store(__nv_bfloat16 *p, const float (&x)[2]) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x[0], x[1]);
    }
};

// The output (a + e v) / (b + e) written as v + (a - b v) / (b + e): the same
// quotient, but exact whenever the past does not move the answer -- an empty
// past (a = b = 0, so y_0 = v_0 bit for bit) or a constant power-of-two v
// (a = v b exactly) -- and the approximate reciprocal only perturbs the
// correction term, whose size is |y - v|.
__device__ __forceinline__ float wkv_output(float a, float b, float e, float v) {
    return v + fmaf(-b, v, a) * rcp_approx(b + e);
}

// e^x through the MUFU ex2 unit, for factors that weigh one term against a
// term of weight exactly 1 (arguments <= 0 after max-normalisation): the
// relative error, about 2^-22 plus |x| 2^-24 from rounding x log2(e), only
// matters where e^x is large, i.e. for small |x|.  Not for factors that get
// raised to powers (the per-step decay e^{-w} uses expf).
__device__ __forceinline__ float fast_exp(float x) { return ex2_approx(x * kLog2e); }

// The receptance gate sigma(r) = 1 / (1 + e^{-r}) of eq. (15) of
// "RWKV：基于RNN的LLM".  Saturates cleanly: e^{-r} = inf gives 0, e^{-r} = 0
// gives 1.
__device__ __forceinline__ float gate_sigmoid(float r) {
    return rcp_approx(1.f + ex2_approx(-r * kLog2e));
}

// ---------------------------------------------------------------------------
// WKV, eq. (14) of "RWKV：基于RNN的LLM" (section 二.1, Time-mixing block):
//   y_t = (num_t + e^{u + k_t} v_t) / (den_t + e^{u + k_t}),
//   num_t = sum_{i<t} e^{-(t-1-i) w + k_i} v_i,  den_t = same without v_i.
//
// State: (a, b, p) with (num, den) = (a, b) * e^p, p in natural-log units.
// Stepping the state: (num, den)_{t+1} = e^{-w} (num, den)_t + e^{k_t} (v_t, 1).
//
// Pass 1 (summary of a sub-chunk ending at step `end`, from the empty state):
// one round finds max k and min k (packed pairs for bf16), a second sums
// a = sum_i e^{k_i - (end-i) w - p} v_i and b = the same without v_i against
// the reference p = max k, so every exponent is <= 0.  Any reference is the
// same state; max k only risks that every term of a chunk whose largest key
// is decayed away falls far below 1 -- when b < 2^-60 the chunk is summed
// again against the exact largest exponent p = max_i (k_i - (end-i) w),
// whose term is exactly 1.
//
// Pass 2 (outputs of a sub-chunk from the state before it): one reference
// M = max(p_in, max_i k_i) for the whole sub-chunk, state scaled to e^M, so
// each step is  e = e^{k_t - M} (<= 1),  y = (a + e U v) / (b + e U),
// a <- a D + e v,  b <- b D + e  with per-channel constants U = e^u,
// D = e^{-w}.  The loop-carried dependency is one FMA.  This is exact
// arithmetic reordered; it is used when a bound shows every denominator stays
// above e^-69 (so nothing that matters is flushed to zero) and U is below
// 2^64.  Otherwise the sub-chunk takes the per-step max-stabilised update,
// whose every exponent is <= 0 for any finite input.
// ---------------------------------------------------------------------------
// GATED: the outputs are sigma(r_t) (.) wkv_t (eq. (15) before the output
// projection), r read as a third input tensor alongside k and v.
template <typename IO, int CPT_, bool GATED = false>
struct WkvOp {
    using io_t = IO;
    static constexpr int CPT = CPT_;
    static constexpr int CG = 32 * CPT;
    static constexpr int NV = 3;
    static constexpr int NIN = GATED ? 3 : 2;  // input tensors per tile: k, v (, r)
    static constexpr int kScalarsPerIo = 1;    // tensor-map elements per io_t
    // two bf16 channels per thread: per-element arithmetic in packed fp32 pairs
    static constexpr bool kPacked = sizeof(IO) == 2 && CPT == 2;
    static constexpr bool kGated = GATED;
    static constexpr bool kSerialForm = true;  // has the per-step form of serial_wkv.cuh
    static constexpr int kPackedUnroll = GATED ? WKV_PACKED_UNROLL_GATED : WKV_PACKED_UNROLL;
    static constexpr int kScalarUnroll = WKV_SCALAR_UNROLL;
    struct Param {
        float u, w;  // bonus and decay (natural units)
        float U, D;  // e^u, e^{-w}
    };
    struct State {
        float a, b, p;
    };
    struct Args {
        const IO *x0;  // k [B, T, C]
        const IO *x1;  // v [B, T, C]
        IO *y;         // y [B, T, C]
        const float *w, *u;  // [C]
        const float *s_in;   // [B, 3, C] state before step 0, or nullptr (empty)
        float *s_out;        // [B, 3, C] state after the last step, or nullptr
        const IO *x2;        // r [B, T, C] (GATED only)
    };
    // per-thread facts pass 1 leaves for pass 2 of the same sub-chunk
    struct Scratch {
        float kmax, kmin;
    };

    __device__ __forceinline__ static Param param(const Args &args, int c, int C) {
        Param q{0.f, 0.f, 1.f, 1.f};
        if (c < C) {
            q.u = args.u[c];
            q.w = args.w[c];
            q.U = expf(q.u);
            q.D = expf(-q.w);
        }
        return q;
    }
    __device__ __forceinline__ static State identity() { return {0.f, 0.f, kNoScale}; }
    // The state before step 0: planes a, b, p of s_in for batch row b
    // (sums (num, den) = (a, b) e^p), or the empty past.  a = b = 0 or
    // p = -inf is the empty past whatever the other fields hold.
    __device__ __forceinline__ static State carry0(const Args &args, int b, int c, int C) {
        if (args.s_in == nullptr || c >= C) return identity();
        const float *s = args.s_in + static_cast<size_t>(b) * 3 * C + c;
        return state_in(s[0], s[C], s[2 * C]);
    }
    __device__ __forceinline__ static State state_in(float a, float b, float p) {
        if ((a == 0.f && b == 0.f) || p == -__int_as_float(0x7f800000)) return identity();
        return {a, b, p};
    }
    // the state after the last step, to s_out (when given) in the same planes
    __device__ __forceinline__ static void store_final(const Args &args, int b, int c, int C,
                                                       const State &st) {
        if (args.s_out == nullptr || c >= C) return;
        float *s = args.s_out + static_cast<size_t>(b) * 3 * C + c;
        s[0] = st.a;
        s[C] = st.b;
        s[2 * C] = st.p;
    }
    __device__ __forceinline__ static State nan_state() {
        const float n = __int_as_float(0x7fffffff);
        return {n, n, n};
    }
    __device__ __forceinline__ static float get(const State &s, int q) {
        return q == 0 ? s.a : (q == 1 ? s.b : s.p);
    }
    __device__ __forceinline__ static State make(const float (&v)[NV]) { return {v[0], v[1], v[2]}; }

    // a published state in two floats: rescaled to the integer log-scale
    // ceil(p), which travels in the record's 16 spare tag bits (published
    // states are never empty, so p is finite; |p| beyond 32767 is clamped,
    // inputs that large are outside the operator's domain anyway)
    __device__ __forceinline__ static void pack(const State &s, float &x, float &y,
                                                uint32_t &bits16) {
        const float pi = fminf(fmaxf(ceilf(s.p), -32768.f), 32767.f);
        const float f = fast_exp(s.p - pi);
        x = s.a * f;
        y = s.b * f;
        bits16 = static_cast<uint32_t>(static_cast<int>(pi) + 32768);
    }
    __device__ __forceinline__ static State unpack(float x, float y, uint32_t bits16) {
        return {x, y, static_cast<float>(static_cast<int>(bits16) - 32768)};
    }

    __device__ __forceinline__ static State combine(const State &l, const State &r, float r_len,
                                                    const Param &q) {
        const float pd = fmaf(-r_len, q.w, l.p);
        const float m = fmaxf(pd, r.p);
        const float fl = fast_exp(pd - m), fr = fast_exp(r.p - m);
        return {fmaf(l.a, fl, r.a * fr), fmaf(l.b, fl, r.b * fr), m};
    }

    // ---- pass 1 ------------------------------------------------------------
    // Exponent argument (x - r) in log2 units for ex2.  fp32 keeps the
    // subtraction exact before scaling, so the error is a few ulp of |x - r|
    // (small for the terms that matter); bf16 folds both into one FMA, whose
    // error of about 2^-24 (|x| + |r|) is far below bf16 rounding.
    __device__ __forceinline__ static float exp_arg(float x, float r, float r2) {
        if constexpr (sizeof(IO) == 2)
            return fmaf(x, kLog2e, -r2);
        else
            return (x - r) * kLog2e;
    }

    // first sweep: largest and smallest key of each channel over n rows
    template <int LS>
    __device__ __forceinline__ static void key_range(const IO *p0, int n, float (&kx)[CPT],
                                                     float (&kn)[CPT]) {
        if constexpr (sizeof(IO) == 2 && CPT == 2) {
            // bf16 pairs: max and min are exact in bf16, two channels per op
            const __nv_bfloat16 ninf = __ushort_as_bfloat16(0xff80u), pinf = __ushort_as_bfloat16(0x7f80u);
            __nv_bfloat162 hx = __halves2bfloat162(ninf, ninf), hn = __halves2bfloat162(pinf, pinf);
            if (n == LS) {
#pragma unroll(kPackedUnroll)
                for (int i = 0; i < LS; ++i) {
                    const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(p0 + i * CG);
                    hx = __hmax2(hx, k2);
                    hn = __hmin2(hn, k2);
                }
            } else {
                for (int i = 0; i < n; ++i) {
                    const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(p0 + i * CG);
                    hx = __hmax2(hx, k2);
                    hn = __hmin2(hn, k2);
                }
            }
            const float2 fx = __bfloat1622float2(hx), fn = __bfloat1622float2(hn);
            kx[0] = fx.x;
            kx[1] = fx.y;
            kn[0] = fn.x;
            kn[1] = fn.y;
        } else {
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                kx[j] = kNoScale;
                kn[j] = -kNoScale;
            }
            if (n == LS) {
#pragma unroll(kScalarUnroll)
                for (int i = 0; i < LS; ++i) {
                    float k[CPT];
                    Vec<IO, CPT>::load(p0 + i * CG, k);
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        kx[j] = fmaxf(kx[j], k[j]);
                        kn[j] = fminf(kn[j], k[j]);
                    }
                }
            } else {
                for (int i = 0; i < n; ++i) {
                    float k[CPT];
                    Vec<IO, CPT>::load(p0 + i * CG, k);
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        kx[j] = fmaxf(kx[j], k[j]);
                        kn[j] = fminf(kn[j], k[j]);
                    }
                }
            }
        }
    }

    // second sweep: a = sum_i e^{k_i - (end-i) w - ref} v_i, b = the same without
    // v_i, over n rows ending at row n-1
    // (U: unroll factor of the scalar full-sub-chunk loop; the register-
    // resident kernels' rare re-sum path keeps 8, its code small)
    template <int LS, int U = kScalarUnroll>
    __device__ __forceinline__ static void chunk_sums(const IO *p0, const IO *p1, int n,
                                                      const Param (&q)[CPT],
                                                      const float (&ref)[CPT], float (&a)[CPT],
                                                      float (&b)[CPT]) {
        float ref2[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            ref2[j] = ref[j] * kLog2e;
            a[j] = 0.f;
            b[j] = 0.f;
        }
        if constexpr (kPacked) {
            // both channels in packed fp32 pairs: one instruction per pair,
            // each component rounded as the scalar fmaf / fadd
            const float2 w2 = make_float2(q[0].w, q[1].w), l2e = make_float2(kLog2e, kLog2e);
            const float2 nref2 = make_float2(-ref2[0], -ref2[1]);
            float2 a2 = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
            const auto one = [&](int i, float ci) {
                float k[CPT], v[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, k);
                Vec<IO, CPT>::load(p1 + i * CG, v);
                const float2 x = __ffma2_rn(make_float2(ci, ci), w2, make_float2(k[0], k[1]));
                const float2 arg = __ffma2_rn(x, l2e, nref2);
                const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                a2 = __ffma2_rn(e, make_float2(v[0], v[1]), a2);
                b2 = __fadd2_rn(b2, e);
            };
            if (n == LS) {
#pragma unroll(kPackedUnroll)
                for (int i = 0; i < LS; ++i) one(i, static_cast<float>(i - (LS - 1)));
            } else {
                for (int i = 0; i < n; ++i) one(i, static_cast<float>(i - (n - 1)));
            }
            a[0] = a2.x;
            a[1] = a2.y;
            b[0] = b2.x;
            b[1] = b2.y;
            return;
        }
        if (n == LS) {
#pragma unroll(U)
            for (int i = 0; i < LS; ++i) {
                float k[CPT], v[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, k);
                Vec<IO, CPT>::load(p1 + i * CG, v);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const float x = fmaf(static_cast<float>(i - (LS - 1)), q[j].w, k[j]);
                    const float e = ex2_approx(exp_arg(x, ref[j], ref2[j]));
                    a[j] = fmaf(e, v[j], a[j]);
                    b[j] += e;
                }
            }
        } else {
            for (int i = 0; i < n; ++i) {
                float k[CPT], v[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, k);
                Vec<IO, CPT>::load(p1 + i * CG, v);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const float x = fmaf(static_cast<float>(i - (n - 1)), q[j].w, k[j]);
                    const float e = ex2_approx(exp_arg(x, ref[j], ref2[j]));
                    a[j] = fmaf(e, v[j], a[j]);
                    b[j] += e;
                }
            }
        }
    }

    // the exact largest exponent max_i (k_i - (end-i) w) of one channel
    __device__ __forceinline__ static float largest_exponent(const IO *p0, int n, int j,
                                                             const Param &q) {
        float m = kNoScale;
        for (int i = 0; i < n; ++i) {
            float k[CPT];
            Vec<IO, CPT>::load(p0 + i * CG, k);
            m = fmaxf(m, fmaf(static_cast<float>(i - (n - 1)), q.w, k[j]));
        }
        return m;
    }

    template <int LS>
    __device__ __forceinline__ static void summarize(const IO *p0, const IO *p1, int n,
                                                     const Param (&q)[CPT], State (&out)[CPT],
                                                     Scratch (&sc)[CPT]) {
        if (n <= 0) {
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                out[j] = identity();
                sc[j] = {kNoScale, -kNoScale};
            }
            return;
        }
        float kx[CPT], kn[CPT], a[CPT], b[CPT];
        key_range<LS>(p0, n, kx, kn);
        chunk_sums<LS>(p0, p1, n, q, kx, a, b);
        float ref[CPT];
        bool redo = false;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            ref[j] = kx[j];
            if (!(b[j] >= 0x1p-60f)) {  // the chunk's weight sits far below max k
                ref[j] = largest_exponent(p0, n, j, q[j]);
                redo = true;
            }
        }
        if (redo) {
            float a2[CPT], b2[CPT];
            chunk_sums<LS>(p0, p1, n, q, ref, a2, b2);
#pragma unroll
            for (int j = 0; j < CPT; ++j)
                if (ref[j] != kx[j]) {
                    a[j] = a2[j];
                    b[j] = b2[j];
                }
        }
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            out[j] = {a[j], b[j], ref[j]};
            sc[j] = {kx[j], kn[j]};
        }
    }

    // ---- pass 2 ------------------------------------------------------------
    // exact per-step update (max-stabilised), one channel
    __device__ __forceinline__ static float step_exact(State &s, float k, float v,
                                                       const Param &q) {
        const float x = q.u + k;
        const float d = s.p - x;
        const float e = ex2_approx(-fabsf(d) * kLog2e);
        const bool old_wins = d >= 0.f;
        const float fo = old_wins ? 1.f : e, fn = old_wins ? e : 1.f;
        // (fo a + fn v) / (fo b + fn) with fo, fn as the state's and the token's weights
        const float y = wkv_output(fo * s.a, fo * s.b, fn, v);
        const float pd = s.p - q.w;
        const float d2 = pd - k;
        const float e2 = ex2_approx(-fabsf(d2) * kLog2e);
        const bool old2 = d2 >= 0.f;
        const float go = old2 ? 1.f : e2, gn = old2 ? e2 : 1.f;
        s.a = fmaf(s.a, go, gn * v);
        s.b = fmaf(s.b, go, gn);
        s.p = fmaxf(pd, k);
        return y;
    }

    // outputs go to out[i * ostride] (shared or global memory); when `valid`
    // is false this thread's channels are past C and nothing is stored
    // (p2: the r rows when GATED, else unused)
    template <int LS>
    __device__ __forceinline__ static void sweep(const State (&carry)[CPT], const IO *p0,
                                                 const IO *p1, const IO *p2, int n,
                                                 const Param (&q)[CPT], const Scratch (&sc)[CPT],
                                                 IO *out, size_t ostride, bool valid) {
        // reference per channel, and whether the fixed-reference form is safe
        float M[CPT], M2[CPT], A[CPT], Bs[CPT];
        bool fast = true;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            M[j] = fmaxf(carry[j].p, sc[j].kmax);
            M2[j] = M[j] * kLog2e;
            const float s = fast_exp(carry[j].p - M[j]);
            A[j] = carry[j].a * s;
            Bs[j] = carry[j].b * s;
            // den_t >= e^{u + k_t - M} once e^{k_t - M}, evaluated on its own
            // before the multiplication by e^u, cannot flush to zero (so
            // k_t - M >= -69 as well when u >= 0); and den_t >= b_in e^{p_in - M - t w}
            const bool by_token = sc[j].kmin + fminf(q[j].u, 0.f) - M[j] >= -69.f;
            const bool by_carry =
                carry[j].b >= 1.f && carry[j].p - M[j] - static_cast<float>(n) * q[j].w >= -69.f;
            fast = fast && (by_token || by_carry) && q[j].u <= 44.f;
        }
        if constexpr (kPacked) {
            if (fast) {
                packed_sweep<LS>(p0, p1, p2, n, q, M2, A, Bs, out, ostride, valid);
                return;
            }
        }
        if (fast) {
            if (n == LS) {
#pragma unroll(kScalarUnroll)
                for (int i = 0; i < LS; ++i)
                    fast_step(p0 + i * CG, p1 + i * CG, p2 + i * CG, out + i * ostride, valid, M,
                              M2, A, Bs, q);
            } else {
                for (int i = 0; i < n; ++i)
                    fast_step(p0 + i * CG, p1 + i * CG, p2 + i * CG, out + i * ostride, valid, M,
                              M2, A, Bs, q);
            }
        } else {
            State s[CPT];
#pragma unroll
            for (int j = 0; j < CPT; ++j) s[j] = carry[j];
            for (int i = 0; i < n; ++i) {
                float k[CPT], v[CPT], y[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, k);
                Vec<IO, CPT>::load(p1 + i * CG, v);
#pragma unroll
                for (int j = 0; j < CPT; ++j) y[j] = step_exact(s[j], k[j], v[j], q[j]);
                if constexpr (GATED) apply_gate(p2 + i * CG, y);
                if (valid) Vec<IO, CPT>::store(out + i * ostride, y);
            }
        }
    }

    // y <- sigma(r) (.) y for this thread's channels, r read at pr
    __device__ __forceinline__ static void apply_gate(const IO *pr, float (&y)[CPT]) {
        float r[CPT];
        Vec<IO, CPT>::load(pr, r);
#pragma unroll
        for (int j = 0; j < CPT; ++j) y[j] *= gate_sigmoid(r[j]);
    }

    // the fixed-reference steps of sweep for two channels in packed fp32 pairs
    // (same per-component arithmetic as fast_step)
    template <int LS>
    __device__ __forceinline__ static void packed_sweep(const IO *p0, const IO *p1, const IO *p2,
                                                        int n, const Param (&q)[CPT],
                                                        const float (&M2)[CPT], float (&A)[CPT],
                                                        float (&Bs)[CPT], IO *out, size_t ostride,
                                                        bool valid) {
        const float2 l2e = make_float2(kLog2e, kLog2e), nM2 = make_float2(-M2[0], -M2[1]);
        const float2 U = make_float2(q[0].U, q[1].U), D = make_float2(q[0].D, q[1].D);
        float2 a = make_float2(A[0], A[1]), bs = make_float2(Bs[0], Bs[1]);
        const auto one = [&](int i) {
            float k[CPT], v[CPT];
            Vec<IO, CPT>::load(p0 + i * CG, k);
            Vec<IO, CPT>::load(p1 + i * CG, v);
            const float2 v2 = make_float2(v[0], v[1]);
            const float2 arg = __ffma2_rn(make_float2(k[0], k[1]), l2e, nM2);
            const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            // v + (A - Bs v) / (Bs + e U), as wkv_output
            const float2 t = __ffma2_rn(make_float2(-bs.x, -bs.y), v2, a);
            const float2 d = __ffma2_rn(e, U, bs);
            const float2 y2 = __ffma2_rn(t, make_float2(rcp_approx(d.x), rcp_approx(d.y)), v2);
            a = __ffma2_rn(a, D, __fmul2_rn(e, v2));
            bs = __ffma2_rn(bs, D, e);
            float y[CPT] = {y2.x, y2.y};
            if constexpr (GATED) apply_gate(p2 + i * CG, y);
            if (valid) Vec<IO, CPT>::store(out + i * ostride, y);
        };
        if (n == LS) {
#pragma unroll(kPackedUnroll)
            for (int i = 0; i < LS; ++i) one(i);
        } else {
            for (int i = 0; i < n; ++i) one(i);
        }
        A[0] = a.x;
        A[1] = a.y;
        Bs[0] = bs.x;
        Bs[1] = bs.y;
    }

    __device__ __forceinline__ static void fast_step(const IO *pk, const IO *pv, const IO *pr,
                                                     IO *py, bool valid, const float (&M)[CPT],
                                                     const float (&M2)[CPT], float (&A)[CPT],
                                                     float (&Bs)[CPT], const Param (&q)[CPT]) {
        float k[CPT], v[CPT], y[CPT];
        Vec<IO, CPT>::load(pk, k);
        Vec<IO, CPT>::load(pv, v);
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const float e = ex2_approx(exp_arg(k[j], M[j], M2[j]));
            // (A + e U v) / (Bs + e U) in the residual form of wkv_output, the
            // denominator in one FMA
            y[j] = v[j] + fmaf(-Bs[j], v[j], A[j]) * rcp_approx(fmaf(e, q[j].U, Bs[j]));
            A[j] = fmaf(A[j], q[j].D, e * v[j]);
            Bs[j] = fmaf(Bs[j], q[j].D, e);
        }
        if constexpr (GATED) apply_gate(pr, y);
        if (valid) Vec<IO, CPT>::store(py, y);
    }
};

// ---------------------------------------------------------------------------
// Diagonal linear scan h_t = a_t h_{t-1} + b_t ("Were RNNs All We Needed?",
// model-architecture section).  Chunk summary: (A, H) = (product of the a's,
// state produced from h = 0); the state h followed by a chunk (A, H) is
// A h + H.
// ---------------------------------------------------------------------------
template <typename IO, int CPT_>
struct ScanOpT {
    using io_t = IO;
    static constexpr int CPT = CPT_;
    static constexpr int kScanUnroll = sizeof(IO) == 2 ? WKV_SCAN_UNROLL_BF16 : WKV_SCAN_UNROLL;
    static constexpr int CG = 32 * CPT;
    static constexpr int NV = 2;
    static constexpr int NIN = 2;
    static constexpr int kScalarsPerIo = 1;
    static constexpr bool kGated = false;
    static constexpr bool kSerialForm = false;
    struct Param {};
    struct State {
        float A, H;
    };
    struct Args {
        const IO *x0;     // a [B, T, D]
        const IO *x1;     // b [B, T, D]
        IO *y;            // h [B, T, D]
        const float *h0;  // [B, D] fp32, or nullptr
    };
    struct Scratch {};

    __device__ __forceinline__ static Param param(const Args &, int, int) { return {}; }
    __device__ __forceinline__ static State identity() { return {1.f, 0.f}; }
    __device__ __forceinline__ static State carry0(const Args &args, int b, int c, int C) {
        State s{1.f, 0.f};
        if (args.h0 != nullptr && c < C) s.H = args.h0[static_cast<size_t>(b) * C + c];
        return s;
    }
    __device__ __forceinline__ static void store_final(const Args &, int, int, int, const State &) {}
    __device__ __forceinline__ static State nan_state() {
        const float n = __int_as_float(0x7fffffff);
        return {n, n};
    }
    __device__ __forceinline__ static float get(const State &s, int q) { return q == 0 ? s.A : s.H; }
    __device__ __forceinline__ static State make(const float (&v)[NV]) { return {v[0], v[1]}; }
    __device__ __forceinline__ static void pack(const State &s, float &x, float &y,
                                                uint32_t &bits16) {
        x = s.A;
        y = s.H;
        bits16 = 0u;
    }
    __device__ __forceinline__ static State unpack(float x, float y, uint32_t) { return {x, y}; }
    __device__ __forceinline__ static State combine(const State &l, const State &r, float,
                                                    const Param &) {
        return {l.A * r.A, fmaf(r.A, l.H, r.H)};
    }

    template <int LS>
    __device__ __forceinline__ static void summarize(const IO *p0, const IO *p1, int n,
                                                     const Param (&)[CPT], State (&out)[CPT],
                                                     Scratch (&)[CPT]) {
        float A[CPT], H[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            A[j] = 1.f;
            H[j] = 0.f;
        }
        if (n == LS) {
#pragma unroll(kScanUnroll)
            for (int i = 0; i < LS; ++i) {
                float a[CPT], b[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, a);
                Vec<IO, CPT>::load(p1 + i * CG, b);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    H[j] = fmaf(a[j], H[j], b[j]);
                    A[j] *= a[j];
                }
            }
        } else {
            for (int i = 0; i < n; ++i) {
                float a[CPT], b[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, a);
                Vec<IO, CPT>::load(p1 + i * CG, b);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    H[j] = fmaf(a[j], H[j], b[j]);
                    A[j] *= a[j];
                }
            }
        }
#pragma unroll
        for (int j = 0; j < CPT; ++j) out[j] = {A[j], H[j]};
    }

    template <int LS>
    __device__ __forceinline__ static void sweep(const State (&carry)[CPT], const IO *p0,
                                                 const IO *p1, const IO *, int n,
                                                 const Param (&)[CPT], const Scratch (&)[CPT],
                                                 IO *out, size_t ostride, bool valid) {
        float H[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) H[j] = carry[j].H;
        if (n == LS) {
#pragma unroll(kScanUnroll)
            for (int i = 0; i < LS; ++i) {
                float a[CPT], b[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, a);
                Vec<IO, CPT>::load(p1 + i * CG, b);
#pragma unroll
                for (int j = 0; j < CPT; ++j) H[j] = fmaf(a[j], H[j], b[j]);
                if (valid) Vec<IO, CPT>::store(out + i * ostride, H);
            }
        } else {
            for (int i = 0; i < n; ++i) {
                float a[CPT], b[CPT];
                Vec<IO, CPT>::load(p0 + i * CG, a);
                Vec<IO, CPT>::load(p1 + i * CG, b);
#pragma unroll
                for (int j = 0; j < CPT; ++j) H[j] = fmaf(a[j], H[j], b[j]);
                if (valid) Vec<IO, CPT>::store(out + i * ostride, H);
            }
        }
    }
};

// fp32 I/O, one channel per thread; bf16 I/O, two (128-byte tile rows either way)
using ScanOp = ScanOpT<float, 1>;
using ScanOpBf16 = ScanOpT<__nv_bfloat16, 2>;

}  // namespace wkvb
