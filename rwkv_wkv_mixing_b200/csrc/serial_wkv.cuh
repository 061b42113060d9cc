// WKV for short sequences and single-token decoding: each thread owns VW
// consecutive channels of one batch row and walks the steps in order with
// the RNN-mode state update (RWKV evolution article, section RWKV-V4;
// sequential decoding, section 三 of "RWKV：基于RNN的LLM").  Each step reads
// k_t, v_t, writes y_t and keeps the states (a, b, p) in registers; they come
// from s_in (or are empty) and go to s_out.
//
// With a handful of steps there is nothing to parallelise over time: the
// chunked kernels' tiles, look-back and workspace would only add latency.
// The work is a pure stream -- per channel and step 2 loads (3 with the
// receptance gate) and 1 store, plus 3 state words in and out -- so the
// kernel is built for bytes in flight: VW = 4 channels per thread turns every
// access into one 16-byte
// (fp32) or 8-byte (bf16) vector access, and consecutive threads own
// consecutive channel groups, so each warp access is one contiguous run.
// The per-step update is the max-stabilised one the chunked kernels use for
// hard inputs, exact for any finite input.
#pragma once

#include <cuda_bf16.h>

#include "wkv_ops.cuh"

namespace wkvb {

constexpr int kSerialThreads = 256;

// Any WkvOp instantiation: only its per-channel functions are used.  VW = 4
// needs C % 4 == 0, k / v / y aligned to 4 elements and s_in / s_out to 16
// bytes; VW = 1 takes anything.
template <class Op, int VW>
__global__ void __launch_bounds__(kSerialThreads)
    wkv_serial_kernel(const typename Op::Args args, int B, int T, int C) {
    using IO = typename Op::io_t;
    const int groups = C / VW;
    const long long i = static_cast<long long>(blockIdx.x) * kSerialThreads + threadIdx.x;
    if (i >= static_cast<long long>(B) * groups) return;
    const int b = static_cast<int>(i / groups);
    const int c0 = static_cast<int>(i - static_cast<long long>(b) * groups) * VW;

    typename Op::Param q[VW];
    typename Op::State s[VW];
#pragma unroll
    for (int j = 0; j < VW; ++j) q[j] = Op::param(args, c0 + j, C);
    const size_t sbase = static_cast<size_t>(b) * 3 * C + c0;
    if (args.s_in != nullptr) {
        float a[VW], bb[VW], p[VW];
        Vec<float, VW>::load(args.s_in + sbase, a);
        Vec<float, VW>::load(args.s_in + sbase + C, bb);
        Vec<float, VW>::load(args.s_in + sbase + 2 * static_cast<size_t>(C), p);
#pragma unroll
        for (int j = 0; j < VW; ++j) s[j] = Op::state_in(a[j], bb[j], p[j]);
    } else {
#pragma unroll
        for (int j = 0; j < VW; ++j) s[j] = Op::identity();
    }

    const size_t base = static_cast<size_t>(b) * T * C + c0;
    for (int t = 0; t < T; ++t) {
        const size_t o = base + static_cast<size_t>(t) * C;
        float k[VW], v[VW], y[VW];
        Vec<IO, VW>::load(args.x0 + o, k);
        Vec<IO, VW>::load(args.x1 + o, v);
#pragma unroll
        for (int j = 0; j < VW; ++j) y[j] = Op::step_exact(s[j], k[j], v[j], q[j]);
        if constexpr (Op::kGated) {  // sigma(r) (.) wkv
            float r[VW];
            Vec<IO, VW>::load(args.x2 + o, r);
#pragma unroll
            for (int j = 0; j < VW; ++j) y[j] *= gate_sigmoid(r[j]);
        }
        Vec<IO, VW>::store(args.y + o, y);
    }

    if (args.s_out != nullptr) {
        float a[VW], bb[VW], p[VW];
#pragma unroll
        for (int j = 0; j < VW; ++j) {
            a[j] = s[j].a;
            bb[j] = s[j].b;
            p[j] = s[j].p;
        }
        Vec<float, VW>::store(args.s_out + sbase, a);
        Vec<float, VW>::store(args.s_out + sbase + C, bb);
        Vec<float, VW>::store(args.s_out + sbase + 2 * static_cast<size_t>(C), p);
    }
}

}  // namespace wkvb
