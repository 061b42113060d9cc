// Token shift: the interpolation between each token and the one before it
// that feeds the time-mixing projections, eqs. (11)-(13) of "RWKV：基于RNN的LLM"
// (section 二.1):
//
//     out[m, b, t, c] = mu[m, c] * x[b, t, c] + (1 - mu[m, c]) * x[b, t-1, c]
//
// for NMIX mixing vectors at once (k, v, r of the time-mixing block; k, r of
// channel mixing), with x[b, -1] = x_prev[b] (the last token of the previous
// call, the layer's saved "last_x") or 0.  The last token x[b, T-1] goes to
// x_last for the next call.
//
// Pure streaming: each thread owns VW consecutive channels of one batch row
// over a chunk of kChunk steps, keeps x_{t-1} in registers, so x is read from
// HBM once (plus one halo step per chunk) and each output once.  Consecutive
// threads own consecutive channel groups: every warp access is one
// contiguous run of 16-byte (fp32) or 8-byte (bf16) vectors.
#pragma once

#include <cuda_bf16.h>

#include "wkv_ops.cuh"

namespace wkvb {

constexpr int kShiftThreads = 256;
constexpr int kShiftChunk = 16;  // steps per thread

template <typename IO, int VW, int NMIX>
__global__ void __launch_bounds__(kShiftThreads)
    token_shift_kernel(const IO *__restrict__ x, const IO *x_prev, const float *__restrict__ mu,
                       IO *__restrict__ out, IO *x_last, int B, int T, int C) {
    const int groups = C / VW;
    const int chunks = (T + kShiftChunk - 1) / kShiftChunk;
    const long long i = static_cast<long long>(blockIdx.x) * kShiftThreads + threadIdx.x;
    if (i >= static_cast<long long>(B) * chunks * groups) return;
    const int cg = static_cast<int>(i % groups);
    const long long rest = i / groups;
    const int chunk = static_cast<int>(rest % chunks);
    const int b = static_cast<int>(rest / chunks);
    const int c0 = cg * VW;
    const int t0 = chunk * kShiftChunk;
    const int t1 = min(T, t0 + kShiftChunk);
    const size_t row = static_cast<size_t>(b) * T * C + c0;   // x[b, 0, c0]
    const size_t plane = static_cast<size_t>(B) * T * C;      // one output tensor

    float m[NMIX][VW], m1[NMIX][VW];
#pragma unroll
    for (int q = 0; q < NMIX; ++q) {
        Vec<float, VW>::load(mu + static_cast<size_t>(q) * C + c0, m[q]);
#pragma unroll
        for (int j = 0; j < VW; ++j) m1[q][j] = 1.f - m[q][j];
    }

    float prev[VW];
    if (t0 > 0) {
        Vec<IO, VW>::load(x + row + static_cast<size_t>(t0 - 1) * C, prev);
    } else if (x_prev != nullptr) {
        Vec<IO, VW>::load(x_prev + static_cast<size_t>(b) * C + c0, prev);
    } else {
#pragma unroll
        for (int j = 0; j < VW; ++j) prev[j] = 0.f;
    }
    if (chunk == 0 && x_last != nullptr) {
        // the thread that read x_prev writes x_last, after that read: the two
        // may be one buffer
        float last[VW];
        Vec<IO, VW>::load(x + row + static_cast<size_t>(T - 1) * C, last);
        Vec<IO, VW>::store(x_last + static_cast<size_t>(b) * C + c0, last);
    }

#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        float cur[VW];
        const size_t o = row + static_cast<size_t>(t) * C;
        Vec<IO, VW>::load(x + o, cur);
#pragma unroll
        for (int q = 0; q < NMIX; ++q) {
            float y[VW];
            // mu x_t + (1 - mu) x_{t-1}: mu = 1 and mu = 0 give x_t and x_{t-1}
            // exactly
#pragma unroll
            for (int j = 0; j < VW; ++j) y[j] = fmaf(m[q][j], cur[j], m1[q][j] * prev[j]);
            Vec<IO, VW>::store(out + q * plane + o, y);
        }
#pragma unroll
        for (int j = 0; j < VW; ++j) prev[j] = cur[j];
    }
}

}  // namespace wkvb
