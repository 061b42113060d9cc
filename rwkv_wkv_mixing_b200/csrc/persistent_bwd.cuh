// WKV gradients on persistent, TMA-fed kernels for sm_100a (shapes a tensor
// map can describe; any other shape takes the per-segment kernels of
// wkv_backward.cuh, whose header states the gradient formulas used here).
//
// Time is cut into segments of 32 steps.  One gradient step is four launches
// over two passes of k, v and gy:
//  1. wkv_bwd_states_kernel: 128-step x 32-channel tiles, in time order per
//     chain, the forward state carried between tiles by the decoupled
//     look-back of the forward kernel (the same record and combine).  Each
//     compute warp owns one 32-step segment of a tile: it writes the forward
//     state before its segment, computes y_t and ln D_t of the segment from
//     it, and writes the segment's reverse summary (the sums over its own
//     outputs, from the zero state).  k and v come through the ring of
//     stages; a group's gy tile, needed only in pass 2, is loaded by TMA into
//     the group's own buffer when the group starts the tile, so a stage goes
//     back after pass 1 and four of them fit.  k, v and gy are read once.
//  2. wkv_bwd_rev_carry_kernel (wkv_backward.cuh), backwards over segments:
//     the reverse state after each segment.
//  3. wkv_bwd_grads_tiles_kernel: every 32-step x 32-channel tile on its own,
//     its two carries read from the scratch: y_t, ln D_t again from the
//     forward state, then the reverse pass from the reverse state; gk and gv
//     are written over the staged k and v and leave by TMA stores, the gw and
//     gu of the segment go to the scratch.  k, v, gy are read a second time,
//     gk and gv written once.
//  4. wkv_bwd_reduce_one_kernel, or for more than 1024 rows x segments
//     wkv_bwd_reduce_kernel (wkv_backward.cuh): gw, gu added in a fixed order.
// HBM traffic per element: 32 bytes of k, v, gy, gk, gv, plus 1.25 bytes of
// segment states (8 floats written, 8 read, 5 read and written by the
// reverse scan, 2 partials, per 32 steps).
//
// The chunk identity behind the carries is the Upper/Lower split of a linear
// recurrence (review of "Resurrecting Recurrent Neural Networks for Long
// Sequences", parallelisation section); the operator is eq. (14) of
// "RWKV：基于RNN的LLM" (section 二.1).  Every wait is bounded, as in the
// forward kernels: a wait that gives up records WKV_ERR_TIMEOUT in the status
// word, leaves NaN in what depends on it and lets the launch finish.
#pragma once

#include <cstdint>

#include "persistent_wkv.cuh"
#include "wkv_backward.cuh"

namespace wkvb {

constexpr int kBwdSegSteps = 32;  // steps per segment: one compute warp's share of a tile

// 1: a gradients warp hands a stage back after its next tile's stores are
// issued; 0: it waits for its stores to read the stage at once (measured
// faster: 62 against 67 us a gradient step on B=8 T=1024 C=768 -- a warp
// holding two stages of the in-order ring stalls the producer)
#ifndef WKV_BWD_DEFER_RELEASE
#define WKV_BWD_DEFER_RELEASE 0
#endif

struct BwdTileArgs {
    const float *w, *u;       // [C]
    const float *k, *v;       // [B, T, C] (read back by the rare exact sweep)
    float *fwd;               // [B, S, 3, C] forward state before each segment
    float *rev;               // [B, S, 5, C] reverse summary of each segment, then
                              // (after the reverse scan) the state after it
    float *partial;           // [B, S, 2, C] gw, gu of each segment
    int S;                    // segments per row, ceil(T / kBwdSegSteps)
};

// ---------------------------------------------------------------------------
// 1. forward states and reverse summaries
// ---------------------------------------------------------------------------
template <int LT, int NWG, int NC, int NSTAGE>
struct BwdStatesCfg {
    static constexpr int kLT = LT;
    static constexpr int CG = 32, LS = LT / NWG;
    static constexpr int NGW = NWG + 1;  // warps per group: NWG compute, 1 carry
    static constexpr int kThreads = (1 + NC * NGW) * 32;
    static constexpr size_t kTileElems = static_cast<size_t>(LT) * CG;
    // a stage: the k and v tiles, then the tile's u and w ([CG] fp32 each)
    static constexpr size_t kParamOffset = 2 * kTileElems * sizeof(float);
    static constexpr size_t kStageBytes = kParamOffset + 2 * CG * sizeof(float);
    static constexpr int kHops = WKV_REG_LOOKBACK_HOPS;
    // per group: the gy tile (loaded by TMA when the group starts a tile,
    // read in pass 2), then two slots (double-buffered) of the compute warps' summaries
    // [NWG][3][CG], of the carry [3][CG] and of the tile aggregate [3][CG]
    static constexpr size_t kGyBytes = kTileElems * sizeof(float);
    static constexpr size_t kSumFloats = static_cast<size_t>(NWG) * 3 * CG;
    static constexpr size_t kCarryFloats = static_cast<size_t>(3) * CG;
    static constexpr size_t kGroupBytes =
        kGyBytes + 2 * (kSumFloats + 2 * kCarryFloats) * sizeof(float);
    static constexpr size_t kSmemBytes = NSTAGE * kStageBytes + NC * kGroupBytes;
    // named barriers per group: tile assigned, carries written, aggregate
    // written; plus one for all consumers at the start
    static constexpr int kBarsPerGroup = 3;
    static_assert(LS == kBwdSegSteps, "a compute warp's sub-chunk is one segment");
    static_assert(LT % NWG == 0 && LT <= 256, "tile length");
    static_assert(NSTAGE >= 2, "at least one stage being read while one loads");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
    static_assert(kStageBytes % 128 == 0 && kParamOffset % 16 == 0 && kGyBytes % 128 == 0,
                  "stage alignment");
    static_assert(2 + kBarsPerGroup * NC <= 16, "named barrier ids: 0, per group, one for all");
};

// The reverse sums over a segment's own outputs can run at the forward
// pass's fixed reference M: with D_t = den_t e^M, each output enters them as
// g_t e^{-L_t} = g_t r_t e^{-M}, r_t = 1 / den_t, so sums kept in units of
// e^{-M} need no exponential at all.  Safe when every den_t >= e^-30 (the
// forward bound at that floor): then r_t <= e^30 and no sum of a segment's
// terms can overflow for |g|, |v| below 1e15.
constexpr float kRevFixedFloor = -30.f;

// y_t of the segment from the state before it, in place of the weights in R
// (R.e[i] <- y_i).  Returns true when the segment takes the fixed reference
// M = max(p_in, max k) of the forward kernel's pass 2 with every denominator
// above e^-30: then R.v[i] <- r_i = 1 / den_i.  Otherwise R.v[i] <- ln D_i:
// at the same reference when the forward kernel's own bound (e^-69) holds,
// else from the per-step max-stabilised form, keys and values read back from
// global memory (batch row b, rows t.., channel c; zeros when the channel
// does not exist).
template <int LS, bool FULL>
__device__ __forceinline__ bool rows_forward_outputs(LaneRows<LS> &R,
                                                     const WkvOp<float, 1>::State &cin, int n,
                                                     const WkvOp<float, 1>::Param &q,
                                                     const BwdTileArgs &a, const Geometry &g,
                                                     int b, int t, int c, float &M) {
    M = fmaxf(cin.p, R.kmax);
    if (sweep_is_safe(R.kmin, M, cin, q, n)) {
        const bool rev_fixed = sweep_is_safe(R.kmin, M, cin, q, n, kRevFixedFloor);
        const float s = fast_exp(R.kmax - M), f = fast_exp(cin.p - M);
        float A = cin.a * f, Bs = cin.b * f;
        if (rev_fixed) {
#pragma unroll
            for (int i = 0; i < LS; ++i)
                if (FULL || i < n) {
                    const float e = R.e[i] * s, v = R.v[i];
                    const float r = rcp_approx(fmaf(e, q.U, Bs));
                    R.e[i] = v + fmaf(-Bs, v, A) * r;
                    R.v[i] = r;
                    A = fmaf(A, q.D, e * v);
                    Bs = fmaf(Bs, q.D, e);
                }
        } else {
#pragma unroll
            for (int i = 0; i < LS; ++i)
                if (FULL || i < n) {
                    const float e = R.e[i] * s, v = R.v[i];
                    const float den = fmaf(e, q.U, Bs);
                    R.e[i] = v + fmaf(-Bs, v, A) * rcp_approx(den);
                    R.v[i] = M + __logf(den);
                    A = fmaf(A, q.D, e * v);
                    Bs = fmaf(Bs, q.D, e);
                }
        }
        return rev_fixed;
    }
    // the rare path: keys and values of rows t.. of batch row b, channel c
    const size_t C = static_cast<size_t>(g.C);
    const bool cvalid = c < g.C;
    const size_t row0 = (static_cast<size_t>(b) * g.T + t) * C + (cvalid ? c : 0);
    const float *kp = a.k + row0, *vp = a.v + row0;
    FwdState st{cin.a, cin.b, cin.p};
#pragma unroll
    for (int i = 0; i < LS; ++i)
        if (FULL || i < n) {
            const float k = cvalid ? kp[i * C] : 0.f, v = cvalid ? vp[i * C] : 0.f;
            const Pair f = max_pair(st.p, q.u + k);
            const float den = fmaf(f.fx, st.d, f.fy);  // in [1, T + 1]
            R.e[i] = fmaf(f.fx, st.a, f.fy * v) * __fdividef(1.f, den);
            R.v[i] = f.q + __logf(den);
            fwd_step(st, k, v, q.w);
        }
    return false;
}

// The segment's reverse summary from the zero state: R holds y_t and, at the
// fixed reference M, r_t (the sums come out in units of e^{-M}: rho = M);
// otherwise ln D_t, and the per-step min-stabilised steps.  gp[i * 32]: the
// upstream gradient g_t.
template <int LS, bool FULL>
__device__ __forceinline__ RevState rows_reverse_summary(const LaneRows<LS> &R, const float *gp,
                                                         int n, const WkvOp<float, 1>::Param &q,
                                                         bool fixed, float M) {
    if (fixed) {
        float P = 0.f, Q = 0.f, Rs = 0.f, R2 = 0.f;
#pragma unroll
        for (int i = LS - 1; i >= 0; --i)
            if (FULL || i < n) {
                const float gr = gp[i * 32] * R.v[i];
                Rs = q.D * (Rs + P);
                R2 = q.D * (R2 + Q);
                P = fmaf(q.D, P, gr);
                Q = fmaf(q.D, Q, gr * R.e[i]);
            }
        return {P, Q, Rs, R2, M};
    }
    RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
#pragma unroll
    for (int i = LS - 1; i >= 0; --i)
        if (FULL || i < n) rev_step(z, gp[i * 32], R.e[i], R.v[i], q.w);
    return z;
}

template <int LT, int NWG, int NC, int NSTAGE>
__global__ void __launch_bounds__(BwdStatesCfg<LT, NWG, NC, NSTAGE>::kThreads, 1)
    wkv_bwd_states_kernel(const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v,
                          const __grid_constant__ CUtensorMap map_gy, const BwdTileArgs a,
                          const Geometry g, const Workspace ws) {
    using Cfg = BwdStatesCfg<LT, NWG, NC, NSTAGE>;
    using Op = WkvOp<float, 1, false>;
    using State = Op::State;
    using Param = Op::Param;
    constexpr int CG = Cfg::CG, LS = Cfg::LS, NV = 3, NGW = Cfg::NGW;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *s_stage = smem;  // [NSTAGE] x (k, v tiles, u[CG], w[CG])
    unsigned char *s_groups = smem + NSTAGE * Cfg::kStageBytes;  // [NC] x kGroupBytes
    __shared__ __align__(8) uint64_t full_bar[NSTAGE];
    __shared__ __align__(8) uint64_t empty_bar[NSTAGE];
    // per group and slot: the compute warps have read the slot's carries
    __shared__ __align__(8) uint64_t free_bar[NC][2];
    // per group: its gy tile has landed (phase i: the group's i-th tile)
    __shared__ __align__(8) uint64_t gy_bar[NC];
    __shared__ int s_gy_loads[NC];     // gy tiles each group has asked for
    __shared__ int s_meta[NSTAGE];     // tile id per stage, -1 = no more tiles
    __shared__ int s_fill_it[NSTAGE];  // ring iteration the stage was last filled for
    __shared__ int s_last_it[NSTAGE];  // last ring iteration loaded into each stage
    __shared__ int s_tile[NC][2];      // each group's tile per slot (-1 none left, -2 abort)
    __shared__ int s_it[NC][2];        // ... and its ring iteration
    __shared__ int s_count[NC][2];     // compute warps of the group that have summarised
    __shared__ int s_next_it;          // next ring iteration a group may take
    __shared__ unsigned long long s_epoch;
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool chained = g.n_seg > 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
            s_last_it[s] = -1;
            s_fill_it[s] = -1;
        }
        for (int q = 0; q < NC; ++q) {
            for (int k = 0; k < 2; ++k) {
                mbar_init(&free_bar[q][k], NWG);
                s_count[q][k] = 0;
            }
            mbar_init(&gy_bar[q], 1);
            s_gy_loads[q] = 0;
        }
        fence_mbar_init();
        s_abort = 0;
        s_next_it = 0;
    }
    // nothing global is read before the previous grid in the stream is done
    grid_dependency_wait();
    __syncthreads();
    volatile int *abort_flag = &s_abort;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&map_k);
            prefetch_tensormap(&map_v);
            prefetch_tensormap(&map_gy);
            int sentinels = 0;
            int next_static = static_cast<int>(blockIdx.x);
            for (int it = 0; sentinels < NC; ++it) {
                const int s = it % NSTAGE;
                if (!wait_phase(&empty_bar[s], ((it / NSTAGE) & 1) ^ 1, abort_flag, ws)) break;
                int tile = -1;
                if (sentinels == 0) {
                    if (chained) {
                        // tickets in the order blocks ask for them: a tile only
                        // ever waits for tiles already being worked on
                        const unsigned t = atomicAdd(ws.ticket, 1u);
                        tile = t < static_cast<unsigned>(g.tiles) ? static_cast<int>(t) : -1;
                    } else {
                        tile = next_static < g.tiles ? next_static : -1;
                        next_static += static_cast<int>(gridDim.x);
                    }
                }
                s_meta[s] = tile;
                *static_cast<volatile int *>(&s_fill_it[s]) = it;
                if (tile < 0) {
                    ++sentinels;
                    mbar_arrive(&full_bar[s]);
                } else {
                    const int seg = tile / g.tiles_per_seg;
                    const int rem = tile - seg * g.tiles_per_seg;
                    const int b = rem / g.n_cg;
                    const int c0 = (rem - b * g.n_cg) * CG;
                    unsigned char *dst = s_stage + static_cast<size_t>(s) * Cfg::kStageBytes;
                    const uint32_t pbytes =
                        static_cast<uint32_t>(min(CG, g.C - c0)) * static_cast<uint32_t>(sizeof(float));
                    s_last_it[s] = it;
                    mbar_arrive_expect_tx(&full_bar[s],
                                          static_cast<uint32_t>(Cfg::kParamOffset) + 2 * pbytes);
                    tma_load_3d(dst, &map_k, &full_bar[s], c0, seg * LT, b);
                    tma_load_3d(dst + Cfg::kTileElems * sizeof(float), &map_v, &full_bar[s], c0,
                                seg * LT, b);
                    float *dp = reinterpret_cast<float *>(dst + Cfg::kParamOffset);
                    bulk_load(dp, a.u + c0, pbytes, &full_bar[s]);
                    bulk_load(dp + CG, a.w + c0, pbytes, &full_bar[s]);
                }
            }
            // every tile of this block is loaded or assigned: the next grid in
            // the stream may start launching its blocks (its own
            // griddepcontrol.wait still waits for this grid to complete)
            allow_dependent_launch();
        }
        __syncwarp();
    } else {
        // ---------------- groups ----------------
        if (threadIdx.x == 32) s_epoch = chained ? epoch_of(ws) : 0ull;
        named_bar_sync(1 + Cfg::kBarsPerGroup * NC, NC * NGW * 32);
        const unsigned long long epoch = s_epoch;
        const int cw = warp - 1;
        const int grp = cw / NGW, wg = cw - grp * NGW;
        const int bar_tile = 1 + Cfg::kBarsPerGroup * grp, bar_carry = bar_tile + 1,
                  bar_agg = bar_tile + 2;
        unsigned char *gbase = s_groups + static_cast<size_t>(grp) * Cfg::kGroupBytes;
        float *g_gy = reinterpret_cast<float *>(gbase);
        float *g_sum0 = g_gy + Cfg::kTileElems;            // [2][NWG][NV][CG]
        float *g_carry0 = g_sum0 + 2 * Cfg::kSumFloats;    // [2][NV][CG]
        float *g_agg0 = g_carry0 + 2 * Cfg::kCarryFloats;  // [2][NV][CG]

        if (wg == NWG) {
            // ---------------- carry warp ----------------
            bool aborted = false;
            for (int i = 0;; ++i) {
                const int k = i & 1;
                const uint32_t ph = (i >> 1) & 1;
                float *g_carry = g_carry0 + k * Cfg::kCarryFloats;
                const float *g_agg = g_agg0 + k * Cfg::kCarryFloats;
                const bool ok = !aborted && warp_wait_phase(&free_bar[grp][k], ph ^ 1, abort_flag, ws);
                if (lane == 0) {
                    int tile = -2, it = 0;
                    if (ok) {
                        it = atomicAdd(&s_next_it, 1);
                        const int s = it % NSTAGE;
                        tile = wait_fill(&full_bar[s], &s_fill_it[s], it, (it / NSTAGE) & 1, abort_flag,
                                         ws)
                                   ? s_meta[s]
                                   : -2;
                    }
                    s_tile[grp][k] = tile;
                    s_it[grp][k] = it;
                }
                __syncwarp();
                const int tile = *static_cast<volatile int *>(&s_tile[grp][k]);
                if (tile < 0) {
                    named_bar_arrive(bar_tile, (NWG + 1) * 32);  // the compute warps leave
                    break;
                }
                const int it = s_it[grp][k];
                const int s = it % NSTAGE;
                for (int n = 0; n < (1 << 20) && !mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1); ++n) {
                }
                const int seg = tile / g.tiles_per_seg;
                const int rem = tile - seg * g.tiles_per_seg;
                const int b = rem / g.n_cg;
                const int c = (rem - b * g.n_cg) * CG + lane;
                const Param prm = staged_param(
                    reinterpret_cast<const float *>(s_stage + static_cast<size_t>(s) * Cfg::kStageBytes +
                                                    Cfg::kParamOffset),
                    lane, c, g.C);
                (void)b;
                __syncwarp();
                named_bar_arrive(bar_tile, (NWG + 1) * 32);  // the compute warps start

                // the state before the tile: empty for the first segment, else
                // the decoupled look-back over the tiles before it
                const bool last = seg == g.n_seg - 1;
                State X = Op::identity();
                if (chained && seg > 0 &&
                    !lookback_channel<Op, LT, 1, Cfg::kHops>(ws, g, tile, epoch, prm, lane, 0, X,
                                                             static_cast<const ChannelPrefetch<1> *>(
                                                                 nullptr))) {
                    atomicExch(ws.status, kStatusTimeout);  // this lane gave up
                    X = Op::nan_state();
                }
                named_bar_sync(bar_agg, 64);  // with the folding warp's arrival
                if (chained && !last) {
                    float vals[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) vals[q] = g_agg[q * CG + lane];
                    publish_channel<Op, CG>(ws, g, tile,
                                            Op::combine(X, Op::make(vals), static_cast<float>(LT), prm),
                                            0, kFlagIncl, epoch, lane);
                }
#pragma unroll
                for (int q = 0; q < NV; ++q) g_carry[q * CG + lane] = Op::get(X, q);
                __syncwarp();
                named_bar_arrive(bar_carry, (NWG + 1) * 32);  // the compute warps go on
            }
        } else {
            // ---------------- compute warps ----------------
            for (int i = 0;; ++i) {
                const int k = i & 1;
                float *g_sum = g_sum0 + k * Cfg::kSumFloats;
                const float *g_carry = g_carry0 + k * Cfg::kCarryFloats;
                named_bar_sync(bar_tile, (NWG + 1) * 32);
                const int tile = *static_cast<volatile int *>(&s_tile[grp][k]);
                if (tile < 0) break;
                const int it = s_it[grp][k];
                const int s = it % NSTAGE;
                for (int n = 0; n < (1 << 20) && !mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1); ++n) {
                }
                const int seg = tile / g.tiles_per_seg;
                const int rem = tile - seg * g.tiles_per_seg;
                const int b = rem / g.n_cg;
                const int t0 = seg * LT;
                const int c = (rem - b * g.n_cg) * CG + lane;
                const unsigned char *st_base = s_stage + static_cast<size_t>(s) * Cfg::kStageBytes;
                const float *s_k = reinterpret_cast<const float *>(st_base);
                const float *s_v = s_k + Cfg::kTileElems;
                const Param prm = staged_param(
                    reinterpret_cast<const float *>(st_base + Cfg::kParamOffset), lane, c, g.C);
                // the tile's gy into the group's buffer, landing during pass 1
                // and the carry: every compute warp of the group is past pass
                // 2 of the previous tile here (the barrier above), so nothing
                // reads the buffer any more
                if (wg == 0 && lane == 0) {
                    fence_proxy_async_smem();  // those reads before the async-proxy write
                    s_gy_loads[grp] = i + 1;
                    mbar_arrive_expect_tx(&gy_bar[grp], static_cast<uint32_t>(Cfg::kGyBytes));
                    tma_load_3d(g_gy, &map_gy, &gy_bar[grp], c - lane, t0, b);
                }

                // pass 1: the segment into registers, weights and summary
                const int s0 = wg * LS;
                const int nval = max(0, min(LS, g.T - (t0 + s0)));
                LaneRows<LS> R;
                {
                    const float *pk = s_k + s0 * CG + lane, *pv = s_v + s0 * CG + lane;
                    State st = Op::identity();
                    if (nval == LS)
                        rows_pass1<LS, true>(pk, pv, nval, prm, R, st);
                    else if (nval > 0)
                        rows_pass1<LS, false>(pk, pv, nval, prm, R, st);
#pragma unroll
                    for (int q = 0; q < NV; ++q) g_sum[(wg * NV + q) * CG + lane] = Op::get(st, q);
                }
                // the warp that summarises last folds the group's summaries
                __syncwarp();
                int order = 0;
                if (lane == 0) {
                    __threadfence_block();
                    order = atomicAdd(&s_count[grp][k], 1);
                }
                order = __shfl_sync(0xffffffffu, order, 0);
                if (order == NWG - 1) {
                    __syncwarp();
                    __threadfence_block();  // every warp's summary (written before its count)
                    float *g_agg = g_agg0 + k * Cfg::kCarryFloats;
                    State acc = Op::identity();
                    for (int w = 0; w < NWG; ++w) {
                        float vals[NV];
                        float *slot = g_sum + w * NV * CG + lane;
#pragma unroll
                        for (int q = 0; q < NV; ++q) vals[q] = slot[q * CG];
#pragma unroll
                        for (int q = 0; q < NV; ++q) slot[q * CG] = Op::get(acc, q);
                        const int len = max(0, min(LS, g.T - (t0 + w * LS)));
                        acc = Op::combine(acc, Op::make(vals), static_cast<float>(len), prm);
                    }
                    if (chained && seg > 0 && seg < g.n_seg - 1)
                        publish_channel<Op, CG>(ws, g, tile, acc, 0, kFlagAgg, epoch, lane);
#pragma unroll
                    for (int q = 0; q < NV; ++q) g_agg[q * CG + lane] = Op::get(acc, q);
                    __syncwarp();
                    if (lane == 0) {
                        s_count[grp][k] = 0;
                        mbar_arrive(&empty_bar[s]);  // every compute warp is done with the stage
                    }
                    named_bar_arrive(bar_agg, 64);   // the carry warp may finish the carry
                }

                // the state before this warp's segment
                named_bar_sync(bar_carry, (NWG + 1) * 32);
                State cur;
                {
                    float vals[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) vals[q] = g_carry[q * CG + lane];
                    cur = Op::make(vals);
                    if (wg > 0) {  // the segments before this warp's, all full
#pragma unroll
                        for (int q = 0; q < NV; ++q) vals[q] = g_sum[(wg * NV + q) * CG + lane];
                        cur = Op::combine(cur, Op::make(vals), static_cast<float>(wg * LS), prm);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_bar[grp][k]);  // the slot may be reused

                // pass 2: the forward state before the segment, y_t and ln D_t,
                // and the segment's reverse summary, to the scratch (gy from
                // the group's buffer once it has landed)
                if (!warp_wait_phase(&gy_bar[grp], static_cast<uint32_t>(i & 1), abort_flag, ws))
                    continue;  // the block is giving up: the next barrier sends the warps home
                if (nval > 0) {
                    // segment (b, (t0 + s0) / LS) of the scratch
                    const int segi = b * a.S + (t0 + s0) / LS;
                    if (c < g.C) {
                        const size_t C = static_cast<size_t>(g.C);
                        float *f = a.fwd + static_cast<size_t>(segi) * 3 * C + c;
                        f[0] = cur.a;
                        f[C] = cur.b;
                        f[2 * C] = cur.p;
                    }
                    const float *pg = g_gy + s0 * CG + lane;
                    RevState z;
                    float M;
                    if (nval == LS) {
                        const bool fx = rows_forward_outputs<LS, true>(R, cur, nval, prm, a, g, b,
                                                                       t0 + s0, c, M);
                        z = rows_reverse_summary<LS, true>(R, pg, nval, prm, fx, M);
                    } else {
                        const bool fx = rows_forward_outputs<LS, false>(R, cur, nval, prm, a, g, b,
                                                                        t0 + s0, c, M);
                        z = rows_reverse_summary<LS, false>(R, pg, nval, prm, fx, M);
                    }
                    if (c < g.C) store_rev(a.rev + static_cast<size_t>(segi) * 5 * g.C + c, g.C, z);
                }
            }
        }
        __syncwarp();
    }

    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        // an aborted block must not exit with tile loads still landing in its
        // shared memory: wait (bounded) for the last load of every stage and
        // every group's last gy tile
        for (int s = 0; s < NSTAGE; ++s) {
            const int it = s_last_it[s];
            if (it < 0) continue;
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1)) {
                if (global_timer_ns() - t0 > kBarrierWaitNs) break;
            }
        }
        for (int q = 0; q < NC; ++q) {
            const int n = s_gy_loads[q];
            if (n == 0) continue;
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&gy_bar[q], static_cast<uint32_t>((n - 1) & 1))) {
                if (global_timer_ns() - t0 > kBarrierWaitNs) break;
            }
        }
    }
    allow_dependent_launch();
    finish_launch(ws, chained, static_cast<int>(threadIdx.x), gridDim.x);
}

// ---------------------------------------------------------------------------
// 3. gradients, one 32-step x 32-channel tile per compute warp
// ---------------------------------------------------------------------------
template <int NCW, int NSTAGE>
struct BwdGradsCfg {
    static constexpr int CG = 32, LT = kBwdSegSteps;
    static constexpr int kThreads = (1 + NCW) * 32;
    static constexpr size_t kTileElems = static_cast<size_t>(LT) * CG;
    static constexpr size_t kTileBytes = kTileElems * sizeof(float);
    static constexpr size_t kStageBytes = 3 * kTileBytes;  // k, v, gy
    static constexpr size_t kSmemBytes = NSTAGE * kStageBytes;
    static_assert(NSTAGE > NCW, "one stage per compute warp plus at least one being loaded");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
    static_assert(kStageBytes % 128 == 0, "stage alignment");
};

// Per-step values of one lane's tile for the reverse pass, in registers:
// at the fixed reference M, E = e^{k_t - M}, X = r_t = 1 / den_t and Y = y_t;
// otherwise E = beta_{t,t}, X = ln D_t and Y = y_t.
// WKV_BWD_KEEP_E 0: E is not held; the reverse pass evaluates it again from
// the staged key (one more exponential a step, 32 fewer registers: eleven
// compute warps without spills, as fast as seven holding it)
#ifndef WKV_BWD_KEEP_E
#define WKV_BWD_KEEP_E 0
#endif
template <int LT>
struct TileRows {
#if WKV_BWD_KEEP_E
    float E[LT];
#endif
    float X[LT], Y[LT];
};

// The forward pass over the tile's n steps from the state before it (sk, sv:
// this lane's column of the staged k and v) and the state after it, z.  A
// full tile whose forward kernel bound holds takes the fixed reference
// M = max(p_in, max k); it returns true, with E, X, Y at M, when every
// denominator is also above e^-30 and z's scale e^{M - rho} below e^30 (the
// reverse pass then runs at M too).  Every other tile ends in the per-step
// form's values and returns false.
template <int LT, bool FULL>
__device__ __forceinline__ bool grads_forward(const float *sk, const float *sv, int n,
                                              const FwdState &cin, const RevState &z,
                                              const WkvOp<float, 1>::Param &q, TileRows<LT> &R,
                                              float &M) {
    constexpr int CG = 32;
    M = 0.f;
    if constexpr (FULL) {
        float kx = kNoScale, kn = -kNoScale;
#pragma unroll
        for (int i = 0; i < LT; ++i) {
            const float k = sk[i * CG];
            kx = fmaxf(kx, k);
            kn = fminf(kn, k);
        }
        const WkvOp<float, 1>::State cs{cin.a, cin.d, cin.p};
        M = fmaxf(cin.p, kx);
        if (sweep_is_safe(kn, M, cs, q, n)) {
            const bool rev_fixed =
                sweep_is_safe(kn, M, cs, q, n, kRevFixedFloor) && M - z.rho <= 30.f;
            const float f = fast_exp(cin.p - M);
            float A = cin.a * f, Bs = cin.d * f;
            if (rev_fixed) {
#pragma unroll
                for (int i = 0; i < LT; ++i) {
                    const float k = sk[i * CG], v = sv[i * CG];
                    const float e = ex2_approx((k - M) * kLog2e);
                    const float r = rcp_approx(fmaf(e, q.U, Bs));
#if WKV_BWD_KEEP_E
                    R.E[i] = e;
#endif
                    R.X[i] = r;
                    R.Y[i] = v + fmaf(-Bs, v, A) * r;
                    A = fmaf(A, q.D, e * v);
                    Bs = fmaf(Bs, q.D, e);
                }
            } else {
#pragma unroll
                for (int i = 0; i < LT; ++i) {
                    const float k = sk[i * CG], v = sv[i * CG];
                    const float e = ex2_approx((k - M) * kLog2e);
                    const float den = fmaf(e, q.U, Bs);
                    const float r = rcp_approx(den);
#if WKV_BWD_KEEP_E
                    R.E[i] = q.U * e * r;  // beta_{t,t}
#endif
                    R.X[i] = M + __logf(den);
                    R.Y[i] = v + fmaf(-Bs, v, A) * r;
                    A = fmaf(A, q.D, e * v);
                    Bs = fmaf(Bs, q.D, e);
                }
            }
            return rev_fixed;
        }
    }
    FwdState st = cin;
#pragma unroll
    for (int i = 0; i < LT; ++i)
        if (FULL || i < n) {
            const float k = sk[i * CG], v = sv[i * CG];
            const Pair f = max_pair(st.p, q.u + k);
            const float den = fmaf(f.fx, st.d, f.fy);  // in [1, T + 1]
            const float rden = __fdividef(1.f, den);
            R.Y[i] = fmaf(f.fx, st.a, f.fy * v) * rden;
            R.X[i] = f.q + __logf(den);
#if WKV_BWD_KEEP_E
            R.E[i] = f.fy * rden;
#endif
            fwd_step(st, k, v, q.w);
        }
    return false;
}

// The reverse pass from the state after the tile: gk over sk, gv over sv,
// and the tile's gw, gu.  At the fixed reference M the four sums run in
// units of e^{-M} (z converted by e^{M - rho} <= e^30; far below 1 it
// flushes to 0, the carried sums then weighing less than e^-87 of theirs)
// and e^{k_j} times a sum is E_j times it: no exponential per step.
// Otherwise the per-step min-stabilised steps, e^{k_j - rho} <= 1 from the
// staged key.
template <int LT, bool FULL>
__device__ __forceinline__ void grads_reverse(float *sk, float *sv, const float *sg, int n,
                                              RevState z, const WkvOp<float, 1>::Param &q,
                                              const TileRows<LT> &R, bool fixed, float M,
                                              float &gw, float &gu) {
    constexpr int CG = 32;
    gw = 0.f;
    gu = 0.f;
    if (fixed) {
        const float f = fast_exp(M - z.rho);
        float P = z.P * f, Q = z.Q * f, Rs = z.R * f, R2 = z.R2 * f;
#pragma unroll
        for (int i = LT - 1; i >= 0; --i)
            if (FULL || i < n) {
                const float vj = sv[i * CG], gj = sg[i * CG];
#if WKV_BWD_KEEP_E
                const float e = R.E[i];
#else
                const float e = ex2_approx((sk[i * CG] - M) * kLog2e);
#endif
                const float gr = gj * R.X[i], y = R.Y[i];
                const float diag = q.U * gr;  // g_j beta_{j,j} / e_j
                const float dv = vj - y;
                sv[i * CG] = e * (diag + P);
                sk[i * CG] = e * fmaf(diag, dv, fmaf(vj, P, -Q));
                gu = fmaf(e * diag, dv, gu);
                gw = fmaf(-e, fmaf(vj, Rs, -R2), gw);
                Rs = q.D * (Rs + P);
                R2 = q.D * (R2 + Q);
                P = fmaf(q.D, P, gr);
                Q = fmaf(q.D, Q, gr * y);
            }
        return;
    }
#pragma unroll
    for (int i = LT - 1; i >= 0; --i)
        if (FULL || i < n) {
            const float kj = sk[i * CG], vj = sv[i * CG], gj = sg[i * CG];
            const float sc = fast_exp(kj - z.rho);  // e^{k_j - rho}, <= 1
#if WKV_BWD_KEEP_E
            const float diag = R.E[i] * gj;         // g_j beta_{j,j}
#else
            const float diag = fast_exp(q.u + kj - R.X[i]) * gj;
#endif
            const float dv = vj - R.Y[i];
            sv[i * CG] = fmaf(sc, z.P, diag);
            sk[i * CG] = fmaf(diag, dv, sc * fmaf(vj, z.P, -z.Q));
            gu = fmaf(diag, dv, gu);
            gw = fmaf(-sc, fmaf(vj, z.R, -z.R2), gw);
            rev_step(z, gj, R.Y[i], R.X[i], q.w);
        }
}

template <int NCW, int NSTAGE>
__global__ void __launch_bounds__(BwdGradsCfg<NCW, NSTAGE>::kThreads, 1)
    wkv_bwd_grads_tiles_kernel(const __grid_constant__ CUtensorMap map_k,
                               const __grid_constant__ CUtensorMap map_v,
                               const __grid_constant__ CUtensorMap map_gy,
                               const __grid_constant__ CUtensorMap map_gk,
                               const __grid_constant__ CUtensorMap map_gv, const BwdTileArgs a,
                               const Geometry g, const Workspace ws) {
    using Cfg = BwdGradsCfg<NCW, NSTAGE>;
    using Param = WkvOp<float, 1>::Param;
    constexpr int CG = Cfg::CG, LT = Cfg::LT;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full_bar[NSTAGE];
    __shared__ __align__(8) uint64_t empty_bar[NSTAGE];
    __shared__ int s_fill_it[NSTAGE];  // ring iteration the stage was last filled for
    __shared__ int s_last_it[NSTAGE];  // last ring iteration loaded into each stage
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
            s_last_it[s] = -1;
            s_fill_it[s] = -1;
        }
        fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();
    volatile int *abort_flag = &s_abort;

    // ring iteration `it` of this block holds tile tiles-1-j, j = block + it *
    // grid: the tiles go latest-first, those the states kernel read last
    const auto tile_of = [&](int it) -> int {
        const long long j = static_cast<long long>(blockIdx.x) + static_cast<long long>(it) * gridDim.x;
        return j < g.tiles ? g.tiles - 1 - static_cast<int>(j) : -1;
    };

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&map_k);
            prefetch_tensormap(&map_v);
            prefetch_tensormap(&map_gy);
            prefetch_tensormap(&map_gk);
            prefetch_tensormap(&map_gv);
            for (int it = 0;; ++it) {
                const int tile = tile_of(it);
                if (tile < 0) break;
                const int s = it % NSTAGE;
                if (!wait_phase(&empty_bar[s], ((it / NSTAGE) & 1) ^ 1, abort_flag, ws)) break;
                const int seg = tile / g.tiles_per_seg;
                const int rem = tile - seg * g.tiles_per_seg;
                const int b = rem / g.n_cg;
                const int c0 = (rem - b * g.n_cg) * CG;
                unsigned char *dst = smem + static_cast<size_t>(s) * Cfg::kStageBytes;
                *static_cast<volatile int *>(&s_fill_it[s]) = it;
                s_last_it[s] = it;
                mbar_arrive_expect_tx(&full_bar[s], static_cast<uint32_t>(Cfg::kStageBytes));
                tma_load_3d(dst, &map_k, &full_bar[s], c0, seg * LT, b);
                tma_load_3d(dst + Cfg::kTileBytes, &map_v, &full_bar[s], c0, seg * LT, b);
                tma_load_3d(dst + 2 * Cfg::kTileBytes, &map_gy, &full_bar[s], c0, seg * LT, b);
            }
            // every tile of this block is loaded or assigned: the next grid in
            // the stream may start launching its blocks (its own
            // griddepcontrol.wait still waits for this grid to complete)
            allow_dependent_launch();
        }
        __syncwarp();
    } else {
        // ---------------- compute warps: ring iterations cw, cw + NCW, ... ----
        // The producer loads k, v and gy without waiting for the grids before
        // this one in the stream: the gradient step's first kernels write
        // none of them (only the scratch), and this grid's blocks are
        // launched only after those kernels' blocks have all started, i.e.
        // after the first of them has itself waited for everything before
        // the step.  What this warp reads from the scratch, and every store,
        // comes after the wait for the previous grid to complete.
        grid_dependency_wait();
        const int cw = warp - 1;
        const size_t C = static_cast<size_t>(g.C);
        int held = -1;  // the stage of this warp's stores still in flight
        for (int it = cw;; it += NCW) {
            const int tile = tile_of(it);
            if (tile < 0) break;
            const int seg = tile / g.tiles_per_seg;
            const int rem = tile - seg * g.tiles_per_seg;
            const int b = rem / g.n_cg;
            const int c0 = (rem - b * g.n_cg) * CG;
            const int c = c0 + lane;
            const int t0 = seg * LT;
            const int n = min(LT, g.T - t0);
            const bool cvalid = c < g.C;
            const size_t bs = static_cast<size_t>(b) * a.S + seg;
            // the channel's parameters and the tile's two carries (global,
            // mostly L2), loaded before waiting for the stage
            Param q{0.f, 0.f, 1.f, 1.f};
            FwdState cin{0.f, 0.f, kNoScale};
            RevState z{0.f, 0.f, 0.f, 0.f, -kNoScale};
            if (cvalid) {
                q.u = a.u[c];
                q.w = a.w[c];
                cin = load_fwd(a.fwd + bs * 3 * C + c, g.C);
                z = load_rev(a.rev + bs * 5 * C + c, g.C);
            }
            q.U = expf(q.u);
            q.D = expf(-q.w);
            const int s = it % NSTAGE;
            const uint32_t parity = (it / NSTAGE) & 1;
            int ok = 0;
            if (lane == 0) ok = wait_fill(&full_bar[s], &s_fill_it[s], it, parity, abort_flag, ws) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            // observing the completed phase makes the TMA writes visible here
            for (int m = 0; m < (1 << 20) && !mbar_try_wait(&full_bar[s], parity); ++m) {
            }
            float *st_k = reinterpret_cast<float *>(smem + static_cast<size_t>(s) * Cfg::kStageBytes);
            float *st_v = st_k + Cfg::kTileElems;
            const float *st_g = st_v + Cfg::kTileElems;
            TileRows<LT> R;
            float gw, gu, M;
            if (n == LT) {
                const bool fx = grads_forward<LT, true>(st_k + lane, st_v + lane, n, cin, z, q, R, M);
                grads_reverse<LT, true>(st_k + lane, st_v + lane, st_g + lane, n, z, q, R, fx, M,
                                        gw, gu);
            } else {
                grads_forward<LT, false>(st_k + lane, st_v + lane, n, cin, z, q, R, M);
                grads_reverse<LT, false>(st_k + lane, st_v + lane, st_g + lane, n, z, q, R, false,
                                         M, gw, gu);
            }
            // gk, gv leave from the stage by TMA (rows >= T and channels >= C
            // are clipped); a stage goes back once its stores have read it:
            // the previous tile's, checked after this tile's stores are issued
            // (at most one group of stores in flight per warp)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&map_gk, st_k, c0, t0, b);
                tma_store_3d(&map_gv, st_v, c0, t0, b);
                bulk_commit();
#if WKV_BWD_DEFER_RELEASE
                if (held >= 0) {
                    bulk_wait_read_all_but_one();
                    mbar_arrive(&empty_bar[held]);
                }
#else
                bulk_wait_read_all();
                mbar_arrive(&empty_bar[s]);
#endif
            }
            held = s;
            if (cvalid) {
                float *pp = a.partial + bs * 2 * C + c;
                pp[0] = gw;
                pp[C] = gu;
            }
            __syncwarp();
        }
        // the block's shared memory must outlive the warp's last stores
        if (lane == 0) {
            bulk_wait_read_all();
#if WKV_BWD_DEFER_RELEASE
            if (held >= 0 && !*abort_flag) mbar_arrive(&empty_bar[held]);
#endif
        }
        __syncwarp();
    }

    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        for (int s = 0; s < NSTAGE; ++s) {
            const int it = s_last_it[s];
            if (it < 0) continue;
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1)) {
                if (global_timer_ns() - t0 > kBarrierWaitNs) break;
            }
        }
    }
    allow_dependent_launch();
}

}  // namespace wkvb
