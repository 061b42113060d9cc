// Persistent fp32 WKV forward with register-resident sub-chunks and a carry
// warp per group, for sm_100a (shapes a TMA tensor map can describe).
//
// One thread block per SM for the whole launch.  Warp 0 is the producer: it
// takes tile tickets and streams each tile's k and v (and r for the gate)
// tiles of LT steps x 32 channels, with the tile's u and w, into a ring of
// shared-memory stages (TMA tile loads plus two bulk copies, one mbarrier per
// stage).  The other warps form NC groups of NWG compute warps and one carry
// warp; a group works on one tile at a time:
//
//  * the compute warps copy their sub-chunk of the stage (LS = LT / NWG steps
//    of their lane's channel) into registers once.  Pass 1 turns each key
//    into its weight E_i = e^{k_i - max k} and sums the sub-chunk by Horner's
//    rule, (a, b) <- (a, b) e^{-w} + E_i (v_i, 1), from the registers.  Pass
//    2 scales the same weights to its own reference and re-sweeps the
//    registers from the carried-in state into the group's output tile in
//    shared memory, which one TMA store writes out.  Each element costs one
//    exponential and one shared-memory read.
//  * the compute warp that finishes pass 1 last folds the group's summaries
//    at once: the tile aggregate is published (for the look-backs of later
//    tiles) and the stage is handed back without waiting for anyone.
//  * the carry warp takes the group's tiles (ring iterations, from a shared
//    counter, as the group becomes free) and walks the decoupled look-back
//    for the state before the tile while the compute warps run pass 1; with
//    the aggregate it publishes the state after the tile and hands the
//    compute warps their carries.  Its slots are double-buffered, so it
//    takes the next tile while the compute warps sweep the current one.
//
// Hand-offs between the carry warp and the compute warps are named barriers
// used producer/consumer-wise (one side arrives, the other waits); the carry
// warp's own waits are bounded, and it always arrives -- with "no tile" when
// it gives up -- so no compute warp can be left waiting.
//
// The chunk identity behind pass 1 / carry / pass 2 is the Upper/Lower split
// of a linear recurrence (review of "Resurrecting Recurrent Neural Networks
// for Long Sequences", parallelisation section); the operator is eq. (14) of
// "RWKV：基于RNN的LLM" (section 二.1), its state and combine are WkvOp's.
//
// Every wait is bounded (global-timer deadline on mbarriers, poll budget in
// the look-back); a wait that gives up records WKV_ERR_TIMEOUT in the status
// word, leaves NaN in the affected outputs and lets the launch finish.
#pragma once

#include <cstdint>

#include "persistent_scan.cuh"
#include "ptx.cuh"
#include "scan_common.cuh"
#include "wkv_ops.cuh"

namespace wkvb {

// look-back hops whose records the carry warp loads together
#ifndef WKV_REG_LOOKBACK_HOPS
#define WKV_REG_LOOKBACK_HOPS 4
#endif

// GATED: the outputs are sigma(r_t) (.) wkv_t (eq. (15) of the same page
// before the output projection), r staged with k and v.  The arithmetic and
// the Args are WkvOp's without the gate (Args carries r in x2 either way).
template <int LT, int NWG, int NC, int NSTAGE, bool GATED = false>
struct RegWkvCfg {
    using Op = WkvOp<float, 1, false>;
    static constexpr int NIN = GATED ? 3 : 2;  // input tiles per stage: k, v (, r)
    static constexpr int CG = 32, LS = LT / NWG;
    static constexpr int NGW = NWG + 1;        // warps per group: NWG compute, 1 carry
    static constexpr int kThreads = (1 + NC * NGW) * 32;
    static constexpr size_t kTileElems = static_cast<size_t>(LT) * CG;
    // a stage: the k tile, the v tile (, the r tile), then the tile's u and w
    // ([CG] fp32 each)
    static constexpr size_t kParamOffset = NIN * kTileElems * sizeof(float);
    static constexpr size_t kStageBytes = kParamOffset + 2 * CG * sizeof(float);
    static constexpr int kHops = WKV_REG_LOOKBACK_HOPS;
    // per group: the output tile, then two slots (double-buffered) of the
    // compute warps' summaries [NWG][3][CG], of the carry [3][CG] and of the
    // tile aggregate [3][CG]
    static constexpr size_t kOutBytes = kTileElems * sizeof(float);
    static constexpr size_t kSumFloats = static_cast<size_t>(NWG) * 3 * CG;
    static constexpr size_t kCarryFloats = static_cast<size_t>(3) * CG;
    static constexpr size_t kGroupBytes =
        kOutBytes + 2 * (kSumFloats + 2 * kCarryFloats) * sizeof(float);
    static constexpr size_t kSmemBytes = NSTAGE * kStageBytes + NC * kGroupBytes;
    // named barriers per group: tile assigned, carries written, output tile
    // written, aggregate written; plus one for all consumers at the start
    static constexpr int kBarsPerGroup = 4;
    static_assert(LT % NWG == 0, "tile length must split evenly over a group's compute warps");
    static_assert(LS % 2 == 0 && LS <= 32, "sub-chunks of an even number of steps, at most 32");
    static_assert(LT <= 256, "TMA box rows are limited to 256");
    // a group holds a stage only through pass 1, which waits on nothing, so
    // any ring of two or more stages keeps every group fed eventually
    static_assert(NSTAGE >= 2, "at least one stage being read while one loads");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
    static_assert(kStageBytes % 128 == 0 && kParamOffset % 16 == 0 && kOutBytes % 128 == 0,
                  "stage and output-tile alignment");
    static_assert(2 + kBarsPerGroup * NC <= 16, "named barrier ids: 0, per group, one for all");
};

// ---------------------------------------------------------------------------
// One lane's sub-chunk in registers: per step the key's weight against the
// sub-chunk's largest key, and the value.
// ---------------------------------------------------------------------------
template <int LS>
struct LaneRows {
    float e[LS];  // k_i on load, then E_i = e^{k_i - kmax}
    float v[LS];
    float kmax, kmin;
};

// ---- rare paths -------------------------------------------------------------
// the sub-chunk summed against the exact largest exponent (its largest key
// decayed away, see rows_pass1)
template <int LS>
__device__ __forceinline__ WkvOp<float, 1>::State resum_f32(const float *sk, const float *sv,
                                                            int n, WkvOp<float, 1>::Param q) {
    using Op = WkvOp<float, 1>;
    const Op::Param qq[1] = {q};
    const float ref[1] = {Op::largest_exponent(sk, n, 0, q)};
    float a2[1], b2[1];
    Op::chunk_sums<LS, 8>(sk, sv, n, qq, ref, a2, b2);
    return {a2[0], b2[0], ref[0]};
}

// the per-step max-stabilised sweep, keys and values read back from global
// memory (kp[i * C], vp[i * C]; zeros when the channel does not exist);
// gated, yp[i * ys] holds r_t on entry
template <bool GATED>
__device__ __forceinline__ void sweep_exact_f32(WkvOp<float, 1>::State st, int n,
                                                WkvOp<float, 1>::Param q, const float *kp,
                                                const float *vp, size_t C, bool cvalid, float *yp,
                                                size_t ys) {
    using Op = WkvOp<float, 1>;
    for (int i = 0; i < n; ++i) {
        const float k = cvalid ? kp[i * C] : 0.f, v = cvalid ? vp[i * C] : 0.f;
        float y = Op::step_exact(st, k, v, q);
        if constexpr (GATED) y *= gate_sigmoid(yp[i * ys]);
        yp[i * ys] = y;
    }
}

// ---- pass 1 ----------------------------------------------------------------
// Load the sub-chunk (rows sk[i * 32], sv[i * 32] of the stage, n of them
// valid), find the key range, turn keys into weights and sum the sub-chunk
// by Horner's rule ending at its last valid step.  The summary's reference is
// max k; when the chunk's weight lands below 2^-60 (its largest key decayed
// far away) it is summed again, directly from the stage, against the exact
// largest exponent, as WkvOp::summarize does.
template <int LS, bool FULL>
__device__ __forceinline__ void rows_pass1(const float *sk, const float *sv, int n,
                                           const WkvOp<float, 1>::Param &q, LaneRows<LS> &R,
                                           WkvOp<float, 1>::State &sum) {
    constexpr int CG = 32;
#pragma unroll
    for (int i = 0; i < LS; ++i) {
        R.e[i] = sk[i * CG];
        R.v[i] = sv[i * CG];
    }
    float kx = kNoScale, kn = -kNoScale;
#pragma unroll
    for (int i = 0; i < LS; ++i)
        if (FULL || i < n) {
            kx = fmaxf(kx, R.e[i]);
            kn = fminf(kn, R.e[i]);
        }
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int i = 0; i < LS; ++i)
        if (FULL || i < n) {
            // fp32 keeps k - kmax exact before scaling (a few ulp of the gap)
            const float e = ex2_approx((R.e[i] - kx) * kLog2e);
            R.e[i] = e;
            a = fmaf(a, q.D, e * R.v[i]);
            b = fmaf(b, q.D, e);
        }
    R.kmax = kx;
    R.kmin = kn;
    sum = {a, b, kx};
    if (!(b >= 0x1p-60f)) sum = resum_f32<LS>(sk, sv, n, q);
}

// ---- pass 2 ----------------------------------------------------------------
// Whether the fixed-reference sweep is safe for the channel: every
// denominator stays above e^-69 (so nothing that matters flushes to zero) and
// e^u below 2^64.  den_t >= e^{u + k_t - M} once e^{k_t - M} itself cannot
// flush (k_t - M >= -69 when u >= 0), and den_t >= b_in e^{p_in - M - t w}.
// (`floor`: the log of the least denominator the bound must guarantee.)
__device__ __forceinline__ bool sweep_is_safe(float kmin, float M, const WkvOp<float, 1>::State &cin,
                                              const WkvOp<float, 1>::Param &q, int n,
                                              float floor = -69.f) {
    const bool by_token = kmin + fminf(q.u, 0.f) - M >= floor;
    const bool by_carry = cin.b >= 1.f && cin.p - M - static_cast<float>(n) * q.w >= floor;
    return (by_token || by_carry) && q.u <= 44.f;
}

// Outputs of the sub-chunk from the state before it, to yp[i * ys] (the
// group's output tile).  Fixed reference M = max(p_in, kmax):
// e_t = E_t e^{kmax - M}, y = v + (a - b v) / (b + e U), a <- a D + e v,
// b <- b D + e.  When that is not safe (rare: extreme keys or bonus), the
// per-step max-stabilised update, with keys and values read back from global
// memory (kp[i * C], vp[i * C]; only when the channel exists, `cvalid`).
// GATED: yp[i * ys] holds r_t on entry (copied there in pass 1) and each
// output is multiplied by sigma(r_t) before it replaces it.
template <int LS, bool FULL, bool GATED>
__device__ __forceinline__ void rows_pass2(const LaneRows<LS> &R, const WkvOp<float, 1>::State &cin,
                                           int n, const WkvOp<float, 1>::Param &q, const float *kp,
                                           const float *vp, size_t C, bool cvalid, float *yp,
                                           size_t ys) {
    const float M = fmaxf(cin.p, R.kmax);
    if (sweep_is_safe(R.kmin, M, cin, q, n)) {
        const float s = fast_exp(R.kmax - M), f = fast_exp(cin.p - M);
        float A = cin.a * f, Bs = cin.b * f;
#pragma unroll
        for (int i = 0; i < LS; ++i)
            if (FULL || i < n) {
                const float e = R.e[i] * s, v = R.v[i];
                float y = v + fmaf(-Bs, v, A) * rcp_approx(fmaf(e, q.U, Bs));
                A = fmaf(A, q.D, e * v);
                Bs = fmaf(Bs, q.D, e);
                if constexpr (GATED) y *= gate_sigmoid(yp[i * ys]);
                yp[i * ys] = y;
            }
    } else {
        sweep_exact_f32<GATED>(cin, n, q, kp, vp, C, cvalid, yp, ys);
    }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// Every lane of the warp waits for the phase with the given parity; lane 0
// alone runs the bounded wait, so the warp agrees on the outcome (false in
// every lane if the block is aborting or the deadline passed).  The other
// lanes then observe the completed phase themselves (acquire), which
// returns at once: the barrier cannot move on to a later phase before the
// waiting warp acts.
__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity,
                                                volatile int *abort_flag, const Workspace &ws) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_phase(bar, parity, abort_flag, ws) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok)
        for (int n = 0; n < (1 << 20) && !mbar_try_wait(bar, parity); ++n) {
        }
    return ok != 0;
}

// the tile's u and w from the stage (channels past C: the neutral parameters)
__device__ __forceinline__ WkvOp<float, 1>::Param staged_param(const float *s_par, int lane, int c,
                                                               int C) {
    WkvOp<float, 1>::Param q{0.f, 0.f, 1.f, 1.f};
    if (c < C) {
        q.u = s_par[lane];
        q.w = s_par[32 + lane];
        q.U = expf(q.u);
        q.D = expf(-q.w);
    }
    return q;
}

template <int LT, int NWG, int NC, int NSTAGE, bool GATED = false>
__global__ void __launch_bounds__(RegWkvCfg<LT, NWG, NC, NSTAGE, GATED>::kThreads, 1)
    persistent_wkv_kernel(const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v,
                          const __grid_constant__ CUtensorMap map_y,
                          const __grid_constant__ CUtensorMap map_r,  // GATED only
                          const WkvOp<float, 1>::Args args, const Geometry g, const Workspace ws) {
    using Cfg = RegWkvCfg<LT, NWG, NC, NSTAGE, GATED>;
    using Op = typename Cfg::Op;
    using State = typename Op::State;
    using Param = typename Op::Param;
    constexpr int CG = Cfg::CG, LS = Cfg::LS, NV = 3, NGW = Cfg::NGW;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *s_stage = smem;  // [NSTAGE] x (k tile, v tile (, r tile), u[CG], w[CG])
    unsigned char *s_groups = smem + NSTAGE * Cfg::kStageBytes;  // [NC] x kGroupBytes
    __shared__ __align__(8) uint64_t full_bar[NSTAGE];
    __shared__ __align__(8) uint64_t empty_bar[NSTAGE];
    // per group, double-buffered by the parity of the group's tile count
    // (slot k = tile & 1; phase (tile >> 1) & 1): the compute warps have read
    // the slot's carries, so the carry warp may reuse it
    __shared__ __align__(8) uint64_t free_bar[NC][2];
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
        for (int q = 0; q < NC; ++q)
            for (int k = 0; k < 2; ++k) {
                mbar_init(&free_bar[q][k], NWG);
                s_count[q][k] = 0;
            }
        fence_mbar_init();
        s_abort = 0;
        s_next_it = 0;
    }
    // everything above touched only shared memory; with a programmatic
    // dependency on the previous grid in the stream, nothing global is read
    // before that grid has finished
    grid_dependency_wait();
    __syncthreads();
    volatile int *abort_flag = &s_abort;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&map_k);
            prefetch_tensormap(&map_v);
            prefetch_tensormap(&map_y);
            if (GATED) prefetch_tensormap(&map_r);
            int sentinels = 0;
            int next_static = static_cast<int>(blockIdx.x);
            for (int it = 0; sentinels < NC; ++it) {
                const int s = it % NSTAGE;
                if (!wait_phase(&empty_bar[s], ((it / NSTAGE) & 1) ^ 1, abort_flag, ws)) break;
                int tile = -1;
                if (sentinels == 0) {
                    if (chained) {
                        // tickets go out in the order blocks ask for them, so a
                        // tile only ever waits for tiles already being worked on
                        const unsigned t = atomicAdd(ws.ticket, 1u);
                        tile = t < static_cast<unsigned>(g.tiles) ? static_cast<int>(t) : -1;
                    } else {
                        tile = next_static < g.tiles ? next_static : -1;
                        next_static += static_cast<int>(gridDim.x);
                    }
                }
                s_meta[s] = tile;
                // stamped before the arrive that releases it: a consumer only
                // accepts a completed phase of this stage when the stamp
                // names its own iteration
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
                    // the tile's u and w: channels c0 .. c0 + CG clipped to C
                    // (C * 4 bytes is a multiple of 16 on this path)
                    const uint32_t pbytes =
                        static_cast<uint32_t>(min(CG, g.C - c0)) * static_cast<uint32_t>(sizeof(float));
                    s_last_it[s] = it;
                    mbar_arrive_expect_tx(&full_bar[s],
                                          static_cast<uint32_t>(Cfg::kParamOffset) + 2 * pbytes);
                    tma_load_3d(dst, &map_k, &full_bar[s], c0, seg * LT, b);
                    tma_load_3d(dst + Cfg::kTileElems * sizeof(float), &map_v, &full_bar[s], c0,
                                seg * LT, b);
                    if (GATED)
                        tma_load_3d(dst + 2 * Cfg::kTileElems * sizeof(float), &map_r, &full_bar[s],
                                    c0, seg * LT, b);
                    float *dp = reinterpret_cast<float *>(dst + Cfg::kParamOffset);
                    bulk_load(dp, args.u + c0, pbytes, &full_bar[s]);
                    bulk_load(dp + CG, args.w + c0, pbytes, &full_bar[s]);
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
        // the launch's epoch, read by one consumer thread while the producer
        // already takes tickets and starts loads
        if (threadIdx.x == 32) s_epoch = chained ? epoch_of(ws) : 0ull;
        named_bar_sync(1 + Cfg::kBarsPerGroup * NC, NC * NGW * 32);
        const unsigned long long epoch = s_epoch;
        const int cw = warp - 1;
        const int grp = cw / NGW, wg = cw - grp * NGW;
        // the group's named barriers: the tile is assigned and the carries
        // are written (carry warp -> compute warps), the output tile is
        // written (among the compute warps), the aggregate is written
        // (folding compute warp -> carry warp)
        const int bar_tile = 1 + Cfg::kBarsPerGroup * grp, bar_carry = bar_tile + 1,
                  bar_out = bar_tile + 2, bar_agg = bar_tile + 3;
        unsigned char *gbase = s_groups + static_cast<size_t>(grp) * Cfg::kGroupBytes;
        float *g_out = reinterpret_cast<float *>(gbase);
        float *g_sum0 = g_out + Cfg::kTileElems;           // [2][NWG][NV][CG]
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
                // the slot is free once the compute warps have read tile i - 2's
                // carries (the wait passes at once for the first two tiles)
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
                // observing the completed phase makes the stage's bytes visible
                // here; the tile's u and w are read before the compute warps
                // are let in (the stage goes back once they have summarised)
                for (int n = 0; n < (1 << 20) && !mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1); ++n) {
                }
                const int seg = tile / g.tiles_per_seg;
                const int rem = tile - seg * g.tiles_per_seg;
                const int b = rem / g.n_cg;
                const int t0 = seg * LT;
                const int c = (rem - b * g.n_cg) * CG + lane;
                const Param prm = staged_param(
                    reinterpret_cast<const float *>(s_stage + static_cast<size_t>(s) * Cfg::kStageBytes +
                                                    Cfg::kParamOffset),
                    lane, c, g.C);
                __syncwarp();
                named_bar_arrive(bar_tile, (NWG + 1) * 32);  // the compute warps start

                // the state before the tile: the given state for the first
                // segment, else the decoupled look-back over the tiles before it
                const bool last = seg == g.n_seg - 1;
                State X = seg == 0 ? Op::carry0(args, b, c, g.C) : Op::identity();
                if (chained && seg > 0 &&
                    !lookback_channel<Op, LT, 1, Cfg::kHops>(ws, g, tile, epoch, prm, lane, 0, X,
                                                             static_cast<const ChannelPrefetch<1> *>(
                                                                 nullptr))) {
                    atomicExch(ws.status, kStatusTimeout);  // this lane gave up
                    X = Op::nan_state();
                }
                // the tile aggregate, once the compute warps have folded it
                named_bar_sync(bar_agg, 64);  // with the folding warp's arrival
                float vals[NV];
#pragma unroll
                for (int q = 0; q < NV; ++q) vals[q] = g_agg[q * CG + lane];
                const State agg = Op::make(vals);
                if (chained && !last)
                    publish_channel<Op, CG>(ws, g, tile,
                                            Op::combine(X, agg, static_cast<float>(LT), prm), 0,
                                            kFlagIncl, epoch, lane);
                if (last)  // the state after the last step
                    Op::store_final(args, b, c, g.C,
                                    Op::combine(X, agg, static_cast<float>(min(LT, g.T - t0)), prm));
#pragma unroll
                for (int q = 0; q < NV; ++q) g_carry[q * CG + lane] = Op::get(X, q);
                __syncwarp();
                named_bar_arrive(bar_carry, (NWG + 1) * 32);  // the compute warps sweep
            }
        } else {
            // ---------------- compute warps ----------------
            const bool issuer = wg == 0 && lane == 0;  // issues the group's output stores
            for (int i = 0;; ++i) {
                const int k = i & 1;
                float *g_sum = g_sum0 + k * Cfg::kSumFloats;
                const float *g_carry = g_carry0 + k * Cfg::kCarryFloats;
                named_bar_sync(bar_tile, (NWG + 1) * 32);
                const int tile = *static_cast<volatile int *>(&s_tile[grp][k]);
                if (tile < 0) break;
                const int it = s_it[grp][k];
                const int s = it % NSTAGE;
                // observing the completed phase makes the stage's bytes visible
                // here (the stage is not refilled before this group's fold)
                for (int n = 0; n < (1 << 20) && !mbar_try_wait(&full_bar[s], (it / NSTAGE) & 1); ++n) {
                }
                const int seg = tile / g.tiles_per_seg;
                const int rem = tile - seg * g.tiles_per_seg;
                const int b = rem / g.n_cg;
                const int t0 = seg * LT;
                const int c0 = (rem - b * g.n_cg) * CG;
                const int c = c0 + lane;
                const unsigned char *st_base = s_stage + static_cast<size_t>(s) * Cfg::kStageBytes;
                const float *s_k = reinterpret_cast<const float *>(st_base);
                const float *s_v = s_k + Cfg::kTileElems;
                const Param prm = staged_param(
                    reinterpret_cast<const float *>(st_base + Cfg::kParamOffset), lane, c, g.C);
                // the group's previous output store must have read the output
                // tile before it is written again: in pass 2 (no compute warp
                // gets its carry before the issuer has summarised, which
                // follows this wait), or, gated, already in pass 1 (r is
                // copied there), hence the barrier
                if (issuer) bulk_wait_read_all();
                if constexpr (GATED) named_bar_sync(bar_out, NWG * 32);

                // pass 1: the sub-chunk into registers, weights and summary
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
                if constexpr (GATED) {
                    // r rows of this warp's sub-chunk into the output tile, where
                    // pass 2 reads each one just before the output replaces it
                    const float *pr = s_k + 2 * Cfg::kTileElems + s0 * CG + lane;
                    float *po = g_out + s0 * CG + lane;
#pragma unroll 8
                    for (int ii = 0; ii < LS; ++ii) po[ii * CG] = pr[ii * CG];
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
                    // in time order; each slot becomes its warp's exclusive
                    // prefix for pass 2
                    State a = Op::identity();
                    for (int w = 0; w < NWG; ++w) {
                        float vals[NV];
                        float *slot = g_sum + w * NV * CG + lane;
#pragma unroll
                        for (int q = 0; q < NV; ++q) vals[q] = slot[q * CG];
#pragma unroll
                        for (int q = 0; q < NV; ++q) slot[q * CG] = Op::get(a, q);
                        const int len = max(0, min(LS, g.T - (t0 + w * LS)));
                        a = Op::combine(a, Op::make(vals), static_cast<float>(len), prm);
                    }
                    if (chained && seg > 0 && seg < g.n_seg - 1)
                        publish_channel<Op, CG>(ws, g, tile, a, 0, kFlagAgg, epoch, lane);
#pragma unroll
                    for (int q = 0; q < NV; ++q) g_agg[q * CG + lane] = Op::get(a, q);
                    __syncwarp();
                    if (lane == 0) {
                        s_count[grp][k] = 0;
                        mbar_arrive(&empty_bar[s]);  // every compute warp is done with the stage
                    }
                    named_bar_arrive(bar_agg, 64);   // the carry warp may finish the carry
                }

                // the carry into this warp's sub-chunk
                named_bar_sync(bar_carry, (NWG + 1) * 32);
                State cur;
                {
                    float vals[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) vals[q] = g_carry[q * CG + lane];
                    cur = Op::make(vals);
                    if (wg > 0) {  // the sub-chunks before this warp's, all full
#pragma unroll
                        for (int q = 0; q < NV; ++q) vals[q] = g_sum[(wg * NV + q) * CG + lane];
                        cur = Op::combine(cur, Op::make(vals), static_cast<float>(wg * LS), prm);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_bar[grp][k]);  // the slot may be reused

                // pass 2: outputs from the registers into the output tile (all
                // channels; the TMA store clips channels >= C and steps >= T)
                if (nval > 0) {
                    const size_t row0 = (static_cast<size_t>(b) * g.T + t0 + s0) * g.C + c;
                    const float *kp = args.x0 + row0, *vp = args.x1 + row0;
                    float *yp = g_out + s0 * CG + lane;
                    const bool cvalid = c < g.C;
                    if (nval == LS)
                        rows_pass2<LS, true, GATED>(R, cur, nval, prm, kp, vp, g.C, cvalid, yp, CG);
                    else
                        rows_pass2<LS, false, GATED>(R, cur, nval, prm, kp, vp, g.C, cvalid, yp, CG);
                }
                // the tile's outputs leave by one TMA store (their generic-proxy
                // writes ordered before the store's async-proxy reads)
                fence_proxy_async_smem();
                named_bar_sync(bar_out, NWG * 32);
                if (issuer) {
                    tma_store_3d(&map_y, g_out, c0, t0, b);
                    bulk_commit();
                }
            }
            // the block's shared memory must outlive the group's last store
            if (issuer) bulk_wait_read_all();
        }
        __syncwarp();
    }

    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        // an aborted block must not exit with tile loads still landing in its
        // shared memory: wait (bounded) for the last load of every stage
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
    finish_launch(ws, chained, static_cast<int>(threadIdx.x), gridDim.x);
}

}  // namespace wkvb
