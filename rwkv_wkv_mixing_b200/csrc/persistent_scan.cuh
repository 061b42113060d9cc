// Persistent, warp-specialised chunked scan for sm_100a (shapes a TMA tensor
// map can describe).
//
// One thread block per SM stays resident for the whole launch.  Warp 0 is the
// producer: one lane takes tile tickets and streams each tile's NIN input
// tensors (LT steps x CG channels) into a ring of NSTAGE shared-memory stages
// with TMA tile loads, each stage guarded by a "full" and an "empty" mbarrier.
// The remaining warps form NC consumer groups of NWG warps; group g handles
// ring iterations g, g+NC, g+2NC, ...  For each tile a group runs the same
// two passes and look-back as chunked_scan_kernel -- pass 1 summaries per
// warp, the carry into the tile (aggregate, decoupled look-back, publication)
// by the group's first warp, pass 2 writing outputs over the stage's first
// tensor -- then one thread issues the TMA store of the outputs, waits until
// the store has read the stage, and releases it to the producer.  Outputs
// leave through the async proxy, so the look-back's release fences never wait
// behind a warp's own output stores.
//
// So HBM sees every element once, loads for the next tiles are in flight
// while tiles are being computed, several tiles per SM hide the look-back
// latency, and no thread block is launched per tile.  Every wait is bounded
// (global-timer deadline on mbarriers, poll budget in the look-back); a wait
// that gives up records WKV_ERR_TIMEOUT in the status word and makes every
// loop of the block finish.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "scan_common.cuh"

namespace wkvb {

constexpr unsigned long long kBarrierWaitNs = 4000000000ull;  // 4 s

// look-back records (hops back in time) a group loads before pass 1
#ifndef WKV_LB_PREFETCH
#define WKV_LB_PREFETCH 1
#endif

// stage waits: 0 = suspend in mbarrier try_wait; N > 0 = poll with
// mbarrier test_wait, N ns apart
#ifndef WKV_FILL_POLL
#define WKV_FILL_POLL 0
#endif

// Ops whose per-channel parameters are the two fp32 arrays args.u and
// args.w (the WKV ops) can have them staged with each tile
template <class Op, class = void>
struct StagesParams : std::false_type {};
template <class Op>
struct StagesParams<Op, std::void_t<decltype(Op::kSerialForm)>>
    : std::bool_constant<Op::kSerialForm> {};

template <class Op, int LT, int NWG, int NC, int NSTAGE>
struct PersistentCfg {
    static constexpr int CPT = Op::CPT, NV = Op::NV, CG = 32 * CPT, LS = LT / NWG;
    static constexpr int kThreads = (1 + NC * NWG) * 32;
    static constexpr size_t kTileElems = static_cast<size_t>(LT) * CG;
    static constexpr bool kStaged = StagesParams<Op>::value;
    // a stage: NIN input tiles, then (WKV) the tile's u and w, [CG] fp32 each
    static constexpr size_t kParamOffset = Op::NIN * kTileElems * sizeof(typename Op::io_t);
    static constexpr size_t kStageBytes = kParamOffset + (kStaged ? 2 * CG * sizeof(float) : 0);
    static constexpr size_t kSmemBytes =
        NSTAGE * kStageBytes + static_cast<size_t>(NC) * (NWG + 1) * NV * CG * sizeof(float);
    static_assert(LT % NWG == 0, "tile length must split evenly over a group's warps");
    static_assert(LT <= 256, "TMA box rows are limited to 256");
    static_assert(NSTAGE > NC, "one stage per group plus at least one being loaded");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
    static_assert(kStageBytes % 128 == 0, "stage alignment");
    static_assert(2 + NC <= 16, "named barrier ids: 0, one per group, one for all consumers");
};

// Wait for phase `parity` of `bar`; false if the block is aborting or the
// deadline passed (which starts the abort).
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           const Workspace &ws) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kBarrierWaitNs) {
                *abort_flag = 1;
                if (ws.status != nullptr) atomicExch(ws.status, kStatusTimeout);
                return false;
            }
        }
    }
}

// Wait until `bar` has completed the phase that delivers ring iteration `it`
// into its stage.  Stages are shared by consumer groups, so a fast group can
// start waiting while the barrier still runs a phase two fills back, whose
// parity is the same as the one wanted; the stage's fill stamp (written by
// the producer before it arms the phase) tells the phases apart.
__device__ __forceinline__ bool wait_fill(uint64_t *bar, const int *fill_it, int it,
                                          uint32_t parity, volatile int *abort_flag,
                                          const Workspace &ws) {
    const volatile int *stamp = fill_it;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned n = 0;; ++n) {
        // try_wait suspends the warp in hardware until the phase completes
        // (or a time limit passes), so waiting costs no issue slots; a
        // completed phase whose stamp is not ours is an older fill of the
        // stage: back off until the producer re-arms it for this iteration
#if WKV_FILL_POLL
        if (mbar_test_wait(bar, parity)) {
            if (*stamp == it) return true;
        }
        __nanosleep(WKV_FILL_POLL);
#else
        if (mbar_try_wait(bar, parity)) {
            if (*stamp == it) return true;
            __nanosleep(64);
        }
#endif
        if ((n & 63u) == 63u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kBarrierWaitNs) {
                *abort_flag = 1;
                if (ws.status != nullptr) atomicExch(ws.status, kStatusTimeout);
                return false;
            }
        }
    }
}

template <class Op, int LT, int NWG, int NC, int NSTAGE>
__global__ void __launch_bounds__(PersistentCfg<Op, LT, NWG, NC, NSTAGE>::kThreads, 1)
    persistent_scan_kernel(const __grid_constant__ CUtensorMap map_x0,
                           const __grid_constant__ CUtensorMap map_x1,
                           const __grid_constant__ CUtensorMap map_y,
                           const __grid_constant__ CUtensorMap map_x2,  // NIN == 3 only
                           const typename Op::Args args, const Geometry g, const Workspace ws) {
    using Cfg = PersistentCfg<Op, LT, NWG, NC, NSTAGE>;
    using io_t = typename Op::io_t;
    using State = typename Op::State;
    using Param = typename Op::Param;
    constexpr int CPT = Cfg::CPT, NV = Cfg::NV, CG = Cfg::CG, LS = Cfg::LS;

    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char *s_stage = smem;  // [NSTAGE] x (NIN tiles [LT][CG], then u[CG], w[CG])
    float *s_sum = reinterpret_cast<float *>(smem + NSTAGE * Cfg::kStageBytes);  // [NC][NWG][NV][CG]
    float *s_carry = s_sum + NC * NWG * NV * CG;                                   // [NC][NV][CG]
    __shared__ __align__(8) uint64_t full_bar[NSTAGE];
    __shared__ __align__(8) uint64_t empty_bar[NSTAGE];
    __shared__ int s_meta[NSTAGE];      // tile id per stage, -1 = no more tiles
    __shared__ int s_fill_it[NSTAGE];   // ring iteration the stage was last filled for
    __shared__ int s_last_it[NSTAGE];   // last ring iteration loaded into each stage
    __shared__ int s_gtile[NC];         // each group's current tile, as its leader saw it
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
        fence_mbar_init();
        s_abort = 0;
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
            prefetch_tensormap(&map_x0);
            if constexpr (Op::NIN >= 2) prefetch_tensormap(&map_x1);
            prefetch_tensormap(&map_y);
            if constexpr (Op::NIN == 3) prefetch_tensormap(&map_x2);
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
                        // (one ticket per stage: handing a block consecutive
                        // tickets up front delays the tiles later ones depend on)
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
                    io_t *dst = reinterpret_cast<io_t *>(s_stage + static_cast<size_t>(s) * Cfg::kStageBytes);
                    s_last_it[s] = it;
                    // the tile's u and w, channels c0 .. c0 + CG clipped to C
                    // (C * 4 bytes is a multiple of 16 on the TMA path)
                    uint32_t pbytes = 0;
                    if constexpr (Cfg::kStaged)
                        if (g.params_staged)
                            pbytes = static_cast<uint32_t>(min(CG, g.C - c0)) *
                                     static_cast<uint32_t>(sizeof(float));
                    mbar_arrive_expect_tx(&full_bar[s],
                                          static_cast<uint32_t>(Cfg::kParamOffset) + 2 * pbytes);
                    if constexpr (Cfg::kStaged) {
                        if (pbytes > 0) {
                            float *dp = reinterpret_cast<float *>(
                                s_stage + static_cast<size_t>(s) * Cfg::kStageBytes + Cfg::kParamOffset);
                            bulk_load(dp, args.u + c0, pbytes, &full_bar[s]);
                            bulk_load(dp + CG, args.w + c0, pbytes, &full_bar[s]);
                        }
                    }
                    tma_load_3d(dst, &map_x0, &full_bar[s], c0 * Op::kScalarsPerIo, seg * LT, b);
                    if constexpr (Op::NIN >= 2)
                        tma_load_3d(dst + Cfg::kTileElems, &map_x1, &full_bar[s], c0 * Op::kScalarsPerIo, seg * LT, b);
                    if constexpr (Op::NIN == 3)
                        tma_load_3d(dst + 2 * Cfg::kTileElems, &map_x2, &full_bar[s],
                                    c0 * Op::kScalarsPerIo, seg * LT, b);
                }
            }
            // every tile of this block is loaded or assigned: the next grid in
            // the stream may start launching its blocks (its own
            // griddepcontrol.wait still waits for this grid to complete)
            allow_dependent_launch();
        }
        __syncwarp();
    } else {
        // ---------------- consumer group ----------------
        // the launch's epoch, read by one consumer thread while the producer
        // already takes tickets and starts loads
        if (threadIdx.x == 32) s_epoch = chained ? epoch_of(ws) : 0ull;
        named_bar_sync(NC + 1, NC * NWG * 32);
        const unsigned long long epoch = s_epoch;
        const int cw = warp - 1;
        const int grp = cw / NWG, wg = cw - grp * NWG;
        const int gtid = wg * 32 + lane;
        const int bar_id = 1 + grp;
        float *g_sum = s_sum + grp * NWG * NV * CG;
        float *g_carry = s_carry + grp * NV * CG;
        for (int it = grp;; it += NC) {
            const int s = it % NSTAGE;
            const uint32_t parity = (it / NSTAGE) & 1;
            // the group leader alone decides whether the stage arrived, so the
            // whole group leaves (or stays in) the loop together
            if (gtid == 0)
                s_gtile[grp] = wait_fill(&full_bar[s], &s_fill_it[s], it, parity, abort_flag, ws)
                                   ? s_meta[s]
                                   : -2;
            named_bar_sync(bar_id, NWG * 32);
            const int tile = s_gtile[grp];
            if (tile < 0) break;
            // the phase has completed; observing it makes the TMA writes visible
            // to this thread (the stage cannot be refilled before this group
            // releases it, so the phase stays complete)
            for (int n = 0; n < (1 << 20) && !mbar_try_wait(&full_bar[s], parity); ++n) {
            }
            const int seg = tile / g.tiles_per_seg;
            const int rem = tile - seg * g.tiles_per_seg;
            const int b = rem / g.n_cg;
            const int t0 = seg * LT;
            const int c0 = (rem - b * g.n_cg) * CG;
            io_t *s_x0 = reinterpret_cast<io_t *>(s_stage + static_cast<size_t>(s) * Cfg::kStageBytes);
            // the second input, when there is one; never read otherwise
            const io_t *s_x1 = Op::NIN >= 2 ? s_x0 + Cfg::kTileElems : s_x0;
            // the third input (r) when there is one; never read otherwise
            const io_t *s_x2 = Op::NIN == 3 ? s_x0 + 2 * Cfg::kTileElems : s_x1;

            Param prm[CPT];
            if constexpr (Cfg::kStaged) {
                if (g.params_staged) {
                    // staged with the tile: no global-memory round trip
                    const float *sp = reinterpret_cast<const float *>(
                        s_stage + static_cast<size_t>(s) * Cfg::kStageBytes + Cfg::kParamOffset);
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        prm[j] = Param{0.f, 0.f, 1.f, 1.f};
                        if (c0 + lane * CPT + j < g.C) {
                            prm[j].u = sp[lane * CPT + j];
                            prm[j].w = sp[CG + lane * CPT + j];
                            prm[j].U = expf(prm[j].u);
                            prm[j].D = expf(-prm[j].w);
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < CPT; ++j) prm[j] = Op::param(args, c0 + lane * CPT + j, g.C);
                }
            } else {
#pragma unroll
                for (int j = 0; j < CPT; ++j) prm[j] = Op::param(args, c0 + lane * CPT + j, g.C);
            }

            // the carry warps load the record their look-back reads first now:
            // the tile before this one in time was handed out well before it,
            // so its state is usually published already and lands during pass 1
            const bool lb = chained && seg > 0;
            ChannelPrefetch<WKV_LB_PREFETCH> pf;
#pragma unroll
            for (int j = 0; j < CPT; ++j)
                if (wg == j && lb) lookback_prefetch_channel<Op>(ws, g, tile, lane, j, pf);

            // pass 1
            const int s0 = wg * LS;
            const int nval = max(0, min(LS, g.T - (t0 + s0)));
            io_t *p0 = s_x0 + s0 * CG + lane * CPT;
            const io_t *p1 = s_x1 + s0 * CG + lane * CPT;
            typename Op::Scratch sc[CPT];
            {
                State st[CPT];
                Op::template summarize<LS>(p0, p1, nval, prm, st, sc);
#pragma unroll
                for (int j = 0; j < CPT; ++j)
#pragma unroll
                    for (int q = 0; q < NV; ++q)
                        g_sum[(wg * NV + q) * CG + lane * CPT + j] = Op::get(st[j], q);
            }
            named_bar_sync(bar_id, NWG * 32);

            // carry into the tile: channel j of every lane by the group's warp
            // j, so a lane's CPT channels resolve in parallel
            static_assert(CPT <= NWG, "one carry warp per channel of a lane");
#pragma unroll
            for (int j = 0; j < CPT; ++j) {  // j is a constant in each copy: prm[j] stays in registers
                if (wg != j) continue;
                // fold the warps' summaries in time order; each slot is
                // overwritten with its warp's exclusive prefix (the fold of the
                // sub-chunks before it) for pass 2
                State agg = Op::identity();
                for (int w = 0; w < NWG; ++w) {
                    float vals[NV];
                    float *slot = g_sum + w * NV * CG + lane * CPT + j;
#pragma unroll
                    for (int q = 0; q < NV; ++q) vals[q] = slot[q * CG];
#pragma unroll
                    for (int q = 0; q < NV; ++q) slot[q * CG] = Op::get(agg, q);
                    const int len = max(0, min(LS, g.T - (t0 + w * LS)));
                    agg = Op::combine(agg, Op::make(vals), static_cast<float>(len), prm[j]);
                }
                // the state before step 0 seeds the first segment only
                State X = seg == 0 ? Op::carry0(args, b, c0 + lane * CPT + j, g.C)
                                   : Op::identity();
                if (chained) {
                    const bool last = seg == g.n_seg - 1;
                    if (seg == 0) {
                        publish_channel<Op, CG>(ws, g, tile,
                                                Op::combine(X, agg, static_cast<float>(LT), prm[j]),
                                                j, kFlagIncl, epoch, lane);
                    } else {
                        if (!last) publish_channel<Op, CG>(ws, g, tile, agg, j, kFlagAgg, epoch, lane);
                        if (!lookback_channel<Op, LT>(ws, g, tile, epoch, prm[j], lane, j, X,
                                                      lb ? &pf : nullptr)) {
                            atomicExch(ws.status, kStatusTimeout);  // this lane gave up
                            X = Op::nan_state();
                        }
                        if (!last)
                            publish_channel<Op, CG>(
                                ws, g, tile, Op::combine(X, agg, static_cast<float>(LT), prm[j]), j,
                                kFlagIncl, epoch, lane);
                    }
                }
                if (seg == g.n_seg - 1)  // the state after the last step
                    Op::store_final(args, b, c0 + lane * CPT + j, g.C,
                                    Op::combine(X, agg, static_cast<float>(min(LT, g.T - t0)), prm[j]));
#pragma unroll
                for (int q = 0; q < NV; ++q) g_carry[q * CG + lane * CPT + j] = Op::get(X, q);
            }
            named_bar_sync(bar_id, NWG * 32);

            // pass 2: outputs over the stage's first tensor
            if (nval > 0) {
                State cur[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    float vals[NV];
#pragma unroll
                    for (int q = 0; q < NV; ++q) vals[q] = g_carry[q * CG + lane * CPT + j];
                    cur[j] = Op::make(vals);
                    if (wg > 0) {  // the sub-chunks before this warp's, all full
#pragma unroll
                        for (int q = 0; q < NV; ++q) vals[q] = g_sum[(wg * NV + q) * CG + lane * CPT + j];
                        cur[j] = Op::combine(cur[j], Op::make(vals), static_cast<float>(wg * LS), prm[j]);
                    }
                }
                Op::template sweep<LS>(cur, p0, p1, s_x2 + s0 * CG + lane * CPT, nval, prm, sc,
                                       p0, CG, true);
            }
            fence_proxy_async_smem();
            named_bar_sync(bar_id, NWG * 32);

            // store the tile (rows >= T and channels >= C are clipped), then
            // hand the stage back once the store has read it
            if (gtid == 0) {
                tma_store_3d(&map_y, s_x0, c0 * Op::kScalarsPerIo, t0, b);
                bulk_commit();
                bulk_wait_read_all();
                mbar_arrive(&empty_bar[s]);
            }
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
