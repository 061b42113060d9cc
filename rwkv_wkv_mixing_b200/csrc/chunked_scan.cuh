// Chunked two-pass time scan over [B, T, C] tensors for sm_100a.
//
// One thread block owns one tile: CG consecutive channels x LT consecutive
// steps of one batch row.  The tile's input tensors (NIN of them) are staged in shared
// memory once (TMA tile copies, or element-wise copies when the tensor cannot
// be described by a tensor map), so HBM sees every input element once and
// every output element once.
//
//   pass 1   each warp reduces its LS = LT/NW steps of every channel to a
//            chunk summary (the state the chunk produces from the empty state)
//   carry    warp 0 folds the NW summaries into the tile aggregate and, when
//            the sequence spans several tiles, obtains the state before the
//            tile by a decoupled look-back over the tiles before it in time
//            (Merrill & Garland, "Single-pass Parallel Prefix Scan with
//            Decoupled Look-back"); then publishes its own inclusive state
//   pass 2   each warp re-sweeps its steps from its carried-in state and
//            writes the outputs over the first input tile in shared memory,
//            which is then copied out (TMA store, or element-wise)
//
// The chunk identity behind pass 1 / carry / pass 2 is the Upper/Lower split
// of a linear recurrence (review of "Resurrecting Recurrent Neural Networks
// for Long Sequences", parallelisation section): the state after a chunk is
// the state before it carried across the chunk, plus what the chunk produces
// from the empty state.
//
// Operation-specific arithmetic lives in an Op policy (wkv_ops.cuh):
//   io_t, CPT (channels per thread), NV (floats per state), Param, State,
//   Args {x0, x1, y, ...}, param(), identity(), carry0(), combine(), step1(),
//   step2(), get(), make(), nan_state().
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "scan_common.cuh"

namespace wkvb {

template <class Op, int LT, int NW>
constexpr size_t chunked_scan_smem_bytes() {
    return static_cast<size_t>(Op::NIN) * LT * 32 * Op::CPT * sizeof(typename Op::io_t) +
           static_cast<size_t>(NW + 1) * Op::NV * 32 * Op::CPT * sizeof(float);
}

template <class Op, int LT, int NW>
__global__ void __launch_bounds__(NW * 32, 3)
    chunked_scan_kernel(const __grid_constant__ CUtensorMap map_x0,
                        const __grid_constant__ CUtensorMap map_x1,
                        const __grid_constant__ CUtensorMap map_y,
                        const __grid_constant__ CUtensorMap map_x2,  // NIN == 3 only
                        const typename Op::Args args, const Geometry g, const Workspace ws) {
    using io_t = typename Op::io_t;
    using State = typename Op::State;
    using Param = typename Op::Param;
    constexpr int CPT = Op::CPT, NV = Op::NV, CG = 32 * CPT, LS = LT / NW;
    static_assert(LT % NW == 0, "tile length must split evenly over the warps");
    static_assert(LT <= 256, "TMA box rows are limited to 256");

    extern __shared__ __align__(128) unsigned char smem[];
    io_t *s_x0 = reinterpret_cast<io_t *>(smem);            // [LT][CG], outputs overwrite it
    io_t *s_x1 = s_x0 + (Op::NIN >= 2 ? LT * CG : 0);       // [LT][CG], when NIN >= 2
    io_t *s_x2 = s_x0 + (Op::NIN == 3 ? 2 * LT * CG : 0);   // [LT][CG] r, when NIN == 3
    float *s_sum = reinterpret_cast<float *>(s_x0 + Op::NIN * LT * CG);  // [NW][NV][CG]
    float *s_carry = s_sum + NW * NV * CG;                   // [NV][CG]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_tile;
    __shared__ unsigned long long s_epoch;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool chained = g.n_seg > 1;

    if (tid == 0) {
        int tile = static_cast<int>(blockIdx.x);
        unsigned long long epoch = 0;
        if (chained) {
            // Tickets hand out tiles in the order blocks start running, so
            // every tile this block waits for belongs to a block that is
            // already resident: the look-back always makes progress.
            tile = static_cast<int>(atomicAdd(ws.ticket, 1u));
            epoch = epoch_of(ws);
            if (tile >= g.tiles) {  // counters corrupted: report, do no work
                atomicExch(ws.status, kStatusTimeout);
                tile = -1;
            }
        }
        s_tile = tile;
        s_epoch = epoch;
        if (g.use_tma) {
            mbar_init(&s_bar, 1);
            fence_mbar_init();
        }
    }
    __syncthreads();
    const int tile = s_tile;
    if (tile < 0) {
        finish_launch(ws, chained, tid, static_cast<unsigned>(g.tiles));
        return;
    }
    const unsigned long long epoch = s_epoch;
    const int seg = tile / g.tiles_per_seg;
    const int rem = tile - seg * g.tiles_per_seg;
    const int b = rem / g.n_cg;
    const int t0 = seg * LT;
    const int c0 = (rem - b * g.n_cg) * CG;

    // ---- stage the tile ---------------------------------------------------
    if (g.use_tma) {
        if (tid == 0) {
            mbar_arrive_expect_tx(&s_bar,
                                  static_cast<uint32_t>(Op::NIN * LT * CG * sizeof(io_t)));
            tma_load_3d(s_x0, &map_x0, &s_bar, c0 * Op::kScalarsPerIo, t0, b);
            if constexpr (Op::NIN >= 2) tma_load_3d(s_x1, &map_x1, &s_bar, c0 * Op::kScalarsPerIo, t0, b);
            if constexpr (Op::NIN == 3) tma_load_3d(s_x2, &map_x2, &s_bar, c0 * Op::kScalarsPerIo, t0, b);
        }
    } else {
        for (int i = tid; i < LT * CG; i += NW * 32) {
            const int tl = i / CG, cl = i - (i / CG) * CG;
            const int t = t0 + tl, c = c0 + cl;
            io_t a = io_zero<io_t>(), bb = io_zero<io_t>(), rr = io_zero<io_t>();
            if (t < g.T && c < g.C) {
                const size_t o = (static_cast<size_t>(b) * g.T + t) * g.C + c;
                a = args.x0[o];
                if constexpr (Op::NIN >= 2) bb = args.x1[o];
                if constexpr (Op::NIN == 3) rr = args.x2[o];
            }
            s_x0[i] = a;
            if constexpr (Op::NIN >= 2) s_x1[i] = bb;
            if constexpr (Op::NIN == 3) s_x2[i] = rr;
        }
    }
    Param prm[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) prm[j] = Op::param(args, c0 + lane * CPT + j, g.C);

    if (g.use_tma) {
        long long n = 0;
        while (!mbar_try_wait(&s_bar, 0)) {
            if (++n > (1ll << 22)) {  // the copy never landed: report, do not hang
                if (lane == 0 && ws.status != nullptr) atomicExch(ws.status, kStatusTimeout);
                break;
            }
        }
    } else {
        __syncthreads();
    }

    // ---- pass 1: summary of this warp's sub-chunk ---------------------------
    const int s0 = warp * LS;
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
                s_sum[(warp * NV + q) * CG + lane * CPT + j] = Op::get(st[j], q);
    }
    __syncthreads();

    // ---- carry into the tile (warp 0) ---------------------------------------
    if (warp == 0) {
        // the look-back's first records are loaded now and land while the
        // warp folds and publishes this tile's aggregate
        LookbackPrefetch<Op> pf;
        const bool lb = chained && seg > 0;
        if (lb) lookback_prefetch<Op>(ws, g, tile, lane, pf);
        State agg[CPT], X[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            // fold the warps' summaries in time order; each slot is
            // overwritten with its warp's exclusive prefix (the fold of the
            // sub-chunks before it) for pass 2
            agg[j] = Op::identity();
            for (int s = 0; s < NW; ++s) {
                float vals[NV];
                float *slot = s_sum + s * NV * CG + lane * CPT + j;
#pragma unroll
                for (int q = 0; q < NV; ++q) vals[q] = slot[q * CG];
#pragma unroll
                for (int q = 0; q < NV; ++q) slot[q * CG] = Op::get(agg[j], q);
                const int len = max(0, min(LS, g.T - (t0 + s * LS)));
                agg[j] = Op::combine(agg[j], Op::make(vals), static_cast<float>(len), prm[j]);
            }
            // the state before step 0 seeds the first segment only
            X[j] = seg == 0 ? Op::carry0(args, b, c0 + lane * CPT + j, g.C) : Op::identity();
        }
        if (chained) {
            const bool last = seg == g.n_seg - 1;
            if (seg == 0) {
                State inc[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j)
                    inc[j] = Op::combine(X[j], agg[j], static_cast<float>(LT), prm[j]);
                publish<Op, CG>(ws, g, tile, inc, kFlagIncl, epoch, lane);
            } else {
                if (!last)
                    publish<Op, CG>(ws, g, tile, agg, kFlagAgg, epoch, lane);
                // decoupled look-back over the tiles before this one in time
                State run[CPT];
                if (!lookback<Op, LT>(ws, g, tile, epoch, prm, lane, run, lb ? &pf : nullptr)) {
                    atomicExch(ws.status, kStatusTimeout);  // this lane gave up
#pragma unroll
                    for (int j = 0; j < CPT; ++j) run[j] = Op::nan_state();
                }
#pragma unroll
                for (int j = 0; j < CPT; ++j) X[j] = run[j];
                if (!last) {
                    State inc[CPT];
#pragma unroll
                    for (int j = 0; j < CPT; ++j)
                        inc[j] = Op::combine(X[j], agg[j], static_cast<float>(LT), prm[j]);
                    publish<Op, CG>(ws, g, tile, inc, kFlagIncl, epoch, lane);
                }
            }
        }
        if (seg == g.n_seg - 1) {  // the state after the last step
            const float len = static_cast<float>(min(LT, g.T - t0));
#pragma unroll
            for (int j = 0; j < CPT; ++j)
                Op::store_final(args, b, c0 + lane * CPT + j, g.C,
                                Op::combine(X[j], agg[j], len, prm[j]));
        }
#pragma unroll
        for (int j = 0; j < CPT; ++j)
#pragma unroll
            for (int q = 0; q < NV; ++q) s_carry[q * CG + lane * CPT + j] = Op::get(X[j], q);
    }
    __syncthreads();

    // ---- pass 2: re-sweep from the carried-in state, outputs over s_x0 ------
    if (nval > 0) {
        State cur[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            float vals[NV];
#pragma unroll
            for (int q = 0; q < NV; ++q) vals[q] = s_carry[q * CG + lane * CPT + j];
            cur[j] = Op::make(vals);
            if (warp > 0) {  // the sub-chunks before this warp's, all full
#pragma unroll
                for (int q = 0; q < NV; ++q) vals[q] = s_sum[(warp * NV + q) * CG + lane * CPT + j];
                cur[j] = Op::combine(cur[j], Op::make(vals), static_cast<float>(warp * LS), prm[j]);
            }
        }
        Op::template sweep<LS>(cur, p0, p1, s_x2 + s0 * CG + lane * CPT, nval, prm, sc, p0, CG,
                               true);
    }

    // ---- write the output tile ----------------------------------------------
    if (g.use_tma) {
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&map_y, s_x0, c0 * Op::kScalarsPerIo, t0, b);  // rows >= T, channels >= C are clipped
            bulk_commit();
            bulk_wait_read_all();
        }
    } else {
        __syncthreads();
        for (int i = tid; i < LT * CG; i += NW * 32) {
            const int tl = i / CG, cl = i - (i / CG) * CG;
            const int t = t0 + tl, c = c0 + cl;
            if (t < g.T && c < g.C)
                args.y[(static_cast<size_t>(b) * g.T + t) * g.C + c] = s_x0[i];
        }
    }
    finish_launch(ws, chained, tid, static_cast<unsigned>(g.tiles));
}

}  // namespace wkvb
