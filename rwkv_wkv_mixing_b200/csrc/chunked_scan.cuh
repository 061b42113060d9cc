// Chunked two-pass time scan over [B, T, C] tensors for sm_100a.
//
// One thread block owns one tile: CG consecutive channels x LT consecutive
// steps of one batch row.  The tile's two input tensors are staged in shared
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

namespace wkvb {

constexpr uint32_t kFlagAgg = 1u;   // tile aggregate published
constexpr uint32_t kFlagIncl = 2u;  // state after the tile published
constexpr int kStatusTimeout = 4;   // == WKV_ERR_TIMEOUT

// Device pointers of one look-back workspace.  The three counters live in
// the workspace itself, so a launch needs no per-launch host state (CUDA-graph
// replays stay correct): blocks take tile tickets from `ticket`; the last
// block to finish resets `ticket` and `done` and advances `epoch`, which tags
// every flag this launch publishes so flags left by earlier launches never
// read as ready.  Launches sharing a workspace must run one after another
// (same stream).
struct Workspace {
    unsigned int *ticket;        // next tile ticket of the running launch
    unsigned int *done;          // blocks of the running launch that finished
    unsigned long long *epoch;   // launches completed on this workspace
    int *status;                 // device status word, 0 or an error code
    unsigned long long *flags;   // [tiles] (epoch << 2) | kFlag*
    float *agg;                  // [tiles][NV][CG] tile aggregates
    float *incl;                 // [tiles][NV][CG] states after each tile
};

struct Geometry {
    int B, T, C;           // batch rows, steps, channels
    int n_cg;              // channel groups per row, ceil(C / CG)
    int n_seg;             // time segments per row, ceil(T / LT)
    int tiles_per_seg;     // B * n_cg
    int tiles;             // n_seg * tiles_per_seg == gridDim.x
    int use_tma;           // 1: TMA tile copies; 0: element-wise copies
    long long spin_limit;  // polls of a predecessor's flag before giving up
};

// ---- vector access to CPT consecutive channels in shared memory -----------
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

template <typename io_t>
__device__ __forceinline__ io_t io_zero();
template <>
__device__ __forceinline__ float io_zero<float>() { return 0.f; }
template <>
__device__ __forceinline__ __nv_bfloat16 io_zero<__nv_bfloat16>() {
    return __float2bfloat16_rn(0.f);
}

// ---- publishing a per-tile value for the look-back -------------------------
template <class Op, int CG>
__device__ __forceinline__ void publish(float *base, unsigned long long *flags, int tile,
                                        const typename Op::State (&val)[Op::CPT],
                                        unsigned long long flag, int lane) {
    float *dst = base + static_cast<size_t>(tile) * Op::NV * CG;
#pragma unroll
    for (int j = 0; j < Op::CPT; ++j)
#pragma unroll
        for (int q = 0; q < Op::NV; ++q)
            st_relaxed_gpu(dst + q * CG + lane * Op::CPT + j, Op::get(val[j], q));
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu_u64(flags + tile, flag);
}

// Count this block as finished; the last block of the launch resets the
// ticket counter and advances the epoch for the next launch.  Every block
// has taken its ticket and finished all look-back reads by this point.
__device__ __forceinline__ void finish_launch(const Workspace &ws, const Geometry &g,
                                              bool chained, int tid) {
    if (!chained) return;
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(ws.done, 1u);
        if (prev == static_cast<unsigned int>(g.tiles) - 1u) {
            atomicExch(ws.ticket, 0u);
            atomicExch(ws.done, 0u);
            atomicAdd(ws.epoch, 1ull);
            __threadfence();
        }
    }
}

template <class Op, int LT, int NW>
constexpr size_t chunked_scan_smem_bytes() {
    return 2ull * LT * 32 * Op::CPT * sizeof(typename Op::io_t) +
           static_cast<size_t>(NW + 1) * Op::NV * 32 * Op::CPT * sizeof(float);
}

template <class Op, int LT, int NW>
__global__ void __launch_bounds__(NW * 32)
    chunked_scan_kernel(const __grid_constant__ CUtensorMap map_x0,
                        const __grid_constant__ CUtensorMap map_x1,
                        const __grid_constant__ CUtensorMap map_y,
                        const typename Op::Args args, const Geometry g, const Workspace ws) {
    using io_t = typename Op::io_t;
    using State = typename Op::State;
    using Param = typename Op::Param;
    constexpr int CPT = Op::CPT, NV = Op::NV, CG = 32 * CPT, LS = LT / NW;
    static_assert(LT % NW == 0, "tile length must split evenly over the warps");
    static_assert(LT <= 256, "TMA box rows are limited to 256");

    extern __shared__ __align__(128) unsigned char smem[];
    io_t *s_x0 = reinterpret_cast<io_t *>(smem);            // [LT][CG], outputs overwrite it
    io_t *s_x1 = s_x0 + LT * CG;                            // [LT][CG]
    float *s_sum = reinterpret_cast<float *>(s_x1 + LT * CG);  // [NW][NV][CG]
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
            epoch = ld_relaxed_gpu_u64(ws.epoch);
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
        finish_launch(ws, g, chained, tid);
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
            mbar_arrive_expect_tx(&s_bar, static_cast<uint32_t>(2 * LT * CG * sizeof(io_t)));
            tma_load_3d(s_x0, &map_x0, &s_bar, c0, t0, b);
            tma_load_3d(s_x1, &map_x1, &s_bar, c0, t0, b);
        }
    } else {
        for (int i = tid; i < LT * CG; i += NW * 32) {
            const int tl = i / CG, cl = i - (i / CG) * CG;
            const int t = t0 + tl, c = c0 + cl;
            io_t a = io_zero<io_t>(), bb = io_zero<io_t>();
            if (t < g.T && c < g.C) {
                const size_t o = (static_cast<size_t>(b) * g.T + t) * g.C + c;
                a = args.x0[o];
                bb = args.x1[o];
            }
            s_x0[i] = a;
            s_x1[i] = bb;
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
    const io_t *p0 = s_x0 + s0 * CG + lane * CPT;
    const io_t *p1 = s_x1 + s0 * CG + lane * CPT;
    {
        State st[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) st[j] = Op::identity();
        if (nval == LS) {
#pragma unroll 8
            for (int i = 0; i < LS; ++i) {
                float x0[CPT], x1[CPT];
                Vec<io_t, CPT>::load(p0 + i * CG, x0);
                Vec<io_t, CPT>::load(p1 + i * CG, x1);
#pragma unroll
                for (int j = 0; j < CPT; ++j) Op::step1(st[j], x0[j], x1[j], prm[j]);
            }
        } else {
            for (int i = 0; i < nval; ++i) {
                float x0[CPT], x1[CPT];
                Vec<io_t, CPT>::load(p0 + i * CG, x0);
                Vec<io_t, CPT>::load(p1 + i * CG, x1);
#pragma unroll
                for (int j = 0; j < CPT; ++j) Op::step1(st[j], x0[j], x1[j], prm[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < CPT; ++j)
#pragma unroll
            for (int q = 0; q < NV; ++q)
                s_sum[(warp * NV + q) * CG + lane * CPT + j] = Op::get(st[j], q);
    }
    __syncthreads();

    // ---- carry into the tile (warp 0) ---------------------------------------
    if (warp == 0) {
        State agg[CPT], X[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            agg[j] = Op::identity();
            for (int s = 0; s < NW; ++s) {
                float vals[NV];
#pragma unroll
                for (int q = 0; q < NV; ++q) vals[q] = s_sum[(s * NV + q) * CG + lane * CPT + j];
                const int len = max(0, min(LS, g.T - (t0 + s * LS)));
                agg[j] = Op::combine(agg[j], Op::make(vals), static_cast<float>(len), prm[j]);
            }
            X[j] = Op::carry0(args, b, c0 + lane * CPT + j, g.C);
        }
        if (chained) {
            const bool last = seg == g.n_seg - 1;
            if (seg == 0) {
                State inc[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j)
                    inc[j] = Op::combine(X[j], agg[j], static_cast<float>(LT), prm[j]);
                publish<Op, CG>(ws.incl, ws.flags, tile, inc, (epoch << 2) | kFlagIncl, lane);
            } else {
                if (!last)
                    publish<Op, CG>(ws.agg, ws.flags, tile, agg, (epoch << 2) | kFlagAgg, lane);
                // decoupled look-back over the tiles before this one in time
                State run[CPT];
#pragma unroll
                for (int j = 0; j < CPT; ++j) run[j] = Op::identity();
                float run_len = 0.f;
                int pred = tile - g.tiles_per_seg;
                bool failed = false;
                while (true) {
                    unsigned long long f = 0;
                    if (lane == 0) {
                        long long n = 0;
                        while (true) {
                            f = ld_acquire_gpu_u64(ws.flags + pred);
                            if ((f >> 2) == epoch && (f & 3u) != 0u) break;
                            if (++n > g.spin_limit) {
                                f = 0;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    f = __shfl_sync(0xffffffffu, f, 0);
                    if (f == 0) {
                        failed = true;
                        break;
                    }
                    // each lane acquires the flag itself before reading the data
                    (void)ld_acquire_gpu_u64(ws.flags + pred);
                    const bool inc = (f & 3u) == kFlagIncl;
                    const float *src =
                        (inc ? ws.incl : ws.agg) + static_cast<size_t>(pred) * NV * CG;
#pragma unroll
                    for (int j = 0; j < CPT; ++j) {
                        float vals[NV];
#pragma unroll
                        for (int q = 0; q < NV; ++q)
                            vals[q] = ld_relaxed_gpu(src + q * CG + lane * CPT + j);
                        run[j] = Op::combine(Op::make(vals), run[j], run_len, prm[j]);
                    }
                    if (inc) break;
                    run_len += static_cast<float>(LT);
                    pred -= g.tiles_per_seg;
                    if (pred < 0) {  // cannot happen: every first-segment tile publishes
                        failed = true;
                        break;
                    }
                }
                if (failed) {
                    if (lane == 0) atomicExch(ws.status, kStatusTimeout);
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
                    publish<Op, CG>(ws.incl, ws.flags, tile, inc, (epoch << 2) | kFlagIncl,
                                    lane);
                }
            }
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
            for (int s = 0; s < warp; ++s) {  // earlier sub-chunks are all full
#pragma unroll
                for (int q = 0; q < NV; ++q) vals[q] = s_sum[(s * NV + q) * CG + lane * CPT + j];
                cur[j] = Op::combine(cur[j], Op::make(vals), static_cast<float>(LS), prm[j]);
            }
        }
        io_t *q0 = s_x0 + s0 * CG + lane * CPT;
        if (nval == LS) {
#pragma unroll 8
            for (int i = 0; i < LS; ++i) {
                float x0[CPT], x1[CPT], y[CPT];
                Vec<io_t, CPT>::load(p0 + i * CG, x0);
                Vec<io_t, CPT>::load(p1 + i * CG, x1);
#pragma unroll
                for (int j = 0; j < CPT; ++j) y[j] = Op::step2(cur[j], x0[j], x1[j], prm[j]);
                Vec<io_t, CPT>::store(q0 + i * CG, y);
            }
        } else {
            for (int i = 0; i < nval; ++i) {
                float x0[CPT], x1[CPT], y[CPT];
                Vec<io_t, CPT>::load(p0 + i * CG, x0);
                Vec<io_t, CPT>::load(p1 + i * CG, x1);
#pragma unroll
                for (int j = 0; j < CPT; ++j) y[j] = Op::step2(cur[j], x0[j], x1[j], prm[j]);
                Vec<io_t, CPT>::store(q0 + i * CG, y);
            }
        }
    }

    // ---- write the output tile ----------------------------------------------
    if (g.use_tma) {
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&map_y, s_x0, c0, t0, b);  // rows >= T, channels >= C are clipped
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
    finish_launch(ws, g, chained, tid);
}

}  // namespace wkvb
