// Pieces shared by the two scan kernels: the look-back workspace, problem
// geometry, publishing a tile's value and the decoupled look-back itself.
//
// The tiles of one (batch row, channel group) form a chain in time: tile
// number `seg * S + r` (S = tiles per time segment) follows `(seg-1) * S + r`.
// A tile publishes its aggregate (the state its steps produce from the empty
// state) as soon as it has it, looks back over its predecessors for the state
// before itself, and publishes the state after itself (Merrill & Garland,
// "Single-pass Parallel Prefix Scan with Decoupled Look-back").
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

// Count this block as finished; the last of the `blocks` increments a
// launch makes resets the ticket counter and advances the epoch for the next
// launch.  Every block has taken its tickets and finished all look-back reads
// by this point.
__device__ __forceinline__ void finish_launch(const Workspace &ws, bool chained, int tid,
                                              unsigned blocks) {
    if (!chained) return;
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(ws.done, 1u);
        if (prev == blocks - 1u) {
            atomicExch(ws.ticket, 0u);
            atomicExch(ws.done, 0u);
            atomicAdd(ws.epoch, 1ull);
            __threadfence();
        }
    }
}

// Decoupled look-back for one tile, run by one warp.  The tiles before this
// one in time are tile - S, tile - 2S, ... (S = tiles per time segment).
// Lanes poll the flags of a window of 32 predecessors at once; the window is
// folded (newest first, lanes now acting as channels) up to the nearest
// predecessor that has published the state after itself, or entirely when
// all 32 have published only their aggregates, in which case the next window
// follows.  Returns false if a flag never appeared within the poll budget.
template <class Op, int LT>
__device__ __forceinline__ bool lookback(const Workspace &ws, const Geometry &g, int tile,
                                         unsigned long long epoch,
                                         const typename Op::Param (&prm)[Op::CPT], int lane,
                                         typename Op::State (&run)[Op::CPT]) {
    constexpr int CPT = Op::CPT, NV = Op::NV, CG = 32 * CPT;
    const int S = g.tiles_per_seg;
#pragma unroll
    for (int j = 0; j < CPT; ++j) run[j] = Op::identity();
    float run_len = 0.f;
    int base = tile;
    while (true) {
        const long long q = static_cast<long long>(base) - static_cast<long long>(lane + 1) * S;
        const bool exists = q >= 0;  // this lane's predecessor in time
        unsigned long long f = 0;
        bool rdy = false;
        int last = -1;        // fold lanes 0..last
        bool found = false;   // lane `last` holds a state-after-tile
        long long polls = 0;
        while (true) {
            if (exists && !rdy) {
                f = ld_acquire_gpu_u64(ws.flags + q);
                rdy = (f >> 2) == epoch && (f & 3u) != 0u;
            }
            const unsigned rdym = __ballot_sync(0xffffffffu, rdy);
            const unsigned incm = __ballot_sync(0xffffffffu, rdy && (f & 3u) == kFlagIncl);
            const unsigned exm = __ballot_sync(0xffffffffu, exists);
            if (incm != 0u) {
                const int h = __ffs(incm) - 1;
                const unsigned need = h == 31 ? 0xffffffffu : ((1u << (h + 1)) - 1u);
                if ((rdym & need) == need) {
                    last = h;
                    found = true;
                    break;
                }
            } else if (exm == 0xffffffffu && rdym == 0xffffffffu) {
                last = 31;  // 32 aggregates, none final yet: fold them, look further
                break;
            }
            if (++polls > g.spin_limit) return false;
            __nanosleep(32);
        }
        // every lane fences after its own acquire, so data published before
        // any of the observed flags is visible to the whole warp
        __syncwarp();
        __threadfence();
        // fold the window newest-first; the loads of several hops are issued
        // together so a window costs a few memory latencies, not one per hop
        constexpr int HB = 8 / CPT;  // hops per batch of loads
        for (int h0 = 0; h0 <= last; h0 += HB) {
            float vals[HB][CPT][NV];
#pragma unroll
            for (int hh = 0; hh < HB; ++hh) {
                const int h = h0 + hh;
                const unsigned long long fh = __shfl_sync(0xffffffffu, f, h & 31);
                if (h <= last) {
                    const long long qh =
                        static_cast<long long>(base) - static_cast<long long>(h + 1) * S;
                    const float *src = ((fh & 3u) == kFlagIncl ? ws.incl : ws.agg) +
                                       static_cast<size_t>(qh) * NV * CG;
#pragma unroll
                    for (int j = 0; j < CPT; ++j)
#pragma unroll
                        for (int v = 0; v < NV; ++v)
                            vals[hh][j][v] = ld_relaxed_gpu(src + v * CG + lane * CPT + j);
                }
            }
#pragma unroll
            for (int hh = 0; hh < HB; ++hh) {
                if (h0 + hh <= last) {
#pragma unroll
                    for (int j = 0; j < CPT; ++j)
                        run[j] = Op::combine(Op::make(vals[hh][j]), run[j], run_len, prm[j]);
                    run_len += static_cast<float>(LT);
                }
            }
        }
        if (found) return true;
        base -= 32 * S;  // all 32 existed, so base - 32 S >= 0
    }
}

}  // namespace wkvb
