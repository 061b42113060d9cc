// Pieces shared by the two scan kernels: the look-back workspace, problem
// geometry, publishing a tile's value and the decoupled look-back itself.
//
// The tiles of one (batch row, channel group) form a chain in time: tile
// number `seg * S + r` (S = tiles per time segment) follows `(seg-1) * S + r`.
// A tile publishes its aggregate (the state its steps produce from the empty
// state) as soon as it has it, looks back over its predecessors for the state
// before itself, and publishes the state after itself (Merrill & Garland,
// "Single-pass Parallel Prefix Scan with Decoupled Look-back").
//
// What is published is one 16-byte record per (tile, channel): two state
// floats and a 64-bit tag, written and read with single aligned vector
// accesses.  The tag says whether the record holds the aggregate or the state
// after the tile, carries the launch's epoch (so records left by earlier
// launches never read as current) and 16 bits the operation may use to
// complete its state.  A record is self-contained: no fence orders it against
// anything else, and one load both polls and reads it.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace wkvb {

constexpr uint32_t kFlagAgg = 1u;   // record holds the tile aggregate
constexpr uint32_t kFlagIncl = 2u;  // record holds the state after the tile
constexpr int kStatusTimeout = 4;   // == WKV_ERR_TIMEOUT
constexpr int kEpochBits = 46;      // tag: epoch(46) | op bits(16) | flag(2)

// Device pointers of one look-back workspace.  The counters live in the
// workspace itself, so a launch needs no per-launch host state (CUDA-graph
// replays stay correct): blocks take tile tickets from `ticket`; the last
// block to finish resets `ticket` and `done` and advances `epoch`.  Launches
// sharing a workspace must run one after another (same stream).
struct Workspace {
    unsigned int *ticket;        // next tile ticket of the running launch
    unsigned int *done;          // blocks of the running launch that finished
    unsigned long long *epoch;   // launches completed on this workspace
    int *status;                 // device status word, 0 or an error code
    uint4 *records;              // [tiles][CG] published states
};

struct Geometry {
    int B, T, C;           // batch rows, steps, channels
    int n_cg;              // channel groups per row, ceil(C / CG)
    int n_seg;             // time segments per row, ceil(T / LT)
    int tiles_per_seg;     // B * n_cg
    int tiles;             // n_seg * tiles_per_seg
    int use_tma;           // 1: TMA tile copies; 0: element-wise copies
    long long spin_limit;  // polls of one predecessor record before giving up
    int skip_publish;      // test hook: this tile publishes nothing (-1: none)
    // 1: the producer stages each tile's per-channel parameters (WKV: u and
    // w) with the tile's inputs, so consumers read them from shared memory
    // instead of global memory (needs 16-byte aligned parameter arrays)
    int params_staged = 0;
};

template <typename io_t>
__device__ __forceinline__ io_t io_zero();
template <>
__device__ __forceinline__ float io_zero<float>() { return 0.f; }
template <>
__device__ __forceinline__ float2 io_zero<float2>() { return make_float2(0.f, 0.f); }
template <>
__device__ __forceinline__ __nv_bfloat16 io_zero<__nv_bfloat16>() {
    return __float2bfloat16_rn(0.f);
}

__device__ __forceinline__ unsigned long long epoch_of(const Workspace &ws) {
    return ld_relaxed_gpu_u64(ws.epoch) & ((1ull << kEpochBits) - 1ull);
}

// Publish channel j of this lane's CPT channels of `tile` with the given
// flag.  (The fault-injection test hook can name one tile that never
// publishes, so that the look-back waits behind it run out.)
template <class Op, int CG>
__device__ __forceinline__ void publish_channel(const Workspace &ws, const Geometry &g, int tile,
                                                const typename Op::State &val, int j,
                                                uint32_t flag, unsigned long long epoch,
                                                int lane) {
    if (tile == g.skip_publish) return;
    uint4 *dst = ws.records + static_cast<size_t>(tile) * CG + lane * Op::CPT + j;
    float x, y;
    uint32_t bits16;
    Op::pack(val, x, y, bits16);
    const unsigned long long tag =
        (epoch << 18) | (static_cast<unsigned long long>(bits16 & 0xffffu) << 2) | flag;
    st_relaxed_gpu_v4(dst, make_uint4(__float_as_uint(x), __float_as_uint(y),
                                      static_cast<uint32_t>(tag), static_cast<uint32_t>(tag >> 32)));
}

// all CPT channels of this lane
template <class Op, int CG>
__device__ __forceinline__ void publish(const Workspace &ws, const Geometry &g, int tile,
                                        const typename Op::State (&val)[Op::CPT], uint32_t flag,
                                        unsigned long long epoch, int lane) {
#pragma unroll
    for (int j = 0; j < Op::CPT; ++j) publish_channel<Op, CG>(ws, g, tile, val[j], j, flag, epoch, lane);
}

__device__ __forceinline__ unsigned long long record_tag(uint4 r) {
    return (static_cast<unsigned long long>(r.w) << 32) | r.z;
}

// Count this block as finished; the last of the `blocks` increments a
// launch makes resets the ticket counter and advances the epoch for the next
// launch.  Every block has taken its tickets and finished all look-back reads
// by this point.  Thread `tid` (0) is the one that took the block's tickets:
// its count is a release, so those tickets come before it, and the last
// count acquires every earlier one, so the reset comes after every ticket of
// the launch.  The next launch sees the reset and the new epoch by the
// kernel boundary.
__device__ __forceinline__ void finish_launch(const Workspace &ws, bool chained, int tid,
                                              unsigned blocks) {
    if (!chained) return;
    __syncthreads();
    if (tid == 0) {
        const unsigned int prev = atom_add_acq_rel_gpu(ws.done, 1u);
        if (prev == blocks - 1u) {
            atomicExch(ws.ticket, 0u);
            atomicExch(ws.done, 0u);
            atomicAdd(ws.epoch, 1ull);
        }
    }
}

// The first records a tile's look-back will read, loaded ahead of time: the
// look-back does not depend on the tile's own data, so the carry warp issues
// these loads before it folds and publishes its own aggregate, and they land
// while it does.  H hops of one channel.
template <int H>
struct ChannelPrefetch {
    static constexpr int kHops = H;
    uint4 rec[H];
};

template <class Op, int H>
__device__ __forceinline__ void lookback_prefetch_channel(const Workspace &ws, const Geometry &g,
                                                          int tile, int lane, int j,
                                                          ChannelPrefetch<H> &pf) {
    constexpr int CPT = Op::CPT, CG = 32 * CPT;
    const long long S = g.tiles_per_seg;
#pragma unroll
    for (int i = 0; i < H; ++i) {
        const long long q = static_cast<long long>(tile) - (i + 1) * S;
        pf.rec[i] = make_uint4(0u, 0u, 0u, 0u);
        if (q >= 0) pf.rec[i] = ld_relaxed_gpu_v4(ws.records + q * CG + lane * CPT + j);
    }
}

// every channel of this lane, 4 records in all
template <class Op>
struct LookbackPrefetch {
    ChannelPrefetch<4 / Op::CPT> ch[Op::CPT];
};

template <class Op>
__device__ __forceinline__ void lookback_prefetch(const Workspace &ws, const Geometry &g, int tile,
                                                  int lane, LookbackPrefetch<Op> &pf) {
#pragma unroll
    for (int j = 0; j < Op::CPT; ++j) lookback_prefetch_channel<Op>(ws, g, tile, lane, j, pf.ch[j]);
}

// Decoupled look-back for one tile, channel j of this lane's CPT channels.
// The tiles before this one in time are tile - S, tile - 2S, ... (S = tiles
// per time segment).  The lane folds its channel's records newest first -- a
// tile aggregate moves the fold one tile further back, a state-after-tile
// ends it -- prefetching several hops' records with independent loads.
// Lanes may stop at different hops; each ends with the state before this
// tile.  Returns false if a record never appeared within the poll budget.
template <class Op, int LT, int H, int HB = 4>  // HB: hops per batch of loads
__device__ __forceinline__ bool lookback_channel(const Workspace &ws, const Geometry &g, int tile,
                                                 unsigned long long epoch,
                                                 const typename Op::Param &prm, int lane, int j,
                                                 typename Op::State &run,
                                                 const ChannelPrefetch<H> *pre) {
    constexpr int CPT = Op::CPT, CG = 32 * CPT;
    const long long S = g.tiles_per_seg;
    run = Op::identity();
    float run_len = 0.f;
    long long base = tile;
    bool first = true;
    for (;;) {
        uint4 rec[HB];
#pragma unroll
        for (int i = 0; i < HB; ++i) {
            const long long q = base - (i + 1) * S;
            rec[i] = make_uint4(0u, 0u, 0u, 0u);
            if (first && pre != nullptr && i < H)
                rec[i] = pre->rec[i];   // possibly stale: re-polled below if not ready
            else if (q >= 0)
                rec[i] = ld_relaxed_gpu_v4(ws.records + q * CG + lane * CPT + j);
        }
        first = false;
#pragma unroll
        for (int i = 0; i < HB; ++i) {
            const long long q = base - (i + 1) * S;
            if (q < 0) return false;  // cannot happen: first-segment tiles always end the fold
            uint4 r = rec[i];
            long long polls = 0;
            while (((record_tag(r) >> 18) != epoch) || (record_tag(r) & 3u) == 0u) {
                if (++polls > g.spin_limit) return false;
                __nanosleep(32);
                r = ld_relaxed_gpu_v4(ws.records + q * CG + lane * CPT + j);
            }
            const unsigned long long tag = record_tag(r);
            const typename Op::State val = Op::unpack(
                __uint_as_float(r.x), __uint_as_float(r.y), static_cast<uint32_t>(tag >> 2) & 0xffffu);
            run = Op::combine(val, run, run_len, prm);
            run_len += static_cast<float>(LT);
            if ((tag & 3u) == kFlagIncl) return true;
        }
        base -= HB * S;
    }
}

// all CPT channels of this lane, one after another; false (in every lane
// that gave up) if a record never appeared within the poll budget
template <class Op, int LT>
__device__ __forceinline__ bool lookback(const Workspace &ws, const Geometry &g, int tile,
                                         unsigned long long epoch,
                                         const typename Op::Param (&prm)[Op::CPT], int lane,
                                         typename Op::State (&run)[Op::CPT],
                                         const LookbackPrefetch<Op> *pre = nullptr) {
    bool ok = true;
#pragma unroll
    for (int j = 0; j < Op::CPT; ++j) {
        if (!ok) {
            run[j] = Op::identity();
            continue;
        }
        ok = lookback_channel<Op, LT>(ws, g, tile, epoch, prm[j], lane, j, run[j],
                                      pre != nullptr ? &pre->ch[j] : nullptr);
    }
    return ok;
}

}  // namespace wkvb
