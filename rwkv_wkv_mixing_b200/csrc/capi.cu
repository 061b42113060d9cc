// C ABI of libwkv_b200.so: argument checks, tensor maps, per-stream
// workspaces and kernel dispatch.  The declarations and their contracts are
// in include/wkv_b200.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "chunked_scan.cuh"
#include "lru_ops.cuh"
#include "persistent_bwd.cuh"
#include "persistent_scan.cuh"
#include "persistent_wkv.cuh"
#include "serial_wkv.cuh"
#include "wkv_backward.cuh"
#include "token_shift.cuh"
#include "wkv_b200.h"
#include "wkv_ops.cuh"

using namespace wkvb;

namespace {
thread_local std::string t_err;
}

namespace wkvb {
// lets the library's other translation units set the wkv_last_error() message
void set_last_error(const char *msg) { t_err = msg; }
}  // namespace wkvb

namespace {

wkv_status fail(wkv_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_err = buf;
    return st;
}

wkv_status cuda_fail(cudaError_t e, const char *what) {
    return fail(WKV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---- driver entry points (no link-time dependency on libcuda) --------------
struct Driver {
    PFN_cuTensorMapEncodeTiled_v12000 encode_tiled = nullptr;
    PFN_cuMemGetAddressRange_v3020 get_address_range = nullptr;
};

const Driver &driver() {
    static Driver d;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            d.encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            d.get_address_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(p);
        cudaGetLastError();
    });
    return d;
}

// ---- tuning knob: tile length in steps ---------------------------------------
std::atomic<int> g_tile_steps{0};  // 0: chosen per call (tile_steps_for)

// ---- fault-injection test hook (see wkv_set_fault_injection) -----------------
std::atomic<int> g_fault_skip_tile{-1};
std::atomic<long long> g_fault_spin_limit{0};

// ---- argument checks ------------------------------------------------------------
// `p` must be device (or managed) memory of device `dev` holding `bytes`.
wkv_status check_buffer(const void *p, size_t bytes, size_t align, const char *name, int dev) {
    if (p == nullptr) return fail(WKV_ERR_INVALID_ARG, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % align != 0)
        return fail(WKV_ERR_ALIGNMENT, "%s is not %zu-byte aligned", name, align);
    cudaPointerAttributes attr;
    cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(WKV_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorName(e));
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
        return fail(WKV_ERR_INVALID_ARG, "%s is not device memory", name);
    if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
        return fail(WKV_ERR_INVALID_ARG, "%s lives on device %d, current device is %d", name,
                    attr.device, dev);
    const Driver &d = driver();
    if (d.get_address_range != nullptr) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (d.get_address_range(&base, &size, reinterpret_cast<CUdeviceptr>(p)) == CUDA_SUCCESS) {
            const uintptr_t end = static_cast<uintptr_t>(base) + size;
            if (reinterpret_cast<uintptr_t>(p) + bytes > end)
                return fail(WKV_ERR_INVALID_ARG,
                            "%s: %zu bytes needed but its allocation ends %zu bytes after it",
                            name, bytes, static_cast<size_t>(end - reinterpret_cast<uintptr_t>(p)));
        }
    }
    return WKV_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

wkv_status check_sizes(int64_t B, int64_t T, int64_t C, bool *empty) {
    if (B < 0 || T < 0 || C < 0)
        return fail(WKV_ERR_INVALID_ARG, "negative size (B=%lld T=%lld C=%lld)",
                    static_cast<long long>(B), static_cast<long long>(T),
                    static_cast<long long>(C));
    *empty = B == 0 || T == 0 || C == 0;
    if (*empty) return WKV_OK;
    if (B > INT32_MAX || T > INT32_MAX || C > INT32_MAX)
        return fail(WKV_ERR_INVALID_ARG, "each of B, T, C must be below 2^31");
    const unsigned __int128 n = static_cast<unsigned __int128>(B) * T * C;
    if (n >= (static_cast<unsigned __int128>(1) << 62))
        return fail(WKV_ERR_INVALID_ARG, "B*T*C must be below 2^62");
    return WKV_OK;
}

// ---- per-(device, stream) workspaces for the cross-tile look-back -------------
// A workspace is only ever used by launches on its own stream, which run one
// after another; its counters reset themselves on the device (see Workspace in
// chunked_scan.cuh).  When a larger problem needs a larger workspace the old
// buffer is retired, not freed, so CUDA graphs captured earlier keep valid
// pointers; wkv_release_workspaces() frees everything.
struct WsEntry {
    int device = -1;
    cudaStream_t stream = nullptr;
    int kind = 0;  // 0: look-back workspace; 1: gradient scratch; 2: gradient sum counters
    char *base = nullptr;
    size_t bytes = 0;
};

std::mutex g_mu;                  // guards g_ws and g_retired
std::vector<WsEntry *> g_ws;
std::vector<std::pair<int, void *>> g_retired;  // (device, buffer)

// header: [0] u32 ticket, [4] u32 done, [8] u64 epoch, [16] i32 status
constexpr size_t kWsHeader = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// header, then one 16-byte record per (tile, channel)
size_t ws_bytes(size_t tiles, size_t channels_per_tile) {
    return round_up(kWsHeader + tiles * channels_per_tile * sizeof(uint4), 256);
}

WsEntry *find_ws(int dev, cudaStream_t stream, int kind = 0) {
    for (WsEntry *e : g_ws)
        if (e->device == dev && e->stream == stream && e->kind == kind) return e;
    return nullptr;
}

// caller holds g_mu
wkv_status ensure_ws(int dev, cudaStream_t stream, size_t need, WsEntry **out, int kind = 0) {
    WsEntry *e = find_ws(dev, stream, kind);
    if (e != nullptr && e->bytes >= need) {
        *out = e;
        return WKV_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) == cudaSuccess && cap != cudaStreamCaptureStatusNone)
        return fail(WKV_ERR_CUDA,
                    "this call needs a %zu-byte look-back workspace for its stream, which "
                    "cannot be allocated during stream capture: make one call of this size "
                    "on the stream before capturing it", need);
    cudaGetLastError();
    const size_t nb = round_up(e != nullptr && need < 2 * e->bytes ? 2 * e->bytes : need, 1 << 20);
    void *p = nullptr;
    cudaError_t err = cudaMalloc(&p, nb);
    if (err != cudaSuccess) {
        cudaGetLastError();
        return fail(WKV_ERR_OOM, "workspace of %zu bytes: %s", nb, cudaGetErrorName(err));
    }
    err = cudaMemsetAsync(p, 0, nb, stream);
    if (err == cudaSuccess && e != nullptr && e->base != nullptr && kind == 0)
        // a timeout recorded in the buffer being retired (and not yet read by
        // wkv_device_status) carries over: the status word moves, in stream
        // order, after every launch that used the old buffer
        err = cudaMemcpyAsync(static_cast<char *>(p) + 16, e->base + 16, sizeof(int),
                              cudaMemcpyDeviceToDevice, stream);
    if (err != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(err, "cudaMemsetAsync(workspace)");
    }
    if (e == nullptr) {
        e = new WsEntry;
        e->device = dev;
        e->stream = stream;
        e->kind = kind;
        g_ws.push_back(e);
    } else if (e->base != nullptr) {
        g_retired.emplace_back(dev, e->base);
    }
    e->base = static_cast<char *>(p);
    e->bytes = nb;
    *out = e;
    return WKV_OK;
}

// ---- tensor maps ------------------------------------------------------------------
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, size_t es, int64_t B,
              int64_t T, int64_t C, int box_c, int box_t) {
    const Driver &d = driver();
    if (d.encode_tiled == nullptr) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(C * es), static_cast<cuuint64_t>(T * C * es)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_c), static_cast<cuuint32_t>(box_t), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = d.encode_tiled(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// TMA tile copies need 16-byte aligned bases, rows of a multiple of 16 bytes
// and a batch stride below 2^40 bytes.
bool tma_eligible(const void *const *ptrs, int n, size_t es, int64_t T, int64_t C) {
    for (int i = 0; i < n; ++i)
        if (reinterpret_cast<uintptr_t>(ptrs[i]) % 16 != 0) return false;
    if ((C * es) % 16 != 0) return false;
    if (static_cast<unsigned __int128>(T) * C * es >= (static_cast<unsigned __int128>(1) << 40))
        return false;
    return driver().encode_tiled != nullptr;
}

// ---- launch -------------------------------------------------------------------------
constexpr long long kSpinLimit = 1ll << 21;  // look-back polls, ~0.1-1 s

int sm_count(int dev) {
    static std::atomic<int> cache[64];
    if (dev >= 0 && dev < 64 && cache[dev].load() > 0) return cache[dev].load();
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = 148;
    }
    if (dev >= 0 && dev < 64) cache[dev].store(n);
    return n;
}

// Geometry, tensor maps and (for sequences longer than one tile) the
// look-back workspace of one call; `cg` channels and `lt` steps per tile.
struct Plan {
    Geometry g;
    CUtensorMap maps[4];  // x0, x1, y, and x2 for three-input ops
    Workspace ws;
};

template <class Op>
wkv_status make_plan(const typename Op::Args &args, int64_t B, int64_t T, int64_t C, int lt,
                     CUtensorMapDataType dt, cudaStream_t stream, int dev, bool want_tma,
                     Plan *p) {
    constexpr int CG = 32 * Op::CPT;
    using io_t = typename Op::io_t;
    Geometry &g = p->g;
    g.B = static_cast<int>(B);
    g.T = static_cast<int>(T);
    g.C = static_cast<int>(C);
    g.n_cg = static_cast<int>((C + CG - 1) / CG);
    g.n_seg = static_cast<int>((T + lt - 1) / lt);
    const long long tiles_per_seg = B * static_cast<long long>(g.n_cg);
    const long long tiles = tiles_per_seg * g.n_seg;
    if (tiles > INT32_MAX) return fail(WKV_ERR_INVALID_ARG, "problem has too many tiles");
    g.tiles_per_seg = static_cast<int>(tiles_per_seg);
    g.tiles = static_cast<int>(tiles);
    g.spin_limit = g_fault_spin_limit.load() > 0 ? g_fault_spin_limit.load() : kSpinLimit;
    g.skip_publish = g_fault_skip_tile.load();
    std::memset(p->maps, 0, sizeof p->maps);
    g.use_tma = 0;
    if (want_tma) {
        // maps: [0] x0, [1] x1 (two or more inputs), [2] y, [3] x2 (three inputs);
        // an io element is kScalarsPerIo tensor-map elements
        const void *ptrs[4] = {args.x0, nullptr, args.y, nullptr};
        if constexpr (Op::NIN >= 2) ptrs[1] = args.x1;
        if constexpr (Op::NIN == 3) ptrs[3] = args.x2;
        const void *used[4];
        int n = 0;
        for (const void *q : ptrs)
            if (q != nullptr) used[n++] = q;
        constexpr int SP = Op::kScalarsPerIo;
        g.use_tma = tma_eligible(used, n, sizeof(io_t), T, C) ? 1 : 0;
        for (int i = 0; i < 4 && g.use_tma; ++i)
            if (ptrs[i] != nullptr &&
                !make_map(&p->maps[i], ptrs[i], dt, sizeof(io_t) / SP, B, T, C * SP, CG * SP, lt))
                g.use_tma = 0;
    }
    g.params_staged = 0;
    if constexpr (StagesParams<Op>::value)
        g.params_staged = reinterpret_cast<uintptr_t>(args.u) % 16 == 0 &&
                          reinterpret_cast<uintptr_t>(args.w) % 16 == 0;
    std::memset(&p->ws, 0, sizeof p->ws);
    if (g.n_seg > 1) {
        std::lock_guard<std::mutex> lk(g_mu);
        WsEntry *e = nullptr;
        wkv_status st = ensure_ws(dev, stream, ws_bytes(static_cast<size_t>(tiles), CG), &e);
        if (st != WKV_OK) return st;
        Workspace &ws = p->ws;
        ws.ticket = reinterpret_cast<unsigned int *>(e->base);
        ws.done = reinterpret_cast<unsigned int *>(e->base + 4);
        ws.epoch = reinterpret_cast<unsigned long long *>(e->base + 8);
        ws.status = reinterpret_cast<int *>(e->base + 16);
        ws.records = reinterpret_cast<uint4 *>(e->base + kWsHeader);
    }
    return WKV_OK;
}

template <typename K>
wkv_status configure_once(K kern, size_t smem, int dev, std::atomic<uint64_t> &done) {
    if (dev < 64 && (done.load() & (1ull << dev))) return WKV_OK;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    if (dev < 64) done.fetch_or(1ull << dev);
    return WKV_OK;
}

// one thread block per tile; any shape (element-wise copies when no tensor map)
template <class Op, int LT, int NW>
wkv_status launch_chunked(const typename Op::Args &args, int64_t B, int64_t T, int64_t C,
                          CUtensorMapDataType dt, cudaStream_t stream, int dev) {
    Plan p;
    wkv_status st = make_plan<Op>(args, B, T, C, LT, dt, stream, dev, true, &p);
    if (st != WKV_OK) return st;
    constexpr size_t smem = chunked_scan_smem_bytes<Op, LT, NW>();
    auto kern = chunked_scan_kernel<Op, LT, NW>;
    static std::atomic<uint64_t> configured{0};
    if ((st = configure_once(kern, smem, dev, configured)) != WKV_OK) return st;
    cudaGetLastError();  // clear a stale error so the check below is about this launch
    kern<<<static_cast<unsigned>(p.g.tiles), NW * 32, smem, stream>>>(
        p.maps[0], p.maps[1], p.maps[2], p.maps[3], args, p.g, p.ws);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

// persistent pipeline, one block per SM; shapes a tensor map describes
template <class Op, int LT, int NWG, int NC, int NSTAGE>
wkv_status launch_persistent(const typename Op::Args &args, int64_t B, int64_t T, int64_t C,
                             CUtensorMapDataType dt, cudaStream_t stream, int dev) {
    using Cfg = PersistentCfg<Op, LT, NWG, NC, NSTAGE>;
    Plan p;
    wkv_status st = make_plan<Op>(args, B, T, C, LT, dt, stream, dev, true, &p);
    if (st != WKV_OK) return st;
    if (!p.g.use_tma)  // a tensor map could not be made after all
        return launch_chunked<Op, LT, 8>(args, B, T, C, dt, stream, dev);
    auto kern = persistent_scan_kernel<Op, LT, NWG, NC, NSTAGE>;
    static std::atomic<uint64_t> configured{0};
    if ((st = configure_once(kern, Cfg::kSmemBytes, dev, configured)) != WKV_OK) return st;
    const int grid = std::min(p.g.tiles, sm_count(dev));
    // programmatic dependent launch: this grid's blocks may be scheduled while
    // the previous grid in the stream drains; the kernel reads no global
    // memory before griddepcontrol.wait
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaGetLastError();
    cudaError_t err =
        cudaLaunchKernelEx(&cfg, kern, p.maps[0], p.maps[1], p.maps[2], p.maps[3], args, p.g, p.ws);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

// fp32 WKV forward (with or without the gate) with register-resident
// sub-chunks; shapes a tensor map describes.  Same plan and workspace as
// launch_persistent.
template <bool GATED, int LT, int NWG, int NC, int NSTAGE>
wkv_status launch_persistent_wkv(const typename WkvOp<float, 1, GATED>::Args &ga, int64_t B,
                                 int64_t T, int64_t C, CUtensorMapDataType dt, cudaStream_t stream,
                                 int dev) {
    using Cfg = RegWkvCfg<LT, NWG, NC, NSTAGE, GATED>;
    using GOp = WkvOp<float, 1, GATED>;  // its Args carry r for the plan's maps
    Plan p;
    wkv_status st = make_plan<GOp>(ga, B, T, C, LT, dt, stream, dev, true, &p);
    if (st != WKV_OK) return st;
    if (!p.g.use_tma)  // a tensor map could not be made after all
        return launch_chunked<GOp, LT, 8>(ga, B, T, C, dt, stream, dev);
    const WkvOp<float, 1>::Args args{ga.x0, ga.x1, ga.y, ga.w, ga.u, ga.s_in, ga.s_out, ga.x2};
    auto kern = persistent_wkv_kernel<LT, NWG, NC, NSTAGE, GATED>;
    static std::atomic<uint64_t> configured{0};
    if ((st = configure_once(kern, Cfg::kSmemBytes, dev, configured)) != WKV_OK) return st;
    const int grid = std::min(p.g.tiles, sm_count(dev));
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaGetLastError();
    cudaError_t err =
        cudaLaunchKernelEx(&cfg, kern, p.maps[0], p.maps[1], p.maps[2], p.maps[3], args, p.g, p.ws);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

// Compute warps per group, groups and ring stages of the register-resident
// WKV kernel for each tile length (build-time tuning parameters; each group
// also has a carry warp, and the block a producer warp).
#ifndef WKV_REG_F32_64
#define WKV_REG_F32_64 4, 3, 10
#endif
#ifndef WKV_REG_F32_128
#define WKV_REG_F32_128 4, 3, 5
#endif
#ifndef WKV_REG_F32_256
#define WKV_REG_F32_256 8, 1, 2
#endif
#ifndef WKV_REG_GATED_F32_64
#define WKV_REG_GATED_F32_64 4, 3, 7
#endif
#ifndef WKV_REG_GATED_F32_128
#define WKV_REG_GATED_F32_128 4, 3, 3
#endif

// The register-resident kernel is the faster one for fp32 problems of few
// time segments (it measured ~6 % faster on B=8 T=1024 C=768); for bf16 and
// for long chains of tiles the stage-resident kernel is (its four consumer
// groups hide the carry between tiles better).
constexpr int64_t kRegKernelMaxSegments = 16;

template <bool GATED>
wkv_status dispatch_reg_wkv(const typename WkvOp<float, 1, GATED>::Args &args, int64_t B,
                            int64_t T, int64_t C, int lt, CUtensorMapDataType dt,
                            cudaStream_t stream, int dev) {
    if constexpr (GATED) {
        switch (lt) {
            case 64: return launch_persistent_wkv<true, 64, WKV_REG_GATED_F32_64>(args, B, T, C, dt, stream, dev);
            default: return launch_persistent_wkv<true, 128, WKV_REG_GATED_F32_128>(args, B, T, C, dt, stream, dev);
        }
    } else {
        switch (lt) {
            case 64: return launch_persistent_wkv<false, 64, WKV_REG_F32_64>(args, B, T, C, dt, stream, dev);
            case 256: return launch_persistent_wkv<false, 256, WKV_REG_F32_256>(args, B, T, C, dt, stream, dev);
            default: return launch_persistent_wkv<false, 128, WKV_REG_F32_128>(args, B, T, C, dt, stream, dev);
        }
    }
}

// Warps per group, groups and ring stages of the stage-resident kernel for
// 128-step tiles of two inputs (build-time tuning parameters): bf16 WKV (two
// channels a thread), everything else
#ifndef WKV_PS_128_BF16
#define WKV_PS_128_BF16 4, 4, 6
#endif
#ifndef WKV_PS_128
#define WKV_PS_128 4, 4, 6
#endif
#ifndef WKV_PS_64_BF16
#define WKV_PS_64_BF16 4, 6, 12
#endif
template <class Op, class = void>
struct PackedIo : std::false_type {};
template <class Op>
struct PackedIo<Op, std::void_t<decltype(Op::kPacked)>> : std::bool_constant<Op::kPacked> {};

// 1: the WKV forward takes the register-resident kernel (persistent_wkv.cuh)
// where a tensor map describes the problem; 0: the stage-resident one
#ifndef WKV_USE_REG_KERNEL
#define WKV_USE_REG_KERNEL 1
#endif

// Steps per tile: the knob's value, or when it is 0, 128 unless a time
// segment holds too few tiles to keep the SMs' consumer groups fed -- long
// sequences over few rows and channels -- where 256-step tiles halve the
// length of the carry chain between tiles.
int tile_steps_for(int64_t B, int64_t T, int64_t C, int cg) {
    const int knob = g_tile_steps.load();
    if (knob != 0) return knob;
    const int64_t tiles_per_seg = B * ((C + cg - 1) / cg);
    return (T > 4096 && tiles_per_seg < 64) ? 256 : 128;
}

// Sequences of at most this many steps (single-token decoding included) run
// on the serial kernel: one thread per (row, channel), no tiles, no workspace.
constexpr int64_t kSerialMaxSteps = 16;

template <class Op>
wkv_status launch_serial(const typename Op::Args &args, int64_t B, int64_t T, int64_t C,
                         cudaStream_t stream) {
    // four channels per thread when every access can be a 4-element vector
    const size_t vb = 4 * sizeof(typename Op::io_t);
    const auto al = [](const void *p, size_t a) {
        return p == nullptr || reinterpret_cast<uintptr_t>(p) % a == 0;
    };
    const bool vec4 = C % 4 == 0 && al(args.x0, vb) && al(args.x1, vb) && al(args.y, vb) &&
                      al(args.x2, vb) && al(args.s_in, 16) && al(args.s_out, 16);
    const int vw = vec4 ? 4 : 1;
    const int64_t blocks = (B * (C / vw) + kSerialThreads - 1) / kSerialThreads;
    if (vec4)
        wkv_serial_kernel<Op, 4><<<static_cast<unsigned>(blocks), kSerialThreads, 0, stream>>>(
            args, static_cast<int>(B), static_cast<int>(T), static_cast<int>(C));
    else
        wkv_serial_kernel<Op, 1><<<static_cast<unsigned>(blocks), kSerialThreads, 0, stream>>>(
            args, static_cast<int>(B), static_cast<int>(T), static_cast<int>(C));
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

template <class Op>
wkv_status dispatch(const typename Op::Args &args, int64_t B, int64_t T, int64_t C,
                    CUtensorMapDataType dt, cudaStream_t stream, int dev) {
    if constexpr (Op::kSerialForm) {
        if (T <= kSerialMaxSteps && (B * C + kSerialThreads - 1) / kSerialThreads <= INT32_MAX)
            return launch_serial<Op>(args, B, T, C, stream);
    }
    const void *ptrs[4] = {args.x0, args.y, nullptr, nullptr};
    int nptr = 2;
    if constexpr (Op::NIN >= 2) ptrs[nptr++] = args.x1;
    if constexpr (Op::NIN == 3) ptrs[nptr++] = args.x2;
    const bool tma = tma_eligible(ptrs, nptr, sizeof(typename Op::io_t), T, C);
    const int lt = tile_steps_for(B, T, C, 32 * Op::CPT);
    if constexpr (Op::kSerialForm && sizeof(typename Op::io_t) == 4 && WKV_USE_REG_KERNEL) {
        // the fp32 WKV forward (with or without the gate) over few time
        // segments: register-resident sub-chunks (u and w staged with each
        // tile by 16-byte bulk copies; three 256-step input tiles per stage
        // do not fit twice in shared memory, so the gate keeps 64 and 128)
        const auto al16 = [](const void *p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
        if (tma && lt >= 64 && (T + lt - 1) / lt <= kRegKernelMaxSegments && al16(args.u) &&
            al16(args.w) && !(Op::kGated && lt == 256))
            return dispatch_reg_wkv<Op::kGated>(args, B, T, C, lt, dt, stream, dev);
    }
    if constexpr (Op::NIN == 3) {
        // a third input tile per stage: fewer stages and groups fit in shared memory
        switch (lt) {
            case 8: return launch_chunked<Op, 8, 8>(args, B, T, C, dt, stream, dev);
            case 32: return launch_chunked<Op, 32, 8>(args, B, T, C, dt, stream, dev);
            case 64:
                return tma ? launch_persistent<Op, 64, 4, 4, 6>(args, B, T, C, dt, stream, dev)
                           : launch_chunked<Op, 64, 8>(args, B, T, C, dt, stream, dev);
            case 256:
                return tma ? launch_persistent<Op, 256, 8, 1, 2>(args, B, T, C, dt, stream, dev)
                           : launch_chunked<Op, 256, 8>(args, B, T, C, dt, stream, dev);
            default:
                return tma ? launch_persistent<Op, 128, 4, 3, 4>(args, B, T, C, dt, stream, dev)
                           : launch_chunked<Op, 128, 8>(args, B, T, C, dt, stream, dev);
        }
    } else {
        switch (lt) {
            case 8: return launch_chunked<Op, 8, 8>(args, B, T, C, dt, stream, dev);
            case 32: return launch_chunked<Op, 32, 8>(args, B, T, C, dt, stream, dev);
            case 64:
                if constexpr (PackedIo<Op>::value)
                    return tma ? launch_persistent<Op, 64, WKV_PS_64_BF16>(args, B, T, C, dt, stream, dev)
                               : launch_chunked<Op, 64, 8>(args, B, T, C, dt, stream, dev);
                else
                    return tma ? launch_persistent<Op, 64, 4, 6, 12>(args, B, T, C, dt, stream, dev)
                               : launch_chunked<Op, 64, 8>(args, B, T, C, dt, stream, dev);
            case 256:
                return tma ? launch_persistent<Op, 256, 8, 2, 3>(args, B, T, C, dt, stream, dev)
                           : launch_chunked<Op, 256, 8>(args, B, T, C, dt, stream, dev);
            default:
                if constexpr (PackedIo<Op>::value)
                    return tma ? launch_persistent<Op, 128, WKV_PS_128_BF16>(args, B, T, C, dt, stream, dev)
                               : launch_chunked<Op, 128, 8>(args, B, T, C, dt, stream, dev);
                else
                    return tma ? launch_persistent<Op, 128, WKV_PS_128>(args, B, T, C, dt, stream, dev)
                               : launch_chunked<Op, 128, 8>(args, B, T, C, dt, stream, dev);
        }
    }
}

wkv_status current_device(int *dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    return WKV_OK;
}

template <typename IO, bool GATED = false>
wkv_status wkv_common(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                      const IO *k, const IO *v, IO *y, const float *s_in, float *s_out,
                      cudaStream_t stream, CUtensorMapDataType dt, const IO *r = nullptr) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, C, &empty);
    if (st != WKV_OK || empty) return st;
    int dev = 0;
    if ((st = current_device(&dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * C * sizeof(IO);
    const size_t nc = static_cast<size_t>(C) * sizeof(float);
    if ((st = check_buffer(w, nc, 4, "w", dev)) != WKV_OK) return st;
    if ((st = check_buffer(u, nc, 4, "u", dev)) != WKV_OK) return st;
    if ((st = check_buffer(k, n, sizeof(IO), "k", dev)) != WKV_OK) return st;
    if ((st = check_buffer(v, n, sizeof(IO), "v", dev)) != WKV_OK) return st;
    if ((st = check_buffer(y, n, sizeof(IO), "y", dev)) != WKV_OK) return st;
    if (overlaps(y, n, k, n) || overlaps(y, n, v, n) || overlaps(y, n, w, nc) ||
        overlaps(y, n, u, nc))
        return fail(WKV_ERR_INVALID_ARG, "y overlaps an input");
    if (GATED) {
        if ((st = check_buffer(r, n, sizeof(IO), "r", dev)) != WKV_OK) return st;
        if (overlaps(y, n, r, n)) return fail(WKV_ERR_INVALID_ARG, "y overlaps r");
    }
    const size_t ns = static_cast<size_t>(B) * 3 * C * sizeof(float);
    if (s_in != nullptr && (st = check_buffer(s_in, ns, 4, "s_in", dev)) != WKV_OK) return st;
    if (s_out != nullptr) {
        if ((st = check_buffer(s_out, ns, 4, "s_out", dev)) != WKV_OK) return st;
        if (overlaps(s_out, ns, k, n) || overlaps(s_out, ns, v, n) || overlaps(s_out, ns, y, n) ||
            overlaps(s_out, ns, w, nc) || overlaps(s_out, ns, u, nc) ||
            overlaps(s_out, ns, r, GATED ? n : 0))
            return fail(WKV_ERR_INVALID_ARG, "s_out overlaps k, v, r, y, w or u");
        if (s_in != nullptr && s_in != s_out && overlaps(s_out, ns, s_in, ns))
            return fail(WKV_ERR_INVALID_ARG, "s_out overlaps s_in without being the same buffer");
    }
    if (overlaps(y, n, s_in, s_in ? ns : 0))
        return fail(WKV_ERR_INVALID_ARG, "y overlaps s_in");
    using Op = WkvOp<IO, sizeof(IO) == 2 ? 2 : 1, GATED>;
    typename Op::Args args{k, v, y, w, u, s_in, s_out, GATED ? r : nullptr};
    return dispatch<Op>(args, B, T, C, dt, stream, dev);
}

// ---- token shift ----------------------------------------------------------------
template <typename IO, int VW>
wkv_status launch_shift(int n_mix, const IO *x, const IO *x_prev, const float *mu, IO *out,
                        IO *x_last, int64_t B, int64_t T, int64_t C, cudaStream_t stream) {
    const int64_t chunks = (T + kShiftChunk - 1) / kShiftChunk;
    const int64_t threads = B * chunks * (C / VW);
    const int64_t blocks = (threads + kShiftThreads - 1) / kShiftThreads;
    if (blocks > INT32_MAX) return fail(WKV_ERR_INVALID_ARG, "problem too large for one launch");
    const dim3 grid(static_cast<unsigned>(blocks));
    const int b = static_cast<int>(B), t = static_cast<int>(T), c = static_cast<int>(C);
    switch (n_mix) {
        case 1: token_shift_kernel<IO, VW, 1><<<grid, kShiftThreads, 0, stream>>>(x, x_prev, mu, out, x_last, b, t, c); break;
        case 2: token_shift_kernel<IO, VW, 2><<<grid, kShiftThreads, 0, stream>>>(x, x_prev, mu, out, x_last, b, t, c); break;
        case 3: token_shift_kernel<IO, VW, 3><<<grid, kShiftThreads, 0, stream>>>(x, x_prev, mu, out, x_last, b, t, c); break;
        default: token_shift_kernel<IO, VW, 4><<<grid, kShiftThreads, 0, stream>>>(x, x_prev, mu, out, x_last, b, t, c); break;
    }
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

template <typename IO>
wkv_status shift_common(int64_t B, int64_t T, int64_t C, int64_t n_mix, const IO *x,
                        const IO *x_prev, const float *mu, IO *out, IO *x_last,
                        cudaStream_t stream) {
    t_err.clear();
    if (n_mix < 1 || n_mix > 4) return fail(WKV_ERR_INVALID_ARG, "n_mix must be 1..4");
    bool empty = false;
    wkv_status st = check_sizes(B, T, C, &empty);
    if (st != WKV_OK || empty) return st;
    int dev = 0;
    if ((st = current_device(&dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * C * sizeof(IO);
    const size_t nrow = static_cast<size_t>(B) * C * sizeof(IO);
    const size_t nmu = static_cast<size_t>(n_mix) * C * sizeof(float);
    const size_t nout = static_cast<size_t>(n_mix) * n;
    if ((st = check_buffer(x, n, sizeof(IO), "x", dev)) != WKV_OK) return st;
    if ((st = check_buffer(mu, nmu, 4, "mu", dev)) != WKV_OK) return st;
    if ((st = check_buffer(out, nout, sizeof(IO), "out", dev)) != WKV_OK) return st;
    if (x_prev != nullptr && (st = check_buffer(x_prev, nrow, sizeof(IO), "x_prev", dev)) != WKV_OK)
        return st;
    if (x_last != nullptr && (st = check_buffer(x_last, nrow, sizeof(IO), "x_last", dev)) != WKV_OK)
        return st;
    if (overlaps(out, nout, x, n) || overlaps(out, nout, mu, nmu) ||
        overlaps(out, nout, x_prev, x_prev ? nrow : 0) ||
        overlaps(out, nout, x_last, x_last ? nrow : 0))
        return fail(WKV_ERR_INVALID_ARG, "out overlaps x, mu, x_prev or x_last");
    if (x_last != nullptr) {
        if (overlaps(x_last, nrow, x, n) || overlaps(x_last, nrow, mu, nmu))
            return fail(WKV_ERR_INVALID_ARG, "x_last overlaps x or mu");
        if (x_prev != nullptr && x_prev != x_last && overlaps(x_last, nrow, x_prev, nrow))
            return fail(WKV_ERR_INVALID_ARG, "x_last overlaps x_prev without being the same buffer");
    }
    const auto al = [](const void *p, size_t a) {
        return p == nullptr || reinterpret_cast<uintptr_t>(p) % a == 0;
    };
    const size_t vb = 4 * sizeof(IO);
    const bool vec4 = C % 4 == 0 && al(x, vb) && al(x_prev, vb) && al(out, vb) &&
                      al(x_last, vb) && al(mu, 16);
    const int nm = static_cast<int>(n_mix);
    return vec4 ? launch_shift<IO, 4>(nm, x, x_prev, mu, out, x_last, B, T, C, stream)
                : launch_shift<IO, 1>(nm, x, x_prev, mu, out, x_last, B, T, C, stream);
}

template <typename IO>
wkv_status scan_common(int64_t B, int64_t T, int64_t D, const IO *a, const IO *b,
                       const float *h0, IO *h, cudaStream_t stream, CUtensorMapDataType dt) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, D, &empty);
    if (st != WKV_OK || empty) return st;
    int dev = 0;
    if ((st = current_device(&dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * D * sizeof(IO);
    const size_t n0 = static_cast<size_t>(B) * D * sizeof(float);
    if ((st = check_buffer(a, n, sizeof(IO), "a", dev)) != WKV_OK) return st;
    if ((st = check_buffer(b, n, sizeof(IO), "b", dev)) != WKV_OK) return st;
    if (h0 != nullptr && (st = check_buffer(h0, n0, 4, "h0", dev)) != WKV_OK) return st;
    if ((st = check_buffer(h, n, sizeof(IO), "h", dev)) != WKV_OK) return st;
    if (overlaps(h, n, a, n) || overlaps(h, n, b, n) || overlaps(h, n, h0, h0 ? n0 : 0))
        return fail(WKV_ERR_INVALID_ARG, "h overlaps an input");
    using Op = ScanOpT<IO, sizeof(IO) == 2 ? 2 : 1>;
    typename Op::Args args{a, b, h, h0};
    return dispatch<Op>(args, B, T, D, dt, stream, dev);
}

#include "capi_host.cuh"

#include "capi_backward.cuh"

}  // namespace

extern "C" {

wkv_status wkv_forward_host(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                            const float *k, const float *v, float *y) {
    return wkv_host_common<float>(B, T, C, w, u, k, v, y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

wkv_status wkv_forward_bf16_host(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                                 const wkv_bf16_t *k, const wkv_bf16_t *v, wkv_bf16_t *y) {
    return wkv_host_common<__nv_bfloat16>(B, T, C, w, u, k, v, y,
                                          CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

wkv_status diag_scan_host(int64_t B, int64_t T, int64_t D, const float *a, const float *b,
                          const float *h0, float *h) {
    return scan_host_impl(B, T, D, a, b, h0, h);
}

}  // extern "C"

extern "C" {

wkv_status wkv_forward(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                       const float *k, const float *v, float *y, cudaStream_t stream) {
    return wkv_common<float>(B, T, C, w, u, k, v, y, nullptr, nullptr, stream,
                             CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

wkv_status wkv_forward_bf16(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                            const wkv_bf16_t *k, const wkv_bf16_t *v, wkv_bf16_t *y,
                            cudaStream_t stream) {
    return wkv_common<__nv_bfloat16>(B, T, C, w, u, reinterpret_cast<const __nv_bfloat16 *>(k),
                                     reinterpret_cast<const __nv_bfloat16 *>(v),
                                     reinterpret_cast<__nv_bfloat16 *>(y), nullptr, nullptr,
                                     stream, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

wkv_status wkv_forward_state(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                             const float *k, const float *v, float *y, const float *s_in,
                             float *s_out, cudaStream_t stream) {
    return wkv_common<float>(B, T, C, w, u, k, v, y, s_in, s_out, stream,
                             CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

wkv_status wkv_forward_bf16_state(int64_t B, int64_t T, int64_t C, const float *w,
                                  const float *u, const wkv_bf16_t *k, const wkv_bf16_t *v,
                                  wkv_bf16_t *y, const float *s_in, float *s_out,
                                  cudaStream_t stream) {
    return wkv_common<__nv_bfloat16>(B, T, C, w, u, reinterpret_cast<const __nv_bfloat16 *>(k),
                                     reinterpret_cast<const __nv_bfloat16 *>(v),
                                     reinterpret_cast<__nv_bfloat16 *>(y), s_in, s_out, stream,
                                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

wkv_status wkv_forward_gated(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                             const float *k, const float *v, const float *r, float *y,
                             const float *s_in, float *s_out, cudaStream_t stream) {
    return wkv_common<float, true>(B, T, C, w, u, k, v, y, s_in, s_out, stream,
                                   CU_TENSOR_MAP_DATA_TYPE_FLOAT32, r);
}

wkv_status wkv_forward_bf16_gated(int64_t B, int64_t T, int64_t C, const float *w,
                                  const float *u, const wkv_bf16_t *k, const wkv_bf16_t *v,
                                  const wkv_bf16_t *r, wkv_bf16_t *y, const float *s_in,
                                  float *s_out, cudaStream_t stream) {
    return wkv_common<__nv_bfloat16, true>(
        B, T, C, w, u, reinterpret_cast<const __nv_bfloat16 *>(k),
        reinterpret_cast<const __nv_bfloat16 *>(v), reinterpret_cast<__nv_bfloat16 *>(y), s_in,
        s_out, stream, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, reinterpret_cast<const __nv_bfloat16 *>(r));
}

wkv_status wkv_token_shift(int64_t B, int64_t T, int64_t C, int64_t n_mix, const float *x,
                           const float *x_prev, const float *mu, float *out, float *x_last,
                           cudaStream_t stream) {
    return shift_common<float>(B, T, C, n_mix, x, x_prev, mu, out, x_last, stream);
}

wkv_status wkv_token_shift_bf16(int64_t B, int64_t T, int64_t C, int64_t n_mix,
                                const wkv_bf16_t *x, const wkv_bf16_t *x_prev, const float *mu,
                                wkv_bf16_t *out, wkv_bf16_t *x_last, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return shift_common<bf>(B, T, C, n_mix, reinterpret_cast<const bf *>(x),
                            reinterpret_cast<const bf *>(x_prev), mu, reinterpret_cast<bf *>(out),
                            reinterpret_cast<bf *>(x_last), stream);
}

wkv_status wkv_backward(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                        const float *k, const float *v, const float *gy, float *gk, float *gv,
                        float *gw, float *gu, cudaStream_t stream) {
    return backward_impl(B, T, C, w, u, k, v, gy, gk, gv, gw, gu, stream);
}

wkv_status lru_scan(int64_t B, int64_t T, int64_t D, const float *nu_log,
                    const float *theta_log, const float *gamma, const float *u,
                    const float *x0, float *x, cudaStream_t stream) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, D, &empty);
    if (st != WKV_OK || empty) return st;
    int dev = 0;
    if ((st = current_device(&dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * D * 8;   // complex64 elements
    const size_t n0 = static_cast<size_t>(B) * D * 8;
    const size_t nd = static_cast<size_t>(D) * 4;
    if ((st = check_buffer(nu_log, nd, 4, "nu_log", dev)) != WKV_OK) return st;
    if ((st = check_buffer(theta_log, nd, 4, "theta_log", dev)) != WKV_OK) return st;
    if (gamma != nullptr && (st = check_buffer(gamma, nd, 4, "gamma", dev)) != WKV_OK) return st;
    if ((st = check_buffer(u, n, 8, "u", dev)) != WKV_OK) return st;
    if (x0 != nullptr && (st = check_buffer(x0, n0, 8, "x0", dev)) != WKV_OK) return st;
    if ((st = check_buffer(x, n, 8, "x", dev)) != WKV_OK) return st;
    if (overlaps(x, n, u, n) || overlaps(x, n, x0, x0 ? n0 : 0) || overlaps(x, n, nu_log, nd) ||
        overlaps(x, n, theta_log, nd) || overlaps(x, n, gamma, gamma ? nd : 0))
        return fail(WKV_ERR_INVALID_ARG, "x overlaps an input");
    LruOp::Args args{reinterpret_cast<const float2 *>(u), nullptr, reinterpret_cast<float2 *>(x),
                     nu_log, theta_log, gamma, reinterpret_cast<const float2 *>(x0)};
    return dispatch<LruOp>(args, B, T, D, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, stream, dev);
}

wkv_status diag_scan(int64_t B, int64_t T, int64_t D, const float *a, const float *b,
                     const float *h0, float *h, cudaStream_t stream) {
    return scan_common<float>(B, T, D, a, b, h0, h, stream, CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
}

wkv_status diag_scan_bf16(int64_t B, int64_t T, int64_t D, const wkv_bf16_t *a,
                          const wkv_bf16_t *b, const float *h0, wkv_bf16_t *h,
                          cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return scan_common<bf>(B, T, D, reinterpret_cast<const bf *>(a),
                           reinterpret_cast<const bf *>(b), h0, reinterpret_cast<bf *>(h), stream,
                           CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

wkv_status wkv_device_status(cudaStream_t stream) {
    t_err.clear();
    int dev = 0;
    wkv_status st = current_device(&dev);
    if (st != WKV_OK) return st;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    std::lock_guard<std::mutex> lk(g_mu);
    WsEntry *w = find_ws(dev, stream);
    if (w == nullptr || w->base == nullptr) return WKV_OK;
    int code = 0;
    e = cudaMemcpy(&code, w->base + 16, sizeof code, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
    if (code != 0) {
        e = cudaMemset(w->base + 16, 0, sizeof code);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
        return fail(static_cast<wkv_status>(code),
                    "a device-side wait gave up; the affected outputs are NaN");
    }
    return WKV_OK;
}

const char *wkv_last_error(void) { return t_err.c_str(); }

wkv_status wkv_release_workspaces(void) {
    t_err.clear();
    int dev = 0;
    wkv_status st = current_device(&dev);
    if (st != WKV_OK) return st;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    for (auto it = g_ws.begin(); it != g_ws.end();) {
        if ((*it)->device == dev) {
            if ((*it)->base) cudaFree((*it)->base);
            delete *it;
            it = g_ws.erase(it);
        } else {
            ++it;
        }
    }
    for (auto it = g_retired.begin(); it != g_retired.end();) {
        if (it->first == dev) {
            cudaFree(it->second);
            it = g_retired.erase(it);
        } else {
            ++it;
        }
    }
    return WKV_OK;
}

wkv_status wkv_set_tile_steps(int steps) {
    t_err.clear();
    if (steps != 0 && steps != 8 && steps != 32 && steps != 64 && steps != 128 && steps != 256)
        return fail(WKV_ERR_INVALID_ARG, "tile steps must be 0 (automatic), 8, 32, 64, 128 or 256");
    g_tile_steps.store(steps);
    return WKV_OK;
}

int wkv_get_tile_steps(void) { return g_tile_steps.load(); }

int wkv_tile_steps_for(int64_t B, int64_t T, int64_t C, int elem_bytes) {
    if (B < 1 || T < 1 || C < 1 || (elem_bytes != 2 && elem_bytes != 4)) return 0;
    return tile_steps_for(B, T, C, elem_bytes == 2 ? 64 : 32);
}

wkv_status wkv_set_fault_injection(int skip_tile, long long spin_limit) {
    t_err.clear();
    if (skip_tile < -1 || spin_limit < 0)
        return fail(WKV_ERR_INVALID_ARG, "skip_tile must be >= -1 and spin_limit >= 0");
    g_fault_skip_tile.store(skip_tile);
    g_fault_spin_limit.store(spin_limit);
    return WKV_OK;
}

}  // extern "C"
