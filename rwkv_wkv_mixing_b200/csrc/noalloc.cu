// wkv_forward_noalloc: the fp32 WKV forward for callers that cannot allocate
// device memory.  Its cross-tile scratch (look-back flags, tile aggregates,
// counters) lives in one fixed-size file-scope device array instead of a
// cudaMalloc'd workspace.  The declaration and contract are in
// include/wkv_b200.h.
//
// This file is its own CUDA module: the array is only created on a device
// once this entry point is first used there, and stays until the process
// exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "chunked_scan.cuh"
#include "persistent_scan.cuh"
#include "wkv_b200.h"
#include "wkv_ops.cuh"

namespace wkvb {
void set_last_error(const char *msg);  // capi.cu: the message wkv_last_error() returns
}

using namespace wkvb;

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(16) << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;
constexpr int kTileSteps = 128;  // tile length of both kernel variants used here
constexpr size_t kHeader = 256;  // [0] ticket, [4] done, [8] epoch, [16] status
constexpr size_t kMaxTiles = (kScratchBytes - kHeader) / (32 * sizeof(uint4));  // 32767

// the scratch; host code must not pass this name to a kernel (it is a host
// stand-in), only the device address cudaGetSymbolAddress returns
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// a distinct Op type, so the kernels below are instantiated in this module
// only and never share a host launch stub with the library's other kernels
struct NoAllocWkvOp : WkvOp<float, 1> {};
using Op = NoAllocWkvOp;
using Persistent = PersistentCfg<Op, kTileSteps, 4, 4, 6>;
constexpr int kChunkedWarps = 8;

wkv_status fail(wkv_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    set_last_error(buf);
    return st;
}

wkv_status cuda_fail(cudaError_t e, const char *what) {
    return fail(WKV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// one-time set-up per device: the scratch's device address and the kernels'
// shared-memory limits, made with that device current
struct DeviceSlot {
    std::once_flag once;
    unsigned char *scratch = nullptr;
    cudaError_t err = cudaSuccess;
    const char *what = "";
};
DeviceSlot g_slots[kMaxDevices];

void set_up_device(DeviceSlot *slot) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
        slot->err = e;
        slot->what = "cudaGetSymbolAddress(scratch)";
        cudaGetLastError();
        return;
    }
    e = cudaFuncSetAttribute(persistent_scan_kernel<Op, kTileSteps, 4, 4, 6>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Persistent::kSmemBytes));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(chunked_scan_kernel<Op, kTileSteps, kChunkedWarps>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(chunked_scan_smem_bytes<Op, kTileSteps, kChunkedWarps>()));
    if (e != cudaSuccess) {
        slot->err = e;
        slot->what = "cudaFuncSetAttribute";
        cudaGetLastError();
        return;
    }
    slot->scratch = static_cast<unsigned char *>(p);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        cudaGetLastError();
    });
    return fn;
}

bool make_map(CUtensorMap *m, const float *ptr, int64_t B, int64_t T, int64_t C) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(C * 4), static_cast<cuuint64_t>(T * C * 4)};
    cuuint32_t box[3] = {32u, static_cast<cuuint32_t>(kTileSteps), 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

wkv_status check_ptr(const void *p, const char *name, int dev) {
    if (p == nullptr) return fail(WKV_ERR_INVALID_ARG, "%s is NULL", name);
    if (reinterpret_cast<uintptr_t>(p) % 4 != 0)
        return fail(WKV_ERR_ALIGNMENT, "%s is not 4-byte aligned", name);
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
    return WKV_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace

extern "C" wkv_status wkv_forward_noalloc(int64_t B, int64_t T, int64_t C, const float *w,
                                          const float *u, const float *k, const float *v,
                                          float *y, cudaStream_t stream) {
    set_last_error("");
    if (B < 0 || T < 0 || C < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
    if (B == 0 || T == 0 || C == 0) return WKV_OK;
    if (B > INT32_MAX || T > INT32_MAX || C > INT32_MAX)
        return fail(WKV_ERR_INVALID_ARG, "each of B, T, C must be below 2^31");
    if (static_cast<unsigned __int128>(B) * T * C >= (static_cast<unsigned __int128>(1) << 62))
        return fail(WKV_ERR_INVALID_ARG, "B*T*C must be below 2^62");
    // tiles of 32 channels x kTileSteps steps, and the scratch they need: a
    // header and one 16-byte record per (tile, channel)
    const long long n_cg = (C + 31) / 32, n_seg = (T + kTileSteps - 1) / kTileSteps;
    const long long tiles = B * n_cg * n_seg;
    const size_t need = n_seg > 1 ? kHeader + static_cast<size_t>(tiles) * 32 * sizeof(uint4) : 0;
    if (tiles > INT32_MAX || need > kScratchBytes)
        return fail(WKV_ERR_INVALID_ARG,
                    "wkv_forward_noalloc: B=%lld T=%lld C=%lld needs %zu bytes of scratch, more "
                    "than its fixed %zu-byte device array (at most %zu tiles of 32 channels x %d "
                    "steps); use wkv_forward",
                    static_cast<long long>(B), static_cast<long long>(T),
                    static_cast<long long>(C), need, kScratchBytes, kMaxTiles, kTileSteps);

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(WKV_ERR_INVALID_ARG, "device index too large");
    DeviceSlot &slot = g_slots[dev];
    std::call_once(slot.once, set_up_device, &slot);
    if (slot.scratch == nullptr) return cuda_fail(slot.err, slot.what);

    wkv_status st;
    if ((st = check_ptr(w, "w", dev)) != WKV_OK) return st;
    if ((st = check_ptr(u, "u", dev)) != WKV_OK) return st;
    if ((st = check_ptr(k, "k", dev)) != WKV_OK) return st;
    if ((st = check_ptr(v, "v", dev)) != WKV_OK) return st;
    if ((st = check_ptr(y, "y", dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * C * sizeof(float);
    const size_t nc = static_cast<size_t>(C) * sizeof(float);
    if (overlaps(y, n, k, n) || overlaps(y, n, v, n) || overlaps(y, n, w, nc) ||
        overlaps(y, n, u, nc))
        return fail(WKV_ERR_INVALID_ARG, "y overlaps an input");

    Geometry g;
    g.B = static_cast<int>(B);
    g.T = static_cast<int>(T);
    g.C = static_cast<int>(C);
    g.n_cg = static_cast<int>(n_cg);
    g.n_seg = static_cast<int>(n_seg);
    g.tiles_per_seg = static_cast<int>(B * n_cg);
    g.tiles = static_cast<int>(tiles);
    g.spin_limit = 1ll << 21;
    g.skip_publish = -1;

    Workspace ws;
    std::memset(&ws, 0, sizeof ws);
    if (need > 0) {
        // the array keeps the last call's contents: start the counters, the
        // status word and this call's records from zero (a memset, not an
        // allocation), so nothing a previous call left behind can be read
        unsigned char *base = slot.scratch;
        e = cudaMemsetAsync(base, 0, need, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(scratch)");
        ws.ticket = reinterpret_cast<unsigned int *>(base);
        ws.done = reinterpret_cast<unsigned int *>(base + 4);
        ws.epoch = reinterpret_cast<unsigned long long *>(base + 8);
        ws.status = reinterpret_cast<int *>(base + 16);
        ws.records = reinterpret_cast<uint4 *>(base + kHeader);
    }

    CUtensorMap maps[4];  // k, v, y; the fourth (a gate input) is unused here
    std::memset(maps, 0, sizeof maps);
    const bool tma = reinterpret_cast<uintptr_t>(k) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(v) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(y) % 16 == 0 && C % 4 == 0 &&
                     static_cast<unsigned __int128>(T) * C * 4 <
                         (static_cast<unsigned __int128>(1) << 40) &&
                     make_map(&maps[0], k, B, T, C) && make_map(&maps[1], v, B, T, C) &&
                     make_map(&maps[2], y, B, T, C);
    g.use_tma = tma ? 1 : 0;
    Op::Args args{k, v, y, w, u};
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    cudaGetLastError();
    if (tma) {
        const int grid = g.tiles < sms ? g.tiles : sms;
        persistent_scan_kernel<Op, kTileSteps, 4, 4, 6>
            <<<grid, Persistent::kThreads, Persistent::kSmemBytes, stream>>>(
                maps[0], maps[1], maps[2], maps[3], args, g, ws);
    } else {
        chunked_scan_kernel<Op, kTileSteps, kChunkedWarps>
            <<<static_cast<unsigned>(g.tiles), kChunkedWarps * 32,
               chunked_scan_smem_bytes<Op, kTileSteps, kChunkedWarps>(), stream>>>(
                maps[0], maps[1], maps[2], maps[3], args, g, ws);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return WKV_OK;
}
