// Host-buffer entry points (wkv_forward_host, wkv_forward_bf16_host,
// diag_scan_host): the chunked copy / compute pipeline over internal streams.
// Included by capi.cu inside its anonymous namespace, after the shared host
// infrastructure and the device-side dispatch it calls; kept apart so that
// the device kernels' code does not change with it.
#pragma once

// ---- host-buffer entry points: a chunked copy / compute pipeline ------------
// The problem is cut into independent chunks -- batch rows, or channel slices
// when there are too few rows -- and chunk c runs on internal stream c % 3:
// host-to-device copies of its inputs, the kernel, the device-to-host copy of
// its outputs.  The copy engines work both directions at once, so one chunk's
// upload overlaps another's compute and download.
constexpr int kPipeStreams = 3;
constexpr int kPipeChunks = 8;

struct HostPipe {
    int device = -1;
    cudaStream_t s[kPipeStreams] = {};
    char *stage = nullptr;  // kPipeStreams slices of `slice` bytes
    size_t slice = 0;
    int *status = nullptr;  // pinned host copies of each stream's device status word
};

std::mutex g_pipe_mu;  // serialises host-buffer calls (and guards g_pipes)
std::vector<HostPipe *> g_pipes;

// caller holds g_pipe_mu
wkv_status get_pipe(int dev, size_t slice, HostPipe **out) {
    HostPipe *p = nullptr;
    for (HostPipe *q : g_pipes)
        if (q->device == dev) p = q;
    if (p == nullptr) {
        p = new HostPipe;
        p->device = dev;
        for (int i = 0; i < kPipeStreams; ++i) {
            cudaError_t e = cudaStreamCreateWithFlags(&p->s[i], cudaStreamNonBlocking);
            if (e != cudaSuccess) {
                for (int j = 0; j < i; ++j) cudaStreamDestroy(p->s[j]);
                delete p;
                return cuda_fail(e, "cudaStreamCreate");
            }
        }
        void *h = nullptr;
        cudaError_t e = cudaHostAlloc(&h, kPipeStreams * sizeof(int), cudaHostAllocDefault);
        if (e != cudaSuccess) {
            for (int j = 0; j < kPipeStreams; ++j) cudaStreamDestroy(p->s[j]);
            delete p;
            cudaGetLastError();
            return fail(WKV_ERR_OOM, "host-pipeline status words: %s", cudaGetErrorName(e));
        }
        p->status = static_cast<int *>(h);
        g_pipes.push_back(p);
    }
    if (p->slice < slice) {
        if (p->stage != nullptr) {
            for (int i = 0; i < kPipeStreams; ++i) cudaStreamSynchronize(p->s[i]);
            cudaFree(p->stage);
            p->stage = nullptr;
            p->slice = 0;
        }
        void *m = nullptr;
        cudaError_t e = cudaMalloc(&m, slice * kPipeStreams);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(WKV_ERR_OOM, "host-pipeline staging of %zu bytes: %s",
                        slice * kPipeStreams, cudaGetErrorName(e));
        }
        p->stage = static_cast<char *>(m);
        p->slice = slice;
    }
    *out = p;
    return WKV_OK;
}

wkv_status check_host(const void *ptr, const char *name) {
    if (ptr == nullptr) return fail(WKV_ERR_INVALID_ARG, "%s is NULL", name);
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(WKV_ERR_INVALID_ARG, "%s: %s", name, cudaGetErrorName(e));
    }
    if (a.type == cudaMemoryTypeDevice)
        return fail(WKV_ERR_INVALID_ARG,
                    "%s is device memory; the _host entry points take host buffers", name);
    return WKV_OK;
}

// One chunk: rows [r0, r0 + rows) x channels [c0, c0 + cols) of [B, T, C].
struct Chunk {
    int64_t r0, rows, c0, cols;
};

// Chunks of at least about kPipeMinChunkBytes of input each (a chunk's copies
// and launch carry a fixed cost that small chunks do not repay), at most
// kPipeChunks (the last chunk's download is the part nothing overlaps).
#ifndef WKV_PIPE_MIN_CHUNK_BYTES
#define WKV_PIPE_MIN_CHUNK_BYTES (16ll << 20)
#endif
constexpr long long kPipeMinChunkBytes = WKV_PIPE_MIN_CHUNK_BYTES;

std::vector<Chunk> plan_chunks(int64_t B, int64_t T, int64_t C, size_t es, int n_in) {
    std::vector<Chunk> out;
    const long long in_bytes = static_cast<long long>(n_in) * B * T * C * static_cast<long long>(es);
    const int64_t n = std::max<int64_t>(
        1, std::min<int64_t>(kPipeChunks, (in_bytes + kPipeMinChunkBytes - 1) / kPipeMinChunkBytes));
    if (B >= 2) {
        const int64_t per = (B + n - 1) / n;
        for (int64_t r = 0; r < B; r += per) out.push_back({r, std::min(per, B - r), 0, C});
    } else if (C >= 2 * 64) {
        // channel slices, a multiple of 64 channels (16-byte aligned rows)
        int64_t per = (C + n - 1) / n;
        per = (per + 63) / 64 * 64;
        for (int64_t c = 0; c < C; c += per) out.push_back({0, B, c, std::min(per, C - c)});
    } else {
        out.push_back({0, B, 0, C});
    }
    return out;
}

// copy a chunk of a [B, T, C] host tensor to a dense [rows, T, cols] device
// buffer (or back)
cudaError_t copy_chunk(void *dst, const void *src, const Chunk &ch, int64_t T, int64_t C,
                       size_t es, bool to_device, cudaStream_t st) {
    const size_t row_bytes = static_cast<size_t>(ch.cols) * es;
    if (ch.cols == C) {
        const size_t off = static_cast<size_t>(ch.r0) * T * C * es;
        const size_t bytes = static_cast<size_t>(ch.rows) * T * C * es;
        if (to_device)
            return cudaMemcpyAsync(dst, static_cast<const char *>(src) + off, bytes,
                                   cudaMemcpyHostToDevice, st);
        return cudaMemcpyAsync(static_cast<char *>(dst) + off, src, bytes, cudaMemcpyDeviceToHost,
                               st);
    }
    const size_t height = static_cast<size_t>(ch.rows) * T;
    const size_t host_off = (static_cast<size_t>(ch.r0) * T * C + ch.c0) * es;
    if (to_device)
        return cudaMemcpy2DAsync(dst, row_bytes, static_cast<const char *>(src) + host_off, C * es,
                                 row_bytes, height, cudaMemcpyHostToDevice, st);
    return cudaMemcpy2DAsync(static_cast<char *>(dst) + host_off, C * es, src, row_bytes, row_bytes,
                             height, cudaMemcpyDeviceToHost, st);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Run `Op` over host tensors x0, x1 -> y with per-channel host params p0, p1
// ([C] each, may be NULL) or per-row-and-channel host h0 ([B, C], may be NULL).
template <class Op>
wkv_status run_host(int64_t B, int64_t T, int64_t C, const void *x0, const void *x1, void *y,
                    const float *p0, const float *p1, const float *h0, CUtensorMapDataType dt,
                    typename Op::Args (*make_args)(const void *, const void *, void *,
                                                   const float *, const float *, const float *)) {
    using io_t = typename Op::io_t;
    const size_t es = sizeof(io_t);
    int dev = 0;
    wkv_status st = current_device(&dev);
    if (st != WKV_OK) return st;
    const std::vector<Chunk> chunks = plan_chunks(B, T, C, es, 2);
    size_t max_elems = 0;
    for (const Chunk &ch : chunks)
        max_elems = std::max(max_elems, static_cast<size_t>(ch.rows) * T * ch.cols);
    // one slice: x0, x1, y of a chunk, then its params (2 x cols) and h0 (rows x cols)
    const size_t t_bytes = align256(max_elems * es);
    const size_t slice = 3 * t_bytes + align256(2 * C * sizeof(float)) +
                         align256(static_cast<size_t>(B) * C * sizeof(float));
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    HostPipe *pipe = nullptr;
    if ((st = get_pipe(dev, slice, &pipe)) != WKV_OK) return st;
    cudaGetLastError();
    cudaError_t e = cudaSuccess;
    for (size_t c = 0; c < chunks.size() && e == cudaSuccess; ++c) {
        const Chunk &ch = chunks[c];
        cudaStream_t sc = pipe->s[c % kPipeStreams];
        char *base = pipe->stage + (c % kPipeStreams) * pipe->slice;
        void *dx0 = base, *dx1 = base + t_bytes, *dy = base + 2 * t_bytes;
        float *dp = reinterpret_cast<float *>(base + 3 * t_bytes);
        float *dh = reinterpret_cast<float *>(base + 3 * t_bytes + align256(2 * C * sizeof(float)));
        e = copy_chunk(dx0, x0, ch, T, C, es, true, sc);
        if (e == cudaSuccess) e = copy_chunk(dx1, x1, ch, T, C, es, true, sc);
        if (e == cudaSuccess && p0 != nullptr)
            e = cudaMemcpyAsync(dp, p0 + ch.c0, ch.cols * sizeof(float), cudaMemcpyHostToDevice, sc);
        if (e == cudaSuccess && p1 != nullptr)
            e = cudaMemcpyAsync(dp + ch.cols, p1 + ch.c0, ch.cols * sizeof(float),
                                cudaMemcpyHostToDevice, sc);
        if (e == cudaSuccess && h0 != nullptr)
            e = cudaMemcpy2DAsync(dh, ch.cols * sizeof(float), h0 + ch.r0 * C + ch.c0,
                                  C * sizeof(float), ch.cols * sizeof(float), ch.rows,
                                  cudaMemcpyHostToDevice, sc);
        if (e != cudaSuccess) break;
        const typename Op::Args args = make_args(dx0, dx1, dy, p0 ? dp : nullptr,
                                                 p1 ? dp + ch.cols : nullptr, h0 ? dh : nullptr);
        st = dispatch<Op>(args, ch.rows, T, ch.cols, dt, sc, dev);
        if (st != WKV_OK) break;
        e = copy_chunk(y, dy, ch, T, C, es, false, sc);
    }
    // each stream's device status word (a device-side wait that gave up)
    // comes back with the stream's last copy, not through a blocking copy
    WsEntry *ws_of[kPipeStreams] = {};
    {
        std::lock_guard<std::mutex> lk2(g_mu);
        for (int i = 0; i < kPipeStreams; ++i) {
            pipe->status[i] = 0;
            WsEntry *w = find_ws(dev, pipe->s[i]);
            if (w == nullptr || w->base == nullptr) continue;
            ws_of[i] = w;
            cudaError_t ce = cudaMemcpyAsync(&pipe->status[i], w->base + 16, sizeof(int),
                                             cudaMemcpyDeviceToHost, pipe->s[i]);
            if (e == cudaSuccess) e = ce;
        }
    }
    // whatever happened, nothing may still be using the staging on return
    for (int i = 0; i < kPipeStreams; ++i) {
        cudaError_t se = cudaStreamSynchronize(pipe->s[i]);
        if (e == cudaSuccess) e = se;
    }
    if (st != WKV_OK) return st;
    if (e != cudaSuccess) return cuda_fail(e, "host-buffer pipeline");
    for (int i = 0; i < kPipeStreams; ++i) {
        const int code = pipe->status[i];
        if (code != 0 && ws_of[i] != nullptr) {
            cudaMemset(ws_of[i]->base + 16, 0, sizeof code);
            return fail(static_cast<wkv_status>(code),
                        "a device-side wait gave up; the affected outputs are NaN");
        }
    }
    return WKV_OK;
}

template <typename IO>
typename WkvOp<IO, sizeof(IO) == 2 ? 2 : 1>::Args wkv_host_args(const void *x0, const void *x1,
                                                               void *y, const float *w,
                                                               const float *u, const float *) {
    return {static_cast<const IO *>(x0), static_cast<const IO *>(x1), static_cast<IO *>(y), w, u};
}

ScanOp::Args scan_host_args(const void *x0, const void *x1, void *y, const float *,
                            const float *, const float *h0) {
    return {static_cast<const float *>(x0), static_cast<const float *>(x1), static_cast<float *>(y),
            h0};
}

template <typename IO>
wkv_status wkv_host_common(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                           const void *k, const void *v, void *y, CUtensorMapDataType dt) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, C, &empty);
    if (st != WKV_OK || empty) return st;
    const char *names[5] = {"w", "u", "k", "v", "y"};
    const void *ptrs[5] = {w, u, k, v, y};
    for (int i = 0; i < 5; ++i)
        if ((st = check_host(ptrs[i], names[i])) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * C * sizeof(IO);
    if (overlaps(y, n, k, n) || overlaps(y, n, v, n))
        return fail(WKV_ERR_INVALID_ARG, "y overlaps an input");
    using Op = WkvOp<IO, sizeof(IO) == 2 ? 2 : 1>;
    return run_host<Op>(B, T, C, k, v, y, w, u, nullptr, dt, &wkv_host_args<IO>);
}

wkv_status scan_host_impl(int64_t B, int64_t T, int64_t D, const float *a, const float *b,
                          const float *h0, float *h) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, D, &empty);
    if (st != WKV_OK || empty) return st;
    if ((st = check_host(a, "a")) != WKV_OK || (st = check_host(b, "b")) != WKV_OK ||
        (st = check_host(h, "h")) != WKV_OK)
        return st;
    if (h0 != nullptr && (st = check_host(h0, "h0")) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * D * sizeof(float);
    if (overlaps(h, n, a, n) || overlaps(h, n, b, n))
        return fail(WKV_ERR_INVALID_ARG, "h overlaps an input");
    return run_host<ScanOp>(B, T, D, a, b, h, nullptr, nullptr, h0,
                            CU_TENSOR_MAP_DATA_TYPE_FLOAT32, &scan_host_args);
}
