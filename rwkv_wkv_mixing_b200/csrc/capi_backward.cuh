// Host side of the WKV gradients (wkv_backward): the tiled path's launch
// configuration and launches (persistent_bwd.cuh), the per-segment path's
// (wkv_backward.cuh), argument checks and the scratch.  Included by capi.cu
// inside its anonymous namespace, after the shared host infrastructure
// (errors, argument checks, workspaces, tensor maps, launch helpers); the
// kernel headers it launches (persistent_bwd.cuh, wkv_backward.cuh) are
// included at the top of capi.cu.  Kept apart so that the forward entry
// points' code does not change with it.
#pragma once

// ---- WKV gradients on the tiled path (persistent_bwd.cuh) -------------------------
// 1: shapes a tensor map describes take the tiled gradient kernels; 0: every
// shape takes the per-segment kernels of wkv_backward.cuh
#ifndef WKV_BWD_TILED
#define WKV_BWD_TILED 1
#endif
// states kernel: 128-step tiles, three groups of four compute warps (one
// 32-step segment each) and a carry warp, four stages of k and v (each
// group's gy tile in its own buffer; five were 14 % slower on B=1 T=32768:
// more tiles of one chain in flight); gradients kernel:
// eleven compute warps (168 registers: three warps per SM sub-partition),
// sixteen 32-step stages of k, v and gy
#ifndef WKV_BWD_STATES_CFG
#define WKV_BWD_STATES_CFG 128, 4, 3, 4
#endif
#ifndef WKV_BWD_GRADS_CFG
#define WKV_BWD_GRADS_CFG 11, 16
#endif
using BwdStates = BwdStatesCfg<WKV_BWD_STATES_CFG>;
using BwdGrads = BwdGradsCfg<WKV_BWD_GRADS_CFG>;
constexpr int kBwdStatesLT = BwdStates::kLT;

Geometry bwd_geometry(int64_t B, int64_t T, int64_t C, int lt) {
    Geometry g{};
    g.B = static_cast<int>(B);
    g.T = static_cast<int>(T);
    g.C = static_cast<int>(C);
    g.n_cg = static_cast<int>((C + 31) / 32);
    g.n_seg = static_cast<int>((T + lt - 1) / lt);
    g.tiles_per_seg = static_cast<int>(B * g.n_cg);
    g.tiles = g.n_seg * g.tiles_per_seg;
    g.use_tma = 1;
    g.spin_limit = g_fault_spin_limit.load() > 0 ? g_fault_spin_limit.load() : kSpinLimit;
    g.skip_publish = g_fault_skip_tile.load();
    g.params_staged = 1;
    return g;
}

template <typename K, typename... A>
wkv_status launch_pdl(K kern, int grid, int threads, size_t smem, cudaStream_t stream, A... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaGetLastError();
    cudaError_t err = cudaLaunchKernelEx(&cfg, kern, args...);
    if (err == cudaSuccess) err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}

// The four launches of one gradient step on the tiled path, or *done = false
// (nothing launched) when a tensor map cannot be made for these buffers.
wkv_status launch_bwd_tiled(const WkvBwdArgs &a, int64_t B, int64_t T, int64_t C,
                            cudaStream_t stream, int dev, bool *done) {
    *done = false;
    const auto dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    // [0..2] k, v, gy in 128-step boxes (states kernel); [3..7] k, v, gy, gk,
    // gv in 32-step boxes (gradients kernel)
    CUtensorMap m[8];
    std::memset(m, 0, sizeof m);
    const void *src[8] = {a.k, a.v, a.gy, a.k, a.v, a.gy, a.gk, a.gv};
    for (int i = 0; i < 8; ++i)
        if (!make_map(&m[i], src[i], dt, sizeof(float), B, T, C, 32,
                      i < 3 ? kBwdStatesLT : kBwdSegSteps))
            return WKV_OK;
    const Geometry gs = bwd_geometry(B, T, C, kBwdStatesLT);
    Geometry gg = bwd_geometry(B, T, C, kBwdSegSteps);
    gg.skip_publish = -1;
    // the look-back workspace of this stream (its status word reports the
    // timeouts of both persistent kernels)
    Workspace ws;
    std::memset(&ws, 0, sizeof ws);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        WsEntry *e = nullptr;
        wkv_status st = ensure_ws(dev, stream, ws_bytes(static_cast<size_t>(gs.tiles), 32), &e);
        if (st != WKV_OK) return st;
        ws.ticket = reinterpret_cast<unsigned int *>(e->base);
        ws.done = reinterpret_cast<unsigned int *>(e->base + 4);
        ws.epoch = reinterpret_cast<unsigned long long *>(e->base + 8);
        ws.status = reinterpret_cast<int *>(e->base + 16);
        ws.records = reinterpret_cast<uint4 *>(e->base + kWsHeader);
    }
    const BwdTileArgs ta{a.w, a.u, a.k, a.v, a.fwd, a.rev, a.partial, a.S};
    auto ks = wkv_bwd_states_kernel<WKV_BWD_STATES_CFG>;
    auto kg = wkv_bwd_grads_tiles_kernel<WKV_BWD_GRADS_CFG>;
    static std::atomic<uint64_t> conf_s{0}, conf_g{0};
    wkv_status st = configure_once(ks, BwdStates::kSmemBytes, dev, conf_s);
    if (st == WKV_OK) st = configure_once(kg, BwdGrads::kSmemBytes, dev, conf_g);
    if (st != WKV_OK) return st;
    *done = true;
    const int sms = sm_count(dev);
    if ((st = launch_pdl(ks, std::min(gs.tiles, sms), BwdStates::kThreads, BwdStates::kSmemBytes,
                         stream, m[0], m[1], m[2], ta, gs, ws)) != WKV_OK)
        return st;
    const int n_cg = static_cast<int>((C + 31) / 32);
    if ((st = launch_pdl(wkv_bwd_rev_carry_kernel, static_cast<int>(B) * n_cg, 32 * kCarryWarps, 0,
                         stream, a)) != WKV_OK)
        return st;
    if ((st = launch_pdl(kg, std::min(gg.tiles, sms), BwdGrads::kThreads, BwdGrads::kSmemBytes,
                         stream, m[3], m[4], m[5], m[6], m[7], ta, gg, ws)) != WKV_OK)
        return st;
    // gw, gu: one level while the (row, segment)s are few, else two
    if (static_cast<int64_t>(a.B) * a.S <= kReduceOneLevelRows)
        return launch_pdl(wkv_bwd_reduce_one_kernel, n_cg, 32 * kReduceOneWarps, 0, stream, a);
    return launch_pdl(wkv_bwd_reduce_kernel, n_cg * kReduceParts, 32 * kReduceWarps, 0, stream, a);
}

wkv_status backward_impl(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                         const float *k, const float *v, const float *gy, float *gk, float *gv,
                         float *gw, float *gu, cudaStream_t stream) {
    t_err.clear();
    bool empty = false;
    wkv_status st = check_sizes(B, T, C, &empty);
    if (st != WKV_OK) return st;
    if (empty) {
        if (B == 0 || T == 0) {  // no outputs: gw, gu are empty sums (C may be > 0)
            if (C > 0) {
                int dev0 = 0;
                if ((st = current_device(&dev0)) != WKV_OK) return st;
                const size_t nc0 = static_cast<size_t>(C) * sizeof(float);
                if ((st = check_buffer(gw, nc0, 4, "gw", dev0)) != WKV_OK) return st;
                if ((st = check_buffer(gu, nc0, 4, "gu", dev0)) != WKV_OK) return st;
                cudaError_t e = cudaMemsetAsync(gw, 0, nc0, stream);
                if (e == cudaSuccess) e = cudaMemsetAsync(gu, 0, nc0, stream);
                if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(gw, gu)");
            }
        }
        return WKV_OK;
    }
    int dev = 0;
    if ((st = current_device(&dev)) != WKV_OK) return st;
    const size_t n = static_cast<size_t>(B) * T * C * sizeof(float);
    const size_t nc = static_cast<size_t>(C) * sizeof(float);
    const struct { const void *p; size_t bytes; const char *name; } in[] = {
        {w, nc, "w"}, {u, nc, "u"}, {k, n, "k"}, {v, n, "v"}, {gy, n, "gy"}};
    const struct { const void *p; size_t bytes; const char *name; } out[] = {
        {gk, n, "gk"}, {gv, n, "gv"}, {gw, nc, "gw"}, {gu, nc, "gu"}};
    for (const auto &x : in)
        if ((st = check_buffer(x.p, x.bytes, 4, x.name, dev)) != WKV_OK) return st;
    for (const auto &x : out)
        if ((st = check_buffer(x.p, x.bytes, 4, x.name, dev)) != WKV_OK) return st;
    for (size_t i = 0; i < 4; ++i) {
        for (const auto &x : in)
            if (overlaps(out[i].p, out[i].bytes, x.p, x.bytes))
                return fail(WKV_ERR_INVALID_ARG, "%s overlaps input %s", out[i].name, x.name);
        for (size_t j = i + 1; j < 4; ++j)
            if (overlaps(out[i].p, out[i].bytes, out[j].p, out[j].bytes))
                return fail(WKV_ERR_INVALID_ARG, "%s overlaps %s", out[i].name, out[j].name);
    }
    // tiled path: every buffer 16-byte aligned, rows of a multiple of 16 bytes
    const void *tptrs[7] = {k, v, gy, gk, gv, u, w};
    const bool tiled = WKV_BWD_TILED && tma_eligible(tptrs, 7, sizeof(float), T, C);
    // segments of kSeg steps for the per-segment kernels, kBwdSegSteps on the
    // tiled path; the scratch is sized for the shorter ones, so a call that
    // meant to go tiled can still take the per-segment kernels
    const int64_t S16 = (T + kSeg - 1) / kSeg;
    const int64_t seg_threads = B * S16 * C;
    if ((seg_threads + kBwdThreads - 1) / kBwdThreads > INT32_MAX)
        return fail(WKV_ERR_INVALID_ARG, "B*C*T too large for one launch");
    // scratch per (row, segment, channel): the forward (3) and reverse (5)
    // summaries, then carries, and the gw, gu partials (2); then the
    // first-level sums of gw, gu.  The sum's counters, one per 32 channels,
    // have a workspace of their own: zero when allocated, and every launch
    // leaves them at zero.
    const int64_t n_cg = (C + 31) / 32;
    const size_t ns = static_cast<size_t>(B) * S16 * C;
    const size_t nred = static_cast<size_t>(kReduceParts) * 2 * C;
    WsEntry *e = nullptr, *ce = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if ((st = ensure_ws(dev, stream, (10 * ns + nred) * sizeof(float), &e, 1)) != WKV_OK)
            return st;
        if ((st = ensure_ws(dev, stream, static_cast<size_t>(n_cg) * sizeof(unsigned), &ce, 2)) !=
            WKV_OK)
            return st;
    }
    float *scratch = reinterpret_cast<float *>(e->base);
    WkvBwdArgs a{w, u, k, v, gy, gk, gv, scratch, scratch + 3 * ns, scratch + 8 * ns, gw, gu,
                 scratch + 10 * ns, reinterpret_cast<unsigned *>(ce->base),
                 static_cast<int>(B), static_cast<int>(T), static_cast<int>(C),
                 static_cast<int>(S16), kSeg};
    if (tiled) {
        WkvBwdArgs at = a;
        at.L = kBwdSegSteps;
        at.S = static_cast<int>((T + kBwdSegSteps - 1) / kBwdSegSteps);
        bool done = false;
        if ((st = launch_bwd_tiled(at, B, T, C, stream, dev, &done)) != WKV_OK || done) return st;
        // no tensor map for these buffers after all: the per-segment kernels
    }
    const unsigned g_seg = static_cast<unsigned>((seg_threads + kBwdThreads - 1) / kBwdThreads);
    const unsigned g_chan = static_cast<unsigned>(B * n_cg);
    const unsigned g_red = static_cast<unsigned>(n_cg * kReduceParts);
    wkv_bwd_fwd_summary_kernel<<<g_seg, kBwdThreads, 0, stream>>>(a);
    wkv_bwd_fwd_carry_kernel<<<g_chan, 32 * kCarryWarps, 0, stream>>>(a);
    wkv_bwd_rev_summary_kernel<<<g_seg, kBwdThreads, 0, stream>>>(a);
    wkv_bwd_rev_carry_kernel<<<g_chan, 32 * kCarryWarps, 0, stream>>>(a);
    wkv_bwd_grads_kernel<<<g_seg, kBwdThreads, 0, stream>>>(a);
    wkv_bwd_reduce_kernel<<<g_red, 32 * kReduceWarps, 0, stream>>>(a);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
    return WKV_OK;
}
