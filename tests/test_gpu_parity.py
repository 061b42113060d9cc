"""CUDA path (through the C ABI) against the float64 CPU oracle.

Element by element on seeded inputs at sizes the oracle finishes in seconds
(spanning several tiles, with ragged tails and odd channel counts that take
the element-wise copy path), and at the full workload sizes in the launch
configuration the benchmark times: every output against the float64
recurrence (the RNN-mode form, pinned to the definition on the CPU), sampled
outputs against the definition itself (eq. (14) of the RWKV page, or the
unrolled scan sum), and invariants checked over every output.

Tolerances: WKV fp32 max|err| <= 1e-5 max|v| (1e-4 max|v| for T >= 65536);
WKV bf16 <= 2e-2 max|v| and, tighter, within one bf16 ulp of the oracle plus
the fp32 bound; diagonal scan <= 1e-5 max|h|.
"""
import numpy as np
import pytest
import torch

import oracle
import pins
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m(cuda_dev):
    import rwkv_wkv_mixing_b200 as mod
    return mod


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda")


def wkv_tol(T, vmax):
    return (1e-4 if T >= 65536 else 1e-5) * vmax


def run_f32(m, w, u, k, v):
    y = m.wkv_forward(dev(w), dev(u), dev(k), dev(v))
    torch.cuda.synchronize()
    return y.double().cpu().numpy()


def run_bf16(m, x):
    y = m.wkv_forward_bf16(dev(x.w), dev(x.u), bf16_dev(x.k_bits), bf16_dev(x.v_bits))
    torch.cuda.synchronize()
    return y.float().double().cpu().numpy()


def run_scan(m, a, b, h0):
    h = m.diag_scan(dev(a), dev(b), None if h0 is None else dev(h0))
    torch.cuda.synchronize()
    return h.double().cpu().numpy()


def assert_full_wkv(got, x, tol, what, bf16=False, chans_per_pass=128):
    """Every output of a [B, T, C] WKV result against oracle.wkv_rnn, a slice
    of channels at a time so the float64 arrays stay a few hundred MB."""
    B, T, C = x.k.shape
    vmax = float(np.abs(x.v).max())
    for c0 in range(0, C, chans_per_pass):
        c1 = min(C, c0 + chans_per_pass)
        sl = lambda a: np.ascontiguousarray(a[:, :, c0:c1])   # noqa: E731
        want = oracle.wkv_rnn(x.w[c0:c1], x.u[c0:c1], sl(x.k), sl(x.v))
        g = np.asarray(got[:, :, c0:c1], dtype=np.float64)
        assert_close(g, want, tol, f"{what} channels {c0}:{c1}")
        if bf16:   # one bf16 rounding (half an ulp) on top of the fp32 bound
            assert np.all(np.abs(g - want) <= np.abs(want) * 2.0 ** -8 + 1e-5 * vmax), \
                f"{what} channels {c0}:{c1}: beyond one bf16 rounding"


def assert_close(got, want, tol, what):
    err = np.abs(got - want)
    i = int(np.argmax(err))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.flat[i] <= tol, (f"{what}: max err {err.flat[i]:.3e} > {tol:.3e} at flat {i} "
                                f"(got {got.flat[i]!r}, want {want.flat[i]!r})")


# ---------------------------------------------------------------------------
# WKV fp32
# ---------------------------------------------------------------------------
def test_wkv_tiny_workload_vs_definition(m):
    x = workloads.make_wkv("wkv_tiny")
    got = run_f32(m, x.w, x.u, x.k, x.v)
    want = oracle.wkv_direct(x.w, x.u, x.k, x.v)
    assert_close(got, want, wkv_tol(x.spec.T, np.abs(x.v).max()), "wkv_tiny")
    assert np.array_equal(got[:, 0, :], x.v[:, 0, :])   # y_0 = v_0 exactly


WKV_SHAPES = [(1, 1, 1), (1, 2, 3), (2, 255, 32), (1, 256, 64), (3, 257, 40), (1, 513, 33),
              (2, 1000, 96), (1, 777, 777), (5, 300, 4), (1, 3000, 8), (2, 2049, 36)]


@pytest.mark.parametrize("B,T,C", WKV_SHAPES)
def test_wkv_f32_shapes_vs_oracle(m, B, T, C):
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=B * 1000 + T + C)
    got = run_f32(m, x.w, x.u, x.k, x.v)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    assert_close(got, want, wkv_tol(T, np.abs(x.v).max()), f"wkv f32 {B}x{T}x{C}")


def test_wkv_f32_unaligned_pointers_take_elementwise_path(m):
    x = workloads.make_wkv("wkv_169m", B=2, T=600, C=64, seed=5)
    n = x.k.size
    kb = torch.empty(n + 1, device="cuda"); kb[1:] = dev(x.k).reshape(-1)
    vb = torch.empty(n + 3, device="cuda"); vb[3:] = dev(x.v).reshape(-1)
    yb = torch.empty(n + 2, device="cuda")
    k, v, y = kb[1:].view(x.k.shape), vb[3:].view(x.k.shape), yb[2:].view(x.k.shape)
    assert k.data_ptr() % 16 != 0
    m.wkv_forward(dev(x.w), dev(x.u), k, v, y=y)
    torch.cuda.synchronize()
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    assert_close(y.double().cpu().numpy(), want, wkv_tol(600, np.abs(x.v).max()), "unaligned")


@pytest.mark.parametrize("steps", [8, 32, 64, 128, 256])
def test_wkv_tile_length_does_not_change_results(m, steps):
    """Chunk boundaries move with the tile length; the results must not
    (the Upper/Lower split of the LRU review's parallelisation section)."""
    x = workloads.make_wkv("wkv_169m", B=2, T=1000, C=64, seed=11)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        got = run_f32(m, x.w, x.u, x.k, x.v)
    finally:
        m.wkv_set_tile_steps(old)
    assert_close(got, want, wkv_tol(1000, np.abs(x.v).max()), f"tile steps {steps}")


def test_wkv_f32_passes_the_oracle_pins(m):
    """The same closed forms, worked examples and invariants that pin the
    oracle, at fp32 tolerance."""
    def fn(w, u, k, v):
        return run_f32(m, np.float32(w), np.float32(u), np.float32(k), np.float32(v))

    # the pins' inputs are float64; this path rounds them to float32 first,
    # which alone moves an output by up to ~1e-7 of |v|
    fails = pins.wkv_single_step(fn, tol=1e-6)
    for pin in (pins.wkv_worked_example, pins.wkv_running_mean, pins.wkv_past_mean,
                pins.wkv_geometric, pins.wkv_fast_decay, pins.wkv_large_bonus):
        fails += pin(fn, tol=1e-5)
    assert fails == []


def test_wkv_f32_invariants(m):
    x = workloads.make_wkv("wkv_169m", B=3, T=1500, C=64, seed=21)
    w, u, k, v = x.w, x.u, x.k, x.v
    y = run_f32(m, w, u, k, v)
    vmax = np.abs(v).max()
    lo = np.minimum.accumulate(v, axis=1); hi = np.maximum.accumulate(v, axis=1)
    slack = 4 * np.finfo(np.float32).eps * vmax
    assert np.all(y >= lo - slack) and np.all(y <= hi + slack), "convex bound"
    # constant power-of-two v comes back exactly; another constant within a few
    # ulp (each product e*v rounds; 6 ulp observed, 32 allowed)
    assert np.array_equal(run_f32(m, w, u, k, np.full_like(v, 0.5)), np.full(v.shape, 0.5))
    c = np.float32(0.3)
    yc = run_f32(m, w, u, k, np.full_like(v, c))
    assert np.max(np.abs(yc - c)) <= 32 * np.spacing(c)
    # shift invariance in k and affine equivariance in v, to tolerance
    assert_close(run_f32(m, w, u, k + np.float32(2.5), v), y, wkv_tol(1500, vmax), "k shift")
    assert_close(run_f32(m, w, u, k, 2 * v - 1), 2 * y - 1, 3 * wkv_tol(1500, vmax), "affine")
    assert np.array_equal(y[:, 0, :], v[:, 0, :])


def test_wkv_f32_extreme_values(m):
    """Large |k| (tens, with spikes of +-80), w from 0 to 1e4, |u| up to 50:
    the running-max stabilisation keeps every output finite and accurate."""
    rng = np.random.default_rng(31)
    B, T, C = 2, 700, 32
    k = rng.normal(0, 20, (B, T, C)).astype(np.float32)
    k[:, 100, :] = 80.0; k[:, 400, :] = -80.0
    v = rng.normal(0, 1, (B, T, C)).astype(np.float32)
    w = np.concatenate([np.zeros(4), np.full(4, 1e-6), np.full(4, 1e4),
                        np.exp(rng.uniform(-6, 3, C - 12))]).astype(np.float32)
    u = np.concatenate([np.full(8, 50.0), np.full(8, -50.0), rng.normal(0, 1, C - 16)]).astype(np.float32)
    got = run_f32(m, w, u, k, v)
    want = oracle.wkv_rnn(w, u, k, v)
    assert_close(got, want, wkv_tol(T, np.abs(v).max()), "extreme")


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_wkv_large_bonus_with_a_key_far_below_the_chunk_max(m, bf16):
    """A bonus u between 18 and 44 with a sub-chunk whose first key sits 98
    below its largest: e^{u + k - M} = e^-68 is a fine weight, but e^{k - M}
    on its own (before the multiplication by e^u) would flush to zero, so the
    first step of the sequence (empty past) must not take the fixed-reference
    sweep.  Outputs finite and matching the oracle; y_0 = v_0."""
    rng = np.random.default_rng(41)
    B, T, C = 2, 700, 64
    k = rng.normal(0, 1, (B, T, C))
    k[:, ::16, :] = -68.0         # the first step of every 16- and 32-step sub-chunk
    k[:, 1::16, :] = 30.0         # and the largest key right after it
    v = rng.normal(0, 1, (B, T, C))
    w = np.exp(rng.uniform(-3, 1, C))
    u = np.concatenate([np.full(32, 30.0), rng.uniform(18, 44, C - 32)])
    kf, vf = k.astype(np.float32), v.astype(np.float32)
    wf, uf = w.astype(np.float32), u.astype(np.float32)
    if bf16:
        kb, vb = workloads.bf16_bits(kf), workloads.bf16_bits(vf)
        y = m.wkv_forward_bf16(dev(wf), dev(uf), bf16_dev(kb), bf16_dev(vb))
        kf, vf = workloads.bf16_bits_to_f32(kb), workloads.bf16_bits_to_f32(vb)
    else:
        y = m.wkv_forward(dev(wf), dev(uf), dev(kf), dev(vf))
    torch.cuda.synchronize()
    got = y.float().double().cpu().numpy()
    want = oracle.wkv_rnn(wf, uf, kf, vf)
    vmax = float(np.abs(vf).max())
    assert_close(got, want, (2e-2 if bf16 else 1e-5) * vmax, "large bonus, far key")
    assert np.array_equal(got[:, 0, :], vf[:, 0, :].astype(np.float64))


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_wkv_chunk_whose_largest_key_decays_away(m, bf16):
    """Sub-chunks whose largest key comes first and is decayed far below the
    rest (w = 10, one key of +30 among keys of -30): summed against max k
    every term would sit below 2^-60, so pass 1 re-sums them against the
    exact largest exponent; results still match the oracle."""
    rng = np.random.default_rng(37)
    B, T, C = 2, 600, 64
    k = np.full((B, T, C), -30.0) + rng.normal(0, 0.5, (B, T, C))
    k[:, ::32, :] = 30.0          # the first step of every 32-step sub-chunk
    k[:, 5::97, :16] = 45.0       # and a few late spikes elsewhere
    v = rng.normal(0, 1, (B, T, C))
    w = np.concatenate([np.full(32, 10.0), np.exp(rng.uniform(-3, 3, 32))])
    u = rng.normal(0, 1, C)
    if bf16:
        kb, vb = workloads.bf16_bits(k.astype(np.float32)), workloads.bf16_bits(v.astype(np.float32))
        k, v = workloads.bf16_bits_to_f32(kb), workloads.bf16_bits_to_f32(vb)
        y = m.wkv_forward_bf16(dev(w), dev(u), bf16_dev(kb), bf16_dev(vb))
        torch.cuda.synchronize()
        got = y.float().double().cpu().numpy()
        tol = 2e-2 * np.abs(v).max()
    else:
        k, v = k.astype(np.float32), v.astype(np.float32)
        got = run_f32(m, w.astype(np.float32), u.astype(np.float32), k, v)
        tol = wkv_tol(T, np.abs(v).max())
    want = oracle.wkv_rnn(w.astype(np.float32), u.astype(np.float32), k, v)
    assert_close(got, want, tol, "decayed-away largest key")


def test_wkv_on_side_streams_concurrently(m):
    """Two streams at once: each has its own look-back workspace."""
    xs = [workloads.make_wkv("wkv_169m", B=2, T=2000, C=128, seed=s) for s in (41, 42)]
    streams = [torch.cuda.Stream() for _ in xs]
    ins = [(dev(x.w), dev(x.u), dev(x.k), dev(x.v)) for x in xs]
    torch.cuda.synchronize()
    outs = []
    for s, a in zip(streams, ins):
        with torch.cuda.stream(s):
            outs.append(m.wkv_forward(*a, stream=s))
    torch.cuda.synchronize()
    for s in streams:
        m.wkv_device_status(s)
    for x, y in zip(xs, outs):
        want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
        assert_close(y.double().cpu().numpy(), want, wkv_tol(2000, np.abs(x.v).max()), "stream")


# ---------------------------------------------------------------------------
# WKV bf16 I/O
# ---------------------------------------------------------------------------
BF16_SHAPES = [(1, 1, 2), (2, 300, 64), (1, 513, 40), (3, 257, 30), (2, 1000, 128), (1, 100, 3)]


@pytest.mark.parametrize("B,T,C", BF16_SHAPES)
def test_wkv_bf16_shapes_vs_oracle(m, B, T, C):
    x = workloads.make_wkv("wkv_3b_bf16", B=B, T=T, C=C, seed=B * 1000 + T + C)
    got = run_bf16(m, x)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)     # from the bf16-rounded inputs
    vmax = np.abs(x.v).max()
    assert_close(got, want, 2e-2 * vmax, f"bf16 {B}x{T}x{C}")
    # tighter: one bf16 rounding (half an ulp, 2^-9 relative) on top of fp32 error
    err = np.abs(got - want)
    assert np.all(err <= np.abs(want) * 2.0 ** -8 + 1e-5 * vmax)


def test_wkv_bf16_convex_bound_is_exact(m):
    x = workloads.make_wkv("wkv_3b_bf16", B=2, T=800, C=64, seed=3)
    y = run_bf16(m, x)
    lo = np.minimum.accumulate(x.v, axis=1); hi = np.maximum.accumulate(x.v, axis=1)
    assert np.all(y >= lo) and np.all(y <= hi)
    assert np.array_equal(y[:, 0, :], x.v[:, 0, :])


# ---------------------------------------------------------------------------
# diagonal scan
# ---------------------------------------------------------------------------
SCAN_SHAPES = [(1, 1, 1), (2, 300, 32), (3, 513, 33), (4, 1000, 64), (1, 4097, 8), (2, 256, 5)]


@pytest.mark.parametrize("with_h0", [False, True])
@pytest.mark.parametrize("B,T,D", SCAN_SHAPES)
def test_scan_shapes_vs_oracle(m, B, T, D, with_h0):
    x = workloads.make_scan("scan_mingru", B=B, T=T, D=D, seed=B + T + D, with_h0=with_h0)
    got = run_scan(m, x.a, x.b, x.h0)
    want = oracle.scan_rnn(x.a, x.b, x.h0)
    assert_close(got, want, 1e-5 * max(np.abs(want).max(), 1e-30), f"scan {B}x{T}x{D}")


def test_scan_passes_the_oracle_pins(m):
    def fn(a, b, h0):
        return run_scan(m, np.float32(a), np.float32(b), None if h0 is None else np.float32(h0))

    fails = []
    fails += pins.scan_worked_example(fn, tol=1e-6)
    fails += pins.scan_closed_forms(fn, tol=1e-4, exact_tol=1e-6)
    fails += pins.scan_chaining(fn, tol=1e-5)
    fails += pins.scan_mingru_convex(fn, tol=1e-6)
    assert fails == []


@pytest.mark.parametrize("steps", [8, 64, 256])
def test_scan_tile_length_does_not_change_results(m, steps):
    x = workloads.make_scan("scan_mingru", B=2, T=1100, D=40, seed=7, with_h0=True)
    want = oracle.scan_rnn(x.a, x.b, x.h0)
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        got = run_scan(m, x.a, x.b, x.h0)
    finally:
        m.wkv_set_tile_steps(old)
    assert_close(got, want, 1e-5 * np.abs(want).max(), f"scan tile steps {steps}")


# ---------------------------------------------------------------------------
# argument checks that reach the C library
# ---------------------------------------------------------------------------
def test_c_abi_rejects_bad_pointers(m):
    lib = m.lib
    k = torch.zeros(2, 8, 4, device="cuda"); w = torch.zeros(4, device="cuda")
    host = np.zeros(64, dtype=np.float32)
    hp = host.ctypes.data
    s = None
    # host memory where device memory is required
    assert lib.wkv_forward(2, 8, 4, w.data_ptr(), w.data_ptr(), hp, k.data_ptr(),
                           torch.empty_like(k).data_ptr(), s) == m.WKV_ERR_INVALID_ARG
    # output aliasing an input
    assert lib.wkv_forward(2, 8, 4, w.data_ptr(), w.data_ptr(), k.data_ptr(), k.data_ptr(),
                           k.data_ptr(), s) == m.WKV_ERR_INVALID_ARG
    # misaligned fp32 pointer
    raw = torch.zeros(2 * 8 * 4 * 4 + 8, dtype=torch.uint8, device="cuda")
    assert lib.wkv_forward(2, 8, 4, w.data_ptr(), w.data_ptr(), raw.data_ptr() + 1,
                           k.data_ptr(), torch.empty_like(k).data_ptr(), s) == m.WKV_ERR_ALIGNMENT
    # NULL
    assert lib.diag_scan(2, 8, 4, None, k.data_ptr(), None, torch.empty_like(k).data_ptr(),
                         s) == m.WKV_ERR_INVALID_ARG
    m.wkv_device_status()


# ---------------------------------------------------------------------------
# full-size workloads, in the configuration the benchmark launches
# ---------------------------------------------------------------------------
def _sample_points(rng, B, T, channels, n):
    """n points: half anywhere, a quarter near the end of the sequence and a
    quarter within two steps of a 256-step tile edge."""
    n_any, n_end = n // 2, n // 4
    n_edge = n - n_any - n_end
    b = rng.integers(0, B, n)
    c = rng.choice(channels, n)
    edges = (rng.integers(0, max(T // 256, 1), n_edge) + 1) * 256 + rng.integers(-2, 2, n_edge)
    t = np.concatenate([rng.integers(0, T, n_any),
                        T - 1 - rng.integers(0, min(T, 300), n_end),
                        np.clip(edges, 0, T - 1)])
    return b, t, c


@pytest.mark.parametrize("name", ["wkv_169m", "wkv_3b_bf16", "wkv_long"])
def test_wkv_full_size_workload(m, name):
    x = workloads.make_wkv(name)
    B, T, C = x.k.shape
    if x.spec.dtype == "bf16":
        y = m.wkv_forward_bf16(dev(x.w), dev(x.u), bf16_dev(x.k_bits), bf16_dev(x.v_bits))
    else:
        y = m.wkv_forward(dev(x.w), dev(x.u), dev(x.k), dev(x.v))
    m.wkv_device_status()
    vmax = float(np.abs(x.v).max())
    # every output: finite and inside the running [min v, max v] envelope
    vd = dev(x.v)
    yf = y.float()
    lo = torch.cummin(vd, dim=1).values; hi = torch.cummax(vd, dim=1).values
    slack = 0.0 if x.spec.dtype == "bf16" else 4 * 1.2e-7 * vmax
    assert bool(torch.isfinite(yf).all())
    assert bool((yf >= lo - slack).all()) and bool((yf <= hi + slack).all())
    assert torch.equal(yf[:, 0, :], vd[:, 0, :])
    del lo, hi, vd
    # sampled outputs against the definition, channel subset passed to the oracle
    rng = np.random.default_rng(0)
    chans = np.sort(rng.choice(C, min(C, 24), replace=False))
    b, t, cidx = _sample_points(rng, B, T, np.arange(chans.size), 2000)
    sub_k = np.ascontiguousarray(x.k[:, :, chans]); sub_v = np.ascontiguousarray(x.v[:, :, chans])
    flat = (b * T + t) * chans.size + cidx
    want = oracle.wkv_direct_points(x.w[chans], x.u[chans], sub_k, sub_v, flat)
    got = yf[torch.from_numpy(b).cuda(), torch.from_numpy(t).cuda(),
             torch.from_numpy(chans[cidx]).cuda()].double().cpu().numpy()
    tol = 2e-2 * vmax if x.spec.dtype == "bf16" else wkv_tol(T, vmax)
    assert_close(got, want, tol, name)
    # every output against the float64 recurrence
    assert_full_wkv(yf.cpu().numpy(), x, tol, name, bf16=x.spec.dtype == "bf16")


def test_scan_full_size_workload(m):
    x = workloads.make_scan("scan_mingru")
    B, T, D = x.a.shape
    h = m.diag_scan(dev(x.a), dev(x.b), None)
    m.wkv_device_status()
    # minGRU form: each h_t is a convex combination of h0 = 0 and h~_0..h~_t
    ht = dev(x.h_tilde)
    lo = torch.clamp(torch.cummin(ht, dim=1).values, max=0.0)
    hi = torch.clamp(torch.cummax(ht, dim=1).values, min=0.0)
    hmax = float(torch.abs(h).max())
    assert bool(torch.isfinite(h).all())
    assert bool((h >= lo - 1e-5 * hmax).all()) and bool((h <= hi + 1e-5 * hmax).all())
    del ht, lo, hi
    rng = np.random.default_rng(1)
    b, t, d = _sample_points(rng, B, T, np.arange(D), 2000)
    flat = (b * T + t) * D + d
    want = oracle.scan_direct_points(x.a, x.b, None, flat)
    got = h[torch.from_numpy(b).cuda(), torch.from_numpy(t).cuda(),
            torch.from_numpy(d).cuda()].double().cpu().numpy()
    assert_close(got, want, 1e-5 * hmax, "scan_mingru")
    # every output against the float64 recurrence
    want_full = oracle.scan_rnn(x.a, x.b, None)
    assert_close(h.double().cpu().numpy(), want_full, 1e-5 * float(np.abs(want_full).max()),
                 "scan_mingru every output")


# ---------------------------------------------------------------------------
# CUDA graphs: the look-back counters live on the device and reset themselves,
# so replaying a captured call gives the right answer every time
# ---------------------------------------------------------------------------
def test_wkv_graph_capture_and_replay(m):
    x = workloads.make_wkv("wkv_169m", B=2, T=1500, C=96, seed=51)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    y = torch.empty_like(k)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        m.wkv_forward(w, u, k, v, y=y, stream=s)   # sizes the workspace before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(3):
            m.wkv_forward(w, u, k, v, y=y, stream=s)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    tol = wkv_tol(1500, np.abs(x.v).max())
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert_close(y.double().cpu().numpy(), want, tol, "graph replay")
    m.wkv_device_status(s)


def test_persistent_and_blockwise_kernels_agree(m):
    """Tile length 32 runs one thread block per tile; 128 runs the persistent
    pipeline.  Both must match the oracle on a chained, ragged problem."""
    x = workloads.make_wkv("wkv_3b_bf16", B=3, T=1111, C=192, seed=61)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    old = m.wkv_get_tile_steps()
    outs = {}
    try:
        for steps in (32, 128):
            m.wkv_set_tile_steps(steps)
            outs[steps] = run_bf16(m, x)
    finally:
        m.wkv_set_tile_steps(old)
    for steps, got in outs.items():
        assert_close(got, want, 2e-2 * np.abs(x.v).max(), f"bf16 tile steps {steps}")


# ---------------------------------------------------------------------------
# many launches queued back to back: the persistent pipeline's stage hand-off
# and the look-back counters must hold up launch after launch
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("op", ["wkv", "wkv_bf16", "scan"])
def test_many_back_to_back_launches(m, op):
    n_out, n_launch = 32, 256
    if op == "scan":
        x = workloads.make_scan("scan_mingru", B=8, T=2048, D=256, seed=71)
        a, b = dev(x.a), dev(x.b)
        want = torch.from_numpy(oracle.scan_rnn(x.a, x.b, None)).to("cuda")
        tol = 1e-5 * float(want.abs().max())
        outs = [torch.empty_like(a) for _ in range(n_out)]
        for i in range(n_launch):
            m.diag_scan(a, b, None, h=outs[i % n_out])
    else:
        name = "wkv_3b_bf16" if op == "wkv_bf16" else "wkv_169m"
        x = workloads.make_wkv(name, B=4, T=2048, C=256, seed=72)
        w, u = dev(x.w), dev(x.u)
        if op == "wkv_bf16":
            k, v = bf16_dev(x.k_bits), bf16_dev(x.v_bits)
            fn, tol = m.wkv_forward_bf16, 2e-2 * float(np.abs(x.v).max())
        else:
            k, v = dev(x.k), dev(x.v)
            fn, tol = m.wkv_forward, wkv_tol(2048, float(np.abs(x.v).max()))
        want = torch.from_numpy(oracle.wkv_rnn(x.w, x.u, x.k, x.v)).to("cuda")
        outs = [torch.empty_like(k) for _ in range(n_out)]
        for i in range(n_launch):
            fn(w, u, k, v, y=outs[i % n_out])
    m.wkv_device_status()
    worst = max(float((o.double() - want).abs().max()) for o in outs)
    assert worst <= tol, f"{op}: worst max err over {n_out} outputs {worst} > {tol}"


# ---------------------------------------------------------------------------
# host-buffer entry points (chunked, overlapped copy / compute pipeline)
# ---------------------------------------------------------------------------
# (calls are cut into chunks of at least 16 MB of input, up to 8 of them)
@pytest.mark.parametrize("B,T,C,pinned", [(8, 2048, 512, True),   # 4 chunks of batch rows
                                          (1, 16384, 1024, True),  # 8 channel slices, 2-D copies
                                          (3, 4000, 512, False),  # pageable memory, 3 chunks
                                          (8, 700, 96, True),     # one chunk
                                          (1, 50, 33, True)])     # one chunk, any shape
def test_wkv_host_entry_point(m, B, T, C, pinned):
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=B + T + C)
    h = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory() if pinned \
        else torch.from_numpy(np.ascontiguousarray(a))   # noqa: E731
    y = m.wkv_forward_host(h(x.w), h(x.u), h(x.k), h(x.v))
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    assert_close(y.double().numpy(), want, wkv_tol(T, np.abs(x.v).max()), f"host {B}x{T}x{C}")


def test_wkv_bf16_host_entry_point(m):
    x = workloads.make_wkv("wkv_3b_bf16", B=1, T=900, C=384, seed=81)
    kb = torch.from_numpy(x.k_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    vb = torch.from_numpy(x.v_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    y = m.wkv_forward_bf16_host(torch.from_numpy(x.w), torch.from_numpy(x.u), kb, vb)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    assert_close(y.float().double().numpy(), want, 2e-2 * np.abs(x.v).max(), "bf16 host")


@pytest.mark.parametrize("B,T,D", [(16, 600, 64), (16, 4096, 256), (1, 16384, 512)])
def test_scan_host_entry_point(m, B, T, D):
    x = workloads.make_scan("scan_mingru", B=B, T=T, D=D, seed=91, with_h0=True)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()   # noqa: E731
    hh = m.diag_scan_host(t(x.a), t(x.b), t(x.h0))
    want = oracle.scan_rnn(x.a, x.b, x.h0)
    assert_close(hh.double().numpy(), want, 1e-5 * np.abs(want).max(), "scan host")


def test_host_entry_point_rejects_device_memory(m):
    k = torch.zeros(1, 4, 4, device="cuda")
    w = torch.zeros(4)
    assert m.lib.wkv_forward_host(1, 4, 4, w.data_ptr(), w.data_ptr(), k.data_ptr(),
                                  k.data_ptr(), k.data_ptr()) == m.WKV_ERR_INVALID_ARG
