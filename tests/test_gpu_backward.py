"""WKV gradients on the GPU through the C ABI against the float64 oracle
(the recurrence form, itself pinned to the definition, autodiff and central
differences).

Tolerance: each gradient array within 1e-4 of its own largest magnitude
(fp32 sums over up to T terms of a softmax-weighted mean); gw and gu, sums
over B T terms, within 2e-4 (1e-3 for keys of N(0, 15)).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m(cuda_dev):
    import rwkv_wkv_mixing_b200 as mod
    return mod


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda")


def check(got, want, rel, what):
    got = np.asarray(got, np.float64)
    scale = max(float(np.abs(want).max()), 1e-30)
    err = np.abs(got - want)
    i = int(np.argmax(err))
    assert np.all(np.isfinite(got)), f"{what}: non-finite"
    assert err.flat[i] <= rel * scale, (f"{what}: max err {err.flat[i]:.3e} > {rel * scale:.3e} "
                                        f"at {i} (got {got.flat[i]!r}, want {want.flat[i]!r})")


def run(m, x, gy):
    out = m.wkv_backward(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(gy))
    torch.cuda.synchronize()
    return [t.double().cpu().numpy() for t in out]


def compare(m, x, gy, what, sums_rel=2e-4):
    got = run(m, x, gy)
    want = oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, gy.astype(np.float32))
    for name, g, wv, rel in zip(("gk", "gv", "gw", "gu"), got, want,
                                (1e-4, 1e-4, sums_rel, sums_rel)):
        check(g, wv, rel, f"{what} {name}")


# C = 33 and 130 (rows not a multiple of 16 bytes) take the per-segment
# kernels; the others the tiled ones (128-step tiles, 32-step segments):
# one segment, one partial tile, several tiles with ragged tails in time
# and channels, long chains; B=9 T=3800 has 1071 rows x segments, beyond
# the one-level gw, gu sum (1024), so its two-level sum runs on the tiled path
SHAPES = [(1, 1, 4), (2, 5, 32), (2, 64, 40), (3, 300, 33), (1, 1024, 64), (4, 700, 130),
          (1, 4100, 40), (2, 257, 96), (1, 31, 8), (2, 129, 36), (1, 128, 32), (3, 2000, 100),
          (2, 4129, 64), (9, 3800, 64)]


@pytest.mark.parametrize("B,T,C", SHAPES)
def test_backward_vs_oracle(m, B, T, C):
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=B * 7 + T + C)
    gy = np.random.default_rng(T + C).normal(0, 1, x.k.shape).astype(np.float32)
    compare(m, x, gy, f"backward {B}x{T}x{C}")


def test_backward_small_vs_definition(m):
    """Against the O(T^2) definition form directly."""
    x = workloads.make_wkv("wkv_tiny", B=2, T=64, C=16, seed=3)
    gy = np.random.default_rng(3).normal(0, 1, x.k.shape).astype(np.float32)
    got = run(m, x, gy)
    want = oracle.wkv_backward_direct(x.w, x.u, x.k, x.v, gy)
    for name, g, wv in zip(("gk", "gv", "gw", "gu"), got, want):
        check(g, wv, 1e-4, f"definition {name}")


def test_backward_long_keys(m):
    """wkv_long's distributions (k ~ N(0,3), slow decays) over 4096 steps."""
    x = workloads.make_wkv("wkv_long", B=1, T=4096, C=64, seed=5)
    gy = np.random.default_rng(5).normal(0, 1, x.k.shape).astype(np.float32)
    compare(m, x, gy, "backward long keys")


def test_backward_extreme_values(m):
    rng = np.random.default_rng(6)
    B, T, C = 2, 400, 32
    k = rng.normal(0, 15, (B, T, C)).astype(np.float32)
    v = rng.normal(0, 1, (B, T, C)).astype(np.float32)
    w = np.concatenate([np.zeros(4), np.full(4, 1e-5), np.full(4, 40.0),
                        np.exp(rng.uniform(-5, 2, C - 12))]).astype(np.float32)
    u = rng.normal(0, 3, C).astype(np.float32)
    gy = rng.normal(0, 1, (B, T, C)).astype(np.float32)

    class X:
        pass
    x = X()
    x.w, x.u, x.k, x.v = w, u, k, v
    # keys of N(0, 15) let single steps dominate the sums over B T steps in
    # gw and gu, whose fp32 accumulation then keeps ~1e-3 of their size
    compare(m, x, gy, "backward extreme", sums_rel=1e-3)


def test_backward_repeated_calls_with_a_forward_between(m):
    """The gradient step's kernels keep counters (the forward look-back's
    tickets and epoch, the gw/gu sum's counters) in per-stream workspaces the
    forward kernels share: calls back to back, with a forward call in
    between, must each find them reset."""
    x = workloads.make_wkv("wkv_169m", B=2, T=1000, C=96, seed=21)
    gy = np.random.default_rng(21).normal(0, 1, x.k.shape).astype(np.float32)
    want = oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, gy)
    w, u, k, v, g = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(gy)
    for call in range(3):
        out = m.wkv_backward(w, u, k, v, g)
        m.wkv_forward(w, u, k, v)
        torch.cuda.synchronize()
        for name, got, wv, rel in zip(("gk", "gv", "gw", "gu"), out, want,
                                      (1e-4, 1e-4, 2e-4, 2e-4)):
            check(got.double().cpu().numpy(), wv, rel, f"call {call} {name}")
    m.wkv_device_status()  # raises if a device-side wait gave up


def test_backward_inputs_written_just_before_each_call(m):
    """The gradient pass starts loading k, v and gy before waiting for the
    step's first kernels (which write only the scratch): each call's gy
    (and k) comes from a kernel launched on the same stream right before the
    call, different every time, and without a synchronisation between the
    calls; every call must see its own inputs.  gk, gv, gw, gu are linear
    in gy, and scaling by a power of two is exact in floating point."""
    x = workloads.make_wkv("wkv_169m", B=2, T=1000, C=96, seed=23)
    gy0 = np.random.default_rng(23).normal(0, 1, x.k.shape).astype(np.float32)
    want = oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, gy0)
    w, u, k0, v, g0 = dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(gy0)
    k = torch.empty_like(k0)
    g = torch.empty_like(g0)
    outs = []
    for call in range(6):
        k.copy_(k0 + 0.0)             # rewritten by a kernel just before the call
        torch.mul(g0, float(2 ** call), out=g)
        outs.append([t.clone() for t in m.wkv_backward(w, u, k, v, g)])
        k.zero_()                     # and overwritten right after it
        g.fill_(float("nan"))
    torch.cuda.synchronize()
    for call, out in enumerate(outs):
        for name, got, wv, rel in zip(("gk", "gv", "gw", "gu"), out, want,
                                      (1e-4, 1e-4, 2e-4, 2e-4)):
            check(got.double().cpu().numpy() / 2 ** call, wv, rel, f"call {call} {name}")
    m.wkv_device_status()


def test_backward_on_two_streams_concurrently(m):
    """Two gradient steps in flight at once on two streams: each stream has
    its own scratch, look-back workspace and sum counters."""
    xs = [workloads.make_wkv("wkv_169m", B=2, T=1500, C=64, seed=s) for s in (31, 32)]
    gys = [np.random.default_rng(s).normal(0, 1, x.k.shape).astype(np.float32)
           for s, x in zip((31, 32), xs)]
    ins = [(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(g)) for x, g in zip(xs, gys)]
    streams = [torch.cuda.Stream() for _ in xs]
    torch.cuda.synchronize()
    outs = []
    for rep in range(3):
        for st, a in zip(streams, ins):
            with torch.cuda.stream(st):
                outs.append((rep, [t for t in m.wkv_backward(*a, stream=st)]))
    torch.cuda.synchronize()
    for st in streams:
        m.wkv_device_status(st)
    wants = [oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, g) for x, g in zip(xs, gys)]
    for i, (rep, out) in enumerate(outs):
        want = wants[i % 2]
        for name, got, wv, rel in zip(("gk", "gv", "gw", "gu"), out, want,
                                      (1e-4, 1e-4, 2e-4, 2e-4)):
            check(got.double().cpu().numpy(), wv, rel, f"stream {i % 2} call {rep} {name}")


def test_backward_every_reverse_frame(m):
    """Keys spread wide enough (N(0, 10)) that some 32-step segments keep the
    forward pass's fixed reference but not the reverse one (a denominator
    between e^-69 and e^-30), fast decays (w up to e^2) that leave the state
    after a segment far above the segment's frame, and plain channels beside
    them: every combination of fixed and per-step passes in one launch."""
    rng = np.random.default_rng(11)
    B, T, C = 2, 640, 64
    k = rng.normal(0, 1, (B, T, C)).astype(np.float32)
    k[:, :, ::2] *= 10.0
    v = rng.normal(0, 1, (B, T, C)).astype(np.float32)
    w = np.exp(rng.uniform(-3, 2, C)).astype(np.float32)
    u = rng.normal(0, 1, C).astype(np.float32)
    gy = rng.normal(0, 1, (B, T, C)).astype(np.float32)

    class X:
        pass
    x = X()
    x.w, x.u, x.k, x.v = w, u, k, v
    compare(m, x, gy, "backward reverse frames", sums_rel=1e-3)


def test_backward_identities_at_full_size(m):
    """wkv_169m (B=8 T=1024 C=768): every gradient against the float64
    recurrence; the k-shift identity sum_j gk_j = 0 and the constant identity
    sum_j gv_j = sum_t gy_t per row and channel; and the decay identity
    gw = sum_j j gk_j - gu over all channels (w enters row t's logits of
    eq. (14) as j w - (t-1) w, and a softmax ignores a row constant)."""
    x = workloads.make_wkv("wkv_169m")
    gy = np.random.default_rng(7).normal(0, 1, x.k.shape).astype(np.float32)
    gk, gv, gw, gu = run(m, x, gy)
    T = x.spec.T
    assert np.max(np.abs(gk.sum(axis=1))) <= 1e-3 * np.abs(gk).max() * np.sqrt(T)
    assert np.allclose(gv.sum(axis=1), gy.astype(np.float64).sum(axis=1),
                       atol=1e-3 * np.abs(gv).max() * np.sqrt(T))
    j = np.arange(T, dtype=np.float64)[None, :, None]
    moment = (j * gk).sum(axis=(0, 1)) - gu
    # the moment weighs gk's fp32 errors by j <= T over B T terms of either
    # sign: errors of 5e-6 max|gk| at random give about this much (a dropped
    # term or a wrong sign in gw moves it by the size of gw, ~60x more here)
    tol = 1e-5 * np.abs(gk).max() * T * np.sqrt(x.spec.B * T) + 2e-4 * np.abs(gw).max()
    assert np.max(np.abs(moment - gw)) <= tol, f"decay identity off by {np.max(np.abs(moment - gw))}"
    want = oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, gy)
    for name, g, wv, rel in zip(("gk", "gv", "gw", "gu"), (gk, gv, gw, gu), want,
                                (1e-4, 1e-4, 2e-4, 2e-4)):
        check(g, wv, rel, f"full size {name}")


def test_backward_argument_errors(m):
    x = workloads.make_wkv("wkv_169m", B=1, T=10, C=32, seed=1)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    gy = torch.ones_like(k)
    gv, gw, gu = torch.empty_like(k), torch.empty_like(w), torch.empty_like(u)
    st = m.lib.wkv_backward(1, 10, 32, w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(),
                            gy.data_ptr(), k.data_ptr(), gv.data_ptr(), gw.data_ptr(),
                            gu.data_ptr(), None)   # gk written over k
    assert st == m.WKV_ERR_INVALID_ARG
    st = m.lib.wkv_backward(0, 10, 32, w.data_ptr(), u.data_ptr(), None, None, None, None, None,
                            gw.data_ptr(), gu.data_ptr(), None)
    torch.cuda.synchronize()
    assert st == m.WKV_OK and float(gw.abs().max()) == 0.0 and float(gu.abs().max()) == 0.0
