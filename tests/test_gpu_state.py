"""WKV with a state in and out (streaming and RNN-mode decoding) on the GPU,
through the C ABI, against the float64 oracle started from the same state.

Outputs are compared element by element; a state is compared by what fixes
it whatever its scaling: the past mean a / b and ln den = p + ln b.  With a
state the outputs are convex combinations of v and the state's mean, so the
spec tolerance scale max|v| becomes max(max|v|, max|a / b|).
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


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to("cuda")


def scale(v, s_in):
    sc = float(np.abs(v).max())
    if s_in is not None:
        sc = max(sc, float(np.abs(s_in[:, 0] / s_in[:, 1]).max()))
    return sc


def assert_close(got, want, tol, what):
    err = np.abs(np.asarray(got, np.float64) - want)
    i = int(np.argmax(err))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.flat[i] <= tol, (f"{what}: max err {err.flat[i]:.3e} > {tol:.3e} at flat {i} "
                                f"(got {np.asarray(got).flat[i]!r}, want {want.flat[i]!r})")


def assert_state_close(got, want, tol_mean, what):
    gm, gl = oracle.state_mean_logden(got)
    wm, wl = oracle.state_mean_logden(want)
    assert np.all(got[:, 1] > 0), f"{what}: state out has b <= 0"
    assert_close(gm, wm, tol_mean, f"{what} state mean")
    # ln den: fp32 holds p to about 6e-8 |p|, the sums to a few ulp
    assert_close(gl, wl, 2e-5 + 1e-6 * float(np.abs(wl).max()), f"{what} state ln den")


def run_state(m, x, s_in, bf16=False):
    s = None if s_in is None else dev(s_in)
    if bf16:
        y, s_out = m.wkv_forward_bf16_state(dev(x.w), dev(x.u), bf16_dev(x.k_bits),
                                            bf16_dev(x.v_bits), s)
        y = y.float()
    else:
        y, s_out = m.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), s)
    torch.cuda.synchronize()
    return y.double().cpu().numpy(), s_out.double().cpu().numpy()


# serial kernel (T <= 16), tiled kernels with one and several tiles, ragged
# tails in T and C, odd C (element-wise tile path)
STATE_SHAPES = [(1, 1, 1), (4, 1, 96), (3, 5, 40), (2, 16, 64), (2, 17, 64), (1, 128, 32),
                (2, 300, 96), (3, 1000, 40), (1, 2049, 33), (2, 777, 160)]


@pytest.mark.parametrize("B,T,C", STATE_SHAPES)
def test_wkv_state_f32_vs_oracle(m, B, T, C):
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=7 * B + T + C)
    s_in = workloads.make_wkv_state(B, C, seed=T)
    y, s_out = run_state(m, x, s_in)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(y, want_y, tol, f"state f32 {B}x{T}x{C} y")
    assert_state_close(s_out, want_s, tol, f"state f32 {B}x{T}x{C}")


@pytest.mark.parametrize("B,T,C", [(2, 1, 64), (3, 9, 40), (2, 3, 33), (2, 600, 128),
                                   (1, 1500, 72)])
def test_wkv_state_bf16_vs_oracle(m, B, T, C):
    x = workloads.make_wkv("wkv_3b_bf16", B=B, T=T, C=C, seed=B + T + C)
    s_in = workloads.make_wkv_state(B, C, seed=T + 1)
    y, s_out = run_state(m, x, s_in, bf16=True)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    sc = scale(x.v, s_in)
    assert_close(y, want_y, 2e-2 * sc, f"state bf16 {B}x{T}x{C} y")
    # the state never passes through bf16: fp32 bounds
    assert_state_close(s_out, want_s, 1e-5 * sc, f"state bf16 {B}x{T}x{C}")


@pytest.mark.parametrize("T", [1, 4, 16])
def test_serial_path_with_unaligned_pointers(m, T):
    """Buffers one element off 16-byte alignment take the one-channel-per-
    thread form of the short-sequence kernel; same results."""
    B, C = 3, 64
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=90 + T)
    s_in = workloads.make_wkv_state(B, C, seed=90 + T)
    n, ns = x.k.size, s_in.size
    kb = torch.empty(n + 1, device="cuda"); kb[1:] = dev(x.k).reshape(-1)
    yb = torch.empty(n + 1, device="cuda")
    sb = torch.empty(ns + 1, device="cuda"); sb[1:] = dev(s_in).reshape(-1)
    k, y, s = kb[1:].view(x.k.shape), yb[1:].view(x.k.shape), sb[1:].view(s_in.shape)
    assert k.data_ptr() % 16 != 0 and s.data_ptr() % 16 != 0
    m.wkv_forward_state(dev(x.w), dev(x.u), k, dev(x.v), s, y=y, s_out=s)
    torch.cuda.synchronize()
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(y.double().cpu().numpy(), want_y, tol, f"unaligned serial T={T} y")
    assert_state_close(s.double().cpu().numpy(), want_s, tol, f"unaligned serial T={T}")


def test_no_state_is_wkv_forward(m):
    """No state and the explicit empty state take wkv_forward's arithmetic:
    bit for bit while at most two tiles follow one another in time (with
    more, the look-back may fold a different but equivalent set of records
    from run to run, which moves the last bits), within rounding beyond."""
    for T in (7, 250, 1000):
        x = workloads.make_wkv("wkv_169m", B=2, T=T, C=64, seed=T)
        y0 = m.wkv_forward(dev(x.w), dev(x.u), dev(x.k), dev(x.v))
        y1, _ = m.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), None)
        s0 = torch.zeros(2, 3, 64, device="cuda")
        s0[:, 2] = -float("inf")
        y2, _ = m.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), s0)
        torch.cuda.synchronize()
        if T <= 256:
            assert torch.equal(y0, y1) and torch.equal(y0, y2), f"T={T}"
        else:
            tol = 2e-6 * float(np.abs(x.v).max())
            assert float((y0 - y1).abs().max()) <= tol and float((y0 - y2).abs().max()) <= tol


def test_state_out_vs_definition_without_state_in(m):
    """The state after T steps from the empty past is the definition's past
    sums at t = T (no current token)."""
    x = workloads.make_wkv("wkv_169m", B=2, T=700, C=48, seed=3)
    _, s_out = run_state(m, x, None)
    _, want = oracle.wkv_direct_state(x.w, x.u, x.k, x.v)
    assert_state_close(s_out, want, 1e-5 * scale(x.v, None), "state out from empty")


@pytest.mark.parametrize("steps", [8, 32, 64, 128, 256])
def test_state_tile_length_does_not_change_results(m, steps):
    x = workloads.make_wkv("wkv_169m", B=2, T=1000, C=64, seed=12)
    s_in = workloads.make_wkv_state(2, 64, seed=12)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        y, s_out = run_state(m, x, s_in)
    finally:
        m.wkv_set_tile_steps(old)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(y, want_y, tol, f"tile steps {steps} y")
    assert_state_close(s_out, want_s, tol, f"tile steps {steps}")


def test_streaming_in_pieces_equals_one_call(m):
    """A sequence fed in pieces (state handed on, in place) gives the outputs
    and final state of one call over all steps, against the oracle."""
    B, T, C = 2, 2000, 96
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=31)
    s_in = workloads.make_wkv_state(B, C, seed=31)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    s = dev(s_in)
    ys = []
    for a, b in ((0, 1), (1, 13), (13, 140), (140, 1111), (1111, 1112), (1112, 2000)):
        y, _ = m.wkv_forward_state(w, u, k[:, a:b].contiguous(), v[:, a:b].contiguous(), s, s_out=s)
        ys.append(y)
    torch.cuda.synchronize()
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(torch.cat(ys, 1).double().cpu().numpy(), want_y, tol, "pieces y")
    assert_state_close(s.double().cpu().numpy(), want_s, tol, "pieces")


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_rnn_mode_decoding_one_token_per_call(m, bf16):
    """64 single-token steps with the state updated in place equal the
    recurrence over the 64 tokens."""
    B, T, C = 8, 64, 200
    spec = "wkv_3b_bf16" if bf16 else "wkv_169m"
    x = workloads.make_wkv(spec, B=B, T=T, C=C, seed=41)
    s_in = workloads.make_wkv_state(B, C, seed=41)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    w, u = dev(x.w), dev(x.u)
    if bf16:
        k, v = bf16_dev(x.k_bits), bf16_dev(x.v_bits)
        fn = m.wkv_forward_bf16_state
    else:
        k, v = dev(x.k), dev(x.v)
        fn = m.wkv_forward_state
    s = dev(s_in)
    ys = []
    for t in range(T):
        y, _ = fn(w, u, k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous(), s, s_out=s)
        ys.append(y)
    torch.cuda.synchronize()
    got = torch.cat(ys, 1).float().double().cpu().numpy()
    sc = scale(x.v, s_in)
    assert_close(got, want_y, (2e-2 if bf16 else 1e-5) * sc, "decode y")
    assert_state_close(s.double().cpu().numpy(), want_s, 1e-5 * sc, "decode")


def test_in_place_state_on_the_tiled_path(m):
    x = workloads.make_wkv("wkv_169m", B=3, T=900, C=64, seed=51)
    s_in = workloads.make_wkv_state(3, 64, seed=51)
    s = dev(s_in)
    y, s_ret = m.wkv_forward_state(dev(x.w), dev(x.u), dev(x.k), dev(x.v), s, s_out=s)
    torch.cuda.synchronize()
    assert s_ret.data_ptr() == s.data_ptr()
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(y.double().cpu().numpy(), want_y, tol, "in place y")
    assert_state_close(s.double().cpu().numpy(), want_s, tol, "in place")


def test_large_state_scales_and_decay_only(m):
    """A state far larger than the tokens (p = 80) dominates: outputs stay at
    its mean until its weight e^{80 - t w} falls to the tokens' level."""
    B, T, C = 1, 400, 64
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=61)
    s_in = workloads.make_wkv_state(B, C, seed=61)
    s_in[:, 2] = 80.0
    y, s_out = run_state(m, x, s_in)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(y, want_y, tol, "large state y")
    assert_state_close(s_out, want_s, tol, "large state")


def test_full_size_wkv_long_from_a_state(m):
    """wkv_long (B=1 T=131072 C=1024) from a drawn state, in the benchmark's
    launch configuration: sampled outputs against the definition and the
    final state against the recurrence."""
    x = workloads.make_wkv("wkv_long")
    s_in = workloads.make_wkv_state(1, 1024, seed=71)
    y, s_out = run_state(m, x, s_in)
    rng = np.random.default_rng(72)
    pts = rng.integers(0, x.k.size, 1500)
    pts = np.concatenate([pts, [0, 1023, x.k.size - 1]])
    want = oracle.wkv_direct_points(x.w, x.u, x.k, x.v, pts, s_in=s_in)
    tol = 1e-4 * scale(x.v, s_in)
    assert_close(y.reshape(-1)[pts], want, tol, "wkv_long state points")
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, s_in)
    assert_state_close(s_out, want_s, tol, "wkv_long final")
    assert_close(y, want_y, tol, "wkv_long state every output")


def test_decode_workload_vs_oracle(m):
    x = workloads.make_wkv("wkv_decode")
    y, s_out = run_state(m, x, x.s_in)
    want_y, want_s = oracle.wkv_rnn_state(x.w, x.u, x.k, x.v, x.s_in)
    tol = 1e-5 * scale(x.v, x.s_in)
    assert_close(y, want_y, tol, "wkv_decode y")
    assert_state_close(s_out, want_s, tol, "wkv_decode")


def test_state_argument_errors(m):
    x = workloads.make_wkv("wkv_169m", B=2, T=40, C=64, seed=81)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    y = torch.empty_like(k)
    with pytest.raises(ValueError):
        m.wkv_forward_state(w, u, k, v, torch.zeros(2, 3, 63, device="cuda"))
    big = torch.zeros(2 * 3 * 64 + 64, device="cuda")
    s_in = big[:2 * 3 * 64].view(2, 3, 64)
    s_out = big[64:].view(2, 3, 64)            # overlaps s_in without being it
    with pytest.raises(m.WkvError) as e:
        m.wkv_forward_state(w, u, k, v, s_in, y=y, s_out=s_out)
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    # s_out inside k
    with pytest.raises(m.WkvError) as e:
        m.wkv_forward_state(w, u, k, v, None, y=y, s_out=k.view(-1)[:384].view(2, 3, 64))
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    # a host pointer as the state (raw C call, past the binding's checks)
    host = torch.zeros(2, 3, 64)
    st = m.lib.wkv_forward_state(2, 40, 64, w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), y.data_ptr(), host.data_ptr(), None, None)
    assert st == m.WKV_ERR_INVALID_ARG
