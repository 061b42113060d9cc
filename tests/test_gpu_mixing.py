"""The elementwise steps around WKV in the time-mixing block, on the GPU
through the C ABI, against the float64 oracle: the receptance gate fused into
the WKV output (sigma(r) (.) wkv, eq. (15) of the RWKV page) and the token
shift mu x_t + (1 - mu) x_{t-1} (eqs. (11)-(13)).

Tolerances: gated WKV as WKV (fp32 1e-5 max|v|, bf16 2e-2 max|v|; with a
state the scale also covers the state's mean); token shift fp32 1e-6 max|x|
(a convex combination, a few roundings), bf16 one bf16 rounding of the
output on top (2^-8 max|x|); mu = 0 and mu = 1 bit-exact.
"""
import dataclasses

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


def assert_close(got, want, tol, what):
    got = np.asarray(got, np.float64)
    err = np.abs(got - want)
    i = int(np.argmax(err))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.flat[i] <= tol, (f"{what}: max err {err.flat[i]:.3e} > {tol:.3e} at flat {i} "
                                f"(got {got.flat[i]!r}, want {want.flat[i]!r})")


def gated(name, **kw):
    spec = dataclasses.replace(workloads.WORKLOADS[name], gated=True)
    return workloads.make_wkv(spec, **kw)


def run_gated(m, x, s_in=None, bf16=False):
    s = None if s_in is None else dev(s_in)
    s_out = None if s_in is None else torch.empty_like(s)
    if bf16:
        y = m.wkv_forward_gated(dev(x.w), dev(x.u), bf16_dev(x.k_bits), bf16_dev(x.v_bits),
                                bf16_dev(x.r_bits), s_in=s, s_out=s_out).float()
    else:
        y = m.wkv_forward_gated(dev(x.w), dev(x.u), dev(x.k), dev(x.v), dev(x.r), s_in=s,
                                s_out=s_out)
    torch.cuda.synchronize()
    return y.double().cpu().numpy(), None if s_out is None else s_out.double().cpu().numpy()


def scale(v, s_in=None):
    sc = float(np.abs(v).max())
    if s_in is not None:
        sc = max(sc, float(np.abs(s_in[:, 0] / s_in[:, 1]).max()))
    return sc


# ---------------------------------------------------------------------------
# gated WKV
# ---------------------------------------------------------------------------
GATED_SHAPES = [(1, 1, 32), (2, 7, 40), (2, 16, 64), (3, 17, 64), (2, 128, 96), (2, 300, 64),
                (1, 1000, 160), (2, 777, 33), (1, 2049, 96)]


@pytest.mark.parametrize("B,T,C", GATED_SHAPES)
def test_gated_f32_vs_oracle(m, B, T, C):
    x = gated("wkv_169m", B=B, T=T, C=C, seed=B * 100 + T + C)
    got, _ = run_gated(m, x)
    want, _ = oracle.wkv_gated(x.w, x.u, x.k, x.v, x.r)
    assert_close(got, want, 1e-5 * scale(x.v), f"gated f32 {B}x{T}x{C}")


@pytest.mark.parametrize("B,T,C", [(2, 5, 64), (2, 600, 128), (1, 1500, 72), (3, 300, 40)])
def test_gated_bf16_vs_oracle(m, B, T, C):
    x = gated("wkv_3b_bf16", B=B, T=T, C=C, seed=B + T + C)
    got, _ = run_gated(m, x, bf16=True)
    want, _ = oracle.wkv_gated(x.w, x.u, x.k, x.v, x.r)
    assert_close(got, want, 2e-2 * scale(x.v), f"gated bf16 {B}x{T}x{C}")


@pytest.mark.parametrize("B,T,C", [(2, 1, 64), (2, 9, 40), (2, 700, 96)])
def test_gated_with_state_vs_oracle(m, B, T, C):
    x = gated("wkv_169m", B=B, T=T, C=C, seed=3 * T + C)
    s_in = workloads.make_wkv_state(B, C, seed=T + 5)
    got, s_out = run_gated(m, x, s_in)
    want, want_s = oracle.wkv_gated(x.w, x.u, x.k, x.v, x.r, s_in)
    tol = 1e-5 * scale(x.v, s_in)
    assert_close(got, want, tol, f"gated state {B}x{T}x{C}")
    gm, gl = oracle.state_mean_logden(s_out)
    wm, wl = oracle.state_mean_logden(want_s)
    assert_close(gm, wm, tol, "gated state mean")
    assert_close(gl, wl, 2e-5 + 1e-6 * float(np.abs(wl).max()), "gated state ln den")


@pytest.mark.parametrize("steps", [8, 32, 64, 128, 256])
def test_gated_tile_lengths(m, steps):
    x = gated("wkv_169m", B=2, T=1000, C=64, seed=77)
    want, _ = oracle.wkv_gated(x.w, x.u, x.k, x.v, x.r)
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        got, _ = run_gated(m, x)
    finally:
        m.wkv_set_tile_steps(old)
    assert_close(got, want, 1e-5 * scale(x.v), f"gated tile steps {steps}")


@pytest.mark.parametrize("T", [10, 200])
def test_gate_saturates(m, T):
    """r = +100 passes wkv through bit for bit (sigma rounds to 1); r = -100
    closes the gate to 0."""
    x = gated("wkv_169m", B=2, T=T, C=64, seed=T)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    y = m.wkv_forward(w, u, k, v)
    y_open = m.wkv_forward_gated(w, u, k, v, torch.full_like(k, 100.0))
    y_shut = m.wkv_forward_gated(w, u, k, v, torch.full_like(k, -100.0))
    torch.cuda.synchronize()
    assert torch.equal(y_open, y)
    assert float(y_shut.abs().max()) == 0.0


def test_gated_full_size_3b_bf16(m):
    """The benchmarked gated workload (B=8 T=4096 C=2560, bf16): sampled
    outputs against sigma(r) times the definition."""
    x = workloads.make_wkv("wkv_3b_gated_bf16")
    got, _ = run_gated(m, x, bf16=True)
    rng = np.random.default_rng(5)
    pts = np.concatenate([rng.integers(0, x.k.size, 1500), [0, x.k.size - 1]])
    want = oracle.sigmoid(x.r.reshape(-1)[pts]) * oracle.wkv_direct_points(x.w, x.u, x.k, x.v, pts)
    assert_close(got.reshape(-1)[pts], want, 2e-2 * scale(x.v), "gated 3b bf16 points")
    # every output against sigma(r) times the float64 recurrence, one batch row at a time
    for b in range(x.k.shape[0]):
        row = lambda a: np.ascontiguousarray(a[b:b + 1])   # noqa: E731
        want_row, _ = oracle.wkv_gated(x.w, x.u, row(x.k), row(x.v), row(x.r))
        assert_close(got[b:b + 1], want_row, 2e-2 * scale(x.v), f"gated 3b bf16 row {b}")


def test_gated_argument_errors(m):
    x = gated("wkv_169m", B=1, T=40, C=64, seed=1)
    w, u, k, v = dev(x.w), dev(x.u), dev(x.k), dev(x.v)
    with pytest.raises(m.WkvError) as e:   # y is r
        m.wkv_forward_gated(w, u, k, v, k.clone(), y=v)
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    r = dev(x.r)
    with pytest.raises(m.WkvError) as e:   # output written over r
        m.wkv_forward_gated(w, u, k, v, r, y=r)
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        m.wkv_forward_gated(w, u, k, v, r[:, :20].contiguous())


# ---------------------------------------------------------------------------
# token shift
# ---------------------------------------------------------------------------
def run_shift(m, s, with_prev=True, n_mix=None, bf16=False, want_last=True):
    if bf16:
        x = bf16_dev(s.x_bits)
        xp = bf16_dev(s.x_prev_bits) if with_prev else None
    else:
        x = dev(s.x)
        xp = dev(s.x_prev) if with_prev else None
    mu = dev(s.mu)
    last = torch.empty((s.x.shape[0], s.x.shape[2]), dtype=x.dtype, device="cuda") \
        if want_last else None
    out = m.token_shift(x, mu, xp, x_last=last)
    torch.cuda.synchronize()
    return (out.float().double().cpu().numpy(),
            None if last is None else last.float().double().cpu().numpy())


SHIFT_SHAPES = [(1, 1, 4, 3), (2, 1, 64, 1), (2, 15, 40, 2), (2, 16, 64, 3), (3, 17, 64, 4),
                (2, 300, 96, 3), (1, 1000, 33, 2), (2, 257, 7, 3)]


@pytest.mark.parametrize("B,T,C,n_mix", SHIFT_SHAPES)
@pytest.mark.parametrize("with_prev", [True, False], ids=["prev", "noprev"])
def test_token_shift_f32_vs_oracle(m, B, T, C, n_mix, with_prev):
    spec = dataclasses.replace(workloads.WORKLOADS["shift_3b_bf16"], dtype="f32")
    s = workloads.make_token_shift(spec, B=B, T=T, C=C, n_mix=n_mix, seed=B + T + C + n_mix)
    got, last = run_shift(m, s, with_prev)
    want, want_last = oracle.token_shift(s.x, s.mu, s.x_prev if with_prev else None)
    assert_close(got, want, 1e-6 * float(np.abs(s.x).max()), f"shift {B}x{T}x{C} m{n_mix}")
    assert np.array_equal(last, want_last)


@pytest.mark.parametrize("B,T,C,n_mix", [(2, 16, 64, 3), (2, 300, 96, 3), (1, 77, 6, 2)])
def test_token_shift_bf16_vs_oracle(m, B, T, C, n_mix):
    s = workloads.make_token_shift("shift_3b_bf16", B=B, T=T, C=C, n_mix=n_mix, seed=T)
    got, last = run_shift(m, s, bf16=True)
    want, want_last = oracle.token_shift(s.x, s.mu, s.x_prev)
    assert_close(got, want, 2.0 ** -8 * float(np.abs(s.x).max()), f"shift bf16 {B}x{T}x{C}")
    assert np.array_equal(last, want_last)


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_token_shift_exact_cases(m, bf16):
    """mu = 1 gives x and mu = 0 gives the shifted x, bit for bit."""
    s = workloads.make_token_shift("shift_3b_bf16", B=2, T=40, C=64, n_mix=2, seed=9)
    s.mu[0] = 1.0
    s.mu[1] = 0.0
    got, _ = run_shift(m, s, bf16=bf16)
    shifted = np.concatenate([s.x_prev[:, None], s.x[:, :-1]], axis=1)
    assert np.array_equal(got[0], s.x)
    assert np.array_equal(got[1], shifted)


def test_token_shift_chaining_in_place(m):
    """Two calls handing the last token on through one buffer (x_last is
    x_prev) equal one call, bit for bit."""
    s = workloads.make_token_shift("shift_3b_bf16", B=3, T=100, C=96, n_mix=3, seed=4)
    x, mu = dev(s.x), dev(s.mu)
    full = m.token_shift(x, mu, dev(s.x_prev))
    carry = dev(s.x_prev)
    a = m.token_shift(x[:, :37].contiguous(), mu, carry, x_last=carry)
    b = m.token_shift(x[:, 37:].contiguous(), mu, carry, x_last=carry)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a, b], dim=2), full)
    assert torch.equal(carry, x[:, -1])


def test_token_shift_full_size_3b_bf16(m):
    s = workloads.make_token_shift("shift_3b_bf16")
    got, last = run_shift(m, s, bf16=True)
    want, want_last = oracle.token_shift(s.x, s.mu, s.x_prev)
    assert_close(got, want, 2.0 ** -8 * float(np.abs(s.x).max()), "shift 3b bf16")
    assert np.array_equal(last, want_last)


def test_token_shift_argument_errors(m):
    s = workloads.make_token_shift("shift_3b_bf16", B=2, T=10, C=64, n_mix=3, seed=2)
    x, mu = dev(s.x), dev(s.mu)
    with pytest.raises(ValueError):
        m.token_shift(x, torch.zeros(5, 64, device="cuda"))
    out = torch.empty(3, 2, 10, 64, device="cuda")
    with pytest.raises(m.WkvError) as e:   # x_last inside x
        m.token_shift(x, mu, out=out, x_last=x.view(-1)[:2 * 64].view(2, 64))
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    st = m.lib.wkv_token_shift(2, 10, 64, 0, x.data_ptr(), None, mu.data_ptr(), out.data_ptr(),
                               None, None)
    assert st == m.WKV_ERR_INVALID_ARG
