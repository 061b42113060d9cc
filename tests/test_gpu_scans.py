"""Scan variants on the GPU through the C ABI against the float64 oracle:
the diagonal scan with bf16 storage, the minLSTM-form workload, and the
LRU's complex diagonal recurrence.

Tolerances: fp32 scans max|err| <= 1e-5 max|h| (as the fp32 diagonal scan);
bf16 storage adds one bf16 rounding of each output on top: 2^-8 max|h|.
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


def assert_close(got, want, tol, what):
    got = np.asarray(got)
    err = np.abs(got - want)
    i = int(np.argmax(err))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.flat[i] <= tol, (f"{what}: max err {err.flat[i]:.3e} > {tol:.3e} at flat {i} "
                                f"(got {got.flat[i]!r}, want {want.flat[i]!r})")


# ---------------------------------------------------------------------------
# bf16 storage
# ---------------------------------------------------------------------------
SCAN_SHAPES = [(1, 1, 8), (2, 7, 64), (2, 128, 64), (3, 300, 72), (1, 1000, 136), (2, 513, 6),
               (1, 2049, 256)]


@pytest.mark.parametrize("B,T,D", SCAN_SHAPES)
@pytest.mark.parametrize("with_h0", [False, True], ids=["h0none", "h0"])
def test_scan_bf16_vs_oracle(m, B, T, D, with_h0):
    x = workloads.make_scan("scan_mingru_bf16", B=B, T=T, D=D, seed=B + T + D, with_h0=with_h0)
    h = m.diag_scan(bf16_dev(x.a_bits), bf16_dev(x.b_bits), None if x.h0 is None else dev(x.h0))
    torch.cuda.synchronize()
    want = oracle.scan_rnn(x.a, x.b, x.h0)
    got = h.float().double().cpu().numpy()
    assert_close(got, want, 2.0 ** -8 * float(np.abs(want).max()), f"scan bf16 {B}x{T}x{D}")


@pytest.mark.parametrize("steps", [8, 32, 64, 128, 256])
def test_scan_bf16_tile_lengths(m, steps):
    x = workloads.make_scan("scan_mingru_bf16", B=2, T=1000, D=128, seed=5, with_h0=True)
    want = oracle.scan_rnn(x.a, x.b, x.h0)
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        h = m.diag_scan(bf16_dev(x.a_bits), bf16_dev(x.b_bits), dev(x.h0))
        torch.cuda.synchronize()
    finally:
        m.wkv_set_tile_steps(old)
    assert_close(h.float().double().cpu().numpy(), want, 2.0 ** -8 * float(np.abs(want).max()),
                 f"scan bf16 tile steps {steps}")


def test_scan_bf16_full_size(m):
    """The bf16 minGRU workload at full size (B=64 T=4096 D=256): sampled
    outputs against the unrolled sum, and the convex bound everywhere."""
    x = workloads.make_scan("scan_mingru_bf16")
    h = m.diag_scan(bf16_dev(x.a_bits), bf16_dev(x.b_bits))
    torch.cuda.synchronize()
    got = h.float().double().cpu().numpy()
    rng = np.random.default_rng(3)
    pts = np.concatenate([rng.integers(0, x.a.size, 1500), [0, x.a.size - 1]])
    want = oracle.scan_direct_points(x.a, x.b, None, pts)
    scale = float(np.abs(x.h_tilde).max())
    assert_close(got.reshape(-1)[pts], want, 2.0 ** -8 * scale, "scan bf16 full-size points")
    # every output against the float64 recurrence over the bf16-rounded inputs
    want_full = oracle.scan_rnn(x.a, x.b, None)
    assert_close(got, want_full, 2.0 ** -8 * scale, "scan bf16 full-size every output")


# ---------------------------------------------------------------------------
# minLSTM form
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,T,D", [(2, 300, 64), (1, 2000, 256)])
def test_minlstm_scan_vs_oracle(m, B, T, D):
    x = workloads.make_scan("scan_minlstm", B=B, T=T, D=D, seed=T)
    h = m.diag_scan(dev(x.a), dev(x.b))
    torch.cuda.synchronize()
    want = oracle.scan_rnn(x.a, x.b, None)
    assert_close(h.double().cpu().numpy(), want, 1e-5 * float(np.abs(want).max()),
                 f"minlstm {B}x{T}x{D}")


def test_minlstm_full_size(m):
    """scan_minlstm (B=64 T=4096 D=256): sampled points against the unrolled
    sum; every output inside the running range of the candidates and 0."""
    x = workloads.make_scan("scan_minlstm")
    h = m.diag_scan(dev(x.a), dev(x.b))
    torch.cuda.synchronize()
    got = h.double().cpu().numpy()
    rng = np.random.default_rng(4)
    pts = np.concatenate([rng.integers(0, x.a.size, 1500), [0, x.a.size - 1]])
    want = oracle.scan_direct_points(x.a, x.b, None, pts)
    assert_close(got.reshape(-1)[pts], want, 1e-5 * float(np.abs(x.h_tilde).max()),
                 "minlstm full-size points")
    want_full = oracle.scan_rnn(x.a, x.b, None)
    assert_close(got, want_full, 1e-5 * float(np.abs(want_full).max()),
                 "minlstm full-size every output")
    lo = np.minimum(np.minimum.accumulate(x.h_tilde, axis=1), 0.0)
    hi = np.maximum(np.maximum.accumulate(x.h_tilde, axis=1), 0.0)
    tol = 1e-5 * float(np.abs(x.h_tilde).max())
    assert np.all(got >= lo - tol) and np.all(got <= hi + tol)


# ---------------------------------------------------------------------------
# LRU complex recurrence
# ---------------------------------------------------------------------------
def run_lru(m, x):
    u = torch.view_as_complex(dev(x.u))
    x0 = None if x.x0 is None else torch.view_as_complex(dev(x.x0))
    gamma = dev(x.gamma)
    out = m.lru_scan(dev(x.nu_log), dev(x.theta_log), u, gamma=gamma, x0=x0)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.complex128)


LRU_SHAPES = [(1, 1, 2), (2, 7, 32), (2, 128, 64), (3, 300, 40), (1, 1000, 130), (2, 513, 5),
              (1, 3000, 64)]


@pytest.mark.parametrize("B,T,D", LRU_SHAPES)
@pytest.mark.parametrize("with_x0", [False, True], ids=["x0none", "x0"])
def test_lru_vs_oracle(m, B, T, D, with_x0):
    x = workloads.make_lru("lru_256", B=B, T=T, D=D, seed=B + T + D, with_x0=with_x0)
    got = run_lru(m, x)
    want = oracle.lru_scan(x.nu_log, x.theta_log, x.gamma, x.u_complex(), x.x0_complex())
    assert_close(got, want, 1e-5 * float(np.abs(want).max()), f"lru {B}x{T}x{D}")


@pytest.mark.parametrize("steps", [8, 32, 64, 128, 256])
def test_lru_tile_lengths(m, steps):
    x = workloads.make_lru("lru_256", B=2, T=1000, D=64, seed=9, with_x0=True)
    want = oracle.lru_scan(x.nu_log, x.theta_log, x.gamma, x.u_complex(), x.x0_complex())
    old = m.wkv_get_tile_steps()
    try:
        m.wkv_set_tile_steps(steps)
        got = run_lru(m, x)
    finally:
        m.wkv_set_tile_steps(old)
    assert_close(got, want, 1e-5 * float(np.abs(want).max()), f"lru tile steps {steps}")


def test_lru_long_phase_accuracy(m):
    """A long sequence (T = 40000) with r close to 1 and large theta: the
    carry across thousands of steps turns the phase through ~10^5 radians,
    which single precision could not reduce; sampled outputs against the
    unrolled sum."""
    x = workloads.make_lru("lru_256", B=1, T=40000, D=16, seed=11, with_x0=True)
    x.nu_log[:] = np.log(1e-4)          # r = e^{-1e-4}: memory of ~10^4 steps
    x.theta_log[:] = np.log(np.linspace(0.5, 6.0, 16)).astype(np.float32)
    got = run_lru(m, x)
    rng = np.random.default_rng(12)
    pts = np.concatenate([rng.integers(0, got.size, 300), [got.size - 1]])
    want = oracle.lru_direct_points(x.nu_log, x.theta_log, x.gamma, x.u_complex(),
                                    x.x0_complex(), pts)
    scale = float(np.abs(want).max())
    assert_close(got.reshape(-1)[pts], want, 1e-4 * scale, "lru long phase")


def test_lru_full_size(m):
    x = workloads.make_lru("lru_256")
    got = run_lru(m, x)
    rng = np.random.default_rng(13)
    pts = np.concatenate([rng.integers(0, got.size, 400), [0, got.size - 1]])
    want = oracle.lru_direct_points(x.nu_log, x.theta_log, x.gamma, x.u_complex(), None, pts)
    assert_close(got.reshape(-1)[pts], want, 1e-5 * float(np.abs(want).max()) + 1e-6,
                 "lru full-size points")
    # every output against the complex128 recurrence, eight batch rows at a
    # time; the tolerance scales with the largest |x| of the whole output
    uc = x.u_complex()
    errs, scale = [], 0.0
    for b0 in range(0, uc.shape[0], 8):
        want_full = oracle.lru_scan(x.nu_log, x.theta_log, x.gamma, uc[b0:b0 + 8])
        assert np.all(np.isfinite(got[b0:b0 + 8])), f"rows {b0}:{b0 + 8}: non-finite output"
        errs.append(float(np.abs(got[b0:b0 + 8] - want_full).max()))
        scale = max(scale, float(np.abs(want_full).max()))
    tol = 1e-5 * scale + 1e-6
    assert max(errs) <= tol, f"lru full-size every output: max err {max(errs):.3e} > {tol:.3e}"


def test_lru_argument_errors(m):
    x = workloads.make_lru("lru_256", B=1, T=10, D=8)
    u = torch.view_as_complex(dev(x.u))
    with pytest.raises(m.WkvError) as e:   # output written over the input
        m.lru_scan(dev(x.nu_log), dev(x.theta_log), u, x=u)
    assert e.value.status == m.WKV_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        m.lru_scan(dev(x.nu_log[:4]), dev(x.theta_log), u)
