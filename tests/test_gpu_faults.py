"""Failure detection on the GPU without faulting it.

A test hook makes one tile never publish its state, so the look-back waits of
the tiles after it in time run out.  Every wait in the kernels is bounded: the
waits give up after a short poll budget, the launch finishes, the affected
outputs are NaN (and only those), wkv_device_status reports WKV_ERR_TIMEOUT,
and the next call on the same context is correct again.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture
def m(cuda_dev):
    import rwkv_wkv_mixing_b200 as mod
    yield mod
    mod.wkv_set_fault_injection(-1, 0)
    mod.wkv_set_tile_steps(0)


@pytest.mark.parametrize("steps", [128, 32])   # persistent pipeline, block per tile
def test_a_tile_that_never_publishes_times_out_cleanly(m, steps):
    B, T, C = 1, 1024, 64            # two 32-channel groups -> two chains in time
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=101)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda")   # noqa: E731
    w, u, k, v = d(x.w), d(x.u), d(x.k), d(x.v)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    tol = 1e-5 * float(np.abs(x.v).max())
    m.wkv_set_tile_steps(steps)
    m.wkv_device_status()             # start from a clean status word

    # tiles are numbered segment-major, 2 per segment: tile 4 = segment 2 of
    # channel group 0; it computes its own outputs but never publishes
    m.wkv_set_fault_injection(4, 4096)
    y = m.wkv_forward(w, u, k, v)
    with pytest.raises(m.WkvError) as err:
        m.wkv_device_status()
    assert err.value.status == m.WKV_ERR_TIMEOUT
    got = y.double().cpu().numpy()
    cut = 3 * steps                   # first step of segment 3
    assert np.isnan(got[:, cut:, :32]).all(), "outputs behind the silent tile must be NaN"
    assert np.abs(got[:, :cut, :] - want[:, :cut, :]).max() <= tol
    assert np.abs(got[:, :, 32:] - want[:, :, 32:]).max() <= tol

    # the context is still usable: the same call without the fault is correct
    m.wkv_set_fault_injection(-1, 0)
    y = m.wkv_forward(w, u, k, v)
    m.wkv_device_status()
    assert np.abs(y.double().cpu().numpy() - want).max() <= tol


def test_gradients_time_out_cleanly_when_a_tile_never_publishes(m):
    """The gradient step's first pass carries the forward state between
    128-step tiles by the same look-back: a silent tile makes the waits
    behind it run out; its channels' gradients come out NaN (the reverse
    sums then carry the NaN back to the start of the chain), the other
    channels' are exact, the status word says so, and the next call is
    correct again."""
    B, T, C = 1, 1024, 64            # two 32-channel chains of eight tiles
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=103)
    gy = np.random.default_rng(103).normal(0, 1, x.k.shape).astype(np.float32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda")   # noqa: E731
    w, u, k, v, g = d(x.w), d(x.u), d(x.k), d(x.v), d(gy)
    want = oracle.wkv_backward_rnn(x.w, x.u, x.k, x.v, gy)
    m.wkv_device_status()
    m.wkv_set_fault_injection(4, 4096)   # segment 2 of channel group 0 stays silent
    got = [t.double().cpu().numpy() for t in m.wkv_backward(w, u, k, v, g)]
    with pytest.raises(m.WkvError) as err:
        m.wkv_device_status()
    assert err.value.status == m.WKV_ERR_TIMEOUT
    for name, gv_, wv, rel in zip(("gk", "gv", "gw", "gu"), got, want, (1e-4, 1e-4, 2e-4, 2e-4)):
        assert np.isnan(gv_[..., :32]).all(), f"{name}: the silent chain's gradients must be NaN"
        scale = float(np.abs(wv[..., 32:]).max())
        assert np.abs(gv_[..., 32:] - wv[..., 32:]).max() <= rel * scale, name
    m.wkv_set_fault_injection(-1, 0)
    got = [t.double().cpu().numpy() for t in m.wkv_backward(w, u, k, v, g)]
    m.wkv_device_status()
    for name, gv_, wv, rel in zip(("gk", "gv", "gw", "gu"), got, want, (1e-4, 1e-4, 2e-4, 2e-4)):
        assert np.abs(gv_ - wv).max() <= rel * float(np.abs(wv).max()), name


def test_fault_injection_arguments_are_checked(m):
    assert m.lib.wkv_set_fault_injection(-2, 0) == m.WKV_ERR_INVALID_ARG
    assert m.lib.wkv_set_fault_injection(0, -1) == m.WKV_ERR_INVALID_ARG
    assert m.lib.wkv_set_fault_injection(-1, 0) == m.WKV_OK


def test_host_entry_point_reports_a_timeout(m):
    """The host-buffer entry point reads each internal stream's status word
    back with the stream's work and returns WKV_ERR_TIMEOUT for the call
    whose wait gave up; the next call is correct again."""
    B, T, C = 1, 1024, 64            # one chunk: the tile numbering of a direct call
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=102)
    h = lambda a: torch.from_numpy(np.ascontiguousarray(a))   # noqa: E731
    w, u, k, v = h(x.w), h(x.u), h(x.k), h(x.v)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    m.wkv_set_tile_steps(128)
    m.wkv_set_fault_injection(4, 4096)
    with pytest.raises(m.WkvError) as err:
        m.wkv_forward_host(w, u, k, v)
    assert err.value.status == m.WKV_ERR_TIMEOUT
    m.wkv_set_fault_injection(-1, 0)
    y = m.wkv_forward_host(w, u, k, v)
    assert np.abs(y.double().numpy() - want).max() <= 1e-5 * float(np.abs(x.v).max())


def test_a_timeout_survives_the_workspace_growing(m):
    """A timeout recorded on a stream, then a larger call on the same stream
    that needs a larger look-back workspace (the old one is retired): the
    status word moves to the new workspace, so wkv_device_status still
    reports the timeout, once."""
    s = torch.cuda.Stream()
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda")   # noqa: E731
    small = workloads.make_wkv("wkv_169m", B=1, T=1024, C=64, seed=103)
    big = workloads.make_wkv("wkv_169m", B=8, T=4096, C=1024, seed=104)  # > 1 MiB of records
    m.wkv_set_tile_steps(128)
    with torch.cuda.stream(s):
        m.wkv_set_fault_injection(4, 4096)
        m.wkv_forward(d(small.w), d(small.u), d(small.k), d(small.v), stream=s)
        m.wkv_set_fault_injection(-1, 0)
        y = m.wkv_forward(d(big.w), d(big.u), d(big.k), d(big.v), stream=s)
    with pytest.raises(m.WkvError) as err:
        m.wkv_device_status(s)
    assert err.value.status == m.WKV_ERR_TIMEOUT
    m.wkv_device_status(s)            # read and cleared
    # the larger call itself was not affected
    sl = lambda a: np.ascontiguousarray(a[:, :, :64])   # noqa: E731
    want = oracle.wkv_rnn(big.w[:64], big.u[:64], sl(big.k), sl(big.v))
    got = y[:, :, :64].double().cpu().numpy()
    assert np.abs(got - want).max() <= 1e-5 * float(np.abs(big.v).max())
