"""wkv_forward_noalloc: the fp32 WKV forward for callers that cannot allocate
device memory (an engine that has reserved the GPU's memory for its own pool,
a plugin interface that hands an operator only its inputs and outputs, a
latency-critical path that must not pay for cudaMalloc or the synchronisation
it can cause).  Its scratch is a fixed device array shared by every call.

Checked through the C ABI on two calls in a row (the second call must clean
up after the first), each against the float64 oracle (the RNN-mode
recurrence of eq. (14) of "RWKV：基于RNN的LLM") at the fp32 tolerance
1e-5 * max|v|, and against the allocating entry point, wkv_forward, at the
same tolerance.  Named to be collected last, and written to pass both alone
in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_dev):
    import rwkv_wkv_mixing_b200 as m
    fn = m.lib.wkv_forward_noalloc
    p, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [i64, i64, i64, p, p, p, p, p, p]
    fn.restype = ctypes.c_int
    return m


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


@pytest.mark.parametrize("B,T,C", [(2, 1000, 96),    # chained tiles, TMA path
                                   (3, 700, 33),     # chained tiles, element-wise path
                                   (1, 100, 64)])    # one tile in time, no scratch
def test_noalloc_matches_oracle_and_allocating_entry_point_twice(lib, B, T, C):
    x = workloads.make_wkv("wkv_169m", B=B, T=T, C=C, seed=B * 7 + T + C)
    w, u, k, v = _dev(x.w), _dev(x.u), _dev(x.k), _dev(x.v)
    want = oracle.wkv_rnn(x.w, x.u, x.k, x.v)   # float64, computed on the CPU
    ref = lib.wkv_forward(w, u, k, v)
    torch.cuda.synchronize()
    tol = 1e-5 * float(np.abs(x.v).max())
    stream = torch.cuda.current_stream()
    for call in range(2):
        y = torch.full_like(k, float("nan"))
        st = lib.lib.wkv_forward_noalloc(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                         v.data_ptr(), y.data_ptr(),
                                         ctypes.c_void_p(stream.cuda_stream))
        assert st == lib.WKV_OK, lib.wkv_last_error()
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        err = float(np.abs(got - want).max())
        assert err <= tol, f"call {call}: max err vs the oracle {err} > {tol}"
        err = float((y.double() - ref.double()).abs().max())
        assert err <= tol, f"call {call}: max err vs wkv_forward {err} > {tol}"


def test_noalloc_rejects_a_problem_beyond_its_scratch(lib):
    # 1 x 4096 x 40960: 1280 channel groups x 32 tiles in time = 40960 tiles > 32767
    B, T, C = 1, 4096, 40960
    k = torch.zeros(B, T, C, device="cuda")
    w = torch.zeros(C, device="cuda")
    y = torch.empty_like(k)
    st = lib.lib.wkv_forward_noalloc(B, T, C, w.data_ptr(), w.data_ptr(), k.data_ptr(),
                                     k.data_ptr(), y.data_ptr(), None)
    assert st == lib.WKV_ERR_INVALID_ARG
    assert "scratch" in lib.wkv_last_error()
