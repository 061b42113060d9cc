"""CPU oracle for the RWKV-4 WKV operator and the diagonal linear scan.

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` are the only callers.  The CUDA
library never imports or links anything here, and nothing here imports the
CUDA library: the two share no code.  Only the seeded input generators in
``workloads`` feed both.

Pieces (all float64; each cites the page it follows):

* ``wkv_direct``          -- eq. (14) of "RWKV：基于RNN的LLM" (section 二.1,
  Time-mixing block) evaluated literally, O(T^2) per channel (C code).
* ``wkv_direct_points``   -- the same definition at chosen (b, t, c) points,
  O(t) each, for full-size workloads (C code).
* ``wkv_direct_np``       -- eq. (14) again, as a masked log-sum-exp over a
  [T, T] logit matrix in numpy; small inputs only.
* ``wkv_rnn``             -- the RNN-mode state update (RWKV evolution
  article, section RWKV-V4), max-stabilised; the full-tensor oracle and the
  timed CPU baseline (C code, OpenMP over channels).
* ``wkv_direct_state`` / ``wkv_rnn_state`` -- the same two forms starting
  from a given state (the past sums before step 0, RNN mode) and returning
  the state after the last step; ``wkv_direct_points(..., s_in=)`` likewise.
  A state is [B, 3, C]: planes a, b, p with (num, den) = (a, b) e^p.
* ``token_shift``         -- the token-shift interpolation that feeds the
  time-mixing projections, mu x_t + (1 - mu) x_{t-1} (eqs. (11)-(13) of
  "RWKV：基于RNN的LLM", section 二.1; x_{-1} is the layer's saved last token,
  "last_x", of the HarmonyOS RWKV article's time-mixing code section, or 0).
* ``lru_scan``            -- the LRU's complex diagonal recurrence
  x_t = lambda x_{t-1} + gamma u_t with lambda = e^{-e^{nu_log} + i e^{theta_log}}
  (review of "Resurrecting Recurrent Neural Networks for Long Sequences",
  linear-RNN section), complex128; ``lru_direct_points`` is its unrolled sum
  x_t = gamma sum_k lambda^{t-k} u_k (+ lambda^{t+1} x_{-1}).
* ``sigmoid`` / ``wkv_gated`` -- the receptance gate sigma(r_t) (.) wkv_t of
  eq. (15) of the same page and of the LRU review's RWKV variant.
* ``wkv_backward_direct`` / ``wkv_backward_rnn`` -- gradients of eq. (14)
  with respect to k, v, w and u (the pages give none): the derivative of a
  softmax-weighted mean written out per output (O(T^2)), and the same by a
  forward and a reverse recurrence (O(T)).
* ``wkv_slru_ratio_np``   -- the "RWKV = ratio of two SLRUs" form from the
  review of "Resurrecting Recurrent Neural Networks for Long Sequences"
  (section on the RWKV variant), unstabilised; |k| small only.
* ``scan_rnn``            -- h_t = a_t h_{t-1} + b_t ("Were RNNs All We
  Needed?" article, scan form) (C code).
* ``scan_direct_points``  -- the unrolled sum of the same scan at chosen points
  (LRU review, linear-RNN section) (C code).

Parity status: every function above is pinned by the ``-m "not gpu"`` tests
(closed forms, invariants, brute force, cross-formulation agreement); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

__all__ = [
    "build", "max_threads", "wkv_direct", "wkv_direct_points", "wkv_direct_np",
    "wkv_rnn", "wkv_slru_ratio_np", "scan_rnn", "scan_direct_points",
    "wkv_direct_state", "wkv_rnn_state", "state_mean_logden",
    "token_shift", "sigmoid", "wkv_gated", "lru_lambda", "lru_scan", "lru_direct_points",
    "wkv_backward_direct", "wkv_backward_rnn",
]


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            i64, p = ctypes.c_int64, ctypes.c_void_p
            lib.oracle_max_threads.restype = ctypes.c_int
            for name, args in {
                "oracle_wkv_direct": [i64, i64, i64, p, p, p, p, p, ctypes.c_int],
                "oracle_wkv_direct_points": [i64, i64, i64, p, p, p, p, i64, p, p, ctypes.c_int],
                "oracle_wkv_rnn": [i64, i64, i64, p, p, p, p, p, ctypes.c_int],
                "oracle_wkv_direct_s": [i64, i64, i64, p, p, p, p, p, p, p, ctypes.c_int],
                "oracle_wkv_direct_points_s": [i64, i64, i64, p, p, p, p, p, i64, p, p,
                                               ctypes.c_int],
                "oracle_wkv_rnn_s": [i64, i64, i64, p, p, p, p, p, p, p, ctypes.c_int],
                "oracle_wkv_backward_direct": [i64, i64, i64, p, p, p, p, p, p, p, p, p,
                                               ctypes.c_int],
                "oracle_wkv_backward_rnn": [i64, i64, i64, p, p, p, p, p, p, p, p, p,
                                            ctypes.c_int],
                "oracle_scan_rnn": [i64, i64, i64, p, p, p, p, ctypes.c_int],
                "oracle_scan_direct_points": [i64, i64, i64, p, p, p, i64, p, p, ctypes.c_int],
            }.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = None
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_get().oracle_max_threads())


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return x.ctypes.data_as(ctypes.c_void_p)


def _wkv_args(w, u, k, v):
    k, v = _f64(k), _f64(v)
    if k.ndim != 3 or k.shape != v.shape:
        raise ValueError("k and v must be [B, T, C] of one shape")
    B, T, C = k.shape
    w, u = _f64(w).reshape(-1), _f64(u).reshape(-1)
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    return B, T, C, w, u, k, v


def wkv_direct(w, u, k, v, nthreads: int = 0) -> np.ndarray:
    """Eq. (14) at every output, O(T^2) per channel."""
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    y = np.empty((B, T, C), dtype=np.float64)
    _get().oracle_wkv_direct(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y), nthreads)
    return y


def _state_arg(s, B, C):
    if s is None:
        return None
    s = _f64(s)
    if s.shape != (B, 3, C):
        raise ValueError("a state must be [B, 3, C]")
    return s


def _optr(x):
    return None if x is None else _ptr(x)


def wkv_direct_points(w, u, k, v, points, nthreads: int = 0, s_in=None) -> np.ndarray:
    """Eq. (14) at the flat output indices ``points`` (b*T*C + t*C + c),
    from the state ``s_in`` ([B, 3, C]) or the empty past."""
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    s_in = _state_arg(s_in, B, C)
    pts = np.ascontiguousarray(points, dtype=np.int64).reshape(-1)
    if pts.size and (pts.min() < 0 or pts.max() >= B * T * C):
        raise IndexError("point out of range")
    out = np.empty(pts.size, dtype=np.float64)
    _get().oracle_wkv_direct_points_s(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v),
                                      _optr(s_in), pts.size, _ptr(pts), _ptr(out), nthreads)
    return out


def wkv_direct_state(w, u, k, v, s_in=None, nthreads: int = 0):
    """Eq. (14) at every output from the state ``s_in`` (None: empty past);
    returns (y, s_out), s_out the past sums after the last step with p the
    largest logit.  O(T^2) per channel."""
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    s_in = _state_arg(s_in, B, C)
    y = np.empty((B, T, C), dtype=np.float64)
    s_out = np.empty((B, 3, C), dtype=np.float64)
    _get().oracle_wkv_direct_s(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _optr(s_in),
                               _ptr(y), _ptr(s_out), nthreads)
    return y, s_out


def wkv_rnn_state(w, u, k, v, s_in=None, nthreads: int = 0):
    """RNN-mode recurrence from the state ``s_in`` (None: empty past);
    returns (y, s_out)."""
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    s_in = _state_arg(s_in, B, C)
    y = np.empty((B, T, C), dtype=np.float64)
    s_out = np.empty((B, 3, C), dtype=np.float64)
    _get().oracle_wkv_rnn_s(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _optr(s_in),
                            _ptr(y), _ptr(s_out), nthreads)
    return y, s_out


def state_mean_logden(s):
    """What a state (a, b, p) fixes whatever its scaling: the mean a / b of
    the past values and ln den = p + ln b.  Two states are the same state
    exactly when both agree."""
    s = np.asarray(s, dtype=np.float64)
    a, b, p = s[:, 0], s[:, 1], s[:, 2]
    with np.errstate(divide="ignore", invalid="ignore"):
        return a / b, p + np.log(b)


def wkv_rnn(w, u, k, v, nthreads: int = 0) -> np.ndarray:
    """RNN-mode recurrence, max-stabilised, float64; all outputs."""
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    y = np.empty((B, T, C), dtype=np.float64)
    _get().oracle_wkv_rnn(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y), nthreads)
    return y


def wkv_direct_np(w, u, k, v) -> np.ndarray:
    """Eq. (14) as a masked softmax over a [T, T] logit matrix (numpy).

    logit[t, i] = -(t-1-i) w + k_i for i < t, u + k_t on the diagonal, and no
    weight for i > t; the output is the logit-softmax-weighted mean of v_i.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64).reshape(-1)
    u = np.asarray(u, dtype=np.float64).reshape(-1)
    B, T, C = k.shape
    t_idx = np.arange(T)[:, None]
    i_idx = np.arange(T)[None, :]
    dist = (t_idx - 1 - i_idx).astype(np.float64)            # t-1-i
    logit = -dist[None, :, :, None] * w[None, None, None, :] + k[:, None, :, :]   # [B,T,T,C]
    diag = u[None, None, :] + k                              # [B,T,C]
    eye = (t_idx == i_idx)
    logit = np.where(eye[None, :, :, None], diag[:, :, None, :], logit)
    logit = np.where((i_idx > t_idx)[None, :, :, None], -np.inf, logit)
    m = logit.max(axis=2, keepdims=True)
    e = np.exp(logit - m)
    return (e * v[:, None, :, :]).sum(axis=2) / e.sum(axis=2)


def wkv_slru_ratio_np(w, u, k, v) -> np.ndarray:
    """Ratio of two real diagonal linear RNNs (LRU review, RWKV variant):

        Y_t = lam Y_{t-1} + e^{k_t} v_t,    Z_t = lam Z_{t-1} + e^{k_t},
        y_t = (Y_t + (gam lam - 1) e^{k_t} v_t) / (Z_t + (gam lam - 1) e^{k_t}),

    with lam = e^{-w} and gam = e^{u}; the sigma(r) gate of that page is not
    part of WKV.  No stabilisation, so only for inputs with small |k|.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lam = np.exp(-np.asarray(w, dtype=np.float64).reshape(-1))
    gam = np.exp(np.asarray(u, dtype=np.float64).reshape(-1))
    B, T, C = k.shape
    Y = np.zeros((B, C))
    Z = np.zeros((B, C))
    out = np.empty((B, T, C))
    for t in range(T):
        ek = np.exp(k[:, t, :])
        Y = lam * Y + ek * v[:, t, :]
        Z = lam * Z + ek
        out[:, t, :] = (Y + (gam * lam - 1.0) * ek * v[:, t, :]) / (Z + (gam * lam - 1.0) * ek)
    return out


def _scan_args(a, b, h0):
    a, b = _f64(a), _f64(b)
    if a.ndim != 3 or a.shape != b.shape:
        raise ValueError("a and b must be [B, T, D] of one shape")
    B, T, D = a.shape
    if h0 is not None:
        h0 = _f64(h0)
        if h0.shape != (B, D):
            raise ValueError("h0 must be [B, D]")
    return B, T, D, a, b, h0


def scan_rnn(a, b, h0=None, nthreads: int = 0) -> np.ndarray:
    """h_t = a_t h_{t-1} + b_t with h_{-1} = h0 (zeros if None), float64."""
    B, T, D, a, b, h0 = _scan_args(a, b, h0)
    h = np.empty((B, T, D), dtype=np.float64)
    _get().oracle_scan_rnn(B, T, D, _ptr(a), _ptr(b), None if h0 is None else _ptr(h0),
                           _ptr(h), nthreads)
    return h


def scan_direct_points(a, b, h0, points, nthreads: int = 0) -> np.ndarray:
    """Unrolled scan sum at the flat output indices ``points``."""
    B, T, D, a, b, h0 = _scan_args(a, b, h0)
    pts = np.ascontiguousarray(points, dtype=np.int64).reshape(-1)
    if pts.size and (pts.min() < 0 or pts.max() >= B * T * D):
        raise IndexError("point out of range")
    out = np.empty(pts.size, dtype=np.float64)
    _get().oracle_scan_direct_points(B, T, D, _ptr(a), _ptr(b),
                                     None if h0 is None else _ptr(h0),
                                     pts.size, _ptr(pts), _ptr(out), nthreads)
    return out


# ---------------------------------------------------------------------------
# The elementwise steps around WKV in the time-mixing block
# ---------------------------------------------------------------------------
def token_shift(x, mu, x_prev=None):
    """Token shift ("RWKV：基于RNN的LLM", section 二.1, eqs. (11)-(13)): for
    each mixing vector mu_m (rows of ``mu``, [n_mix, C]),

        out[m, b, t] = mu_m * x[b, t] + (1 - mu_m) * x[b, t-1],

    with x[b, -1] = x_prev[b] (the token before this call, [B, C]) or 0.
    Returns (out [n_mix, B, T, C], x_last [B, C] = x[:, T-1]), float64.
    The pages print eqs. (16)-(17) with a minus before (1 - mu); the plus of
    eqs. (11)-(13) is the reading taken everywhere."""
    x = np.asarray(x, dtype=np.float64)
    mu = np.asarray(mu, dtype=np.float64)
    if mu.ndim == 1:
        mu = mu[None]
    B, T, C = x.shape
    if mu.shape[1] != C:
        raise ValueError("mu must be [n_mix, C]")
    prev = np.zeros((B, 1, C)) if x_prev is None else \
        np.asarray(x_prev, dtype=np.float64).reshape(B, 1, C)
    shifted = np.concatenate([prev, x[:, :-1]], axis=1)        # x_{t-1}
    out = np.stack([m * x + (1.0 - m) * shifted for m in mu])  # [n_mix, B, T, C]
    return out, x[:, -1].copy()


def sigmoid(r):
    """The logistic function 1 / (1 + e^{-r}), float64."""
    r = np.asarray(r, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-r))


def wkv_gated(w, u, k, v, r, s_in=None):
    """sigma(r_t) (.) wkv_t (eq. (15) of "RWKV：基于RNN的LLM" before the output
    projection; the LRU review's RWKV variant), wkv from the RNN-mode oracle,
    optionally from a state.  Returns (out, s_out)."""
    y, s_out = wkv_rnn_state(w, u, k, v, s_in)
    return sigmoid(r) * y, s_out


# ---------------------------------------------------------------------------
# LRU: complex diagonal linear recurrence
# ---------------------------------------------------------------------------
def lru_lambda(nu_log, theta_log):
    """lambda = r e^{i theta} with r = e^{-nu}, nu = e^{nu_log}, theta = e^{theta_log}
    (the LRU review's parameterisation, linear-RNN section)."""
    nu = np.exp(np.asarray(nu_log, dtype=np.float64))
    theta = np.exp(np.asarray(theta_log, dtype=np.float64))
    return np.exp(-nu) * np.exp(1j * theta)


def lru_scan(nu_log, theta_log, gamma, u, x0=None):
    """x_t = lambda x_{t-1} + gamma u_t per channel, x_{-1} = x0 (0 if None).
    u: complex [B, T, D] (or real); gamma: [D] real or None (1).  Returns
    complex128 [B, T, D]."""
    lam = lru_lambda(nu_log, theta_log)
    u = np.asarray(u)
    B, T, D = u.shape
    g = np.ones(D) if gamma is None else np.asarray(gamma, dtype=np.float64)
    x = np.zeros((B, D), dtype=np.complex128) if x0 is None else \
        np.asarray(x0, dtype=np.complex128).reshape(B, D).copy()
    out = np.empty((B, T, D), dtype=np.complex128)
    for t in range(T):
        x = lam * x + g * u[:, t].astype(np.complex128)
        out[:, t] = x
    return out


def lru_direct_points(nu_log, theta_log, gamma, u, x0, points):
    """The unrolled sum x_t = gamma sum_{k<=t} lambda^{t-k} u_k + lambda^{t+1} x_{-1}
    at flat indices b*T*D + t*D + d (powers from exp of the scaled exponent)."""
    nu = np.exp(np.asarray(nu_log, dtype=np.float64))
    theta = np.exp(np.asarray(theta_log, dtype=np.float64))
    u = np.asarray(u).astype(np.complex128)
    B, T, D = u.shape
    g = np.ones(D) if gamma is None else np.asarray(gamma, dtype=np.float64)
    out = np.empty(len(points), dtype=np.complex128)
    for j, f in enumerate(np.asarray(points, dtype=np.int64)):
        b, t, d = f // (T * D), (f // D) % T, f % D
        n = t - np.arange(t + 1)                     # t - k for k = 0..t
        pw = np.exp(n * (-nu[d] + 1j * theta[d]))    # lambda^{t-k}
        acc = g[d] * np.sum(pw * u[b, :t + 1, d])
        if x0 is not None:
            acc += np.exp((t + 1) * (-nu[d] + 1j * theta[d])) * complex(np.asarray(x0)[b, d])
        out[j] = acc
    return out


# ---------------------------------------------------------------------------
# WKV gradients
# ---------------------------------------------------------------------------
def _wkv_backward(name, w, u, k, v, gy, nthreads):
    B, T, C, w, u, k, v = _wkv_args(w, u, k, v)
    gy = _f64(gy)
    if gy.shape != k.shape:
        raise ValueError("gy must have the shape of k")
    gk = np.empty_like(k)
    gv = np.empty_like(k)
    gw = np.empty(C)
    gu = np.empty(C)
    getattr(_get(), name)(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy), _ptr(gk),
                          _ptr(gv), _ptr(gw), _ptr(gu), nthreads)
    return gk, gv, gw, gu


def wkv_backward_direct(w, u, k, v, gy, nthreads: int = 0):
    """(gk, gv, gw, gu) for upstream gradient gy, by the definition (O(T^2))."""
    return _wkv_backward("oracle_wkv_backward_direct", w, u, k, v, gy, nthreads)


def wkv_backward_rnn(w, u, k, v, gy, nthreads: int = 0):
    """(gk, gv, gw, gu) by a forward and a reverse recurrence (O(T))."""
    return _wkv_backward("oracle_wkv_backward_rnn", w, u, k, v, gy, nthreads)
