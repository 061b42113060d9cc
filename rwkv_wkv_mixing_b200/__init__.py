"""Python binding of libwkv_b200.so (RWKV-4 WKV forward and the diagonal
linear scan on B200 / sm_100a).

Argument marshalling only: every entry point takes torch CUDA tensors, checks
dtype / shape / contiguity, and calls the C function of the same name with
raw device pointers and the current torch CUDA stream.  All arithmetic runs
in the library's kernels; there is no CPU fallback, and importing this module
raises if the library has not been built.

    y = wkv_forward(w, u, k, v)            # fp32 [B,T,C] k, v; [C] w, u
    y = wkv_forward_bf16(w, u, k, v)       # bf16 k, v -> bf16 y, fp32 state
    y, s = wkv_forward_state(w, u, k, v, s_in)   # + state [B,3,C] in and out
    y = wkv_forward_gated(w, u, k, v, r)   # sigma(r) * wkv, one pass
    out = token_shift(x, mu, x_prev)       # [n_mix,B,T,C] mu x_t + (1-mu) x_{t-1}
    h = diag_scan(a, b, h0=None)           # fp32 [B,T,D]; h0 [B,D] or None
    y = wkv_forward_host(w, u, k, v)       # the same on CPU tensors, copies overlapped
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwkv_b200.so")

WKV_OK = 0
WKV_ERR_INVALID_ARG = 1
WKV_ERR_ALIGNMENT = 2
WKV_ERR_CUDA = 3
WKV_ERR_TIMEOUT = 4
WKV_ERR_OOM = 5
STATUS_NAMES = {0: "WKV_OK", 1: "WKV_ERR_INVALID_ARG", 2: "WKV_ERR_ALIGNMENT",
                3: "WKV_ERR_CUDA", 4: "WKV_ERR_TIMEOUT", 5: "WKV_ERR_OOM"}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python rwkv_wkv_mixing_b200/build.py` (nvcc, sm_100a)")

_i64, _p, _i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
lib = ctypes.CDLL(LIB_PATH)
_SIGS = {
    "wkv_forward": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_bf16": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_noalloc": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_state": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_bf16_state": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_gated": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_bf16_gated": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_token_shift": ([_i64, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_token_shift_bf16": ([_i64, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p], _i32),
    "diag_scan": ([_i64, _i64, _i64, _p, _p, _p, _p, _p], _i32),
    "diag_scan_bf16": ([_i64, _i64, _i64, _p, _p, _p, _p, _p], _i32),
    "lru_scan": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_backward": ([_i64, _i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_host": ([_i64, _i64, _i64, _p, _p, _p, _p, _p], _i32),
    "wkv_forward_bf16_host": ([_i64, _i64, _i64, _p, _p, _p, _p, _p], _i32),
    "diag_scan_host": ([_i64, _i64, _i64, _p, _p, _p, _p], _i32),
    "wkv_device_status": ([_p], _i32),
    "wkv_last_error": ([], ctypes.c_char_p),
    "wkv_release_workspaces": ([], _i32),
    "wkv_set_tile_steps": ([_i32], _i32),
    "wkv_get_tile_steps": ([], _i32),
    "wkv_tile_steps_for": ([_i64, _i64, _i64, _i32], _i32),
    "wkv_set_fault_injection": ([_i32, _i64], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class WkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.wkv_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


def _check(status: int, where: str):
    if status != WKV_OK:
        raise WkvError(status, where)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, ndim):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _wkv(fn_name, io_dtype, w, u, k, v, y, stream):
    import torch
    _need(k, "k", io_dtype, 3)
    _need(v, "v", io_dtype, 3)
    _need(w, "w", torch.float32, 1)
    _need(u, "u", torch.float32, 1)
    if k.shape != v.shape:
        raise ValueError("k and v must have one shape")
    B, T, C = k.shape
    if w.shape[0] != C or u.shape[0] != C:
        raise ValueError("w and u must be [C]")
    if y is None:
        y = torch.empty_like(k)
    else:
        _need(y, "y", io_dtype, 3)
        if y.shape != k.shape:
            raise ValueError("y must have the shape of k")
    _check(getattr(lib, fn_name)(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), y.data_ptr(), _stream_handle(stream)), fn_name)
    return y


def wkv_forward(w, u, k, v, y=None, stream=None):
    """WKV forward, fp32: y[b,t,c] per eq. (14) of the RWKV page."""
    import torch
    return _wkv("wkv_forward", torch.float32, w, u, k, v, y, stream)


def wkv_forward_bf16(w, u, k, v, y=None, stream=None):
    """WKV forward, bf16 k/v/y with fp32 state and fp32 w, u."""
    import torch
    return _wkv("wkv_forward_bf16", torch.bfloat16, w, u, k, v, y, stream)


def _wkv_state(fn_name, io_dtype, w, u, k, v, s_in, y, s_out, stream):
    import torch
    _need(k, "k", io_dtype, 3)
    B, _, C = k.shape
    for t, name in ((s_in, "s_in"), (s_out, "s_out")):
        if t is not None:
            _need(t, name, torch.float32, 3)
            if tuple(t.shape) != (B, 3, C):
                raise ValueError(f"{name} must be [B, 3, C] = {(B, 3, C)}")
    if s_out is None:
        s_out = torch.empty((B, 3, C), dtype=torch.float32, device=k.device)
    _need(v, "v", io_dtype, 3)
    _need(w, "w", torch.float32, 1)
    _need(u, "u", torch.float32, 1)
    if k.shape != v.shape:
        raise ValueError("k and v must have one shape")
    if w.shape[0] != C or u.shape[0] != C:
        raise ValueError("w and u must be [C]")
    if y is None:
        y = torch.empty_like(k)
    else:
        _need(y, "y", io_dtype, 3)
        if y.shape != k.shape:
            raise ValueError("y must have the shape of k")
    _check(getattr(lib, fn_name)(B, k.shape[1], C, w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), y.data_ptr(),
                                 None if s_in is None else s_in.data_ptr(), s_out.data_ptr(),
                                 _stream_handle(stream)), fn_name)
    return y, s_out


def wkv_forward_state(w, u, k, v, s_in=None, y=None, s_out=None, stream=None):
    """WKV forward, fp32, from the state ``s_in`` ([B, 3, C] planes a, b, p:
    past sums (num, den) = (a, b) e^p; None = empty past).  Returns
    (y, s_out), s_out the state after the last step (``s_out=s_in`` updates
    it in place; T = 1 is one RNN-mode decoding step)."""
    import torch
    return _wkv_state("wkv_forward_state", torch.float32, w, u, k, v, s_in, y, s_out, stream)


def wkv_forward_bf16_state(w, u, k, v, s_in=None, y=None, s_out=None, stream=None):
    """wkv_forward_state with bf16 k/v/y; the state stays fp32."""
    import torch
    return _wkv_state("wkv_forward_bf16_state", torch.bfloat16, w, u, k, v, s_in, y, s_out,
                      stream)


def wkv_forward_gated(w, u, k, v, r, y=None, s_in=None, s_out=None, stream=None):
    """sigma(r) (.) wkv in one pass (eq. (15) before the output projection);
    k, v, r, y fp32 or all bf16 (then the bf16 entry point runs).  Optional
    state [B, 3, C] fp32 in (``s_in``) and out (``s_out``, may be s_in)."""
    import torch
    io = k.dtype
    if io not in (torch.float32, torch.bfloat16):
        raise TypeError("k must be float32 or bfloat16")
    _need(k, "k", io, 3)
    _need(v, "v", io, 3)
    _need(r, "r", io, 3)
    _need(w, "w", torch.float32, 1)
    _need(u, "u", torch.float32, 1)
    if k.shape != v.shape or k.shape != r.shape:
        raise ValueError("k, v and r must have one shape")
    B, T, C = k.shape
    if w.shape[0] != C or u.shape[0] != C:
        raise ValueError("w and u must be [C]")
    for t, name in ((s_in, "s_in"), (s_out, "s_out")):
        if t is not None:
            _need(t, name, torch.float32, 3)
            if tuple(t.shape) != (B, 3, C):
                raise ValueError(f"{name} must be [B, 3, C] = {(B, 3, C)}")
    if y is None:
        y = torch.empty_like(k)
    else:
        _need(y, "y", io, 3)
        if y.shape != k.shape:
            raise ValueError("y must have the shape of k")
    fn = "wkv_forward_gated" if io == torch.float32 else "wkv_forward_bf16_gated"
    _check(getattr(lib, fn)(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(),
                            r.data_ptr(), y.data_ptr(),
                            None if s_in is None else s_in.data_ptr(),
                            None if s_out is None else s_out.data_ptr(),
                            _stream_handle(stream)), fn)
    return y


def token_shift(x, mu, x_prev=None, out=None, x_last=None, stream=None):
    """mu[m] x_t + (1 - mu[m]) x_{t-1} for every row m of ``mu`` ([n_mix, C]
    fp32) from one read of x ([B, T, C] fp32 or bf16); x_{-1} = x_prev [B, C]
    (zeros if None).  Returns out [n_mix, B, T, C]; ``x_last`` [B, C], if
    given, receives x[:, T-1] (it may be x_prev)."""
    import torch
    io = x.dtype
    if io not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, "x", io, 3)
    B, T, C = x.shape
    _need(mu, "mu", torch.float32, 2)
    if mu.shape[1] != C or not 1 <= mu.shape[0] <= 4:
        raise ValueError("mu must be [n_mix, C] with 1 <= n_mix <= 4")
    n_mix = mu.shape[0]
    for t, name in ((x_prev, "x_prev"), (x_last, "x_last")):
        if t is not None:
            _need(t, name, io, 2)
            if tuple(t.shape) != (B, C):
                raise ValueError(f"{name} must be [B, C] = {(B, C)}")
    if out is None:
        out = torch.empty((n_mix, B, T, C), dtype=io, device=x.device)
    else:
        _need(out, "out", io, 4)
        if tuple(out.shape) != (n_mix, B, T, C):
            raise ValueError("out must be [n_mix, B, T, C]")
    fn = "wkv_token_shift" if io == torch.float32 else "wkv_token_shift_bf16"
    _check(getattr(lib, fn)(B, T, C, n_mix, x.data_ptr(),
                            None if x_prev is None else x_prev.data_ptr(), mu.data_ptr(),
                            out.data_ptr(), None if x_last is None else x_last.data_ptr(),
                            _stream_handle(stream)), fn)
    return out


def wkv_forward_noalloc(w, u, k, v, y=None, stream=None):
    """WKV forward, fp32, with the library allocating no device memory: its
    scratch is a fixed 16 MiB device array shared by every call on a device
    (serialise calls; problems needing more scratch raise WkvError).  For
    callers that cannot allocate; `y` should then be passed in."""
    import torch
    return _wkv("wkv_forward_noalloc", torch.float32, w, u, k, v, y, stream)


def diag_scan(a, b, h0=None, h=None, stream=None):
    """h_t = a_t * h_{t-1} + b_t per channel, h_{-1} = h0 (zeros if None).
    a, b, h fp32, or all bf16 (fp32 state, bf16 storage); h0 fp32."""
    import torch
    io = a.dtype
    if io not in (torch.float32, torch.bfloat16):
        raise TypeError("a must be float32 or bfloat16")
    _need(a, "a", io, 3)
    _need(b, "b", io, 3)
    if a.shape != b.shape:
        raise ValueError("a and b must have one shape")
    B, T, D = a.shape
    if h0 is not None:
        _need(h0, "h0", torch.float32, 2)
        if tuple(h0.shape) != (B, D):
            raise ValueError("h0 must be [B, D]")
    if h is None:
        h = torch.empty_like(a)
    else:
        _need(h, "h", io, 3)
        if h.shape != a.shape:
            raise ValueError("h must have the shape of a")
    fn = "diag_scan" if io == torch.float32 else "diag_scan_bf16"
    _check(getattr(lib, fn)(B, T, D, a.data_ptr(), b.data_ptr(),
                            None if h0 is None else h0.data_ptr(), h.data_ptr(),
                            _stream_handle(stream)), fn)
    return h


def wkv_backward(w, u, k, v, gy, stream=None):
    """Gradients of wkv_forward (fp32, no state) for upstream gradient gy:
    returns (gk, gv, gw, gu), gw and gu summed over batch rows and steps."""
    import torch
    for t, name in ((k, "k"), (v, "v"), (gy, "gy")):
        _need(t, name, torch.float32, 3)
    _need(w, "w", torch.float32, 1)
    _need(u, "u", torch.float32, 1)
    if k.shape != v.shape or k.shape != gy.shape:
        raise ValueError("k, v and gy must have one shape")
    B, T, C = k.shape
    if w.shape[0] != C or u.shape[0] != C:
        raise ValueError("w and u must be [C]")
    gk, gv = torch.empty_like(k), torch.empty_like(k)
    gw, gu = torch.empty_like(w), torch.empty_like(u)
    _check(lib.wkv_backward(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(),
                            gy.data_ptr(), gk.data_ptr(), gv.data_ptr(), gw.data_ptr(),
                            gu.data_ptr(), _stream_handle(stream)), "wkv_backward")
    return gk, gv, gw, gu


def lru_scan(nu_log, theta_log, u, gamma=None, x0=None, x=None, stream=None):
    """The LRU recurrence x_t = lambda x_{t-1} + gamma u_t per complex channel,
    lambda = e^{-e^{nu_log} + i e^{theta_log}}.  u: complex64 [B, T, D] (or
    float32 [B, T, D, 2]); nu_log, theta_log, gamma: float32 [D]; x0: complex64
    [B, D] or None (zeros).  Returns x like u."""
    import torch
    as_complex = u.dtype == torch.complex64
    ur = torch.view_as_real(u) if as_complex else u
    _need(ur, "u", torch.float32, 4)
    if ur.shape[-1] != 2:
        raise ValueError("u must be complex64 [B, T, D] or float32 [B, T, D, 2]")
    B, T, D, _ = ur.shape
    for t, name in ((nu_log, "nu_log"), (theta_log, "theta_log"), (gamma, "gamma")):
        if t is not None:
            _need(t, name, torch.float32, 1)
            if t.shape[0] != D:
                raise ValueError(f"{name} must be [D]")
    x0r = None
    if x0 is not None:
        x0r = torch.view_as_real(x0) if x0.dtype == torch.complex64 else x0
        _need(x0r, "x0", torch.float32, 3)
        if tuple(x0r.shape) != (B, D, 2):
            raise ValueError("x0 must be [B, D] complex")
    if x is None:
        x = torch.empty_like(u)
    xr = torch.view_as_real(x) if x.dtype == torch.complex64 else x
    _need(xr, "x", torch.float32, 4)
    if xr.shape != ur.shape:
        raise ValueError("x must have the shape of u")
    _check(lib.lru_scan(B, T, D, nu_log.data_ptr(), theta_log.data_ptr(),
                        None if gamma is None else gamma.data_ptr(), ur.data_ptr(),
                        None if x0r is None else x0r.data_ptr(), xr.data_ptr(),
                        _stream_handle(stream)), "lru_scan")
    return x


def _need_host(t, name, dtype, ndim):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a CPU tensor (pinned for overlapped copies)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _wkv_host(fn_name, io_dtype, w, u, k, v, y):
    import torch
    _need_host(k, "k", io_dtype, 3)
    _need_host(v, "v", io_dtype, 3)
    _need_host(w, "w", torch.float32, 1)
    _need_host(u, "u", torch.float32, 1)
    if k.shape != v.shape:
        raise ValueError("k and v must have one shape")
    B, T, C = k.shape
    if w.shape[0] != C or u.shape[0] != C:
        raise ValueError("w and u must be [C]")
    if y is None:
        y = torch.empty_like(k, pin_memory=k.is_pinned())
    else:
        _need_host(y, "y", io_dtype, 3)
        if y.shape != k.shape:
            raise ValueError("y must have the shape of k")
    _check(getattr(lib, fn_name)(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                 v.data_ptr(), y.data_ptr()), fn_name)
    return y


def wkv_forward_host(w, u, k, v, y=None):
    """WKV forward, fp32, on host (CPU) tensors: uploads, computes and
    downloads in an overlapped pipeline; returns when y holds the result."""
    import torch
    return _wkv_host("wkv_forward_host", torch.float32, w, u, k, v, y)


def wkv_forward_bf16_host(w, u, k, v, y=None):
    """WKV forward, bf16 k/v/y on host tensors (fp32 w, u)."""
    import torch
    return _wkv_host("wkv_forward_bf16_host", torch.bfloat16, w, u, k, v, y)


def diag_scan_host(a, b, h0=None, h=None):
    """Diagonal scan on host (CPU) tensors, pipelined; returns h."""
    import torch
    _need_host(a, "a", torch.float32, 3)
    _need_host(b, "b", torch.float32, 3)
    if a.shape != b.shape:
        raise ValueError("a and b must have one shape")
    B, T, D = a.shape
    if h0 is not None:
        _need_host(h0, "h0", torch.float32, 2)
        if tuple(h0.shape) != (B, D):
            raise ValueError("h0 must be [B, D]")
    if h is None:
        h = torch.empty_like(a, pin_memory=a.is_pinned())
    else:
        _need_host(h, "h", torch.float32, 3)
        if h.shape != a.shape:
            raise ValueError("h must have the shape of a")
    _check(lib.diag_scan_host(B, T, D, a.data_ptr(), b.data_ptr(),
                              None if h0 is None else h0.data_ptr(), h.data_ptr()),
           "diag_scan_host")
    return h


def wkv_device_status(stream=None):
    """Synchronise the stream; raise WkvError if a device-side wait gave up."""
    _check(lib.wkv_device_status(_stream_handle(stream)), "wkv_device_status")


def wkv_last_error() -> str:
    return lib.wkv_last_error().decode(errors="replace")


def wkv_release_workspaces():
    _check(lib.wkv_release_workspaces(), "wkv_release_workspaces")


def wkv_set_tile_steps(steps: int):
    _check(lib.wkv_set_tile_steps(int(steps)), "wkv_set_tile_steps")


def wkv_get_tile_steps() -> int:
    """The knob's value; 0 means each call chooses (see wkv_tile_steps_for)."""
    return int(lib.wkv_get_tile_steps())


def wkv_tile_steps_for(B: int, T: int, C: int, elem_bytes: int = 4) -> int:
    """The tile length a call of this shape uses under the current knob."""
    return int(lib.wkv_tile_steps_for(B, T, C, elem_bytes))


def wkv_set_fault_injection(skip_tile: int = -1, spin_limit: int = 0):
    """Test hook: make tile `skip_tile` never publish (its successors' bounded
    waits run out after `spin_limit` polls); (-1, 0) turns it off."""
    _check(lib.wkv_set_fault_injection(int(skip_tile), int(spin_limit)),
           "wkv_set_fault_injection")


__all__ = ["wkv_forward", "wkv_forward_bf16", "wkv_forward_noalloc", "diag_scan",
           "wkv_forward_state", "wkv_forward_bf16_state", "wkv_forward_gated", "token_shift",
           "lru_scan", "wkv_backward",
           "wkv_forward_host", "wkv_forward_bf16_host", "diag_scan_host", "wkv_device_status",
           "wkv_last_error", "wkv_release_workspaces", "wkv_set_tile_steps",
           "wkv_get_tile_steps", "wkv_tile_steps_for", "WkvError", "lib", "LIB_PATH"]
