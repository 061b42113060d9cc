"""Seeded synthetic inputs for the WKV operator and the diagonal linear scan.

This module is shared by the CPU oracle's tests, the CUDA parity tests and
``bench.py``.  It holds none of the operator's arithmetic: it only draws
random numbers, applies the input recipes below (which describe what the
inputs look like, not what the operator computes) and rounds them to the
storage type the GPU path consumes.

Recipe (every workload): ``numpy.random.default_rng(seed)``; values drawn in
float64, in the order listed per workload; then rounded to float32 (round to
nearest even); for bf16 workloads the float32 values of k and v are rounded
once more to bfloat16 (round to nearest even) and the oracle is fed the
rounded values widened back to float.  ``N(mu, sigma)`` takes the standard
deviation as its second argument, ``U(lo, hi)`` is uniform.

Named workloads (shapes from RWKV-4 models and the minGRU scan form):

* ``wkv_tiny``   WKV fp32, B=1 T=64 C=32; k, v ~ N(0,1); w = exp(N(-0.5,0.5));
  u ~ N(0,0.5)
* ``wkv_169m``   WKV fp32, B=8 T=1024 C=768 (RWKV-4-169M width); k, v ~ N(0,1);
  w = exp(U(-3,1)); u ~ N(0,0.5)
* ``wkv_3b_bf16`` WKV bf16 k/v/y with fp32 state, B=8 T=4096 C=2560 (RWKV-4-3B
  width); same distributions as ``wkv_169m``
* ``wkv_long``   WKV fp32, B=1 T=131072 C=1024; k ~ N(0,3), v ~ N(0,1);
  w = exp(U(-6,0)); u ~ N(0,1)
* ``scan_mingru`` diagonal scan fp32, B=64 T=4096 D=256 in minGRU form:
  z = sigmoid(N(0,1)), h~ ~ N(0,1), a = 1 - z, b = z * h~, h0 = 0
* ``scan_mingru_bf16`` the same minGRU-form scan with bf16 a, b, h storage
  (values rounded to bf16 after the float32 recipe)
* ``scan_minlstm`` diagonal scan fp32, B=64 T=4096 D=256 in minLSTM form:
  f = sigmoid(N(0,1)), i = sigmoid(N(0,1)), h~ ~ N(0,1) (drawn in that order),
  a = f / (f + i), b = i / (f + i) * h~, h0 = 0 (the normalised gates of the
  "Were RNNs All We Needed?" article's minLSTM section)
* ``lru_256`` the LRU's complex diagonal recurrence, B=64 T=4096 D=256 complex
  channels (see ``make_lru``)
* ``wkv_3b_gated_bf16`` the receptance-gated WKV sigma(r) (.) wkv with bf16
  k/v/r/y, B=8 T=4096 C=2560; k, v, w, u as ``wkv_3b_bf16``, then r ~ N(0, 2)
* ``shift_3b_bf16`` token shift (3 mixing vectors: k, v, r) on bf16 x,
  B=8 T=4096 C=2560; x ~ N(0, 1), mu ~ U(0, 1) (see ``make_token_shift``)
* ``wkv_169m_bwd`` the WKV gradients at the ``wkv_169m`` shape and
  distributions, then an upstream gradient gy ~ N(0, 1)
* ``wkv_decode`` WKV fp32 RNN-mode decoding, one token per sequence: B=1024
  sequences, T=1, C=2560 (RWKV-4-3B width), k, v, w, u as ``wkv_169m``, plus
  a state per (sequence, channel) from ``make_wkv_state``

States (``make_wkv_state``): [B, 3, C] float32 planes (a, b, p) standing for
the past sums (a, b) e^p.  Drawn with their own generator, seed + 1, in the
order: the past mean m ~ N(0, 1), ln b ~ U(-1, 1), p ~ N(0, p_sigma); then
a = m * b (so a / b = m stays within the range of v).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "WkvSpec", "ScanSpec", "WORKLOADS", "WkvInputs", "ScanInputs",
    "make_wkv", "make_scan", "bf16_round", "bf16_bits", "bf16_bits_to_f32",
    "get_workload", "make_wkv_state", "ShiftSpec", "ShiftInputs", "make_token_shift",
    "LruSpec", "LruInputs", "make_lru",
]


@dataclasses.dataclass(frozen=True)
class WkvSpec:
    """Shape and input distributions of one WKV workload."""
    name: str
    B: int
    T: int
    C: int
    dtype: str = "f32"            # "f32" or "bf16" storage of k, v, y
    k_sigma: float = 1.0          # k ~ N(0, k_sigma)
    v_sigma: float = 1.0          # v ~ N(0, v_sigma)
    w_log: tuple = ("normal", -0.5, 0.5)   # log w ~ N(m, s) or U(lo, hi)
    u_sigma: float = 0.5          # u ~ N(0, u_sigma)
    seed: int = 0
    state: bool = False           # the workload starts from a drawn state
    gated: bool = False           # also draws the receptance r ~ N(0, r_sigma)
    r_sigma: float = 2.0
    backward: bool = False        # gradients: also draws gy ~ N(0, 1)

    @property
    def elements(self) -> int:
        return self.B * self.T * self.C


@dataclasses.dataclass(frozen=True)
class ScanSpec:
    """Shape of one diagonal scan workload (minGRU or minLSTM form)."""
    name: str
    B: int
    T: int
    D: int
    seed: int = 0
    with_h0: bool = False         # minGRU recipe uses h0 = 0 (passed as "none")
    form: str = "mingru"          # "mingru" or "minlstm"
    dtype: str = "f32"            # "f32" or "bf16" storage of a, b, h

    @property
    def elements(self) -> int:
        return self.B * self.T * self.D


WORKLOADS = {
    "wkv_tiny": WkvSpec("wkv_tiny", 1, 64, 32, "f32", 1.0, 1.0, ("normal", -0.5, 0.5), 0.5),
    "wkv_169m": WkvSpec("wkv_169m", 8, 1024, 768, "f32", 1.0, 1.0, ("uniform", -3.0, 1.0), 0.5),
    "wkv_3b_bf16": WkvSpec("wkv_3b_bf16", 8, 4096, 2560, "bf16", 1.0, 1.0, ("uniform", -3.0, 1.0), 0.5),
    "wkv_long": WkvSpec("wkv_long", 1, 131072, 1024, "f32", 3.0, 1.0, ("uniform", -6.0, 0.0), 1.0),
    "scan_mingru": ScanSpec("scan_mingru", 64, 4096, 256),
    "scan_mingru_bf16": ScanSpec("scan_mingru_bf16", 64, 4096, 256, dtype="bf16"),
    "scan_minlstm": ScanSpec("scan_minlstm", 64, 4096, 256, form="minlstm"),
    "wkv_decode": WkvSpec("wkv_decode", 1024, 1, 2560, "f32", 1.0, 1.0, ("uniform", -3.0, 1.0),
                          0.5, state=True),
    "wkv_3b_gated_bf16": WkvSpec("wkv_3b_gated_bf16", 8, 4096, 2560, "bf16", 1.0, 1.0,
                                 ("uniform", -3.0, 1.0), 0.5, gated=True),
    "wkv_169m_bwd": WkvSpec("wkv_169m_bwd", 8, 1024, 768, "f32", 1.0, 1.0,
                            ("uniform", -3.0, 1.0), 0.5, backward=True),
}


@dataclasses.dataclass(frozen=True)
class ShiftSpec:
    """Shape of one token-shift workload."""
    name: str
    B: int
    T: int
    C: int
    n_mix: int = 3
    dtype: str = "f32"
    seed: int = 0

    @property
    def elements(self) -> int:
        return self.B * self.T * self.C


WORKLOADS["shift_3b_bf16"] = ShiftSpec("shift_3b_bf16", 8, 4096, 2560, 3, "bf16")


def get_workload(name: str):
    return WORKLOADS[name]


# ---------------------------------------------------------------------------
# bfloat16 storage helpers (numpy has no bfloat16 type)
# ---------------------------------------------------------------------------
def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.

    Inputs are finite, so the NaN special case is not needed."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    bias = ((bits >> 16) & 1) + 0x7FFF
    return ((bits + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b16: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact widening)."""
    return (np.ascontiguousarray(b16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16, returned as float32."""
    return bf16_bits_to_f32(bf16_bits(x32))


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class WkvInputs:
    """float32 host arrays; for bf16 workloads k and v hold the rounded values
    and ``k_bits``/``v_bits`` the uint16 storage the GPU path reads."""
    spec: WkvSpec
    w: np.ndarray   # [C] float32, w >= 0
    u: np.ndarray   # [C] float32
    k: np.ndarray   # [B, T, C] float32
    v: np.ndarray   # [B, T, C] float32
    k_bits: Optional[np.ndarray] = None
    v_bits: Optional[np.ndarray] = None
    s_in: Optional[np.ndarray] = None   # [B, 3, C] float32 when spec.state
    r: Optional[np.ndarray] = None      # [B, T, C] float32 when spec.gated
    r_bits: Optional[np.ndarray] = None
    gy: Optional[np.ndarray] = None     # [B, T, C] float32 when spec.backward


@dataclasses.dataclass
class ScanInputs:
    spec: ScanSpec
    a: np.ndarray   # [B, T, D] float32 (bf16-rounded values for bf16)
    b: np.ndarray   # [B, T, D] float32 (bf16-rounded values for bf16)
    h0: Optional[np.ndarray]   # [B, D] float32 or None (zeros)
    h_tilde: Optional[np.ndarray] = None   # [B, T, D] float32, the candidate states
    a_bits: Optional[np.ndarray] = None    # bf16 storage for bf16 workloads
    b_bits: Optional[np.ndarray] = None


def _draw_log_w(rng, spec_w, C):
    kind, p0, p1 = spec_w
    if kind == "normal":
        return rng.normal(p0, p1, size=C)
    if kind == "uniform":
        return rng.uniform(p0, p1, size=C)
    raise ValueError(kind)


def make_wkv(spec, *, B=None, T=None, C=None, seed=None) -> WkvInputs:
    """Draw one WKV workload. ``spec`` is a WkvSpec or a workload name; the
    keyword overrides give the same distributions at another shape."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    if B is not None or T is not None or C is not None or seed is not None:
        spec = dataclasses.replace(
            spec, B=spec.B if B is None else B, T=spec.T if T is None else T,
            C=spec.C if C is None else C, seed=spec.seed if seed is None else seed,
            name=f"{spec.name}@{B or spec.B}x{T or spec.T}x{C or spec.C}")
    rng = np.random.default_rng(spec.seed)
    shape = (spec.B, spec.T, spec.C)
    k = rng.normal(0.0, spec.k_sigma, size=shape).astype(np.float32)
    v = rng.normal(0.0, spec.v_sigma, size=shape).astype(np.float32)
    w = np.exp(_draw_log_w(rng, spec.w_log, spec.C)).astype(np.float32)
    u = rng.normal(0.0, spec.u_sigma, size=spec.C).astype(np.float32)
    r = rng.normal(0.0, spec.r_sigma, size=shape).astype(np.float32) if spec.gated else None
    gy = rng.normal(0.0, 1.0, size=shape).astype(np.float32) if spec.backward else None
    s_in = make_wkv_state(spec.B, spec.C, spec.seed) if spec.state else None
    if spec.dtype == "bf16":
        kb, vb = bf16_bits(k), bf16_bits(v)
        rb = bf16_bits(r) if r is not None else None
        return WkvInputs(spec, w, u, bf16_bits_to_f32(kb), bf16_bits_to_f32(vb), kb, vb, s_in,
                         None if rb is None else bf16_bits_to_f32(rb), rb)
    return WkvInputs(spec, w, u, k, v, s_in=s_in, r=r, gy=gy)


@dataclasses.dataclass
class ShiftInputs:
    spec: ShiftSpec
    x: np.ndarray        # [B, T, C] float32 (bf16-rounded values for bf16)
    mu: np.ndarray       # [n_mix, C] float32
    x_prev: np.ndarray   # [B, C] float32 (bf16-rounded for bf16)
    x_bits: Optional[np.ndarray] = None
    x_prev_bits: Optional[np.ndarray] = None


def make_token_shift(spec, *, B=None, T=None, C=None, n_mix=None, seed=None) -> ShiftInputs:
    """Draw one token-shift workload: x ~ N(0, 1) [B, T, C], mu ~ U(0, 1)
    [n_mix, C], x_prev ~ N(0, 1) [B, C], in that order."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    spec = dataclasses.replace(
        spec, B=spec.B if B is None else B, T=spec.T if T is None else T,
        C=spec.C if C is None else C, n_mix=spec.n_mix if n_mix is None else n_mix,
        seed=spec.seed if seed is None else seed)
    rng = np.random.default_rng(spec.seed)
    x = rng.normal(0.0, 1.0, size=(spec.B, spec.T, spec.C)).astype(np.float32)
    mu = rng.uniform(0.0, 1.0, size=(spec.n_mix, spec.C)).astype(np.float32)
    xp = rng.normal(0.0, 1.0, size=(spec.B, spec.C)).astype(np.float32)
    if spec.dtype == "bf16":
        xb, pb = bf16_bits(x), bf16_bits(xp)
        return ShiftInputs(spec, bf16_bits_to_f32(xb), mu, bf16_bits_to_f32(pb), xb, pb)
    return ShiftInputs(spec, x, mu, xp)


def make_wkv_state(B: int, C: int, seed: int = 0, p_sigma: float = 2.0) -> np.ndarray:
    """A random non-empty WKV state [B, 3, C] float32 (planes a, b, p)."""
    rng = np.random.default_rng(seed + 1)
    mean = rng.normal(0.0, 1.0, size=(B, C))
    b = np.exp(rng.uniform(-1.0, 1.0, size=(B, C)))
    p = rng.normal(0.0, p_sigma, size=(B, C))
    return np.stack([mean * b, b, p], axis=1).astype(np.float32)


def make_scan(spec, *, B=None, T=None, D=None, seed=None, with_h0=None) -> ScanInputs:
    """Draw one diagonal-scan workload: minGRU form (a = 1 - z, b = z * h~)
    or minLSTM form (a = f / (f + i), b = i / (f + i) * h~)."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    spec = dataclasses.replace(
        spec, B=spec.B if B is None else B, T=spec.T if T is None else T,
        D=spec.D if D is None else D, seed=spec.seed if seed is None else seed,
        with_h0=spec.with_h0 if with_h0 is None else with_h0)
    rng = np.random.default_rng(spec.seed)
    shape = (spec.B, spec.T, spec.D)
    if spec.form == "minlstm":
        f = 1.0 / (1.0 + np.exp(-rng.normal(0.0, 1.0, size=shape)))
        i = 1.0 / (1.0 + np.exp(-rng.normal(0.0, 1.0, size=shape)))
        h_tilde = rng.normal(0.0, 1.0, size=shape)
        a = (f / (f + i)).astype(np.float32)
        b = (i / (f + i) * h_tilde).astype(np.float32)
    else:
        z = 1.0 / (1.0 + np.exp(-rng.normal(0.0, 1.0, size=shape)))
        h_tilde = rng.normal(0.0, 1.0, size=shape)
        a = (1.0 - z).astype(np.float32)
        b = (z * h_tilde).astype(np.float32)
    h0 = rng.normal(0.0, 1.0, size=(spec.B, spec.D)).astype(np.float32) if spec.with_h0 else None
    if spec.dtype == "bf16":
        ab, bb = bf16_bits(a), bf16_bits(b)
        return ScanInputs(spec, bf16_bits_to_f32(ab), bf16_bits_to_f32(bb), h0,
                          h_tilde.astype(np.float32), ab, bb)
    return ScanInputs(spec, a, b, h0, h_tilde.astype(np.float32))


@dataclasses.dataclass(frozen=True)
class LruSpec:
    """Shape of one LRU (complex diagonal recurrence) workload."""
    name: str
    B: int
    T: int
    D: int
    r_min: float = 0.9
    r_max: float = 0.999
    seed: int = 0
    with_x0: bool = False

    @property
    def elements(self) -> int:
        return self.B * self.T * self.D


WORKLOADS["lru_256"] = LruSpec("lru_256", 64, 4096, 256)


@dataclasses.dataclass
class LruInputs:
    spec: LruSpec
    nu_log: np.ndarray     # [D] float32
    theta_log: np.ndarray  # [D] float32
    gamma: np.ndarray      # [D] float32
    u: np.ndarray          # [B, T, D, 2] float32: real and imaginary parts
    x0: Optional[np.ndarray] = None   # [B, D, 2] float32 or None

    def u_complex(self):
        return self.u[..., 0].astype(np.float64) + 1j * self.u[..., 1].astype(np.float64)

    def x0_complex(self):
        if self.x0 is None:
            return None
        return self.x0[..., 0].astype(np.float64) + 1j * self.x0[..., 1].astype(np.float64)


def make_lru(spec, *, B=None, T=None, D=None, seed=None, with_x0=None) -> LruInputs:
    """Draw one LRU workload with the LRU review's initialisation: r^2 ~
    U[r_min^2, r_max^2], theta ~ U[0, 2 pi], stored as nu_log = ln(-ln r)
    and theta_log = ln theta; gamma = sqrt(1 - r^2); u complex with real and
    imaginary parts ~ N(0, 1/2); drawn in that order (x0 last, same law as u)."""
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    spec = dataclasses.replace(
        spec, B=spec.B if B is None else B, T=spec.T if T is None else T,
        D=spec.D if D is None else D, seed=spec.seed if seed is None else seed,
        with_x0=spec.with_x0 if with_x0 is None else with_x0)
    rng = np.random.default_rng(spec.seed)
    r = np.sqrt(rng.uniform(spec.r_min ** 2, spec.r_max ** 2, size=spec.D))
    theta = rng.uniform(0.0, 2.0 * np.pi, size=spec.D)
    nu_log = np.log(-np.log(r)).astype(np.float32)
    theta_log = np.log(theta).astype(np.float32)
    gamma = np.sqrt(1.0 - r ** 2).astype(np.float32)
    u = rng.normal(0.0, np.sqrt(0.5), size=(spec.B, spec.T, spec.D, 2)).astype(np.float32)
    x0 = rng.normal(0.0, np.sqrt(0.5), size=(spec.B, spec.D, 2)).astype(np.float32) \
        if spec.with_x0 else None
    return LruInputs(spec, nu_log, theta_log, gamma, u, x0)
