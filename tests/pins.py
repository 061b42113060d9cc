"""Pins for WKV and diagonal-scan implementations.

Each check takes an implementation ``fn`` (numpy arrays in, float64 array out)
and returns a list of failure messages.  The values they compare against come
from outside the implementation under test:

* hand-worked examples in exact rational arithmetic (``tests/golden``);
* closed forms of special cases (running mean, geometric series, two-token
  softmax limit, cumulative sum / product);
* invariants the definition fixes (convex combination, shift invariance in k,
  affine equivariance in v, causality).

Used by the oracle's CPU tests (including the planted-mistake tests, which
check that every planted mistake trips at least one pin) and by the GPU
parity tests.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    recs = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            recs[key] = [Fraction(x) for x in vals]
    return recs


def _close(got, want, tol):
    got, want = np.asarray(got), np.asarray(want)
    cplx = np.iscomplexobj(got) or np.iscomplexobj(want)
    got = got.astype(np.complex128 if cplx else np.float64)
    want = want.astype(np.complex128 if cplx else np.float64)
    if got.shape != want.shape:
        return f"shape {got.shape} != {want.shape}"
    err = np.max(np.abs(got - want)) if got.size else 0.0
    if not np.isfinite(err) or err > tol:
        return f"max err {err:.3e} > {tol:.1e}"
    return None


# ---------------------------------------------------------------------------
# WKV pins
# ---------------------------------------------------------------------------
def wkv_worked_example(fn, tol=1e-12):
    g = read_golden("wkv_worked_example.txt")
    w = np.array([-np.log(float(g["w_exp_neg"][0]))])
    u = np.array([np.log(float(g["u_exp"][0]))])
    k = np.log(np.array([float(x) for x in g["k_exp"]]))[None, :, None]
    v = np.array([float(x) for x in g["v"]])[None, :, None]
    want = np.array([float(x) for x in g["y"]])[None, :, None]
    msg = _close(fn(w, u, k, v), want, tol)
    return [f"worked example: {msg}"] if msg else []


def wkv_exact_rational(fn, seed=3, T=7, C=3, tol=1e-12):
    """Brute force in exact rationals: pick e^{k}, e^{-w}, e^{u} rational."""
    rng = np.random.default_rng(seed)
    r = [[Fraction(int(rng.integers(1, 9)), int(rng.integers(1, 9))) for _ in range(C)] for _ in range(T)]
    lam = [Fraction(int(rng.integers(1, 8)), 8) for _ in range(C)]
    gam = [Fraction(int(rng.integers(1, 7)), int(rng.integers(1, 7))) for _ in range(C)]
    vv = [[Fraction(int(rng.integers(-9, 10))) for _ in range(C)] for _ in range(T)]
    want = np.zeros((1, T, C))
    for c in range(C):
        for t in range(T):
            num = gam[c] * r[t][c] * vv[t][c]
            den = gam[c] * r[t][c]
            for i in range(t):
                wt = lam[c] ** (t - 1 - i) * r[i][c]
                num += wt * vv[i][c]
                den += wt
            want[0, t, c] = float(num / den)
    k = np.log(np.array([[float(x) for x in row] for row in r]))[None]
    w = -np.log(np.array([float(x) for x in lam]))
    u = np.log(np.array([float(x) for x in gam]))
    v = np.array([[float(x) for x in row] for row in vv])[None]
    msg = _close(fn(w, u, k, v), want, tol)
    return [f"exact rational: {msg}"] if msg else []


def wkv_single_step(fn, tol=0.0):
    rng = np.random.default_rng(1)
    k = rng.normal(0, 2, (3, 1, 5)); v = rng.normal(0, 1, (3, 1, 5))
    w = np.exp(rng.normal(0, 1, 5)); u = rng.normal(0, 1, 5)
    msg = _close(fn(w, u, k, v), v, tol)
    return [f"T=1 gives v: {msg}"] if msg else []


def wkv_running_mean(fn, tol=1e-12):
    """w = 0, u = 0, constant k: every past token and the current one weigh
    the same, so y_t is the mean of v_0..v_t."""
    rng = np.random.default_rng(2)
    T, C = 40, 4
    v = rng.normal(0, 1, (2, T, C))
    k = np.full((2, T, C), 0.7)
    want = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None]
    msg = _close(fn(np.zeros(C), np.zeros(C), k, v), want, tol)
    return [f"running mean: {msg}"] if msg else []


def wkv_past_mean(fn, tol=1e-9):
    """w = 0, constant k, bonus u -> -inf (u = -40): the current token's
    weight vanishes, y_t (t >= 1) is the mean of v_0..v_{t-1}."""
    rng = np.random.default_rng(4)
    T, C = 30, 3
    v = rng.normal(0, 1, (1, T, C))
    k = np.zeros((1, T, C))
    got = np.asarray(fn(np.zeros(C), np.full(C, -40.0), k, v))
    want = np.cumsum(v, axis=1)[:, :-1, :] / np.arange(1, T)[None, :, None]
    msg = _close(got[:, 1:, :], want, tol)
    return [f"past-only mean: {msg}"] if msg else []


def wkv_geometric(fn, tol=1e-12):
    """k = 0, u = 0, decay lam = e^{-w}, v one-hot at step j: the weight of
    token j at step t > j is lam^{t-1-j}, the denominator is the geometric
    sum (1 - lam^t) / (1 - lam) + 1."""
    T, j = 24, 5
    lam = np.array([0.5, 0.9, 0.25])
    w = -np.log(lam)
    C = lam.size
    v = np.zeros((1, T, C)); v[0, j, :] = 1.0
    k = np.zeros((1, T, C))
    want = np.zeros((1, T, C))
    for t in range(T):
        den = (1 - lam ** t) / (1 - lam) + 1.0
        if t == j:
            want[0, t] = 1.0 / den
        elif t > j:
            want[0, t] = lam ** (t - 1 - j) / den
    msg = _close(fn(w, np.zeros(C), k, v), want, tol)
    return [f"geometric one-hot: {msg}"] if msg else []


def wkv_fast_decay(fn, tol=1e-12):
    """w -> inf (w = 60): only the previous token (weight e^{k_{t-1}}) and
    the current one (weight e^{u + k_t}) survive."""
    rng = np.random.default_rng(5)
    T, C = 20, 4
    k = rng.normal(0, 1, (1, T, C)); v = rng.normal(0, 1, (1, T, C))
    u = rng.normal(0, 0.5, C)
    want = v.copy()
    ep = np.exp(k[:, :-1]); ec = np.exp(u + k[:, 1:])
    want[:, 1:] = (ep * v[:, :-1] + ec * v[:, 1:]) / (ep + ec)
    msg = _close(fn(np.full(C, 60.0), u, k, v), want, tol)
    return [f"fast decay two-token limit: {msg}"] if msg else []


def wkv_large_bonus(fn, tol=1e-12):
    """u -> inf (u = 60) with |k| small: y_t = v_t."""
    rng = np.random.default_rng(6)
    k = rng.normal(0, 1, (1, 16, 3)); v = rng.normal(0, 1, (1, 16, 3))
    msg = _close(fn(np.full(3, 0.1), np.full(3, 60.0), k, v), v, tol)
    return [f"large bonus: {msg}"] if msg else []


def _rand_wkv(seed, B=2, T=48, C=5, ksig=2.0):
    rng = np.random.default_rng(seed)
    return (np.exp(rng.normal(-0.5, 1.0, C)), rng.normal(0, 1, C),
            rng.normal(0, ksig, (B, T, C)), rng.normal(0, 1, (B, T, C)))


def wkv_invariants(fn, rel=1e-11):
    out = []
    w, u, k, v = _rand_wkv(7)
    y = np.asarray(fn(w, u, k, v))
    # convex combination of v_0..v_t
    lo = np.minimum.accumulate(v, axis=1); hi = np.maximum.accumulate(v, axis=1)
    if np.any(y < lo - rel) or np.any(y > hi + rel):
        out.append("convex bound violated")
    # shift invariance in k (common factor of numerator and denominator)
    msg = _close(fn(w, u, k + 3.25, v), y, rel * 10)
    if msg: out.append(f"k-shift invariance: {msg}")
    # affine equivariance in v
    msg = _close(fn(w, u, k, 2.5 * v - 1.5), 2.5 * y - 1.5, rel * 10)
    if msg: out.append(f"affine equivariance: {msg}")
    # constant v gives v
    msg = _close(fn(w, u, k, np.full_like(v, 0.375)), np.full_like(v, 0.375), rel)
    if msg: out.append(f"constant v: {msg}")
    # causality: editing step j leaves every earlier output unchanged
    j = 30
    v2 = v.copy(); k2 = k.copy(); v2[:, j:] += 5.0; k2[:, j:] -= 2.0
    y2 = np.asarray(fn(w, u, k2, v2))
    if not np.array_equal(y2[:, :j], y[:, :j]):
        out.append("causality: future tokens changed past outputs")
    # channels and batch rows are independent
    yb = np.asarray(fn(w[1:3], u[1:3], k[1:, :, 1:3], v[1:, :, 1:3]))
    msg = _close(yb, y[1:, :, 1:3], 0.0)
    if msg: out.append(f"channel/batch independence: {msg}")
    return out


WKV_PINS = [wkv_worked_example, wkv_exact_rational, wkv_single_step, wkv_running_mean,
            wkv_past_mean, wkv_geometric, wkv_fast_decay, wkv_large_bonus, wkv_invariants]


def run_wkv_pins(fn):
    fails = []
    for pin in WKV_PINS:
        try:
            fails += pin(fn)
        except Exception as e:  # a mutant may crash a pin; that counts as caught
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails


# ---------------------------------------------------------------------------
# WKV with a state in and out.  An implementation here is
#     fn(w, u, k, v, s_in) -> (y, s_out)
# with states [B, 3, C] (planes a, b, p: past sums (num, den) = (a, b) e^p) and
# s_in None for the empty past.  A state is compared by what fixes it: the
# mean a / b and ln den = p + ln b.
# ---------------------------------------------------------------------------
def _state_parts(s):
    s = np.asarray(s, dtype=np.float64)
    a, b, p = s[:, 0], s[:, 1], s[:, 2]
    with np.errstate(divide="ignore", invalid="ignore"):
        return a / b, p + np.log(b)


def _close_state(got, want, tol):
    gm, gl = _state_parts(got)
    wm, wl = _state_parts(want)
    return _close(gm, wm, tol) or _close(gl, wl, tol)


def _state_from(num, den):
    """A [1, 3, C] state holding the past sums num, den (den > 0)."""
    num = np.asarray(num, dtype=np.float64).reshape(1, -1)
    den = np.asarray(den, dtype=np.float64).reshape(1, -1)
    return np.stack([num / den, np.ones_like(den), np.log(den)], axis=1)


def wkv_state_worked_example(fn, tol=1e-12):
    g = read_golden("wkv_state_worked_example.txt")
    w = np.array([-np.log(float(g["w_exp_neg"][0]))])
    u = np.array([np.log(float(g["u_exp"][0]))])
    s_in = np.array([[[float(g["state_a"][0])], [float(g["state_b"][0])],
                      [np.log(float(g["state_p_exp"][0]))]]])
    k = np.log(np.array([float(x) for x in g["k_exp"]]))[None, :, None]
    v = np.array([float(x) for x in g["v"]])[None, :, None]
    y, s_out = fn(w, u, k, v, s_in)
    out = []
    msg = _close(y, np.array([float(x) for x in g["y"]])[None, :, None], tol)
    if msg: out.append(f"state worked example, y: {msg}")
    msg = _close_state(s_out, _state_from(float(g["num_out"][0]), float(g["den_out"][0])), tol)
    if msg: out.append(f"state worked example, state out: {msg}")
    return out


def wkv_state_empty(fn, tol=0.0):
    """No state, the explicit empty state (a = b = 0) and the no-state
    forms agree, outputs and state out."""
    w, u, k, v = _rand_wkv(11, B=2, T=20, C=3)
    y0, s0 = fn(w, u, k, v, None)
    out = []
    for p_fill in (-np.inf, 0.0, 7.5):
        s_in = np.zeros((2, 3, 3)); s_in[:, 2] = p_fill
        y1, s1 = fn(w, u, k, v, s_in)
        msg = _close(y1, y0, tol) or _close_state(s1, s0, max(tol, 1e-15))
        if msg: out.append(f"empty state (p = {p_fill}): {msg}")
    return out


def wkv_state_chaining(fn, tol=1e-12):
    """Splitting the steps into calls that hand the state on gives the
    outputs and final state of one call (several split points, T = 1 calls
    included: RNN-mode decoding)."""
    w, u, k, v = _rand_wkv(12, B=2, T=40, C=4)
    y, s = fn(w, u, k, v, None)
    out = []
    for cuts in ([17], [1, 2, 3, 39], [10, 20, 30], list(range(1, 40))):
        ys, st, prev = [], None, 0
        for c in cuts + [40]:
            yy, st = fn(w, u, k[:, prev:c], v[:, prev:c], st)
            ys.append(yy)
            prev = c
        msg = _close(np.concatenate(ys, axis=1), y, tol) or _close_state(st, s, tol)
        if msg: out.append(f"chaining at {cuts[:4]}: {msg}")
    return out


def wkv_state_virtual_token(fn, tol=1e-12):
    """The state after one token (k0, v0) is (num, den) = (e^{k0} v0, e^{k0});
    starting there equals running that token first and dropping its output."""
    w, u, k, v = _rand_wkv(13, B=1, T=25, C=3)
    y_full, s_full = fn(w, u, k, v, None)
    s_in = _state_from(np.exp(k[0, 0]) * v[0, 0], np.exp(k[0, 0]))
    y, s = fn(w, u, k[:, 1:], v[:, 1:], s_in)
    msg = _close(y, y_full[:, 1:], tol) or _close_state(s, s_full, tol)
    return [f"state as a virtual token: {msg}"] if msg else []


def wkv_state_scaling(fn, tol=1e-12):
    """(a, b, p) and (a e^s, b e^s, p - s) are one state: same outputs and
    same state out."""
    w, u, k, v = _rand_wkv(14, B=2, T=16, C=3)
    rng = np.random.default_rng(14)
    s_in = np.stack([rng.normal(0, 1, (2, 3)), np.exp(rng.normal(0, 1, (2, 3))),
                     rng.normal(0, 2, (2, 3))], axis=1)
    y0, s0 = fn(w, u, k, v, s_in)
    out = []
    for sh in (-3.0, 0.5, 12.0):
        s2 = s_in.copy(); s2[:, 0] *= np.exp(sh); s2[:, 1] *= np.exp(sh); s2[:, 2] -= sh
        y1, s1 = fn(w, u, k, v, s2)
        msg = _close(y1, y0, tol) or _close_state(s1, s0, tol)
        if msg: out.append(f"state rescaling by e^{sh}: {msg}")
    return out


def wkv_state_decay_only(fn, tol=1e-12):
    """With k = -inf-like keys (-60) and u = 0 the tokens add nothing next to
    a unit state: the state's mean passes straight through to every output
    and the state out is the state in decayed t times (ln den drops by T w)."""
    C, T = 3, 6
    w = np.array([0.1, 0.7, 2.0]); u = np.zeros(C)
    k = np.full((1, T, C), -60.0); v = np.ones((1, T, C))
    s_in = np.stack([np.array([[0.25, -1.5, 2.0]]), np.ones((1, C)), np.array([[3.0, 0.0, -2.0]])], axis=1)
    # token weight e^{-60} against a state weight of at least e^{-2 - 5 * 2}:
    # the tokens move the results by about e^{-48}, far below tol
    y, s = fn(w, u, k, v, s_in)
    out = []
    msg = _close(y, np.broadcast_to(np.array([0.25, -1.5, 2.0]), (1, T, C)), tol)
    if msg: out.append(f"decay only, y: {msg}")
    want = np.stack([np.array([[0.25, -1.5, 2.0]]), np.ones((1, C)),
                     np.array([[3.0, 0.0, -2.0]]) - T * w[None]], axis=1)
    msg = _close_state(s, want, tol)
    if msg: out.append(f"decay only, state: {msg}")
    return out


WKV_STATE_PINS = [wkv_state_worked_example, wkv_state_empty, wkv_state_chaining,
                  wkv_state_virtual_token, wkv_state_scaling, wkv_state_decay_only]


def run_wkv_state_pins(fn):
    """The state pins, plus every stateless pin on fn(..., None)[0]."""
    fails = []
    for pin in WKV_STATE_PINS:
        try:
            fails += pin(fn)
        except Exception as e:  # a mutant may crash a pin; that counts as caught
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    fails += run_wkv_pins(lambda w, u, k, v: fn(w, u, k, v, None)[0])
    return fails


# ---------------------------------------------------------------------------
# Token shift: fn(x, mu, x_prev) -> (out [n_mix, B, T, C], x_last [B, C])
# ---------------------------------------------------------------------------
def token_shift_worked_example(fn, tol=1e-15):
    g = read_golden("token_shift_worked_example.txt")
    x = np.array([float(a) for a in g["x"]]).reshape(1, 3, 2)
    x_prev = np.array([float(a) for a in g["x_prev"]]).reshape(1, 2)
    mu = np.array([float(a) for a in g["mu"]]).reshape(2, 2)
    out, last = fn(x, mu, x_prev)
    fails = []
    msg = _close(out, np.array([float(a) for a in g["out"]]).reshape(2, 1, 3, 2), tol)
    if msg: fails.append(f"token shift worked example: {msg}")
    msg = _close(last, np.array([float(a) for a in g["x_last"]]).reshape(1, 2), 0.0)
    if msg: fails.append(f"token shift last token: {msg}")
    return fails


def token_shift_special_cases(fn, tol=0.0):
    """mu = 1 keeps x_t, mu = 0 takes x_{t-1} (x_prev at t = 0), mu = 1/2
    averages the two; no x_prev is a zero x_prev."""
    rng = np.random.default_rng(31)
    B, T, C = 2, 9, 5
    x = rng.normal(0, 1, (B, T, C)); xp = rng.normal(0, 1, (B, C))
    mu = np.stack([np.ones(C), np.zeros(C), np.full(C, 0.5)])
    out, last = fn(x, mu, xp)
    shifted = np.concatenate([xp[:, None], x[:, :-1]], axis=1)
    fails = []
    for m, want, name in ((0, x, "mu = 1"), (1, shifted, "mu = 0"),
                          (2, 0.5 * (x + shifted), "mu = 1/2")):
        msg = _close(np.asarray(out)[m], want, tol if m < 2 else 1e-15)
        if msg: fails.append(f"token shift {name}: {msg}")
    msg = _close(last, x[:, -1], 0.0)
    if msg: fails.append(f"token shift last token: {msg}")
    o0, _ = fn(x, mu, None)
    o1, _ = fn(x, mu, np.zeros((B, C)))
    msg = _close(o0, o1, 0.0)
    if msg: fails.append(f"token shift without x_prev: {msg}")
    return fails


def token_shift_chaining(fn, tol=1e-15):
    """Two calls handing on the last token equal one call."""
    rng = np.random.default_rng(32)
    B, T, C = 3, 20, 6
    x = rng.normal(0, 1, (B, T, C)); xp = rng.normal(0, 1, (B, C))
    mu = rng.uniform(0, 1, (3, C))
    out, last = fn(x, mu, xp)
    o1, l1 = fn(x[:, :7], mu, xp)
    o2, l2 = fn(x[:, 7:], mu, l1)
    msg = _close(np.concatenate([o1, o2], axis=2), out, tol) or _close(l2, last, 0.0)
    return [f"token shift chaining: {msg}"] if msg else []


TOKEN_SHIFT_PINS = [token_shift_worked_example, token_shift_special_cases, token_shift_chaining]


def run_token_shift_pins(fn):
    fails = []
    for pin in TOKEN_SHIFT_PINS:
        try:
            fails += pin(fn)
        except Exception as e:
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails


# ---------------------------------------------------------------------------
# Gated WKV: fn(w, u, k, v, r) -> sigma(r) (.) wkv
# ---------------------------------------------------------------------------
def gate_worked_example(fn, tol=1e-12):
    g = read_golden("wkv_gate_worked_example.txt")
    w = np.array([-np.log(float(g["w_exp_neg"][0]))])
    u = np.array([np.log(float(g["u_exp"][0]))])
    k = np.log(np.array([float(x) for x in g["k_exp"]]))[None, :, None]
    v = np.array([float(x) for x in g["v"]])[None, :, None]
    r = np.log(np.array([float(x) for x in g["r_exp"]]))[None, :, None]
    msg = _close(fn(w, u, k, v, r), np.array([float(x) for x in g["out"]])[None, :, None], tol)
    return [f"gate worked example: {msg}"] if msg else []


def gate_limits(fn, tol=1e-12):
    """r = +60 passes wkv through (sigma = 1 in float64); r = 0 halves it;
    sigma(r) + sigma(-r) = 1; r = -60 closes the gate."""
    w, u, k, v = _rand_wkv(33, B=2, T=30, C=4)
    rng = np.random.default_rng(33)
    r = rng.normal(0, 2, k.shape)
    open_ = np.asarray(fn(w, u, k, v, np.full(k.shape, 60.0)))
    fails = [f"gate open, stateless pins: {f}" for f in run_wkv_pins(
        lambda w_, u_, k_, v_: fn(w_, u_, k_, v_, np.full(np.shape(k_), 60.0)))]
    msg = _close(fn(w, u, k, v, np.zeros(k.shape)), 0.5 * open_, tol)
    if msg: fails.append(f"gate at r = 0: {msg}")
    msg = _close(np.asarray(fn(w, u, k, v, r)) + np.asarray(fn(w, u, k, v, -r)), open_, tol)
    if msg: fails.append(f"gate symmetry: {msg}")
    msg = _close(fn(w, u, k, v, np.full(k.shape, -60.0)), np.zeros(k.shape), 1e-25)
    if msg: fails.append(f"gate closed: {msg}")
    return fails


GATE_PINS = [gate_worked_example, gate_limits]


def run_gate_pins(fn):
    fails = []
    for pin in GATE_PINS:
        try:
            fails += pin(fn)
        except Exception as e:
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails


# ---------------------------------------------------------------------------
# LRU scan: fn(nu_log, theta_log, gamma, u, x0) -> complex x [B, T, D]
# ---------------------------------------------------------------------------
def lru_worked_example(fn, tol=1e-14):
    g = read_golden("lru_worked_example.txt")
    nu_log = np.array([np.log(-np.log(float(g["r"][0])))])
    theta_log = np.array([np.log(np.pi * float(g["theta_over_pi"][0]))])
    u = (np.array([float(x) for x in g["u_re"]]) + 1j * np.array([float(x) for x in g["u_im"]]))
    u = u.reshape(1, 3, 1)
    out = []
    for case, x0 in (("case1", None), ("case2", np.array([[float(g["case2_x0_re"][0]) +
                                                           1j * float(g["case2_x0_im"][0])]]))):
        want = np.array([float(x) for x in g[f"{case}_x_re"]]) + \
            1j * np.array([float(x) for x in g[f"{case}_x_im"]])
        got = np.asarray(fn(nu_log, theta_log, np.array([float(g[f"{case}_gamma"][0])]), u, x0))
        msg = _close(got.reshape(-1), want, tol)
        if msg: out.append(f"lru worked example {case}: {msg}")
    return out


def lru_impulse(fn, tol=1e-12):
    """u = delta at t = 0: x_t = gamma lambda^t = gamma r^t (cos t theta + i sin t theta)."""
    D, T = 4, 50
    nu_log = np.log(np.array([0.01, 0.1, 0.5, 2.0]))
    theta_log = np.log(np.array([0.3, 1.0, 2.5, 6.0]))
    gamma = np.array([1.0, 0.5, 2.0, 0.1])
    u = np.zeros((1, T, D), dtype=complex); u[0, 0] = 1.0
    t = np.arange(T)[:, None]
    r, th = np.exp(-np.exp(nu_log)), np.exp(theta_log)
    want = gamma * r ** t * (np.cos(t * th) + 1j * np.sin(t * th))
    msg = _close(np.asarray(fn(nu_log, theta_log, gamma, u, None))[0], want, tol)
    return [f"lru impulse response: {msg}"] if msg else []


def lru_real_case(fn, tol=1e-12, scan=None):
    """theta -> 0 makes lambda real (= e^{-nu}): real and imaginary parts each
    follow the real diagonal scan with a = e^{-nu}, b = gamma u."""
    rng = np.random.default_rng(41)
    B, T, D = 2, 40, 3
    nu_log = rng.normal(-1, 1, D); theta_log = np.full(D, -200.0)
    gamma = rng.uniform(0.5, 1.5, D)
    u = rng.normal(0, 1, (B, T, D)) + 1j * rng.normal(0, 1, (B, T, D))
    x0 = rng.normal(0, 1, (B, D)) + 1j * rng.normal(0, 1, (B, D))
    got = np.asarray(fn(nu_log, theta_log, gamma, u, x0))
    a = np.broadcast_to(np.exp(-np.exp(nu_log)), (B, T, D))
    out = []
    for part, name in ((np.real, "re"), (np.imag, "im")):
        want = scan(a, gamma * part(u), part(x0))
        msg = _close(part(got), want, tol)
        if msg: out.append(f"lru real case ({name}): {msg}")
    return out


def lru_linearity_and_chaining(fn, tol=1e-12):
    rng = np.random.default_rng(42)
    B, T, D = 2, 30, 4
    nu_log, theta_log = rng.normal(-2, 1, D), rng.normal(0, 1, D)
    gamma = rng.uniform(0.5, 1.5, D)
    u = rng.normal(0, 1, (B, T, D)) + 1j * rng.normal(0, 1, (B, T, D))
    x0 = rng.normal(0, 1, (B, D)) + 1j * rng.normal(0, 1, (B, D))
    x = np.asarray(fn(nu_log, theta_log, gamma, u, x0))
    out = []
    rot = np.exp(0.7j)
    msg = _close(np.asarray(fn(nu_log, theta_log, gamma, rot * u, rot * x0)), rot * x, tol)
    if msg: out.append(f"lru rotation equivariance: {msg}")
    x1 = np.asarray(fn(nu_log, theta_log, gamma, u[:, :11], x0))
    x2 = np.asarray(fn(nu_log, theta_log, gamma, u[:, 11:], x1[:, -1]))
    msg = _close(np.concatenate([x1, x2], axis=1), x, tol)
    if msg: out.append(f"lru chaining: {msg}")
    return out


def lru_variance(fn):
    """For iid zero-mean u, E|x_t|^2 = gamma^2 (1 - r^{2(t+1)}) / (1 - r^2) E|u|^2
    (the LRU review's initialisation section); checked statistically."""
    rng = np.random.default_rng(43)
    B, T, D = 4000, 24, 2
    nu_log = np.log(-np.log(np.array([0.9, 0.5])))
    theta_log = np.log(np.array([1.0, 2.0]))
    gamma = np.array([1.0, 0.7])
    u = (rng.normal(0, 1, (B, T, D)) + 1j * rng.normal(0, 1, (B, T, D))) / np.sqrt(2)
    x = np.asarray(fn(nu_log, theta_log, gamma, u, None))
    r = np.array([0.9, 0.5])
    t = np.arange(T)[:, None]
    want = gamma ** 2 * (1 - r ** (2 * (t + 1))) / (1 - r ** 2)
    got = np.mean(np.abs(x) ** 2, axis=0)
    rel = np.max(np.abs(got - want) / want)
    return [] if rel < 0.1 else [f"lru variance formula: rel err {rel:.3f}"]


LRU_PINS = [lru_worked_example, lru_impulse, lru_real_case, lru_linearity_and_chaining,
            lru_variance]


def run_lru_pins(fn, scan):
    fails = []
    for pin in LRU_PINS:
        try:
            fails += pin(fn, scan=scan) if pin is lru_real_case else pin(fn)
        except Exception as e:
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails


# ---------------------------------------------------------------------------
# WKV gradients: fn(w, u, k, v, gy) -> (gk, gv, gw, gu), gw and gu [C]
# ---------------------------------------------------------------------------
def grad_worked_example(fn, tol=1e-12):
    g = read_golden("wkv_grad_worked_example.txt")
    w = np.array([-np.log(float(g["w_exp_neg"][0]))])
    u = np.array([np.log(float(g["u_exp"][0]))])
    k = np.log(np.array([float(x) for x in g["k_exp"]]))[None, :, None]
    v = np.array([float(x) for x in g["v"]])[None, :, None]
    gy = np.array([float(x) for x in g["g"]])[None, :, None]
    gk, gv, gw, gu = fn(w, u, k, v, gy)
    out = []
    for name, got in (("gk", gk), ("gv", gv), ("gw", gw), ("gu", gu)):
        want = np.array([float(x) for x in g[name]])
        msg = _close(np.asarray(got).reshape(-1), want, tol)
        if msg: out.append(f"gradient worked example {name}: {msg}")
    return out


def _torch_grads(w, u, k, v, gy):
    """Reverse-mode autodiff (PyTorch, float64) through eq. (14) written as a
    masked softmax over the [T, T] logits."""
    import torch
    tw, tu, tk, tv = (torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True)
                      for x in (w, u, k, v))
    B, T, C = tk.shape
    t_idx = torch.arange(T)[:, None]
    i_idx = torch.arange(T)[None, :]
    dist = (t_idx - 1 - i_idx).double()
    logit = -dist[None, :, :, None] * tw[None, None, None, :] + tk[:, None, :, :]
    diag = (tu[None, None, :] + tk)[:, :, None, :].expand(B, T, T, C)
    eye = (t_idx == i_idx)[None, :, :, None].expand(B, T, T, C)
    logit = torch.where(eye, diag, logit)
    logit = logit.masked_fill((i_idx > t_idx)[None, :, :, None].expand(B, T, T, C), float("-inf"))
    beta = torch.softmax(logit, dim=2)
    y = (beta * tv[:, None, :, :]).sum(dim=2)
    (y * torch.tensor(np.asarray(gy, dtype=np.float64))).sum().backward()
    return tk.grad.numpy(), tv.grad.numpy(), tw.grad.numpy(), tu.grad.numpy()


def grad_autodiff(fn, tol=1e-11):
    """Against reverse-mode autodiff of the definition on random inputs."""
    w, u, k, v = _rand_wkv(51, B=2, T=24, C=3)
    gy = np.random.default_rng(51).normal(0, 1, k.shape)
    got = fn(w, u, k, v, gy)
    want = _torch_grads(w, u, k, v, gy)
    out = []
    for name, a, b in zip(("gk", "gv", "gw", "gu"), got, want):
        msg = _close(a, b, tol * max(1.0, float(np.abs(b).max())))
        if msg: out.append(f"gradient vs autodiff {name}: {msg}")
    return out


def grad_finite_difference(fn, h=1e-6, tol=1e-7):
    """Central differences of the definition itself (numpy, float64)."""
    w, u, k, v = _rand_wkv(52, B=1, T=6, C=2, ksig=1.0)
    gy = np.random.default_rng(52).normal(0, 1, k.shape)

    def loss(w_, u_, k_, v_):
        T = k_.shape[1]
        tot = 0.0
        for c in range(k_.shape[2]):
            for t in range(T):
                l = np.array([-(t - 1 - j) * w_[c] + k_[0, j, c] for j in range(t)] + [u_[c] + k_[0, t, c]])
                e = np.exp(l - l.max())
                tot += gy[0, t, c] * np.dot(e, v_[0, :t + 1, c]) / e.sum()
        return tot

    gk, gv, gw, gu = fn(w, u, k, v, gy)
    out = []
    for name, arr, grad in (("k", k, gk), ("v", v, gv), ("w", w, gw), ("u", u, gu)):
        for idx in ([(0, 0, 0), (0, 3, 1), (0, 5, 0)] if arr.ndim == 3 else [(0,), (1,)]):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += h
            a2[idx] -= h
            args1 = {"k": (w, u, a1, v), "v": (w, u, k, a1), "w": (a1, u, k, v), "u": (w, a1, k, v)}[name]
            args2 = {"k": (w, u, a2, v), "v": (w, u, k, a2), "w": (a2, u, k, v), "u": (w, a2, k, v)}[name]
            fd = (loss(*args1) - loss(*args2)) / (2 * h)
            if abs(fd - np.asarray(grad)[idx]) > tol:
                out.append(f"gradient vs central difference d{name}{idx}: {np.asarray(grad)[idx]} vs {fd}")
    return out


def grad_identities(fn, tol=1e-11):
    """T = 1: y = v, so gv = gy and the rest vanish.  For any input: the
    outputs are invariant to shifting k, so sum_j gk_j = 0 per row and
    channel; a weighted mean reproduces constants, so sum_j gv_j =
    sum_t gy_t; and the decay's gradient is the keys' first moment less the
    bonus's, gw = sum_j j gk_j - gu."""
    out = []
    rng = np.random.default_rng(53)
    w, u, k, v = _rand_wkv(53, B=2, T=1, C=4)
    gy = rng.normal(0, 1, k.shape)
    gk, gv, gw, gu = fn(w, u, k, v, gy)
    msg = (_close(gv, gy, tol) or _close(gk, np.zeros_like(gk), tol) or
           _close(gw, np.zeros(4), tol) or _close(gu, np.zeros(4), tol))
    if msg: out.append(f"gradient at T = 1: {msg}")
    w, u, k, v = _rand_wkv(54, B=2, T=30, C=4)
    gy = rng.normal(0, 1, k.shape)
    gk, gv, gw, gu = fn(w, u, k, v, gy)
    msg = _close(np.asarray(gk).sum(axis=1), np.zeros((2, 4)), tol * 30)
    if msg: out.append(f"gradient k-shift identity: {msg}")
    msg = _close(np.asarray(gv).sum(axis=1), gy.sum(axis=1), tol * 30)
    if msg: out.append(f"gradient constant identity: {msg}")
    # w enters the logits of output t as j w - (t-1) w for j < t and not at
    # all in the diagonal u + k_t.  A softmax ignores a constant added to a
    # whole row, so moving the row's -(t-1) w onto every logit of the row
    # leaves the weight j on l_{t,j} (j < t) and t - 1 on l_{t,t}; k_j enters
    # l_{t,j} with weight 1 and u the diagonal only, hence
    # gw = sum_j j gk_j - gu (summed over rows; j counted from 0).
    j = np.arange(k.shape[1])[None, :, None]
    moment = (j * np.asarray(gk)).sum(axis=(0, 1)) - np.asarray(gu)
    msg = _close(moment, np.asarray(gw), tol * 30 * max(1.0, float(np.abs(gw).max())))
    if msg: out.append(f"gradient w-shift identity: {msg}")
    return out


GRAD_PINS = [grad_worked_example, grad_autodiff, grad_finite_difference, grad_identities]


def run_grad_pins(fn):
    fails = []
    for pin in GRAD_PINS:
        try:
            fails += pin(fn)
        except Exception as e:
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails


# ---------------------------------------------------------------------------
# diagonal scan pins
# ---------------------------------------------------------------------------
def scan_worked_example(fn, tol=1e-12):
    g = read_golden("scan_worked_example.txt")
    a = np.array([float(x) for x in g["a"]])[None, :, None]
    b = np.array([float(x) for x in g["b"]])[None, :, None]
    h0 = np.array([[float(g["h0"][0])]])
    want = np.array([float(x) for x in g["h"]])[None, :, None]
    msg = _close(fn(a, b, h0), want, tol)
    return [f"worked example: {msg}"] if msg else []


def scan_closed_forms(fn, tol=1e-10, exact_tol=0.0):
    out = []
    rng = np.random.default_rng(11)
    B, T, D = 2, 50, 3
    b = rng.normal(0, 1, (B, T, D))
    h0 = rng.normal(0, 1, (B, D))
    # a = 1: cumulative sum on top of h0
    msg = _close(fn(np.ones((B, T, D)), b, h0), h0[:, None, :] + np.cumsum(b, axis=1), tol)
    if msg: out.append(f"a=1 cumsum: {msg}")
    # a = 0: h = b
    msg = _close(fn(np.zeros((B, T, D)), b, h0), b, exact_tol)
    if msg: out.append(f"a=0: {msg}")
    # b = 0: h_t = h0 * prod_{j<=t} a_j
    a = rng.uniform(0.5, 1.2, (B, T, D))
    msg = _close(fn(a, np.zeros((B, T, D)), h0), h0[:, None, :] * np.cumprod(a, axis=1), tol)
    if msg: out.append(f"b=0 cumprod: {msg}")
    # constant a = lam, constant b = beta, h0 = 0: beta (1 - lam^{t+1}) / (1 - lam)
    lam, beta = 0.8, 1.25
    t = np.arange(T)
    want = np.broadcast_to((beta * (1 - lam ** (t + 1)) / (1 - lam))[None, :, None], (B, T, D))
    msg = _close(fn(np.full((B, T, D), lam), np.full((B, T, D), beta), None), want, tol)
    if msg: out.append(f"geometric series: {msg}")
    # no h0 equals h0 = 0
    msg = _close(fn(a, b, None), fn(a, b, np.zeros((B, D))), 0.0)
    if msg: out.append(f"h0=None vs zeros: {msg}")
    return out


def scan_chaining(fn, tol=1e-12):
    rng = np.random.default_rng(12)
    B, T, D, T1 = 2, 40, 3, 17
    a = rng.uniform(0.3, 1.0, (B, T, D)); b = rng.normal(0, 1, (B, T, D))
    h0 = rng.normal(0, 1, (B, D))
    full = np.asarray(fn(a, b, h0))
    first = np.asarray(fn(a[:, :T1], b[:, :T1], h0))
    second = np.asarray(fn(a[:, T1:], b[:, T1:], first[:, -1, :]))
    msg = _close(np.concatenate([first, second], axis=1), full, tol)
    return [f"chaining: {msg}"] if msg else []


def scan_mingru_convex(fn, tol=1e-12):
    """minGRU form a = 1 - z, b = z h~ with z in (0, 1): each h_t is a convex
    combination of h0 and h~_0..h~_t."""
    rng = np.random.default_rng(13)
    B, T, D = 2, 64, 4
    z = 1 / (1 + np.exp(-rng.normal(0, 1, (B, T, D))))
    ht = rng.normal(0, 1, (B, T, D))
    h0 = rng.normal(0, 1, (B, D))
    h = np.asarray(fn(1 - z, z * ht, h0))
    lo = np.minimum(np.minimum.accumulate(ht, axis=1), h0[:, None, :])
    hi = np.maximum(np.maximum.accumulate(ht, axis=1), h0[:, None, :])
    if np.any(h < lo - tol) or np.any(h > hi + tol):
        return ["minGRU convex bound violated"]
    return []


def scan_linearity(fn, tol=1e-11):
    rng = np.random.default_rng(14)
    B, T, D = 1, 30, 3
    a = rng.uniform(0.2, 1.1, (B, T, D))
    b1, b2 = rng.normal(0, 1, (2, B, T, D))
    msg = _close(fn(a, 2 * b1 - 3 * b2, None), 2 * np.asarray(fn(a, b1, None)) - 3 * np.asarray(fn(a, b2, None)), tol)
    return [f"linearity in b: {msg}"] if msg else []


SCAN_PINS = [scan_worked_example, scan_closed_forms, scan_chaining, scan_mingru_convex, scan_linearity]


def run_scan_pins(fn):
    fails = []
    for pin in SCAN_PINS:
        try:
            fails += pin(fn)
        except Exception as e:
            fails.append(f"{pin.__name__} raised {type(e).__name__}: {e}")
    return fails
