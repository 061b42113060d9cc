"""The CPU oracle against what the pages and the mathematics fix.

Every oracle function must pass every pin in ``pins.py`` (hand-worked
examples in exact rationals, closed forms, invariants), the independent
formulations must agree with each other, and a set of planted mistakes --
the plausible errors an implementation of eq. (14) could make -- must each
trip at least one pin.
"""
import os
import shutil
import subprocess
import ctypes

import numpy as np
import pytest

import oracle
import workloads
import pins


# --- wrappers with the common pin signature -------------------------------
def c_direct(w, u, k, v):
    return oracle.wkv_direct(w, u, k, v)


def c_rnn(w, u, k, v):
    return oracle.wkv_rnn(w, u, k, v)


def c_points(w, u, k, v):
    k = np.asarray(k)
    return oracle.wkv_direct_points(w, u, k, v, np.arange(k.size)).reshape(k.shape)


def np_direct(w, u, k, v):
    return oracle.wkv_direct_np(w, u, k, v)


def slru_ratio(w, u, k, v):
    return oracle.wkv_slru_ratio_np(w, u, k, v)


@pytest.mark.parametrize("fn", [c_direct, c_rnn, c_points, np_direct],
                         ids=["c_direct", "c_rnn", "c_points", "np_direct"])
def test_wkv_oracle_passes_pins(fn):
    assert pins.run_wkv_pins(fn) == []


def test_slru_ratio_form_passes_pins_in_range():
    # The unstabilised two-SLRU form overflows for |u|, w or |k| of tens;
    # check it on the pins whose inputs stay in range.
    # (its T = 1 output is (Y + (gam lam - 1) e^k v) / (Z + ...), exact only up
    # to rounding, hence the small tolerance there)
    for pin in (pins.wkv_worked_example, pins.wkv_exact_rational,
                lambda fn: pins.wkv_single_step(fn, tol=1e-12),
                pins.wkv_running_mean, pins.wkv_geometric, pins.wkv_invariants):
        assert pin(slru_ratio) == [], getattr(pin, "__name__", "single_step")


@pytest.mark.parametrize("seed,B,T,C,ksig", [(0, 2, 64, 7, 1.0), (1, 1, 200, 3, 2.0),
                                             (2, 3, 33, 5, 0.3)])
def test_wkv_formulations_agree(seed, B, T, C, ksig):
    """Definition (C and numpy), RNN mode and the two-SLRU ratio from a
    different page all give the same numbers."""
    rng = np.random.default_rng(seed)
    k = rng.normal(0, ksig, (B, T, C)); v = rng.normal(0, 1, (B, T, C))
    w = np.exp(rng.uniform(-3, 1, C)); u = rng.normal(0, 0.5, C)
    ref = oracle.wkv_direct_np(w, u, k, v)
    for got in (oracle.wkv_direct(w, u, k, v), oracle.wkv_rnn(w, u, k, v),
                oracle.wkv_slru_ratio_np(w, u, k, v)):
        assert np.max(np.abs(got - ref)) < 1e-12


def test_wkv_stabilised_under_large_keys():
    """k ~ N(0, 30): e^{k} alone overflows float64 sums of the raw form; the
    direct and RNN forms keep every exponent <= 0 and agree."""
    rng = np.random.default_rng(9)
    B, T, C = 1, 300, 4
    k = rng.normal(0, 30, (B, T, C)); v = rng.normal(0, 1, (B, T, C))
    k[0, 100, :] = 800.0   # e^{800} is inf in float64
    w = np.array([0.0, 1e-3, 1.0, 50.0]); u = np.array([0.0, -3.0, 2.0, 700.0])
    d = oracle.wkv_direct(w, u, k, v)
    r = oracle.wkv_rnn(w, u, k, v)
    assert np.all(np.isfinite(d)) and np.all(np.isfinite(r))
    assert np.max(np.abs(d - r)) < 1e-12


def test_wkv_points_match_full():
    x = workloads.make_wkv("wkv_tiny")
    full = oracle.wkv_direct(x.w, x.u, x.k, x.v)
    pts = np.random.default_rng(0).choice(x.k.size, 300, replace=False)
    got = oracle.wkv_direct_points(x.w, x.u, x.k, x.v, pts)
    assert np.array_equal(got, full.reshape(-1)[pts])


def test_wkv_tiny_workload_direct_vs_rnn():
    x = workloads.make_wkv("wkv_tiny")
    d = oracle.wkv_direct_np(x.w, x.u, x.k, x.v)
    r = oracle.wkv_rnn(x.w, x.u, x.k, x.v)
    assert np.max(np.abs(d - r)) < 1e-12
    assert np.array_equal(r[:, 0, :], x.v[:, 0, :].astype(np.float64))


def test_eq10_offset_is_eq14_with_shifted_bonus():
    """Eq. (10) of the RWKV page decays by (t-i) w while eq. (14) uses
    (t-1-i) w; the two differ only by a constant factor e^{-w} on every past
    token, i.e. eq. (10) with bonus u equals eq. (14) with bonus u + w."""
    rng = np.random.default_rng(10)
    B, T, C = 1, 40, 3
    k = rng.normal(0, 1, (B, T, C)); v = rng.normal(0, 1, (B, T, C))
    w = np.exp(rng.normal(0, 1, C)); u = rng.normal(0, 1, C)
    eq10 = np.empty((B, T, C))
    for t in range(T):
        i = np.arange(t)
        lg = np.concatenate([-(t - i)[:, None] * w[None] + k[0, :t], (u + k[0, t])[None]], 0)
        e = np.exp(lg - lg.max(0))
        eq10[0, t] = (e * v[0, :t + 1]).sum(0) / e.sum(0)
    assert np.max(np.abs(eq10 - oracle.wkv_direct(w, u + w, k, v))) < 1e-12


# --- planted mistakes in a numpy copy of the definition -------------------
def _direct_variant(kind):
    def fn(w, u, k, v):
        k = np.asarray(k, float); v = np.asarray(v, float)
        w = np.asarray(w, float).reshape(-1); u = np.asarray(u, float).reshape(-1)
        if kind == "swap_kv":
            k, v = v, k
        B, T, C = k.shape
        y = np.empty((B, T, C))
        for t in range(T):
            i = np.arange(t + 1 if kind == "future_token" and t + 1 < T else t)
            off = {"eq10_offset": t - i, "sign_w": -(t - 1 - i)}.get(kind, t - 1 - i)
            past = -off[:, None] * w[None] + k[:, i]
            cur = (k[:, t] if kind == "no_bonus" else u + k[:, t])[:, None]
            if kind == "future_token" and t + 1 < T:
                past = past.copy(); past[:, -1] = k[:, t + 1]   # leaks v_{t+1}
            lg = np.concatenate([past, cur], 1)
            vals = np.concatenate([v[:, i], v[:, t][:, None]], 1)
            e = np.exp(lg - lg.max(1, keepdims=True))
            num = (e * vals).sum(1)
            den = e[:, :-1].sum(1) if kind == "drop_current_den" else e.sum(1)
            if kind == "drop_current_den":
                den = den + (t == 0)
            y[:, t] = num / den
        return y
    return fn


@pytest.mark.parametrize("kind", ["eq10_offset", "sign_w", "no_bonus", "swap_kv",
                                  "future_token", "drop_current_den"])
def test_planted_mistake_in_definition_is_caught(kind):
    assert _direct_variant("none")(np.ones(2), np.zeros(2), np.zeros((1, 3, 2)),
                                   np.ones((1, 3, 2))).shape == (1, 3, 2)
    assert pins.run_wkv_pins(_direct_variant("none")) == []
    assert pins.run_wkv_pins(_direct_variant(kind)) != []


# --- planted mistakes in a copy of the C oracle ---------------------------
C_MUTANTS = {
    "decay_sign": ("double pd = p - wc;", "double pd = p + wc;"),
    "bonus_dropped": ("double x = uc + kt;", "double x = kt;"),
    # past decayed once more at output time: the (t-i) offset of eq. (10)
    "extra_decay_at_output": ("double ep = exp(p - q), ex = exp(x - q);",
                              "double ep = exp(p - wc - q), ex = exp(x - q);"),
    "state_new_weight": ("double f_old = exp(pd - q2), f_new = exp(kt - q2);",
                         "double f_old = exp(pd - q2), f_new = exp(kt - q2 + uc);"),
    "den_uses_v": ("d = f_old * d + f_new;", "d = f_old * d + f_new * vt;"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(C_MUTANTS))
def test_planted_mistake_in_c_oracle_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "wkv_oracle.c")).read()
    old, new = C_MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    mpath = tmp_path / "mut.c"
    mpath.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                           str(mpath), "-lm"])
    lib = ctypes.CDLL(str(so))
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_wkv_rnn.argtypes = [i64, i64, i64, p, p, p, p, p, ctypes.c_int]
    lib.oracle_wkv_rnn.restype = None

    def mut(w, u, k, v):
        k = np.ascontiguousarray(k, float); v = np.ascontiguousarray(v, float)
        w = np.ascontiguousarray(w, float).reshape(-1); u = np.ascontiguousarray(u, float).reshape(-1)
        y = np.empty(k.shape)
        B, T, C = k.shape
        lib.oracle_wkv_rnn(B, T, C, *(x.ctypes.data_as(p) for x in (w, u, k, v, y)), 1)
        return y

    assert pins.run_wkv_pins(mut) != []


# --- WKV with a state in and out -------------------------------------------
def st_direct(w, u, k, v, s):
    return oracle.wkv_direct_state(w, u, k, v, s)


def st_rnn(w, u, k, v, s):
    return oracle.wkv_rnn_state(w, u, k, v, s)


def st_points(w, u, k, v, s):
    k = np.asarray(k)
    y = oracle.wkv_direct_points(w, u, k, v, np.arange(k.size), s_in=s).reshape(k.shape)
    return y, oracle.wkv_direct_state(w, u, k, v, s)[1]


@pytest.mark.parametrize("fn", [st_direct, st_rnn, st_points], ids=["direct", "rnn", "points"])
def test_wkv_state_oracle_passes_pins(fn):
    assert pins.run_wkv_state_pins(fn) == []


def test_wkv_state_forms_agree_on_random_states():
    rng = np.random.default_rng(21)
    B, T, C = 3, 70, 6
    w, u, k, v = (np.exp(rng.uniform(-3, 1, C)), rng.normal(0, 0.5, C),
                  rng.normal(0, 2, (B, T, C)), rng.normal(0, 1, (B, T, C)))
    s_in = np.stack([rng.normal(0, 1, (B, C)), np.exp(rng.normal(0, 1, (B, C))),
                     rng.normal(0, 3, (B, C))], axis=1)
    y1, s1 = oracle.wkv_direct_state(w, u, k, v, s_in)
    y2, s2 = oracle.wkv_rnn_state(w, u, k, v, s_in)
    assert np.max(np.abs(y1 - y2)) < 1e-13
    for x1, x2 in zip(oracle.state_mean_logden(s1), oracle.state_mean_logden(s2)):
        assert np.max(np.abs(x1 - x2)) < 1e-12


C_STATE_MUTANTS = {
    # (anchor, replacement, C function the mutant is called through)
    "state_not_decayed": ("double ls = has_s ? -(double)t * w + s[2 * C] : -INFINITY;",
                          "double ls = has_s ? s[2 * C] : -INFINITY;", "direct"),
    "state_decayed_once_more": ("double ls = has_s ? -(double)t * w + s[2 * C] : -INFINITY;",
                                "double ls = has_s ? -(double)(t + 1) * w + s[2 * C] : -INFINITY;",
                                "direct"),
    "state_b_weights_num": ("n += e * s[0];", "n += e * s[C];", "direct"),
    "state_out_one_step_short": ("past_sums(C, w[c], kb, vb, sb, T, -INFINITY, &m, &num, &den);",
                                 "past_sums(C, w[c], kb, vb, sb, T - 1, -INFINITY, &m, &num, &den);",
                                 "direct"),
    "rnn_state_planes_swapped": ("a = sb[0];\n            d = sb[C];",
                                 "a = sb[C];\n            d = sb[0];", "rnn"),
    "rnn_state_out_decayed": ("so[2 * C] = p;\n        }\n    }\n}\n\nvoid oracle_wkv_rnn(",
                              "so[2 * C] = p - wc;\n        }\n    }\n}\n\nvoid oracle_wkv_rnn(", "rnn"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(C_STATE_MUTANTS))
def test_planted_mistake_in_state_oracle_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "wkv_oracle.c")).read()
    old, new, which = C_STATE_MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    mpath = tmp_path / "mut.c"
    mpath.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                           str(mpath), "-lm"])
    lib = ctypes.CDLL(str(so))
    i64, p = ctypes.c_int64, ctypes.c_void_p
    cfn = getattr(lib, "oracle_wkv_direct_s" if which == "direct" else "oracle_wkv_rnn_s")
    cfn.argtypes = [i64, i64, i64, p, p, p, p, p, p, p, ctypes.c_int]
    cfn.restype = None

    def mut(w, u, k, v, s_in):
        k = np.ascontiguousarray(k, float); v = np.ascontiguousarray(v, float)
        w = np.ascontiguousarray(w, float).reshape(-1); u = np.ascontiguousarray(u, float).reshape(-1)
        B, T, C = k.shape
        sp = None if s_in is None else np.ascontiguousarray(s_in, float)
        y = np.empty(k.shape); s_out = np.empty((B, 3, C))
        cfn(B, T, C, *(x.ctypes.data_as(p) for x in (w, u, k, v)),
            None if sp is None else sp.ctypes.data_as(p), y.ctypes.data_as(p),
            s_out.ctypes.data_as(p), 1)
        return y, s_out

    assert pins.run_wkv_state_pins(mut) != []


# --- token shift and receptance gate ---------------------------------------
def test_token_shift_oracle_passes_pins():
    assert pins.run_token_shift_pins(oracle.token_shift) == []


def _token_shift_variant(kind):
    def fn(x, mu, x_prev):
        x = np.asarray(x, float); mu = np.asarray(mu, float)
        B, T, C = x.shape
        prev = np.zeros((B, 1, C)) if (x_prev is None or kind == "prev_ignored") else \
            np.asarray(x_prev, float).reshape(B, 1, C)
        sh = np.concatenate([prev, x[:, :-1]], axis=1)
        if kind == "shift_two":
            sh = np.concatenate([prev, prev, x[:, :-2]], axis=1)[:, :T]
        outs = []
        for m in mu:
            if kind == "mu_swapped":
                outs.append(m * sh + (1 - m) * x)
            elif kind == "minus_reading":   # eqs. (16)-(17) as printed
                outs.append(m * x - (1 - m) * sh)
            else:
                outs.append(m * x + (1 - m) * sh)
        last = x[:, -2] if kind == "last_off_by_one" else x[:, -1]
        return np.stack(outs), last
    return fn


@pytest.mark.parametrize("kind", ["mu_swapped", "minus_reading", "prev_ignored", "shift_two",
                                  "last_off_by_one"])
def test_planted_mistake_in_token_shift_is_caught(kind):
    assert pins.run_token_shift_pins(_token_shift_variant("none")) == []
    assert pins.run_token_shift_pins(_token_shift_variant(kind)) != []


def _gate(w, u, k, v, r):
    return oracle.wkv_gated(w, u, k, v, r)[0]


def test_gate_oracle_passes_pins():
    assert pins.run_gate_pins(_gate) == []
    assert abs(float(oracle.sigmoid(np.log(3.0))) - 0.75) < 1e-16
    assert float(oracle.sigmoid(-800.0)) == 0.0 and float(oracle.sigmoid(800.0)) == 1.0


@pytest.mark.parametrize("kind", ["tanh", "neg", "ungated", "gate_on_v"])
def test_planted_mistake_in_gate_is_caught(kind):
    def fn(w, u, k, v, r):
        y = oracle.wkv_rnn(w, u, k, v)
        r = np.asarray(r, float)
        if kind == "tanh":
            return np.tanh(r) * y
        if kind == "neg":
            return oracle.sigmoid(-r) * y
        if kind == "ungated":
            return y
        return oracle.wkv_rnn(w, u, k, oracle.sigmoid(r) * np.asarray(v))
    assert pins.run_gate_pins(fn) != []


# --- LRU complex scan ----------------------------------------------------
def _lru_points(nu_log, theta_log, gamma, u, x0):
    u = np.asarray(u)
    pts = np.arange(u.size)
    return oracle.lru_direct_points(nu_log, theta_log, gamma, u, x0, pts).reshape(u.shape)


@pytest.mark.parametrize("fn", [oracle.lru_scan, _lru_points], ids=["recurrence", "unrolled"])
def test_lru_oracle_passes_pins(fn):
    assert pins.run_lru_pins(fn, oracle.scan_rnn) == []


@pytest.mark.parametrize("kind", ["conj", "gamma_on_state", "x0_undecayed", "r_squared"])
def test_planted_mistake_in_lru_is_caught(kind):
    def fn(nu_log, theta_log, gamma, u, x0):
        lam = oracle.lru_lambda(nu_log, theta_log)
        if kind == "conj":
            lam = np.conj(lam)
        if kind == "r_squared":
            lam = lam * np.abs(lam)
        u = np.asarray(u).astype(complex)
        B, T, D = u.shape
        g = np.ones(D) if gamma is None else np.asarray(gamma, float)
        x = np.zeros((B, D), complex) if x0 is None else np.asarray(x0, complex).copy()
        out = np.empty((B, T, D), complex)
        for t in range(T):
            if kind == "gamma_on_state":
                x = g * (lam * x + u[:, t])
            elif kind == "x0_undecayed" and t == 0:
                x = x + g * u[:, t]
            else:
                x = lam * x + g * u[:, t]
            out[:, t] = x
        return out
    assert pins.run_lru_pins(fn, oracle.scan_rnn) != []


# --- diagonal scan ---------------------------------------------------------
def scan_rnn(a, b, h0):
    return oracle.scan_rnn(a, b, h0)


def scan_points(a, b, h0):
    a = np.asarray(a)
    return oracle.scan_direct_points(a, b, h0, np.arange(a.size)).reshape(a.shape)


@pytest.mark.parametrize("fn", [scan_rnn, scan_points], ids=["rnn", "points"])
def test_scan_oracle_passes_pins(fn):
    assert pins.run_scan_pins(fn) == []


@pytest.mark.parametrize("name,mut", [
    ("drop_h0", lambda a, b, h0: oracle.scan_rnn(a, b, None)),
    ("shift_a", lambda a, b, h0: oracle.scan_rnn(np.roll(a, 1, axis=1), b, h0)),
    ("swap_ab", lambda a, b, h0: oracle.scan_rnn(b, a, h0)),
    ("exclusive", lambda a, b, h0: np.concatenate(
        [np.broadcast_to(np.zeros(1) if h0 is None else np.asarray(h0)[:, None, :],
                         (np.asarray(a).shape[0], 1, np.asarray(a).shape[2])),
         oracle.scan_rnn(a, b, h0)[:, :-1]], axis=1)),
])
def test_planted_mistake_in_scan_is_caught(name, mut):
    assert pins.run_scan_pins(mut) != []


def test_scan_rnn_vs_points_on_mingru_workload():
    x = workloads.make_scan("scan_mingru", B=2, T=300, D=8, with_h0=True)
    full = oracle.scan_rnn(x.a, x.b, x.h0)
    pts = np.random.default_rng(1).choice(x.a.size, 400, replace=False)
    got = oracle.scan_direct_points(x.a, x.b, x.h0, pts)
    assert np.max(np.abs(got - full.reshape(-1)[pts])) < 1e-12


def test_scan_variance_formula():
    """Variance of x_t = lam x_{t-1} + u_t for iid zero-mean u (LRU review,
    initialisation section): E x_t^2 = (1 - lam^{2(t+1)}) / (1 - lam^2) E u^2.
    Checked statistically over 40000 independent channels."""
    rng = np.random.default_rng(21)
    B, T, D, lam = 10, 60, 4000, 0.95
    b = rng.normal(0, 1, (B, T, D))
    h = oracle.scan_rnn(np.full((B, T, D), lam), b, None)
    emp = (h ** 2).mean(axis=(0, 2))
    t = np.arange(T)
    want = (1 - lam ** (2 * (t + 1))) / (1 - lam ** 2)
    assert np.max(np.abs(emp / want - 1)) < 0.05


def test_worked_examples_read():
    g = pins.read_golden("wkv_worked_example.txt")
    assert len(g["y"]) == len(g["v"]) == 4
    g = pins.read_golden("scan_worked_example.txt")
    assert len(g["h"]) == len(g["a"]) == 4


def test_minlstm_workload_is_a_convex_scan():
    """minLSTM's normalised gates sum to one (f' + i' = 1), so each state is a
    convex combination of the previous one and the candidate: the scan stays
    within the running range of the candidates (h0 = 0 included)."""
    x = workloads.make_scan("scan_minlstm", B=3, T=200, D=8)
    f_prime = x.a.astype(np.float64)
    i_prime = x.b.astype(np.float64) / x.h_tilde.astype(np.float64)
    assert np.allclose(f_prime + i_prime, 1.0, atol=1e-6)
    h = oracle.scan_rnn(x.a, x.b, None)
    lo = np.minimum(np.minimum.accumulate(x.h_tilde, axis=1), 0.0)
    hi = np.maximum(np.maximum.accumulate(x.h_tilde, axis=1), 0.0)
    assert np.all(h >= lo - 1e-6) and np.all(h <= hi + 1e-6)



# --- WKV gradients ---------------------------------------------------------
@pytest.mark.parametrize("fn", [oracle.wkv_backward_direct, oracle.wkv_backward_rnn],
                         ids=["direct", "rnn"])
def test_wkv_gradient_oracle_passes_pins(fn):
    assert pins.run_grad_pins(fn) == []


def test_wkv_gradient_forms_agree_under_large_keys():
    rng = np.random.default_rng(61)
    B, T, C = 2, 150, 5
    w = np.concatenate([[0.0, 1e-4, 30.0], np.exp(rng.uniform(-3, 2, C - 3))])
    u = rng.normal(0, 2, C)
    k = rng.normal(0, 15, (B, T, C))
    v = rng.normal(0, 1, (B, T, C))
    gy = rng.normal(0, 1, (B, T, C))
    a = oracle.wkv_backward_direct(w, u, k, v, gy)
    b = oracle.wkv_backward_rnn(w, u, k, v, gy)
    for x, y in zip(a, b):
        assert np.all(np.isfinite(y))
        assert np.max(np.abs(x - y)) <= 1e-10 * max(1.0, np.abs(x).max())


C_GRAD_MUTANTS = {
    "R_without_P": ("R = fold * (R + P);", "R = fold * R;"),
    "gw_sign": ("gw_c -= sc * (vj * R - R2);", "gw_c += sc * (vj * R - R2);"),
    "diag_missing_in_gv": ("gvb[j * C] = diag + sc * P;", "gvb[j * C] = sc * P;"),
    "Q_without_y": ("double Qn = fnew * gj * ys[j] + fold * Q;", "double Qn = fnew * gj + fold * Q;"),
    "decay_once_more": ("double r2 = rho + w[c];", "double r2 = rho + 2.0 * w[c];"),
}


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(C_GRAD_MUTANTS))
def test_planted_mistake_in_gradient_oracle_is_caught(name, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "wkv_oracle.c")).read()
    old, new = C_GRAD_MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found"
    mpath = tmp_path / "mut.c"
    mpath.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(so),
                           str(mpath), "-lm"])
    lib = ctypes.CDLL(str(so))
    i64, p = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_wkv_backward_rnn.argtypes = [i64, i64, i64] + [p] * 9 + [ctypes.c_int]
    lib.oracle_wkv_backward_rnn.restype = None

    def mut(w, u, k, v, gy):
        k = np.ascontiguousarray(k, float); v = np.ascontiguousarray(v, float)
        gy = np.ascontiguousarray(gy, float)
        w = np.ascontiguousarray(w, float).reshape(-1); u = np.ascontiguousarray(u, float).reshape(-1)
        B, T, C = k.shape
        gk, gv = np.empty(k.shape), np.empty(k.shape)
        gw, gu = np.empty(C), np.empty(C)
        lib.oracle_wkv_backward_rnn(B, T, C, *(x.ctypes.data_as(p) for x in (w, u, k, v, gy, gk, gv, gw, gu)), 1)
        return gk, gv, gw, gu

    assert pins.run_grad_pins(mut) != []
