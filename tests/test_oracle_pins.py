"""Pins for the CPU oracle: it is checked against what the method and the
mathematics fix, never against itself.

minGRU (page "Mingru Pytorch", Requirements & limits: log-space minGRU):
  - hand-worked sequences with exact dyadic values (tests/golden/);
  - the linear recurrence and the log-space formula, two independent
    statements of the same function, agree to fp64 rounding;
  - closed forms: z = 1 gives h_t = g(hx_t); z = 0 gives h_t = h_0; constant
    inputs give h_t = g + (1 - z)^t (h_0 - g);
  - sigmoid branches against scipy's expit (a library routine);
  - invariants: positivity, the convex-hull bound, splitting T with the
    carried state (the token-by-token mode of the page's second guide).
MinMax (page "MinMax Recurrent Neural Cascades", The model, item 3):
  - a hand-worked trace; brute force over small value sets against the
    unrolled max-min closed form; selection, bound, monotonicity and hold.
"""
import itertools
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _tok(s: str) -> float:
    s = s.strip()
    table = {"ln3": math.log(3.0), "-ln3": -math.log(3.0), "inf": math.inf, "-inf": -math.inf}
    return table[s] if s in table else float(s)


def _read_fixture(name):
    init = None
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in ("h0", "x0"):
                init = None if parts[1] == "none" else float(parts[1])
                continue
            rows.append([_tok(p) for p in parts])
    a = np.array(rows, dtype=np.float64)
    return init, a[:, 0], a[:, 1], a[:, 2]


def _seq(x):
    return np.asarray(x, dtype=np.float64).reshape(1, -1, 1)


def _log_tol(k):
    """Error bound of the log-space formula: its running sum a*_t reaches
    |a*_T| = sum softplus(k), and exp() turns that sum's rounding (a few ulp of
    |a*_T|) into relative error of h."""
    k = np.asarray(k, dtype=np.float64)
    sp = np.maximum(k, 0) + np.log1p(np.exp(-np.abs(k)))
    return max(1e-14, 8.0 * float(np.max(np.sum(sp, axis=1))) * 2.0 ** -52)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-300)))


# ---------------------------------------------------------------- golden

@pytest.mark.parametrize("name", ["mingru_worked_example.txt", "mingru_worked_example_noh0.txt"])
def test_mingru_linear_golden(name):
    h0, k, hx, want = _read_fixture(name)
    h0a = None if h0 is None else np.array([[h0]])
    got = oracle.mingru_linear(_seq(k), _seq(hx), h0a).ravel()
    assert _rel(got, want) <= 4e-16, (got, want)


@pytest.mark.parametrize("name", ["mingru_worked_example.txt", "mingru_worked_example_noh0.txt"])
def test_mingru_log_golden(name):
    # the log-space formula needs finite k; +-50 moves sigmoid by < 2e-22
    h0, k, hx, want = _read_fixture(name)
    k = np.where(np.isinf(k), np.sign(k) * 50.0, k)
    h0a = None if h0 is None else np.array([[h0]])
    got = oracle.mingru_log(_seq(k), _seq(hx), h0a).ravel()
    assert _rel(got, want) <= 1e-14, (got, want)


def test_minmax_golden():
    x0, r, s, want = _read_fixture("minmax_worked_example.txt")
    got = oracle.minmax(_seq(r), _seq(s), np.array([[x0]])).ravel()
    assert np.array_equal(got, want), (got, want)


# ------------------------------------------------- two formulations agree

@pytest.mark.parametrize("with_h0", [False, True])
@pytest.mark.parametrize("k_mean", [0.0, 2.0, -2.0])
def test_linear_and_log_space_agree(with_h0, k_mean):
    rng = np.random.default_rng(7)
    B, T, D = 3, 517, 5
    k = rng.standard_normal((B, T, D)) + k_mean
    hx = rng.standard_normal((B, T, D))
    h0 = rng.uniform(0.1, 1.0, (B, D)) if with_h0 else None
    lin = oracle.mingru_linear(k, hx, h0)
    lg = oracle.mingru_log(k, hx, h0)
    # the log-space sum carries |a*_T| ~ T * softplus(k); its rounding sets the gap
    assert _rel(lg, lin) <= 1e-12


def test_linear_and_log_space_agree_long():
    # long sequence with gates near 1 (k ~ N(2, 1)): |a*_T| reaches ~1e4, so the
    # log-space value carries ~1e4 * 2^-53 of absolute log error
    rng = np.random.default_rng(11)
    k = rng.standard_normal((1, 8192, 3)) + 2.0
    hx = rng.standard_normal((1, 8192, 3))
    h0 = rng.uniform(0.1, 1.0, (1, 3))
    assert _rel(oracle.mingru_log(k, hx, h0), oracle.mingru_linear(k, hx, h0)) <= 1e-10


# ----------------------------------------------------------- closed forms

def test_gate_one_gives_candidate():
    # z = 1 (k = +inf): h_t = g(hx_t) whatever the history
    rng = np.random.default_rng(1)
    hx = rng.standard_normal((2, 64, 4)) * 3
    k = np.full_like(hx, np.inf)
    h = oracle.mingru_linear(k, hx, rng.uniform(0.1, 1, (2, 4)))
    pos = hx >= 0
    assert np.array_equal(h[pos], hx[pos] + 0.5)          # g's positive branch, exact
    assert _rel(h[~pos], expit(hx[~pos])) <= 4e-16        # g's negative branch = sigmoid


def test_large_gate_is_near_candidate():
    rng = np.random.default_rng(2)
    hx = rng.standard_normal((1, 32, 8))
    k = np.full_like(hx, 40.0)                       # 1 - z = sigmoid(-40) ~ 4e-18
    h = oracle.mingru_linear(k, hx, np.ones((1, 8)))
    want = np.where(hx >= 0, hx + 0.5, expit(hx))
    assert _rel(h, want) <= 1e-15
    assert _rel(oracle.mingru_log(k, hx, np.ones((1, 8))), want) <= _log_tol(k)


def test_gate_zero_holds_state():
    # z = 0 (k = -inf): h_t = h_0 exactly; without h_0 the state stays 0
    rng = np.random.default_rng(3)
    hx = rng.standard_normal((2, 50, 3))
    k = np.full_like(hx, -np.inf)
    h0 = rng.uniform(0.1, 1, (2, 3))
    h = oracle.mingru_linear(k, hx, h0)
    assert np.array_equal(h, np.broadcast_to(h0[:, None, :], h.shape))
    assert np.array_equal(oracle.mingru_linear(k, hx), np.zeros_like(hx))


def test_small_gate_is_near_state():
    rng = np.random.default_rng(4)
    hx = rng.standard_normal((1, 40, 3))
    k = np.full_like(hx, -40.0)
    h0 = rng.uniform(0.1, 1, (1, 3))
    want = np.broadcast_to(h0[:, None, :], hx.shape)
    assert _rel(oracle.mingru_linear(k, hx, h0), want) <= 1e-15
    assert _rel(oracle.mingru_log(k, hx, h0), want) <= 1e-14


@pytest.mark.parametrize("kc,hc,h0", [(math.log(3.0), 0.5, 0.2), (0.3, -1.7, 0.9), (-1.1, 2.25, 0.5)])
def test_constant_inputs_closed_form(kc, hc, h0):
    # h_t = g + (1 - z)^t (h_0 - g), t = 1..T, from summing the geometric series
    T = 60
    z = expit(kc)
    gv = hc + 0.5 if hc >= 0 else expit(hc)
    t = np.arange(1, T + 1, dtype=np.float64)
    want = gv + (1.0 - z) ** t * (h0 - gv)
    k = np.full((1, T, 1), kc)
    hx = np.full((1, T, 1), hc)
    h0a = np.array([[h0]])
    assert _rel(oracle.mingru_linear(k, hx, h0a).ravel(), want) <= 1e-13
    assert _rel(oracle.mingru_log(k, hx, h0a).ravel(), want) <= 1e-13


def test_sigmoid_branches_match_library():
    # both branches of the stable sigmoid, through g's negative branch and z
    x = np.concatenate([np.linspace(-30, -1e-3, 200), [-700.0, -1e-300]])
    h = oracle.mingru_linear(np.full((1, x.size, 1), np.inf), _seq(x))
    assert _rel(h.ravel(), expit(x)) <= 4e-16
    kk = np.linspace(-30, 30, 301)
    # z = sigmoid(k) read off the first step with h_0 = 0 and g = 1 (hx = 0.5)
    z = oracle.mingru_linear(kk.reshape(1, 1, -1), np.full((1, 1, kk.size), 0.5)).ravel()
    assert _rel(z, expit(kk)) <= 4e-16


# ------------------------------------------------------------- invariants

def test_positive_and_inside_hull():
    rng = np.random.default_rng(5)
    B, T, D = 2, 400, 6
    k = rng.standard_normal((B, T, D)) * 2
    hx = rng.standard_normal((B, T, D)) * 2
    h0 = rng.uniform(0.1, 1, (B, D))
    h = oracle.mingru_linear(k, hx, h0)
    assert np.all(h > 0)
    g = np.where(hx >= 0, hx + 0.5, expit(hx))
    lo = np.minimum(np.minimum.accumulate(g, axis=1), h0[:, None, :])
    hi = np.maximum(np.maximum.accumulate(g, axis=1), h0[:, None, :])
    assert np.all(h >= lo * (1 - 1e-15)) and np.all(h <= hi * (1 + 1e-15))


@pytest.mark.parametrize("cut", [1, 37, 128, 399])
def test_split_with_carried_state(cut):
    rng = np.random.default_rng(6)
    k = rng.standard_normal((2, 400, 3))
    hx = rng.standard_normal((2, 400, 3))
    h0 = rng.uniform(0.1, 1, (2, 3))
    full = oracle.mingru_linear(k, hx, h0)
    a = oracle.mingru_linear(k[:, :cut], hx[:, :cut], h0)
    b = oracle.mingru_linear(k[:, cut:], hx[:, cut:], a[:, -1, :])
    assert np.array_equal(np.concatenate([a, b], axis=1), full)


def test_token_by_token_equals_parallel():
    rng = np.random.default_rng(8)
    k = rng.standard_normal((2, 30, 4))
    hx = rng.standard_normal((2, 30, 4))
    full = oracle.mingru_linear(k, hx)
    h = None
    for t in range(30):
        h = oracle.mingru_step(k[:, t], hx[:, t], h)
        assert np.array_equal(h, full[:, t])


# ------------------------------------------------------------------ MinMax

def _minmax_unrolled(x0, r, s):
    """x_t = max( min(x0, r_0..r_{t-1}),  max_j min(s_j, r_{j+1}..r_{t-1}) ):
    the recurrence unrolled with min distributed over max (a total order)."""
    out = []
    for t in range(1, len(r) + 1):
        best = min([x0] + list(r[:t]))
        for j in range(t):
            best = max(best, min([s[j]] + list(r[j + 1:t])))
        out.append(best)
    return out


@pytest.mark.parametrize("T", [1, 2, 3])
def test_minmax_brute_force(T):
    vals = [-1.0, 0.5, 1.0, 2.0]
    cases = list(itertools.product(vals, repeat=2 * T + 1))
    n = len(cases)
    x0 = np.array([c[0] for c in cases]).reshape(n, 1)
    r = np.array([c[1:1 + T] for c in cases]).reshape(n, T, 1)
    s = np.array([c[1 + T:] for c in cases]).reshape(n, T, 1)
    got = oracle.minmax(r, s, x0)
    for i, c in enumerate(cases):
        want = _minmax_unrolled(c[0], c[1:1 + T], c[1 + T:])
        assert list(got[i, :, 0]) == want, (c, got[i, :, 0], want)


def test_minmax_selection_bound_monotone_hold():
    rng = np.random.default_rng(9)
    B, T, D = 2, 300, 5
    r = rng.standard_normal((B, T, D)).astype(np.float32).astype(np.float64)
    s = rng.standard_normal((B, T, D)).astype(np.float32).astype(np.float64)
    x0 = rng.standard_normal((B, D))
    x = oracle.minmax(r, s, x0)
    for b in range(B):
        for d in range(D):
            seen = {x0[b, d]}
            for t in range(T):
                seen.add(r[b, t, d])
                seen.add(s[b, t, d])
                assert x[b, t, d] in seen                      # selection
    lo = np.minimum(np.minimum(np.minimum.accumulate(r, 1), np.minimum.accumulate(s, 1)),
                    x0[:, None, :])
    hi = np.maximum(np.maximum(np.maximum.accumulate(r, 1), np.maximum.accumulate(s, 1)),
                    x0[:, None, :])
    assert np.all(x >= lo) and np.all(x <= hi)                # bound
    x_up = oracle.minmax(r, s, x0 + 0.25)
    assert np.all(x_up >= x)                                  # monotone in x0
    x_r = oracle.minmax(r + 0.1, s, x0)
    assert np.all(x_r >= x)                                   # monotone in r
    x_s = oracle.minmax(r, s + 0.1, x0)
    assert np.all(x_s >= x)                                   # monotone in s
    prev = np.concatenate([x0[:, None, :], x[:, :-1, :]], axis=1)
    held = (s <= prev) & (prev <= r)
    assert np.array_equal(x[held], prev[held])                # hold ("perfect memory")


def test_minmax_default_state_is_zero():
    rng = np.random.default_rng(10)
    r = rng.standard_normal((1, 20, 3))
    s = rng.standard_normal((1, 20, 3))
    assert np.array_equal(oracle.minmax(r, s), oracle.minmax(r, s, np.zeros((1, 3))))


def test_empty_shapes():
    for B, T, D in [(0, 5, 3), (2, 0, 3), (2, 5, 0)]:
        z = np.zeros((B, T, D))
        assert oracle.mingru_linear(z, z).shape == (B, T, D)
        assert oracle.minmax(z, z).shape == (B, T, D)
