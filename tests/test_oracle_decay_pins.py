"""Pins of the time-decay oracle (oracle.mingru_decay, mingru_decay_backward).

The page "Your first delta model" (Step 5) gives the decay contract: the
carried state is gated once per token at the token boundary, h <- gamma_t h,
before the token's own write; gamma = exp(-lambda * delta_t); delta_t = 0
gives gamma = exp(0) = 1 (no decay); a gap with lambda * delta_t above about
1e4 wipes the state completely; log1p_delta compresses the gaps.  Pins:

- delta_t = 0 (the page's control schedule) and lambda = 0 reduce exactly to
  the plain minGRU oracle (pinned in test_oracle_pins.py);
- a wiping gap before token t* makes the rest of the sequence independent of
  everything before t*: it equals a fresh scan from t* with a zero state;
- constant inputs and gaps give the geometric closed form
  h_t = b (1 - c^t) / (1 - c) + c^t h0 with c = (1 - z) gamma, b = z g;
- log1p_delta is the same as passing log1p(delta_t);
- gradients: fp64 torch.autograd through a plain loop (including lambda),
  and central finite differences in lambda.
"""
import numpy as np
import pytest
import torch

import oracle


def _data(B, T, D, seed, gap_scale=1.0):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(B, T, D))
    hx = rng.normal(size=(B, T, D))
    h0 = rng.uniform(0.1, 1.0, size=(B, D))
    dt = rng.exponential(gap_scale, size=(B, T))
    lam = rng.uniform(0.0, 2.0, size=D)
    return k, hx, h0, dt, lam


@pytest.mark.parametrize("with_h0", [False, True])
def test_zero_gap_and_zero_rate_are_the_plain_recurrence(with_h0):
    k, hx, h0, dt, lam = _data(2, 50, 6, 1)
    h0 = h0 if with_h0 else None
    plain = oracle.mingru_linear(k, hx, h0)
    np.testing.assert_array_equal(oracle.mingru_decay(k, hx, h0, np.zeros_like(dt), lam), plain)
    np.testing.assert_array_equal(oracle.mingru_decay(k, hx, h0, dt, np.zeros_like(lam)), plain)


def test_wiping_gap_restarts_the_sequence():
    k, hx, h0, dt, lam = _data(2, 40, 5, 2)
    lam = np.full_like(lam, 1.0)
    t_star = 17
    dt[:, t_star] = 2e4                                  # lambda * gap > 1e4
    h = oracle.mingru_decay(k, hx, h0, dt, lam)
    fresh = oracle.mingru_decay(k[:, t_star:], hx[:, t_star:], None, dt[:, t_star:], lam)
    # the first token after the gap starts from a zero state
    np.testing.assert_allclose(h[:, t_star:], fresh, rtol=1e-15, atol=0)
    # a long but finite gap leaves a trace of the old state
    dt2 = dt.copy()
    dt2[:, t_star] = 5.0
    h2 = oracle.mingru_decay(k, hx, h0, dt2, lam)
    assert np.all(h2[:, t_star] != fresh[:, 0])


@pytest.mark.parametrize("k_val,hx_val,gap,lam_val,h0_val", [
    (0.3, 0.7, 0.5, 0.4, 0.8), (-1.2, -0.9, 2.0, 0.1, 0.2), (2.0, 1.5, 0.0, 3.0, 1.0)])
def test_constant_inputs_closed_form(k_val, hx_val, gap, lam_val, h0_val):
    B, T, D = 1, 60, 1
    k = np.full((B, T, D), k_val)
    hx = np.full((B, T, D), hx_val)
    dt = np.full((B, T), gap)
    lam = np.array([lam_val])
    h = oracle.mingru_decay(k, hx, np.full((B, D), h0_val), dt, lam)
    z = 1.0 / (1.0 + np.exp(-k_val))
    g = hx_val + 0.5 if hx_val >= 0 else 1.0 / (1.0 + np.exp(-hx_val))
    c = (1 - z) * np.exp(-lam_val * gap)
    b = z * g
    t = np.arange(1, T + 1)
    want = b * (1 - c ** t) / (1 - c) + c ** t * h0_val
    np.testing.assert_allclose(h[0, :, 0], want, rtol=1e-12)


def test_log1p_delta_compresses_the_gaps():
    k, hx, h0, dt, lam = _data(2, 30, 4, 3, gap_scale=100.0)
    a = oracle.mingru_decay(k, hx, h0, dt, lam, log1p_delta=True)
    b = oracle.mingru_decay(k, hx, h0, np.log1p(dt), lam, log1p_delta=False)
    np.testing.assert_array_equal(a, b)


def _torch_decay(k, hx, h0, dt, lam, log1p_delta):
    u = torch.log1p(dt) if log1p_delta else dt
    prev = h0
    outs = []
    for t in range(k.shape[1]):
        x = lam[None, :] * u[:, t:t + 1]
        gamma = torch.where(x > 1e4, torch.zeros_like(x), torch.exp(-x))
        z = torch.sigmoid(k[:, t])
        g = torch.where(hx[:, t] >= 0, hx[:, t] + 0.5, torch.sigmoid(hx[:, t]))
        prev = (1 - z) * gamma * prev + z * g
        outs.append(prev)
    return torch.stack(outs, 1)


@pytest.mark.parametrize("log1p_delta", [False, True])
def test_decay_backward_matches_autograd(log1p_delta):
    k, hx, h0, dt, lam = _data(3, 25, 5, 4)
    dt[0, 7] = 2e4                                       # one clamped gap
    gy = np.random.default_rng(5).normal(size=k.shape)
    dk, dhx, dh0, dlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy, log1p_delta)
    K, H, H0, L = (torch.tensor(a, requires_grad=True) for a in (k, hx, h0, lam))
    y = _torch_decay(K, H, H0, torch.tensor(dt), L, log1p_delta)
    (y * torch.tensor(gy)).sum().backward()
    for got, want in ((dk, K.grad), (dhx, H.grad), (dh0, H0.grad), (dlam, L.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-11, atol=1e-13)


def test_decay_backward_lambda_finite_differences():
    k, hx, h0, dt, lam = _data(2, 12, 3, 6)
    gy = np.random.default_rng(7).normal(size=k.shape)
    _, _, _, dlam = oracle.mingru_decay_backward(k, hx, h0, dt, lam, gy)
    eps = 1e-6
    for d in range(lam.size):
        p, m = lam.copy(), lam.copy()
        p[d] += eps
        m[d] -= eps
        fd = ((oracle.mingru_decay(k, hx, h0, dt, p) - oracle.mingru_decay(k, hx, h0, dt, m)) * gy).sum() / (2 * eps)
        assert abs(fd - dlam[d]) <= 1e-7 * max(1.0, abs(fd))


def test_decay_backward_without_decay_is_the_plain_gradient():
    k, hx, h0, dt, lam = _data(2, 30, 4, 8)
    gy = np.random.default_rng(9).normal(size=k.shape)
    dk, dhx, dh0, _ = oracle.mingru_decay_backward(k, hx, h0, np.zeros_like(dt), lam, gy)
    pk, phx, ph0 = oracle.mingru_backward(k, hx, h0, gy)
    np.testing.assert_array_equal(dk, pk)
    np.testing.assert_array_equal(dhx, phx)
    np.testing.assert_array_equal(dh0, ph0)
