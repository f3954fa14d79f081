"""Pins of the gradient oracles (oracle.mingru_backward, oracle.minmax_backward)
to things other than the oracle itself.

The pages show both models as trainable PyTorch modules (page "Mingru
Pytorch"; page "MinMax Recurrent Neural Cascades", Key properties: bounded
gradients) but print no derivative, so the gradient is that of the
sequential recurrence.  Pins:

- torch.autograd in float64 differentiating a plain torch loop of the
  forward recurrence (a derivative computed by a library, not retyped);
- central finite differences of the forward oracle (pinned on its own in
  test_oracle_pins.py) on tiny inputs;
- closed forms: one step (T = 1); a one-hot upstream gradient at the last
  step gives dh0 = product of the gates 1 - z_t;
- conservation identities of the two models: minGRU's h_t is a convex
  combination of h0 and the candidates g(hx_s), so with every hx >= 0
  (g' = 1) sum_t gy_t = dh0 + sum_t dhx_t; MinMax's output is a selection
  whose weights (ties split evenly) sum to 1, so sum_t gy_t = dx0 + sum dr + sum ds;
- MinMax ties on small value sets, where autograd's rule for equal operands
  of minimum/maximum decides.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_mingru(k, hx, h0):
    prev = h0 if h0 is not None else torch.zeros_like(k[:, 0])
    outs = []
    for t in range(k.shape[1]):
        z = torch.sigmoid(k[:, t])
        g = torch.where(hx[:, t] >= 0, hx[:, t] + 0.5, torch.sigmoid(hx[:, t]))
        prev = (1 - z) * prev + z * g
        outs.append(prev)
    return torch.stack(outs, 1)


def _torch_minmax(r, s, x0):
    prev = x0 if x0 is not None else torch.zeros_like(r[:, 0])
    outs = []
    for t in range(r.shape[1]):
        prev = torch.maximum(torch.minimum(r[:, t], prev), s[:, t])
        outs.append(prev)
    return torch.stack(outs, 1)


def _autograd(fn, p, q, init, gy):
    P = torch.tensor(p, requires_grad=True)
    Q = torch.tensor(q, requires_grad=True)
    I = torch.tensor(init if init is not None else np.zeros((p.shape[0], p.shape[2])), requires_grad=True)
    y = fn(P, Q, I)
    (y * torch.tensor(gy)).sum().backward()
    return P.grad.numpy(), Q.grad.numpy(), I.grad.numpy()


@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 7, 3), (3, 40, 5)])
@pytest.mark.parametrize("with_h0", [False, True])
@pytest.mark.parametrize("k_mean", [0.0, 3.0, -3.0])
def test_mingru_backward_matches_autograd(shape, with_h0, k_mean):
    rng = np.random.default_rng(sum(shape) + int(with_h0) + int(k_mean * 10) + 100)
    k = rng.normal(k_mean, 2.0, size=shape)
    hx = rng.normal(0.0, 2.0, size=shape)
    gy = rng.normal(size=shape)
    h0 = rng.uniform(-1.0, 1.0, size=(shape[0], shape[2])) if with_h0 else None
    dk, dhx, dh0 = oracle.mingru_backward(k, hx, h0, gy)
    ak, ahx, ah0 = _autograd(_torch_mingru, k, hx, h0, gy)
    for got, want in ((dk, ak), (dhx, ahx), (dh0, ah0)):
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("with_h0", [False, True])
def test_mingru_backward_finite_differences(with_h0):
    rng = np.random.default_rng(5)
    B, T, D = 2, 6, 2
    k = rng.normal(size=(B, T, D))
    hx = rng.normal(size=(B, T, D))
    hx[np.abs(hx) < 1e-3] = 0.5           # keep away from g's kink at 0
    h0 = rng.uniform(0.1, 1.0, size=(B, D)) if with_h0 else None
    gy = rng.normal(size=(B, T, D))
    dk, dhx, dh0 = oracle.mingru_backward(k, hx, h0, gy)
    loss = lambda k_, hx_, h0_: float((oracle.mingru_linear(k_, hx_, h0_) * gy).sum())
    eps = 1e-6
    for arr, grad in ((k, dk), (hx, dhx)):
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = (plus, hx, h0) if arr is k else (k, plus, h0)
            args_m = (minus, hx, h0) if arr is k else (k, minus, h0)
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (idx, fd, grad[idx])
    base = h0 if with_h0 else np.zeros((B, D))
    for idx in np.ndindex(base.shape):
        plus, minus = base.copy(), base.copy()
        plus[idx] += eps
        minus[idx] -= eps
        fd = (loss(k, hx, plus) - loss(k, hx, minus)) / (2 * eps)
        assert abs(fd - dh0[idx]) <= 1e-7 * max(1.0, abs(fd))


def test_mingru_backward_one_step_closed_form():
    rng = np.random.default_rng(6)
    B, D = 3, 8
    k = rng.normal(size=(B, 1, D)) * 3
    hx = rng.normal(size=(B, 1, D)) * 3
    h0 = rng.uniform(0.1, 1.0, size=(B, D))
    gy = rng.normal(size=(B, 1, D))
    dk, dhx, dh0 = oracle.mingru_backward(k, hx, h0, gy)
    z = 1.0 / (1.0 + np.exp(-k[:, 0]))
    x = hx[:, 0]
    g = np.where(x >= 0, x + 0.5, 1.0 / (1.0 + np.exp(-x)))
    gp = np.where(x >= 0, 1.0, np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))) ** 2)
    np.testing.assert_allclose(dk[:, 0], gy[:, 0] * z * (1 - z) * (g - h0), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dhx[:, 0], gy[:, 0] * z * gp, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dh0, gy[:, 0] * (1 - z), rtol=1e-12)


def test_mingru_backward_state_gradient_is_product_of_gates():
    rng = np.random.default_rng(7)
    B, T, D = 2, 30, 4
    k = rng.normal(1.0, 1.0, size=(B, T, D))
    hx = rng.normal(size=(B, T, D))
    gy = np.zeros((B, T, D))
    gy[:, -1] = 1.0                                   # L = h_T
    _, _, dh0 = oracle.mingru_backward(k, hx, rng.uniform(0.1, 1, (B, D)), gy)
    one_minus_z = 1.0 / (1.0 + np.exp(k))
    np.testing.assert_allclose(dh0, one_minus_z.prod(axis=1), rtol=1e-12)


def test_mingru_backward_convex_combination_conserves_gradient():
    rng = np.random.default_rng(8)
    B, T, D = 3, 50, 6
    k = rng.normal(size=(B, T, D))
    hx = np.abs(rng.normal(size=(B, T, D)))          # g' = 1 everywhere
    gy = rng.normal(size=(B, T, D))
    _, dhx, dh0 = oracle.mingru_backward(k, hx, rng.uniform(0.1, 1, (B, D)), gy)
    np.testing.assert_allclose(gy.sum(axis=1), dh0 + dhx.sum(axis=1), rtol=1e-11, atol=1e-11)


def test_mingru_backward_saturated_gates():
    # z = 1 (k = +inf): h_t = g(hx_t) does not depend on k or on earlier states
    B, T, D = 1, 5, 3
    rng = np.random.default_rng(9)
    hx = rng.normal(size=(B, T, D))
    gy = rng.normal(size=(B, T, D))
    dk, dhx, dh0 = oracle.mingru_backward(np.full((B, T, D), np.inf), hx, np.ones((B, D)), gy)
    gp = np.where(hx >= 0, 1.0, np.exp(-np.abs(hx)) / (1.0 + np.exp(-np.abs(hx))) ** 2)
    assert np.all(dk == 0) and np.all(dh0 == 0)
    np.testing.assert_allclose(dhx, gy * gp, rtol=1e-13)
    # z = 0 (k = -inf): h_t = h0; the whole gradient reaches h0
    dk, dhx, dh0 = oracle.mingru_backward(np.full((B, T, D), -np.inf), hx, np.ones((B, D)), gy)
    assert np.all(dk == 0) and np.all(dhx == 0)
    np.testing.assert_allclose(dh0, gy.sum(axis=1), rtol=1e-13)


VALUES = [-1.0, 0.0, 1.0, 2.0]


@pytest.mark.parametrize("seed", range(6))
def test_minmax_backward_matches_autograd_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    B, T, D = 3, 9, 4
    r = rng.choice(VALUES, size=(B, T, D))
    s = rng.choice(VALUES, size=(B, T, D))
    x0 = rng.choice(VALUES, size=(B, D))
    gy = rng.normal(size=(B, T, D))
    got = oracle.minmax_backward(r, s, x0, gy)
    want = _autograd(_torch_minmax, r, s, x0, gy)
    for g_, w_ in zip(got, want):
        np.testing.assert_allclose(g_, w_, rtol=1e-13, atol=1e-15)


def test_minmax_backward_default_state_is_zero():
    rng = np.random.default_rng(11)
    B, T, D = 2, 6, 3
    r, s, gy = (rng.choice(VALUES, size=(B, T, D)) for _ in range(3))
    a = oracle.minmax_backward(r, s, None, gy)
    b = oracle.minmax_backward(r, s, np.zeros((B, D)), gy)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_minmax_backward_finite_differences_away_from_ties():
    # continuous random values: no ties, the map is linear near the point
    rng = np.random.default_rng(12)
    B, T, D = 2, 8, 3
    r = rng.normal(size=(B, T, D))
    s = rng.normal(size=(B, T, D))
    x0 = rng.normal(size=(B, D))
    gy = rng.normal(size=(B, T, D))
    dr, ds, dx0 = oracle.minmax_backward(r, s, x0, gy)
    loss = lambda r_, s_, x_: float((oracle.minmax(r_, s_, x_) * gy).sum())
    eps = 1e-9
    for arr, grad, which in ((r, dr, 0), (s, ds, 1)):
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += eps
            m[idx] -= eps
            args = [[r, s, x0], [r, s, x0]]
            args[0][which], args[1][which] = p, m
            fd = (loss(*args[0]) - loss(*args[1])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-5 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])
    for idx in np.ndindex(x0.shape):
        p, m = x0.copy(), x0.copy()
        p[idx] += eps
        m[idx] -= eps
        fd = (loss(r, s, p) - loss(r, s, m)) / (2 * eps)
        assert abs(fd - dx0[idx]) <= 1e-5 * max(1.0, abs(fd))


@pytest.mark.parametrize("seed", range(4))
def test_minmax_backward_conserves_gradient(seed):
    rng = np.random.default_rng(200 + seed)
    B, T, D = 2, 30, 5
    r = rng.choice(VALUES, size=(B, T, D))
    s = rng.choice(VALUES, size=(B, T, D))
    x0 = rng.choice(VALUES, size=(B, D))
    gy = rng.integers(-8, 9, size=(B, T, D)).astype(np.float64)   # dyadic: exact sums
    dr, ds, dx0 = oracle.minmax_backward(r, s, x0, gy)
    np.testing.assert_array_equal(gy.sum(axis=1), dx0 + dr.sum(axis=1) + ds.sum(axis=1))


def test_minmax_backward_gradient_weights_are_bounded():
    # every coefficient is in [0, 1]: |gradient| <= sum of |gy| over the steps it can reach
    rng = np.random.default_rng(13)
    B, T, D = 2, 40, 4
    r, s = rng.normal(size=(B, T, D)), rng.normal(size=(B, T, D))
    gy = rng.normal(size=(B, T, D))
    dr, ds, dx0 = oracle.minmax_backward(r, s, None, gy)
    bound = np.flip(np.cumsum(np.flip(np.abs(gy), 1), 1), 1)   # sum_{u >= t} |gy_u|
    assert np.all(np.abs(dr) <= bound + 1e-12) and np.all(np.abs(ds) <= bound + 1e-12)
    assert np.all(np.abs(dx0) <= bound[:, 0] + 1e-12)
