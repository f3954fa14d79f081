"""Pins of the projected-scan oracle (oracle.mingru_projected): the minGRU
layer's input projection followed by the scan (page "Mingru Pytorch": the
layer applied to a (B, T, d) input).  The projection is numpy's fp64 matrix
product; the pins check how the oracle splits and orients the weight and
feeds the scan, against sums written out and weights with known products.
"""
import numpy as np
import pytest

import oracle


def test_identity_blocks_feed_the_input_to_both_gates():
    rng = np.random.default_rng(1)
    B, T, D = 2, 40, 8
    x = rng.normal(size=(B, T, D))
    w = np.concatenate([np.eye(D), 2.0 * np.eye(D)], 0)        # k = x, hx = 2 x
    h0 = rng.uniform(0.1, 1, size=(B, D))
    np.testing.assert_array_equal(oracle.mingru_projected(x, w, h0), oracle.mingru_linear(x, 2.0 * x, h0))


def test_zero_weight_closed_form():
    # k = hx = 0: z = 1/2, g(0) = 1/2, so h_t = h_{t-1} / 2 + 1/4 -> 1/2
    B, T, D, d = 1, 30, 4, 16
    x = np.random.default_rng(2).normal(size=(B, T, d))
    h0 = np.full((B, D), 3.0)
    h = oracle.mingru_projected(x, np.zeros((2 * D, d)), h0)
    t = np.arange(1, T + 1)
    want = 0.5 + (3.0 - 0.5) * 0.5 ** t
    np.testing.assert_allclose(h[0, :, 0], want, rtol=1e-15)


@pytest.mark.parametrize("with_h0", [False, True])
def test_projection_written_out(with_h0):
    rng = np.random.default_rng(3)
    B, T, d, D = 2, 5, 3, 2
    x = rng.normal(size=(B, T, d))
    w = rng.normal(size=(2 * D, d))
    h0 = rng.uniform(0.1, 1, size=(B, D)) if with_h0 else None
    k = np.zeros((B, T, D))
    hx = np.zeros((B, T, D))
    for b in range(B):
        for t in range(T):
            for c in range(D):
                k[b, t, c] = sum(x[b, t, j] * w[c, j] for j in range(d))
                hx[b, t, c] = sum(x[b, t, j] * w[D + c, j] for j in range(d))
    np.testing.assert_allclose(oracle.mingru_projected(x, w, h0), oracle.mingru_linear(k, hx, h0), rtol=1e-13)
