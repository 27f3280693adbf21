"""Pins of the oracle's alpha search (CPU only).

L(alpha) = mean over outputs of (Q(W s)(s^-1 X) - W X)^2, s = s_X^alpha
("MIT 6.5940 Fall 2024 Lecture 13: LLM Deployment" reading guide, §AWQ,
slide 28).  The quantizer the loss uses is pinned elsewhere; these tests pin
the composition: the divided activation, the quantized product and its fp16
rounding, the exact target and the mean.
"""
import math

import numpy as np
import pytest

import oracle

F16 = np.float16


def _brute_loss(W, X, alpha, bits=4, mode=oracle.ASYM):
    """The same loss written out with Python loops over scalars."""
    T, K = X.shape
    N = W.shape[0]
    s = []
    for k in range(K):
        m = sum(abs(float(X[t, k])) for t in range(T)) / T
        s.append(float(F16(m ** alpha)))
    q, sc, z = oracle.quantize_pack(W, np.array(s, dtype=F16), 128, bits, mode)
    w_hat = oracle.dequant(q, sc, z)
    total = 0.0
    for t in range(T):
        xd = [float(F16(float(X[t, k]) / s[k])) for k in range(K)]
        for n in range(N):
            yq = float(F16(math.fsum(xd[k] * w_hat[n, k] for k in range(K))))
            y = math.fsum(float(X[t, k]) * float(W[n, k]) for k in range(K))
            total += (yq - y) ** 2
    return total / (T * N)


@pytest.mark.parametrize("alpha", [0.0, 0.5, 1.0])
def test_loss_matches_brute_force(alpha):
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((3, 128)) * 0.02).astype(F16)
    X = rng.standard_normal((4, 128)).astype(F16)
    X[:, 7] *= 20
    got = oracle.awq_loss(W, X, alpha)
    want = _brute_loss(W, X, alpha)
    assert got == pytest.approx(want, rel=1e-12, abs=0.0)


def test_on_grid_weights_and_integer_activations_lose_nothing_at_alpha_zero():
    """alpha = 0 gives s = 1.  Integer weights spanning -8..7 in every group are
    on the 4-bit grid (Delta = 1, z = 8), and with small integer activations
    every output is an integer that fp16 holds exactly, so L(0) = 0."""
    rng = np.random.default_rng(5)
    W = rng.integers(-8, 8, size=(4, 256)).astype(F16)
    W[:, 0], W[:, 1], W[:, 128], W[:, 129] = -8, 7, -8, 7
    X = rng.integers(-3, 4, size=(5, 256)).astype(F16)
    assert oracle.awq_loss(W, X, 0.0) == 0.0
    assert oracle.awq_loss(W, X, 1.0) > 0.0  # scaling moves the weights off the grid


def test_search_returns_the_grid_minimum():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(F16)
    X = rng.standard_normal((8, 256)).astype(F16)
    X[:, 3] *= 20
    alphas = [0.0, 0.25, 0.5, 0.75, 1.0]
    losses, best = oracle.awq_search(W, X, alphas)
    assert len(losses) == len(alphas)
    assert losses[best] == min(losses)
    assert losses == [oracle.awq_loss(W, X, a) for a in alphas]
