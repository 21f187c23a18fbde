"""Pins for the oracle's QLoRA linear forward and backward (nlp-lineage
'QLoRA', section 'The idea', notation paragraph: Y = X·doubleDequant(...) +
X·L1·L2, only L1 and L2 get weight gradients; examadda 'QLoRA', 'The Flow':
no gradient reaches the 4-bit base).

Independent references: torch.autograd in float64 (a library routine that
differentiates the forward formula by itself), central finite differences,
math.fsum dot products, and closed-form special cases.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O


def _problem(M=5, N=24, K=128, r=8, seed=0, scale_lora=1.0):
    rng = np.random.default_rng(seed)
    X = rng.normal(0, 1, (M, K))
    W = rng.normal(0, 0.02, (N, K))
    L1 = rng.normal(0, 1 / 64, (K, r)) * scale_lora
    L2 = rng.normal(0, 0.1, (r, N)) * scale_lora
    dY = rng.normal(0, 1, (M, N))
    return X, W, L1, L2, dY


def test_forward_backward_match_autograd():
    X, W, L1, L2, dY = _problem(scale_lora=30.0)
    s = 0.75
    Y, T = O.linear_fwd(X, W, L1, L2, s)
    dX, dL1, dL2, dT = O.linear_bwd(dY, X, W, L1, L2, s, T)
    tX = torch.tensor(X, requires_grad=True)
    tW = torch.tensor(W, requires_grad=True)
    tL1 = torch.tensor(L1, requires_grad=True)
    tL2 = torch.tensor(L2, requires_grad=True)
    tY = tX @ tW.T + s * (tX @ tL1) @ tL2
    (tY * torch.tensor(dY)).sum().backward()
    assert np.allclose(Y, tY.detach().numpy(), rtol=1e-13, atol=1e-13)
    assert np.allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL1, tL1.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL2, tL2.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_backward_matches_finite_differences():
    X, W, L1, L2, dY = _problem(M=3, N=8, K=64, r=4, seed=3, scale_lora=10.0)
    s = 1.5
    _, T = O.linear_fwd(X, W, L1, L2, s)
    dX, dL1, dL2, _ = O.linear_bwd(dY, X, W, L1, L2, s, T)

    def loss(X_, L1_, L2_):
        return float(np.sum(O.linear_fwd(X_, W, L1_, L2_, s)[0] * dY))

    h = 1e-6
    for (arr, grad, which) in [(X, dX, 0), (L1, dL1, 1), (L2, dL2, 2)]:
        for idx in [(0, 0), (1, 3), (arr.shape[0] - 1, arr.shape[1] - 1)]:
            a, b = arr.copy(), arr.copy()
            a[idx] += h
            b[idx] -= h
            args_a = [X, L1, L2]
            args_b = [X, L1, L2]
            args_a[which], args_b[which] = a, b
            fd = (loss(*args_a) - loss(*args_b)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd))


def test_zero_weight_gives_pure_lora():
    X, W, L1, L2, _ = _problem()
    Y, T = O.linear_fwd(X, np.zeros_like(W), L1, L2, 2.0)
    assert np.array_equal(Y, 2.0 * ((X @ L1) @ L2))


def test_zero_L2_gives_base_and_no_L1_grad():
    X, W, L1, L2, dY = _problem()
    Y, T = O.linear_fwd(X, W, L1, np.zeros_like(L2), 2.0)
    assert np.array_equal(Y, X @ W.T + 0.0)
    dX, dL1, dL2, _ = O.linear_bwd(dY, X, W, L1, np.zeros_like(L2), 2.0, T)
    assert np.all(dL1 == 0)
    assert np.array_equal(dX, dY @ W)


def test_zero_scale_is_plain_linear():
    X, W, L1, L2, dY = _problem()
    Y, _ = O.linear_fwd(X, W, L1, L2, 0.0)
    assert np.array_equal(Y, X @ W.T)


def test_linearity_in_X():
    X, W, L1, L2, _ = _problem()
    Y1, _ = O.linear_fwd(X, W, L1, L2, 0.5)
    Y2, _ = O.linear_fwd(2 * X, W, L1, L2, 0.5)
    assert np.array_equal(Y2, 2 * Y1)


def test_single_token_against_fsum():
    X, W, L1, L2, dY = _problem(M=1, N=6, K=64, r=4)
    s = 0.25
    Y, T = O.linear_fwd(X, W, L1, L2, s)
    for j in range(6):
        t = [math.fsum(X[0, k] * L1[k, i] for k in range(64)) for i in range(4)]
        ref = math.fsum([math.fsum(X[0, k] * W[j, k] for k in range(64))] + [s * t[i] * L2[i, j] for i in range(4)])
        assert abs(Y[0, j] - ref) <= 1e-14 * max(1.0, abs(ref))


def test_planted_sign_mistake_is_caught():
    """A sign error in the backward (dX = dY W - s dT L1^T) must fail the
    autograd pin."""
    X, W, L1, L2, dY = _problem(scale_lora=30.0)
    s = 0.75
    _, T = O.linear_fwd(X, W, L1, L2, s)
    dX, _, _, dT = O.linear_bwd(dY, X, W, L1, L2, s, T)
    bad = dY @ W - s * dT @ L1.T
    tX = torch.tensor(X, requires_grad=True)
    tY = tX @ torch.tensor(W).T + s * (tX @ torch.tensor(L1)) @ torch.tensor(L2)
    (tY * torch.tensor(dY)).sum().backward()
    assert np.allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert not np.allclose(bad, tX.grad.numpy(), rtol=1e-6, atol=1e-6)
