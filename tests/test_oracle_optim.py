"""Pins of the oracle's SGD-with-momentum step and training loop (CPU).

The update is pinned by closed forms of the heavy-ball recursion; the exact
weight gradient by torch autograd of the summed cross-entropy; the loop by
monotone descent of a convex loss under the exact gradient and by descent
under the Dust estimator itself.
"""
import numpy as np
import torch

import oracle
import synth


def test_plain_sgd_when_momentum_is_zero():
    rng = np.random.default_rng(0)
    W, v, G = rng.normal(size=(3, 7, 5))
    W1, v1 = oracle.sgd_momentum(W, v, G, lr=0.3, mu=0.0)
    assert np.array_equal(v1, G)
    assert np.allclose(W1, W - 0.3 * G, rtol=0, atol=1e-15)


def test_constant_gradient_geometric_series():
    # v_n = G (1 - mu^n)/(1 - mu);  W_n = W_0 - lr G (n - mu (1 - mu^n)/(1 - mu)) / (1 - mu)
    rng = np.random.default_rng(1)
    W0, G = rng.normal(size=(2, 4, 3))
    lr, mu, n = 0.07, 0.85, 23
    W, v = W0.copy(), np.zeros_like(W0)
    for _ in range(n):
        W, v = oracle.sgd_momentum(W, v, G, lr, mu)
    geo = (1 - mu ** n) / (1 - mu)
    assert np.allclose(v, G * geo, rtol=1e-13, atol=0)
    assert np.allclose(W, W0 - lr * G * (n - mu * geo) / (1 - mu), rtol=1e-12, atol=1e-14)


def test_exact_weight_grad_matches_autograd():
    rng = np.random.default_rng(2)
    T, d, V = 9, 6, 13
    H = rng.normal(size=(T, d))
    W = rng.normal(size=(V, d)) / np.sqrt(d)
    y = rng.integers(0, V, size=T)
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    z = torch.tensor(H, dtype=torch.float64) @ Wt.T
    torch.nn.functional.cross_entropy(z, torch.tensor(y), reduction="sum").backward()
    assert np.allclose(oracle.exact_weight_grad(H, W, y), Wt.grad.numpy(), rtol=1e-12, atol=1e-13)


def _tiny():
    wl = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_head_inputs(wl)
    prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=wl.K, S=0, sigma=wl.sigma, seed=wl.seed)
    return inp["H"], inp["W"], inp["targets"], prm


def test_exact_gradient_descends_monotonically():
    H, W, y, prm = _tiny()
    r = oracle.train_head(H, W, y, prm, steps=6, lr=0.005, mu=0.5, exact=True)
    assert np.all(np.diff(r["losses"]) < 0), r["losses"]


def test_dust_estimator_trains_the_head():
    # K = 16 full-vocabulary draws per step, fresh noise every step
    H, W, y, prm = _tiny()
    r = oracle.train_head(H, W, y, prm, steps=5, lr=0.05, mu=0.9)
    assert r["losses"][-1] < 0.5 * r["losses"][0], r["losses"]
    # step s uses draw indices [s K, (s+1) K): the first step is the plain estimator
    G0 = oracle.head_grad(H, W, y, prm)["G"]
    W1, _ = oracle.sgd_momentum(W, np.zeros_like(G0), G0, 0.05, 0.9)
    r1 = oracle.train_head(H, W, y, prm, steps=1, lr=0.05, mu=0.9)
    assert np.array_equal(r1["W"], W1)
