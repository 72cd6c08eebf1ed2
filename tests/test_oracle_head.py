"""Pins for the oracle's LM-head estimator.

Each check ties the oracle to something other than itself: torch's
cross-entropy and autograd (the backprop gradient softmax(z) - onehot),
scipy's logsumexp, brute-force finite differences, exact expectations over
enumerated noise, and the cos(K) law of "Dust：无需反向传播的Transformer零阶
预训练", §2 梯度对齐.
"""
import math

import numpy as np
import pytest
import torch
from scipy.optimize import curve_fit
from scipy.special import logsumexp

import oracle


def _problem(T=6, d=5, V=11, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) * scale / math.sqrt(d)
    y = rng.integers(0, V, size=T)
    return H, W, y


def _torch_grad_z(H, W, y):
    """dL_t/dz_t by torch autograd of per-token cross-entropy (fp64)."""
    z = torch.tensor(H @ W.T, dtype=torch.float64, requires_grad=True)
    loss = torch.nn.functional.cross_entropy(z, torch.tensor(y), reduction="sum")
    loss.backward()
    return z.grad.numpy()


def _torch_grad_W(H, W, y):
    Wt = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    z = torch.tensor(H, dtype=torch.float64) @ Wt.T
    torch.nn.functional.cross_entropy(z, torch.tensor(y), reduction="sum").backward()
    return Wt.grad.numpy()


def test_clean_forward_matches_libraries():
    H, W, y = _problem(T=20, d=7, V=300)
    c = oracle.clean_head(H, W, y)
    z = H @ W.T
    np.testing.assert_allclose(c["lse"], logsumexp(z, axis=1), rtol=0, atol=1e-12)
    ce = torch.nn.functional.cross_entropy(torch.tensor(z), torch.tensor(y), reduction="none")
    np.testing.assert_allclose(c["loss"], ce.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(c["p"].sum(axis=1), 1.0, atol=1e-12)


@pytest.mark.parametrize("S", [0, 4])
def test_sigma_zero_gives_zero_reward(S):
    H, W, y = _problem(V=16)
    prm = oracle.Params(T=H.shape[0], d=H.shape[1], V=16, K=8, S=S, sigma=0.0, seed=1)
    out = oracle.head_grad(H, W, y, prm)
    assert np.all(out["rewards"] == 0.0)
    assert np.all(out["g"] == 0.0) and np.all(out["G"] == 0.0)


def test_small_sigma_reward_is_linear_in_the_gradient():
    """r = L - L' -> -sigma eps . dL/dz as sigma -> 0 (first-order Taylor)."""
    H, W, y = _problem(T=4, V=13)
    gz = _torch_grad_z(H, W, y)
    sig = 2.0 ** -20
    prm = oracle.Params(T=4, d=H.shape[1], V=13, K=32, sigma=sig, seed=9)
    out = oracle.head_grad(H, W, y, prm)
    for t in range(4):
        eps = oracle.gaussians(9, t, np.arange(32), np.arange(13), oracle.TAG_HEAD)
        lin = -sig * (eps @ gz[t])
        np.testing.assert_allclose(out["rewards"][t], lin, rtol=0, atol=1e-4 * sig)


def _pm_basis(n, scale):
    """Noise set {+-sqrt(n) e_m}: E[eps eps^T] = I exactly over the set."""
    e = np.concatenate([np.eye(n), -np.eye(n)]) * math.sqrt(n)
    return e * scale


def test_full_vocab_estimate_is_unbiased_exact_expectation():
    H, W, y = _problem(T=5, V=17)
    gz = _torch_grad_z(H, W, y)
    p = oracle.clean_head(H, W, y)["p"]
    sig = 1e-6
    eps = _pm_basis(17, 1.0)
    for t in range(5):
        r, acc = oracle.full_vocab_draws(p[t], y[t], eps, sig)
        g = -acc / (eps.shape[0] * sig)
        np.testing.assert_allclose(g, gz[t], rtol=0, atol=1e-8)


@pytest.mark.parametrize("V,S,a", [(12, 5, 7), (12, 12, 5), (31, 3, 19), (16, 1, 9)])
def test_subset_estimate_is_unbiased_exact_expectation(V, S, a):
    """Average over every offset b and over +-sqrt(S+1) e_m noise gives dL/dz."""
    H, W, y = _problem(T=4, d=3, V=V, seed=V + S)
    gz = _torch_grad_z(H, W, y)
    p = oracle.clean_head(H, W, y)["p"]
    sig = 1e-6
    eps1 = _pm_basis(S + 1, 1.0)
    b = np.repeat(np.arange(V), eps1.shape[0])
    eps = np.tile(eps1, (V, 1))
    for t in range(4):
        r, acc = oracle.subset_draws(p[t], y[t], b, eps, S, a, sig)
        g = -acc / (b.size * sig)
        np.testing.assert_allclose(g, gz[t], rtol=0, atol=1e-7)
        # the literal reading (V/S also on the target) biases the target coordinate
        if S < V:
            _, acc_l = oracle.subset_draws(p[t], y[t], b, eps, S, a, sig, literal_target_scale=True)
            g_l = -acc_l / (b.size * sig)
            np.testing.assert_allclose(g_l[y[t]], gz[t][y[t]] * V / S, rtol=1e-5)


def _subset_linear_variance(grad, y, V, S, a):
    """Per-coordinate variance of one draw of the subset estimator as sigma -> 0.

    One draw with offset b perturbs D = {(a k + b) mod V : k < S} plus the
    target y, each with its own unit Gaussian. To first order in sigma its
    contribution to coordinate j is X_j = s_j eps_j [j in D'] sum_{k in D'}
    eps_k grad_k, with s_j the inverse inclusion probability (V/S off the
    target, 1 on it). With independent unit Gaussians,
    E[eps_j^2 (sum_k eps_k grad_k)^2] = 2 grad_j^2 + sum_{k in D'} grad_k^2;
    b is uniform over V, so E[X_j^2] is an exact average over every b."""
    ex2 = np.zeros(V)
    for b in range(V):
        dset = sorted({(a * k + b) % V for k in range(S)} | {int(y)})
        norm2 = float(sum(grad[k] ** 2 for k in dset))
        for j in dset:
            s = 1.0 if j == y else V / S
            ex2[j] += s * s * (2.0 * grad[j] ** 2 + norm2) / V
    return ex2 - grad ** 2


@pytest.mark.parametrize("V,S,a", [(12, 5, 7), (16, 3, 5)])
def test_assembled_subset_estimator_matches_its_exact_variance(V, S, a):
    """oracle.head_grad with S > 0, end to end (Philox offsets b, slot noise, the
    appended target slot, the V/S and 1 scales, the -1/(K sigma) factor), against
    dL/dz = p - e_y from autograd: the error of g is what the exact per-draw
    variance predicts, E||g - grad||^2 = sum_j Var_j / K, and no coordinate
    is off by more than 5 of its standard deviations. A wrong scale, sign, a
    dropped target term or a reused noise slot biases g by O(1), hundreds of
    standard deviations here."""
    T, K = 8, 200_000
    H, W, y = _problem(T=T, d=3, V=V, seed=40 + V)
    gz = _torch_grad_z(H, W, y)
    prm = oracle.Params(T=T, d=3, V=V, K=K, S=S, sigma=1e-4, seed=17, subset_a=a)
    g = oracle.head_grad(H, W, y, prm)["g"]
    num = den = 0.0
    for t in range(T):
        var = _subset_linear_variance(gz[t], y[t], V, S, a)
        assert np.all(var >= -1e-12)
        z = (g[t] - gz[t]) / np.sqrt(np.maximum(var, 1e-30) / K)
        assert np.abs(z).max() < 5.0, (t, z)
        num += ((g[t] - gz[t]) ** 2).sum()
        den += var.sum() / K
    assert 0.6 < num / den < 1.5, num / den


def test_subset_draws_the_arithmetic_progression_and_the_target():
    V, S, a = 50, 7, 31
    p = np.full(V, 1.0 / V)
    # a unit bump on one slot: only that index's reward term moves
    for b in (0, 13, 49):
        idx = [(a * k + b) % V for k in range(S)]
        assert len(set(idx)) == S
        for k in range(S + 1):
            eps = np.zeros((1, S + 1))
            eps[0, k] = 1.0
            y = 3 if 3 not in idx else next(j for j in range(V) if j not in idx)
            r, acc = oracle.subset_draws(p, y, np.array([b]), eps, S, a, 0.5)
            nz = np.nonzero(acc)[0]
            if k < S:
                assert list(nz) == [idx[k]]
                assert r[0] == pytest.approx(-math.log1p(p[idx[k]] * math.expm1(0.5)))
            else:
                assert list(nz) == [y]          # slot S carries the appended target
                assert r[0] == pytest.approx(0.5 - math.log1p(p[y] * math.expm1(0.5)))


def test_subset_with_S_equal_V_matches_full_vocab():
    V, a = 9, 5
    H, W, y = _problem(T=3, d=4, V=V)
    p = oracle.clean_head(H, W, y)["p"]
    rng = np.random.default_rng(0)
    for t in range(3):
        b = rng.integers(0, V, size=6)
        eps = rng.standard_normal((6, V + 1))
        r_s, acc_s = oracle.subset_draws(p[t], y[t], b, eps, V, a, 0.05)
        eps_full = np.zeros((6, V))
        for i in range(6):
            eps_full[i, (a * np.arange(V) + b[i]) % V] = eps[i, :V]
        r_f, acc_f = oracle.full_vocab_draws(p[t], y[t], eps_full, 0.05)
        np.testing.assert_allclose(r_s, r_f, rtol=0, atol=1e-15)
        np.testing.assert_allclose(acc_s, acc_f, rtol=0, atol=1e-13)


def test_weight_gradient_is_the_outer_product_sum():
    H, W, y = _problem(T=7, d=3, V=10)
    prm = oracle.Params(T=7, d=3, V=10, K=16, sigma=0.1, seed=4)
    out = oracle.head_grad(H, W, y, prm)
    G = np.zeros((10, 3))
    for t in range(7):
        G += np.outer(out["g"][t], H[t])
    np.testing.assert_allclose(out["G"], G, rtol=0, atol=1e-12)
    assert out["G"].shape == W.shape


def test_closed_form_gradient_matches_finite_differences():
    """(p - e_y) h^T, the sigma -> 0, K -> inf limit of G_W, is dL/dW by brute force."""
    H, W, y = _problem(T=5, d=3, V=6)
    p = oracle.clean_head(H, W, y)["p"]
    closed = np.zeros_like(W)
    for t in range(5):
        gz = p[t].copy()
        gz[y[t]] -= 1.0
        closed += np.outer(gz, H[t])
    fd = np.zeros_like(W)
    h = 1e-5
    for v in range(6):
        for e in range(3):
            Wp, Wm = W.copy(), W.copy()
            Wp[v, e] += h
            Wm[v, e] -= h
            fd[v, e] = (oracle.clean_head(H, Wp, y)["loss"].sum()
                        - oracle.clean_head(H, Wm, y)["loss"].sum()) / (2 * h)
    np.testing.assert_allclose(fd, closed, rtol=0, atol=1e-8)
    np.testing.assert_allclose(_torch_grad_W(H, W, y), closed, rtol=0, atol=1e-12)


def test_estimate_converges_to_backprop_gradient():
    """E||g - grad||^2 / ||grad||^2 = (V + 1) / K for full-vocabulary draws."""
    T, V, K = 24, 24, 4096
    H, W, y = _problem(T=T, d=6, V=V, seed=3)
    gz = _torch_grad_z(H, W, y)
    prm = oracle.Params(T=T, d=6, V=V, K=K, sigma=1e-4, seed=21)
    out = oracle.head_grad(H, W, y, prm)
    ratio = (((out["g"] - gz) ** 2).sum(axis=1) / (gz ** 2).sum(axis=1)).mean()
    assert ratio == pytest.approx((V + 1) / K, rel=0.2)
    # the sigma -> 0 estimator with the same draws agrees to O(sigma)
    lin = oracle.head_linear_estimate(H, W, y, prm)
    np.testing.assert_allclose(out["g"], lin, rtol=0, atol=5e-3)
    # and G_W approaches the autograd weight gradient
    gW = _torch_grad_W(H, W, y)
    err = np.linalg.norm(out["G"] - gW) / np.linalg.norm(gW)
    assert err < 3.0 * math.sqrt((V + 1) / K) * math.sqrt(T)


def test_cosine_follows_the_population_law():
    """cos(K) = c_max / sqrt(1 + c/K) with fit RMSE < 0.06 and c near its closed form."""
    T, d, V = 8, 6, 24
    H, W, y = _problem(T=T, d=d, V=V, seed=5)
    gz = _torch_grad_z(H, W, y)
    gW = gz.T @ H
    Ks = np.array([64, 256, 1024, 4096, 16384])
    cos = []
    for K in Ks:
        prm = oracle.Params(T=T, d=d, V=V, K=int(K), sigma=1e-4, seed=33)
        G = oracle.head_grad(H, W, y, prm)["G"]
        cos.append(float((G * gW).sum() / (np.linalg.norm(G) * np.linalg.norm(gW))))
    cos = np.array(cos)
    law = lambda k, cmax, c: cmax / np.sqrt(1.0 + c / k)  # noqa: E731
    (cmax, c), _ = curve_fit(law, Ks, cos, p0=(1.0, 100.0))
    rmse = math.sqrt(np.mean((law(Ks, cmax, c) - cos) ** 2))
    assert rmse < 0.06
    # E||G - gW||^2 = (V + 1)/K * sum_t ||grad_t||^2 ||h_t||^2
    c_closed = (V + 1) * sum((gz[t] @ gz[t]) * (H[t] @ H[t]) for t in range(T)) / (gW * gW).sum()
    assert cmax == pytest.approx(1.0, abs=0.1)
    assert c == pytest.approx(c_closed, rel=0.35)
    assert np.all(np.diff(cos) > 0)
