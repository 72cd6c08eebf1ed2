"""Pins for the oracle's MLP up-projection estimator.

Checked against torch's GELU, bf16 conversion and autograd, brute-force
finite differences and the exact expectation over enumerated noise.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _mlp_problem(T=4, d=5, d_ff=7, V=9, seed=0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, d))
    W_up = rng.standard_normal((d_ff, d)) / math.sqrt(d)
    W_down = rng.standard_normal((d, d_ff)) / math.sqrt(d_ff)
    W_head = rng.standard_normal((V, d)) / math.sqrt(d)
    y = rng.integers(0, V, size=T)
    return X, W_up, W_down, W_head, y


def _torch_loss(X, W_up, W_down, W_head, y, wrt=None):
    tens = {k: torch.tensor(v, dtype=torch.float64) for k, v in
            dict(X=X, W_up=W_up, W_down=W_down, W_head=W_head).items()}
    if wrt and wrt != "u":
        tens[wrt].requires_grad_(True)
    u = tens["X"] @ tens["W_up"].T
    if wrt == "u":
        u = u.detach().requires_grad_(True)
        tens["u"] = u
    a = torch.nn.functional.gelu(u, approximate="none")
    h = tens["X"] + a @ tens["W_down"].T
    z = h @ tens["W_head"].T
    loss = torch.nn.functional.cross_entropy(z, torch.tensor(y), reduction="sum")
    if wrt:
        loss.backward()
        return loss.item(), tens[wrt].grad.numpy()
    return loss.item(), None


def test_gelu_matches_torch():
    x = np.linspace(-8, 8, 4001)
    ref = torch.nn.functional.gelu(torch.tensor(x), approximate="none").numpy()
    np.testing.assert_allclose(oracle.gelu(x), ref, rtol=0, atol=1e-15)


def test_clean_forward_matches_torch():
    X, Wu, Wd, Wh, y = _mlp_problem(T=6)
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    ref, _ = _torch_loss(X, Wu, Wd, Wh, y)
    assert c["loss"].sum() == pytest.approx(ref, abs=1e-12)


def test_sigma_zero_gives_zero_reward():
    X, Wu, Wd, Wh, y = _mlp_problem()
    prm = oracle.Params(T=4, d=5, V=9, d_ff=7, K=6, sigma=0.0, seed=2)
    out = oracle.mlp_grad(X, Wu, Wd, Wh, y, prm)
    assert np.all(out["rewards"] == 0.0) and np.all(out["G"] == 0.0)


def test_estimate_is_unbiased_exact_expectation():
    """Over +-sqrt(d_ff) e_m noise, g equals dL/du from torch autograd (to O(sigma^2))."""
    X, Wu, Wd, Wh, y = _mlp_problem(T=3)
    _, gu = _torch_loss(X, Wu, Wd, Wh, y, wrt="u")
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    d_ff = Wu.shape[0]
    eps = np.concatenate([np.eye(d_ff), -np.eye(d_ff)]) * math.sqrt(d_ff)
    sig = 1e-6
    for t in range(3):
        r, acc = oracle.mlp_draws(c["u"][t], c["p"][t], y[t], eps, Wd, Wh, sig)
        g = -acc / (eps.shape[0] * sig)
        np.testing.assert_allclose(g, gu[t], rtol=0, atol=1e-8)


def test_closed_form_up_gradient_matches_finite_differences():
    """sum_t [GELU'(u) * W_down^T W_head^T (p - e_y)] x^T against brute force."""
    X, Wu, Wd, Wh, y = _mlp_problem(T=3, d=3, d_ff=4, V=5)
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    u, p = c["u"], c["p"]
    dgelu = 0.5 * (1 + np.vectorize(math.erf)(u / math.sqrt(2))) + u * np.exp(-u * u / 2) / math.sqrt(2 * math.pi)
    closed = np.zeros_like(Wu)
    for t in range(3):
        gz = p[t].copy()
        gz[y[t]] -= 1.0
        closed += np.outer(dgelu[t] * (Wd.T @ (Wh.T @ gz)), X[t])
    fd = np.zeros_like(Wu)
    h = 1e-5
    for i in range(Wu.shape[0]):
        for j in range(Wu.shape[1]):
            P, M = Wu.copy(), Wu.copy()
            P[i, j] += h
            M[i, j] -= h
            fd[i, j] = (oracle.clean_mlp(X, P, Wd, Wh, y)["loss"].sum()
                        - oracle.clean_mlp(X, M, Wd, Wh, y)["loss"].sum()) / (2 * h)
    np.testing.assert_allclose(fd, closed, rtol=0, atol=1e-8)
    _, gW = _torch_loss(X, Wu, Wd, Wh, y, wrt="W_up")
    np.testing.assert_allclose(gW, closed, rtol=0, atol=1e-12)


def test_estimate_converges_with_population():
    X, Wu, Wd, Wh, y = _mlp_problem(T=4, d=4, d_ff=6, V=7, seed=3)
    _, gW = _torch_loss(X, Wu, Wd, Wh, y, wrt="W_up")
    errs = []
    for K in (256, 4096):
        prm = oracle.Params(T=4, d=4, V=7, d_ff=6, K=K, sigma=1e-4, seed=8)
        G = oracle.mlp_grad(X, Wu, Wd, Wh, y, prm, draw_chunk=4096)["G"]
        assert G.shape == Wu.shape
        errs.append(np.linalg.norm(G - gW) / np.linalg.norm(gW))
    assert errs[1] < errs[0] / 2.5
    assert errs[1] < 0.25


# ---- down-projection variant ----------------------------------------------

def _dL_dh(X, W_up, W_down, W_head, y):
    """dL/dh for every token from torch autograd (h detached as a leaf)."""
    t = {k: torch.tensor(v, dtype=torch.float64) for k, v in
         dict(X=X, W_up=W_up, W_down=W_down, W_head=W_head).items()}
    a = torch.nn.functional.gelu(t["X"] @ t["W_up"].T, approximate="none")
    h = (t["X"] + a @ t["W_down"].T).detach().requires_grad_(True)
    loss = torch.nn.functional.cross_entropy(h @ t["W_head"].T, torch.tensor(y), reduction="sum")
    loss.backward()
    return h.grad.numpy()


def test_down_estimate_is_unbiased_exact_expectation():
    """Over +-sqrt(d) e_m noise on W_down's output, g equals dL/dh (to O(sigma^2))."""
    X, Wu, Wd, Wh, y = _mlp_problem(T=3)
    gh = _dL_dh(X, Wu, Wd, Wh, y)
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    d = Wh.shape[1]
    eps = np.concatenate([np.eye(d), -np.eye(d)]) * math.sqrt(d)
    sig = 1e-6
    for t in range(3):
        r, acc = oracle.mlp_down_draws(c["p"][t], y[t], eps, Wh, sig)
        np.testing.assert_allclose(-acc / (eps.shape[0] * sig), gh[t], rtol=0, atol=1e-8)


def test_down_weight_gradient_matches_finite_differences_and_autograd():
    """sum_t dL/dh_t a_t^T against brute-force differences of the summed loss in W_down."""
    X, Wu, Wd, Wh, y = _mlp_problem(T=3, d=3, d_ff=4, V=5)
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    closed = _dL_dh(X, Wu, Wd, Wh, y).T @ c["a"]
    fd = np.zeros_like(Wd)
    h = 1e-5
    for i in range(Wd.shape[0]):
        for j in range(Wd.shape[1]):
            P, M = Wd.copy(), Wd.copy()
            P[i, j] += h
            M[i, j] -= h
            fd[i, j] = (oracle.clean_mlp(X, Wu, P, Wh, y)["loss"].sum()
                        - oracle.clean_mlp(X, Wu, M, Wh, y)["loss"].sum()) / (2 * h)
    np.testing.assert_allclose(fd, closed, rtol=0, atol=1e-8)
    _, gW = _torch_loss(X, Wu, Wd, Wh, y, wrt="W_down")
    np.testing.assert_allclose(gW, closed, rtol=0, atol=1e-12)


def test_down_sigma_zero_and_noise_stream():
    X, Wu, Wd, Wh, y = _mlp_problem()
    prm = oracle.Params(T=4, d=5, V=9, d_ff=7, K=6, sigma=0.0, seed=2)
    out = oracle.mlp_down_grad(X, Wu, Wd, Wh, y, prm)
    assert np.all(out["rewards"] == 0.0) and np.all(out["G"] == 0.0)
    # the down-projection draws its noise from its own counter tag
    e_up = oracle.gaussians(2, 0, np.arange(3), np.arange(5), oracle.TAG_MLP_UP)
    e_dn = oracle.gaussians(2, 0, np.arange(3), np.arange(5), oracle.TAG_MLP_DOWN)
    assert not np.allclose(e_up, e_dn)


def test_down_estimate_converges_with_population():
    X, Wu, Wd, Wh, y = _mlp_problem(T=4, d=4, d_ff=6, V=7, seed=3)
    _, gW = _torch_loss(X, Wu, Wd, Wh, y, wrt="W_down")
    errs = []
    for K in (256, 4096):
        prm = oracle.Params(T=4, d=4, V=7, d_ff=6, K=K, sigma=1e-4, seed=8)
        G = oracle.mlp_down_grad(X, Wu, Wd, Wh, y, prm, draw_chunk=4096)["G"]
        assert G.shape == Wd.shape
        errs.append(np.linalg.norm(G - gW) / np.linalg.norm(gW))
    assert errs[1] < errs[0] / 2.5
    assert errs[1] < 0.25


# ---- attention output-projection variant -------------------------------------

def _attn_problem(T=4, d=5, d_o=6, d_ff=7, V=9, seed=0):
    rng = np.random.default_rng(seed + 100)
    X, Wu, Wd, Wh, y = _mlp_problem(T=T, d=d, d_ff=d_ff, V=V, seed=seed)
    R = rng.standard_normal((T, d))                 # residual before the attention write
    O = rng.standard_normal((T, d_o))               # the output projection's input
    W_o = rng.standard_normal((d, d_o)) / math.sqrt(d_o)
    return R, O, W_o, Wu, Wd, Wh, y


def _dL_dx(X, W_up, W_down, W_head, y):
    """dL/dx for the residual entering the MLP block (x a leaf), from autograd."""
    t = {k: torch.tensor(v, dtype=torch.float64) for k, v in
         dict(W_up=W_up, W_down=W_down, W_head=W_head).items()}
    x = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    a = torch.nn.functional.gelu(x @ t["W_up"].T, approximate="none")
    z = (x + a @ t["W_down"].T) @ t["W_head"].T
    torch.nn.functional.cross_entropy(z, torch.tensor(y), reduction="sum").backward()
    return x.grad.numpy()


def test_attn_out_estimate_is_unbiased_exact_expectation():
    """Over +-sqrt(d) e_m noise on x, g equals dL/dx (to O(sigma^2))."""
    R, O, W_o, Wu, Wd, Wh, y = _attn_problem(T=3)
    X = R + O @ W_o.T
    gx = _dL_dx(X, Wu, Wd, Wh, y)
    c = oracle.clean_mlp(X, Wu, Wd, Wh, y)
    d = Wh.shape[1]
    eps = np.concatenate([np.eye(d), -np.eye(d)]) * math.sqrt(d)
    sig = 1e-6
    for t in range(3):
        r, acc = oracle.attn_out_draws(c["u"][t], c["p"][t], y[t], eps, Wu, Wd, Wh, sig)
        np.testing.assert_allclose(-acc / (eps.shape[0] * sig), gx[t], rtol=0, atol=1e-7)


def test_attn_out_weight_gradient_matches_finite_differences():
    """sum_t dL/dx_t o_t^T against brute-force differences in W_o, x = r + W_o o."""
    R, O, W_o, Wu, Wd, Wh, y = _attn_problem(T=3, d=3, d_o=4, d_ff=4, V=5)
    X = R + O @ W_o.T
    closed = _dL_dx(X, Wu, Wd, Wh, y).T @ O
    fd = np.zeros_like(W_o)
    h = 1e-5
    for i in range(W_o.shape[0]):
        for j in range(W_o.shape[1]):
            P, M = W_o.copy(), W_o.copy()
            P[i, j] += h
            M[i, j] -= h
            fd[i, j] = (oracle.clean_mlp(R + O @ P.T, Wu, Wd, Wh, y)["loss"].sum()
                        - oracle.clean_mlp(R + O @ M.T, Wu, Wd, Wh, y)["loss"].sum()) / (2 * h)
    np.testing.assert_allclose(fd, closed, rtol=0, atol=1e-8)


def test_attn_out_sigma_zero_and_convergence():
    R, O, W_o, Wu, Wd, Wh, y = _attn_problem(T=4, d=4, d_o=3, d_ff=6, V=7, seed=3)
    X = R + O @ W_o.T
    prm = oracle.Params(T=4, d=4, V=7, d_ff=6, K=6, sigma=0.0, seed=2)
    out = oracle.attn_out_grad(X, O, Wu, Wd, Wh, y, prm)
    assert np.all(out["rewards"] == 0.0) and np.all(out["G"] == 0.0)
    exact = _dL_dx(X, Wu, Wd, Wh, y).T @ O
    errs = []
    for K in (256, 4096):
        prm = oracle.Params(T=4, d=4, V=7, d_ff=6, K=K, sigma=1e-4, seed=8)
        G = oracle.attn_out_grad(X, O, Wu, Wd, Wh, y, prm, draw_chunk=4096)["G"]
        assert G.shape == (4, 3)
        errs.append(np.linalg.norm(G - exact) / np.linalg.norm(exact))
    # the error falls as 1/sqrt(K) in expectation (4x over these K); one sample each
    assert errs[1] < errs[0] / 2 and errs[1] < 0.1
