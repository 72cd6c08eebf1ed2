"""LM-head variant of the Dust estimator, step by step in fp64.

Follows "Dust：无需反向传播的Transformer零阶预训练" (agentlenshq), §1:
for the head y_t = W h_t the noise sigma*eps goes on the logits of token t,
the perturbed per-token loss is recomputed from the cached clean logits
(减少干扰, "仅头部扰动"), the reward is the loss reduction r = L - L', the
output-error estimate is g_t = -(1/(K sigma)) sum_i r_i eps_i and the weight
gradient is G_W = sum_t g_t h_t^T (无需反向传播的信用分配).

Readings of points the pages leave open:

* loss is natural-log cross-entropy per token; no label smoothing;
* a_t^(i) in the estimate is the unit Gaussian eps (so E[g] -> dL/dz);
* the perturbed loss is formed in the delta form
  L' - L = log1p(sum_j p_j expm1(sigma eps_j)) - sigma eps_y, identical in exact
  arithmetic to LSE(z + sigma eps) - (z_y + sigma eps_y) - L;
* subset draws (the pages: "each draw evaluates a small subset of the
  vocabulary"): slot k < S perturbs index j_k = (a k + b) mod V with a coprime
  to V and b drawn from the draw's counter; the target is always included
  (as slot S with its own noise when it is not among the j_k); only the
  drawn logits move, so LSE' = LSE + log(1 + sum_{j drawn} p_j (e^{sigma eps_j} - 1));
* subset scaling: each coordinate of g is divided by its inclusion
  probability, S/V for non-target indices and 1 for the target (the literal
  "scale by V/S everywhere" reading is available as ``literal_target_scale``);
* sigma = 0 gives rewards 0 and, by convention, g = 0 and G_W = 0.
"""
from __future__ import annotations

import numpy as np

from .params import Params
from .philox import TAG_HEAD, default_subset_a, gaussians, subset_offset


def clean_head(H: np.ndarray, W: np.ndarray, targets: np.ndarray) -> dict:
    """Clean logits z = H W^T, log-sum-exp, per-token loss and softmax p."""
    H = np.asarray(H, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    z = H @ W.T
    zmax = z.max(axis=1)
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
    rows = np.arange(z.shape[0])
    loss = lse - z[rows, y]
    p = np.exp(z - lse[:, None])
    return {"z": z, "lse": lse, "loss": loss, "p": p}


def full_vocab_draws(p_t, y_t, eps, sig):
    """Rewards and sum_i r_i eps_i for draws over the whole vocabulary.

    ``eps`` is (n, V): the unit noise of n draws on token t's logits.
    """
    x = sig * eps
    s = (p_t[None, :] * np.expm1(x)).sum(axis=1)
    r = x[:, y_t] - np.log1p(s)
    acc = (r[:, None] * eps).sum(axis=0)
    return r, acc


def subset_draws(p_t, y_t, b, eps, S, a, sig, literal_target_scale=False):
    """Rewards and the scaled sum of r_i eps_i for vocabulary-subset draws.

    ``b`` is (n,) subset offsets, ``eps`` is (n, S + 1) slot noise (slot S is
    used only when the target is not among the S drawn indices).
    """
    V = p_t.shape[0]
    k = np.arange(S, dtype=np.int64)
    idx = (a * k[None, :] + np.asarray(b, dtype=np.int64)[:, None]) % V   # (n, S)
    eps_win, eps_extra = eps[:, :S], eps[:, S]
    hit = idx == y_t                                                      # target drawn?
    in_win = hit.any(axis=1)
    eps_y = np.where(in_win, (eps_win * hit).sum(axis=1), eps_extra)
    s = (p_t[idx] * np.expm1(sig * eps_win)).sum(axis=1)
    s = s + np.where(in_win, 0.0, p_t[y_t] * np.expm1(sig * eps_extra))
    r = sig * eps_y - np.log1p(s)
    # scale each coordinate by its inverse inclusion probability
    scale_other = V / S
    scale_target = scale_other if literal_target_scale else 1.0
    contrib = r[:, None] * eps_win
    non_target = ~hit
    acc = np.bincount(idx[non_target], weights=contrib[non_target], minlength=V) * scale_other
    acc[y_t] += scale_target * (r * eps_y).sum()
    return r, acc


def head_grad(H, W, targets, prm: Params, draw_chunk: int = 1024) -> dict:
    """Full estimator output: clean loss, rewards (T x K), g (T x V), G_W (V x d)."""
    H = np.asarray(H, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    T, V = H.shape[0], W.shape[0]
    assert W.shape[1] == H.shape[1] and y.shape == (T,)
    clean = clean_head(H, W, y)
    p = clean["p"]
    a = prm.subset_a if prm.subset_a else default_subset_a(V)
    rewards = np.zeros((T, prm.K))
    g = np.zeros((T, V))
    for t in range(T):
        t_abs = t + prm.token_offset
        for i0 in range(0, prm.K, draw_chunk):
            i1 = min(prm.K, i0 + draw_chunk)
            draws = np.arange(i0, i1, dtype=np.int64) + prm.draw_offset
            if prm.full_vocab:
                eps = gaussians(prm.seed, t_abs, draws, np.arange(V), TAG_HEAD, prm.stream_id)
                r, acc = full_vocab_draws(p[t], y[t], eps, prm.sigma32)
            else:
                b = subset_offset(prm.seed, t_abs, draws, V, prm.stream_id)
                eps = gaussians(prm.seed, t_abs, draws, np.arange(prm.S + 1), TAG_HEAD,
                                prm.stream_id)
                r, acc = subset_draws(p[t], y[t], b, eps, prm.S, a, prm.sigma32,
                                      prm.literal_target_scale)
            rewards[t, i0:i1] = r
            g[t] += acc
    if prm.sigma32 == 0.0:
        g[:] = 0.0
    else:
        g *= -1.0 / (prm.K * prm.sigma32)
    G = np.einsum("tv,td->vd", g, H)
    return {"loss": clean["loss"], "lse": clean["lse"], "rewards": rewards, "g": g,
            "G": G, "p": p, "z": clean["z"], "subset_a": a}


def head_linear_estimate(H, W, targets, prm: Params) -> np.ndarray:
    """g of the first-order (sigma -> 0) estimator for the same noise draws.

    To first order in sigma the reward is r = -sigma eps . dL/dz with
    dL/dz = p - e_y, so g_t = (1/K) sum_i (eps_i . (p_t - e_y)) eps_i.
    Full-vocabulary draws only.
    """
    assert prm.full_vocab
    clean = clean_head(H, W, targets)
    p = clean["p"]
    y = np.asarray(targets, dtype=np.int64)
    T, V = p.shape
    g = np.zeros((T, V))
    draws = np.arange(prm.K, dtype=np.int64) + prm.draw_offset
    for t in range(T):
        grad = p[t].copy()
        grad[y[t]] -= 1.0
        eps = gaussians(prm.seed, t + prm.token_offset, draws, np.arange(V), TAG_HEAD, prm.stream_id)
        g[t] = ((eps @ grad)[:, None] * eps).mean(axis=0)
    return g
