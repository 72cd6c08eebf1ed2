"""Hidden-MLP up-projection variant of the Dust estimator, in fp64.

The perturbed layer is the up-projection u = W_up x (d_ff outputs per token).
Per the pages ("Dust：无需反向传播的Transformer零阶预训练", §1: noise on every
linear layer's output per token, layer types perturbed in separate passes
with unperturbed intermediates cached; "不用反向传播训练Transformer：Dust零阶
优化获突破": cache unperturbed intermediates, recompute only what the
perturbation changes), a draw adds sigma*eps to u and recomputes GELU, the
down-projection and the head from the cached x, u and clean logits:

  clean:     u = x W_up^T, a = GELU(u), h = x + a W_down^T, z = h W_head^T
  perturbed: da = GELU(u + sigma eps) - GELU(u), dh = da W_down^T,
             dz = dh W_head^T,
             r  = dz_y - log1p(sum_j p_j expm1(dz_j))       (= L - L')
  estimate:  g_t = -(1/(K sigma)) sum_i r_i eps_i   (d_ff entries)
             G_up = sum_t g_t x_t^T                  (d_ff x d)

Readings: GELU is the exact erf form (the only GELU the pages show is
PyTorch's default ``nn.GELU()`` in the code listing of "Dust：无需反向传播的
Transformer 预训练方法"); there is no LayerNorm and no bias. The pages state no
precision: the inputs (x and the weights) are whatever values the caller
holds, and every intermediate here is exact fp64 (the GPU carries the
activations and per-draw deltas at about 2^-17 relative precision).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

from .params import Params
from .philox import TAG_ATTN_OUT, TAG_MLP_DOWN, TAG_MLP_UP, gaussians


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def clean_mlp(X, W_up, W_down, W_head, targets) -> dict:
    """Clean pass: u, a, h, logits z, log-sum-exp, per-token CE and softmax p."""
    X = np.asarray(X, dtype=np.float64)
    u = X @ np.asarray(W_up, dtype=np.float64).T
    a = gelu(u)
    h = X + a @ np.asarray(W_down, dtype=np.float64).T
    z = h @ np.asarray(W_head, dtype=np.float64).T
    zmax = z.max(axis=1)
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
    y = np.asarray(targets, dtype=np.int64)
    loss = lse - z[np.arange(z.shape[0]), y]
    p = np.exp(z - lse[:, None])
    return {"u": u, "a": a, "h": h, "z": z, "lse": lse, "loss": loss, "p": p}


def mlp_draws(u_t, p_t, y_t, eps, W_down, W_head, sig):
    """Rewards and sum_i r_i eps_i for n draws of noise ``eps`` (n, d_ff) on u_t."""
    da = gelu(u_t[None, :] + sig * eps) - gelu(u_t)[None, :]
    dh = da @ W_down.T
    dz = dh @ W_head.T
    r = dz[:, y_t] - np.log1p((p_t[None, :] * np.expm1(dz)).sum(axis=1))
    acc = (r[:, None] * eps).sum(axis=0)
    return r, acc


def mlp_grad(X, W_up, W_down, W_head, targets, prm: Params, draw_chunk: int = 64) -> dict:
    X = np.asarray(X, dtype=np.float64)
    Wd = np.asarray(W_down, dtype=np.float64)
    Wh = np.asarray(W_head, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    clean = clean_mlp(X, W_up, W_down, W_head, y)
    u, p = clean["u"], clean["p"]
    T, d_ff = u.shape
    sig = prm.sigma32
    rewards = np.zeros((T, prm.K))
    g = np.zeros((T, d_ff))
    for t in range(T):
        t_abs = t + prm.token_offset
        for i0 in range(0, prm.K, draw_chunk):
            i1 = min(prm.K, i0 + draw_chunk)
            draws = np.arange(i0, i1, dtype=np.int64) + prm.draw_offset
            eps = gaussians(prm.seed, t_abs, draws, np.arange(d_ff), TAG_MLP_UP, prm.stream_id)
            r, acc = mlp_draws(u[t], p[t], y[t], eps, Wd, Wh, sig)
            rewards[t, i0:i1] = r
            g[t] += acc
    if sig == 0.0:
        g[:] = 0.0
    else:
        g *= -1.0 / (prm.K * sig)
    G = np.einsum("tc,td->cd", g, X)
    return {"loss": clean["loss"], "lse": clean["lse"], "rewards": rewards, "g": g, "G": G,
            "u": u, "p": p, "z": clean["z"]}


# --------------------------------------------------------------------------
# Down-projection variant: the perturbed layer is y = W_down a (d outputs per
# token, a = GELU(u) its cached input). The same pages' reading (one layer
# type per pass, only what the perturbation changes recomputed): sigma eps
# adds to the block output h, so the head sees dz = sigma eps W_head^T and
#   r   = dz_y - log1p(sum_j p_j expm1(dz_j)),
#   g_t = -(1/(K sigma)) sum_i r_i eps_i      (d entries),
#   G_down = sum_t g_t a_t^T                  (d x d_ff).

def mlp_down_draws(p_t, y_t, eps, W_head, sig):
    """Rewards and sum_i r_i eps_i for n draws of noise ``eps`` (n, d) on W_down's output."""
    dz = (sig * eps) @ W_head.T
    r = dz[:, y_t] - np.log1p((p_t[None, :] * np.expm1(dz)).sum(axis=1))
    acc = (r[:, None] * eps).sum(axis=0)
    return r, acc


def mlp_down_grad(X, W_up, W_down, W_head, targets, prm: Params, draw_chunk: int = 256) -> dict:
    Wh = np.asarray(W_head, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    clean = clean_mlp(X, W_up, W_down, W_head, y)
    a, p = clean["a"], clean["p"]
    T = a.shape[0]
    d = Wh.shape[1]
    sig = prm.sigma32
    rewards = np.zeros((T, prm.K))
    g = np.zeros((T, d))
    for t in range(T):
        t_abs = t + prm.token_offset
        for i0 in range(0, prm.K, draw_chunk):
            i1 = min(prm.K, i0 + draw_chunk)
            draws = np.arange(i0, i1, dtype=np.int64) + prm.draw_offset
            eps = gaussians(prm.seed, t_abs, draws, np.arange(d), TAG_MLP_DOWN, prm.stream_id)
            r, acc = mlp_down_draws(p[t], y[t], eps, Wh, sig)
            rewards[t, i0:i1] = r
            g[t] += acc
    if sig == 0.0:
        g[:] = 0.0
    else:
        g *= -1.0 / (prm.K * sig)
    G = np.einsum("tc,tf->cf", g, a)
    return {"loss": clean["loss"], "lse": clean["lse"], "rewards": rewards, "g": g, "G": G,
            "a": a, "p": p, "z": clean["z"]}


# --------------------------------------------------------------------------
# Attention output-projection variant: the perturbed layer is y = W_o o (d
# outputs per token, o the cached attention output, the layer's input), and y
# is added to the residual stream that enters the MLP block: x = r + W_o o.
# Noise sigma eps on y moves x, so each draw recomputes the MLP block and the
# head from the cached x, u and clean logits (the same per-layer reading):
#   du = sigma eps W_up^T,  da = GELU(u + du) - GELU(u),
#   dh = sigma eps + da W_down^T,  dz = dh W_head^T,
#   r  = dz_y - log1p(sum_j p_j expm1(dz_j)),
#   g_t = -(1/(K sigma)) sum_i r_i eps_i  (d entries),  G_o = sum_t g_t o_t^T.

def attn_out_draws(u_t, p_t, y_t, eps, W_up, W_down, W_head, sig):
    """Rewards and sum_i r_i eps_i for n draws of noise ``eps`` (n, d) on x_t."""
    dx = sig * eps
    du = dx @ W_up.T
    da = gelu(u_t[None, :] + du) - gelu(u_t)[None, :]
    dh = dx + da @ W_down.T
    dz = dh @ W_head.T
    r = dz[:, y_t] - np.log1p((p_t[None, :] * np.expm1(dz)).sum(axis=1))
    acc = (r[:, None] * eps).sum(axis=0)
    return r, acc


def attn_out_grad(X, O, W_up, W_down, W_head, targets, prm: Params, draw_chunk: int = 64) -> dict:
    """X: residual entering the MLP block (T x d); O: the output projection's
    input (T x d_o). Returns the estimator's outputs, G of shape d x d_o."""
    Wu = np.asarray(W_up, dtype=np.float64)
    Wd = np.asarray(W_down, dtype=np.float64)
    Wh = np.asarray(W_head, dtype=np.float64)
    y = np.asarray(targets, dtype=np.int64)
    clean = clean_mlp(X, W_up, W_down, W_head, y)
    u, p = clean["u"], clean["p"]
    T = u.shape[0]
    d = Wh.shape[1]
    sig = prm.sigma32
    rewards = np.zeros((T, prm.K))
    g = np.zeros((T, d))
    for t in range(T):
        t_abs = t + prm.token_offset
        for i0 in range(0, prm.K, draw_chunk):
            i1 = min(prm.K, i0 + draw_chunk)
            draws = np.arange(i0, i1, dtype=np.int64) + prm.draw_offset
            eps = gaussians(prm.seed, t_abs, draws, np.arange(d), TAG_ATTN_OUT, prm.stream_id)
            r, acc = attn_out_draws(u[t], p[t], y[t], eps, Wu, Wd, Wh, sig)
            rewards[t, i0:i1] = r
            g[t] += acc
    if sig == 0.0:
        g[:] = 0.0
    else:
        g *= -1.0 / (prm.K * sig)
    G = np.einsum("tc,tf->cf", g, np.asarray(O, dtype=np.float64))
    return {"loss": clean["loss"], "lse": clean["lse"], "rewards": rewards, "g": g, "G": G,
            "u": u, "p": p, "z": clean["z"]}
