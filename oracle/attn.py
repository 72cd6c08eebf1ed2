"""Attention-internals variant of the Dust estimator, in fp64: noise on the
output of the query, key or value projection.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: "Dust：无需反向传播的Transformer零阶预训练", §1 无需反向传播的信用分配
(the attention internals are estimated like the other linear layers, but the
reward comes from the change of the attention output rather than from the
per-token loss) and §1 减少干扰 (attention-specific jitter: only the attention
output is recomputed for a draw, the rest of the network stays cached);
"不用反向传播训练Transformer：Dust零阶优化获突破", the paragraph on interference
reductions (the effect of a perturbation inside the attention module is
judged from the change of the attention output together with an error
signal).

Readings, where the pages leave the form open:

* the error signal is an output error e_t at the attention output o_t of every
  token (width D = H d_h, heads side by side), supplied by the caller (for
  instance the output-error estimate of the layer that reads o);
* a draw's reward is the first-order loss decrease that the output change
  implies, r = -sum_t <o'_t - o_t, e_t>, summed over every token whose
  attention output the perturbation changes: noise on q_s changes o_s only;
  noise on k_s or v_s changes o_t for t = s and every later t of the same
  sequence;
* no attention-weighted future-token discount (the pages call it optional);
* causal multi-head attention over independent sequences of L tokens,
  scores q.k / sqrt(d_h), no dropout, no bias, no other mask.

Estimate: g_s = -(1/(K sigma)) sum_i r_i eps_i (D entries),
G = sum_s g_s x_s^T (D x d) against the projection's cached input x.

Each draw here recomputes the whole attention of the perturbed token's
sequence from the perturbed Q, K or V with the same function that computes
the clean output, so tokens the perturbation cannot reach come out bit for
bit unchanged.
"""
from __future__ import annotations

import math

import numpy as np

from .params import Params
from .philox import TAG_ATTN_K, TAG_ATTN_Q, TAG_ATTN_V, gaussians

WHICH_TAG = {"q": TAG_ATTN_Q, "k": TAG_ATTN_K, "v": TAG_ATTN_V}


def attention_seq(Q, K, V, H: int):
    """Causal multi-head attention of one sequence (or a batch of them).

    Q, K, V: (..., L, D) with D = H d_h. Returns the output (..., L, D) and the
    probabilities (..., H, L, L)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, D = Q.shape[-2], Q.shape[-1]
    dh = D // H
    lead = Q.shape[:-2]

    def heads(x):  # (..., L, D) -> (..., H, L, dh)
        return np.swapaxes(x.reshape(lead + (L, H, dh)), -3, -2)

    q, k, v = heads(Q), heads(K), heads(V)
    s = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(dh)
    future = np.triu(np.ones((L, L), dtype=bool), 1)
    s = np.where(future, -np.inf, s)
    s = s - s.max(axis=-1, keepdims=True)
    a = np.exp(s)
    a = a / a.sum(axis=-1, keepdims=True)
    o = a @ v                                           # (..., H, L, dh)
    O = np.swapaxes(o, -3, -2).reshape(lead + (L, D))
    return O, a


def attention(Q, K, V, L: int, H: int):
    """Causal attention of T = n L tokens in n independent sequences of L.
    Returns O (T x D) and A (n, H, L, L)."""
    Q = np.asarray(Q, dtype=np.float64)
    T, D = Q.shape
    n = T // L
    O, A = attention_seq(Q.reshape(n, L, D), np.asarray(K, np.float64).reshape(n, L, D),
                         np.asarray(V, np.float64).reshape(n, L, D), H)
    return O.reshape(T, D), A


def perturbed_outputs(Qb, Kb, Vb, H: int, pos: int, which: str, delta):
    """Attention outputs of one sequence with delta (n_draws, D) added to row
    ``pos`` of Q, K or V: (n_draws, L, D)."""
    n = delta.shape[0]
    mats = {"q": Qb, "k": Kb, "v": Vb}
    batch = {}
    for key, m in mats.items():
        m = np.broadcast_to(np.asarray(m, dtype=np.float64), (n,) + m.shape).copy()
        if key == which:
            m[:, pos, :] += delta
        batch[key] = m
    O, _ = attention_seq(batch["q"], batch["k"], batch["v"], H)
    return O


def attn_draws(Qb, Kb, Vb, Ob, Eb, H: int, pos: int, which: str, eps, sig: float):
    """Rewards and sum_i r_i eps_i for n draws of noise ``eps`` (n, D) on row
    ``pos`` of one sequence's Q, K or V."""
    O1 = perturbed_outputs(Qb, Kb, Vb, H, pos, which, sig * eps)
    dO = O1 - Ob[None]
    r = -(dO * Eb[None]).sum(axis=(1, 2))
    acc = (r[:, None] * eps).sum(axis=0)
    return r, acc


def attn_grad(X, Q, K, V, E, L: int, H: int, which: str, prm: Params,
              draw_chunk: int = 64) -> dict:
    """The estimator for noise on the output of the ``which`` projection
    ("q", "k" or "v"). X: the projection's input (T x d); Q, K, V: the cached
    projections (T x D); E: the error signal at the attention output (T x D).
    Returns rewards (T x K), g (T x D), G (D x d), the clean output O and the
    attention probabilities A."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    E = np.asarray(E, dtype=np.float64)
    T, D = Q.shape
    if T % L:
        raise ValueError("T must be a multiple of L")
    O, A = attention(Q, K, V, L, H)
    sig = prm.sigma32
    tag = WHICH_TAG[which]
    rewards = np.zeros((T, prm.K))
    g = np.zeros((T, D))
    for s in range(T):
        b, pos = divmod(s, L)
        rows = slice(b * L, (b + 1) * L)
        t_abs = s + prm.token_offset
        for i0 in range(0, prm.K, draw_chunk):
            i1 = min(prm.K, i0 + draw_chunk)
            draws = np.arange(i0, i1, dtype=np.int64) + prm.draw_offset
            eps = gaussians(prm.seed, t_abs, draws, np.arange(D), tag, prm.stream_id)
            r, acc = attn_draws(Q[rows], K[rows], V[rows], O[rows], E[rows], H, pos, which,
                                eps, sig)
            rewards[s, i0:i1] = r
            g[s] += acc
    if sig == 0.0:
        g[:] = 0.0
    else:
        g *= -1.0 / (prm.K * sig)
    G = np.einsum("tc,tf->cf", g, np.asarray(X, dtype=np.float64))
    return {"rewards": rewards, "g": g, "G": G, "O": O, "A": A}
