"""SGD with momentum on the LM-head weights, and a multi-step loop, in fp64.

The pages report their pretraining runs under SGD with momentum ("Dust：无需
反向传播的Transformer零阶预训练", §2 实证发现, the heading of the pretraining
results) without stating the form, the learning rate or the momentum. The
reading taken here is the heavy-ball form with no dampening, no Nesterov
step and no weight decay:

    v <- mu v + G,      W <- W - lr v,

with G the estimator's weight gradient (the sum over tokens, so lr absorbs any
1/T). In the loop, step s draws its noise at draw indices [s K, (s+1) K) of
the same seed, so every step has fresh, independent noise; the weights the
estimator sees are the bf16 rounding of the fp32 master weights when the
workload is bf16 (the product keeps an fp32 master copy and a bf16 copy).
"""
from __future__ import annotations

from dataclasses import replace

import numpy as np

from .head import clean_head, head_grad
from .params import Params


def sgd_momentum(W, v, G, lr: float, mu: float):
    """One heavy-ball step: returns (W', v') with v' = mu v + G, W' = W - lr v'."""
    v_new = mu * np.asarray(v, dtype=np.float64) + np.asarray(G, dtype=np.float64)
    W_new = np.asarray(W, dtype=np.float64) - lr * v_new
    return W_new, v_new


def exact_weight_grad(H, W, targets) -> np.ndarray:
    """dL/dW for L = sum_t CE_t: (softmax(z) - onehot(y))^T H."""
    c = clean_head(H, W, targets)
    g = c["p"].copy()
    g[np.arange(g.shape[0]), np.asarray(targets, dtype=np.int64)] -= 1.0
    return g.T @ np.asarray(H, dtype=np.float64)


def train_head(H, W0, targets, prm: Params, steps: int, lr: float, mu: float,
               round_weights=None, exact: bool = False) -> dict:
    """``steps`` SGD-momentum steps on the head weights from W0.

    round_weights maps the master weights to the values the estimator reads
    (e.g. bf16 rounding); ``exact`` swaps the estimator for the exact gradient.
    Returns the per-step clean mean loss (before each update), the final
    master weights and the momentum buffer."""
    W = np.asarray(W0, dtype=np.float64).copy()
    v = np.zeros_like(W)
    losses = []
    for s in range(steps):
        Wr = round_weights(W) if round_weights is not None else W
        if exact:
            G = exact_weight_grad(H, Wr, targets)
            loss = clean_head(H, Wr, targets)["loss"]
        else:
            out = head_grad(H, Wr, targets, replace(prm, draw_offset=prm.draw_offset + s * prm.K))
            G, loss = out["G"], out["loss"]
        losses.append(float(np.mean(loss)))
        W, v = sgd_momentum(W, v, G, lr, mu)
    return {"losses": np.array(losses), "W": W, "v": v}
