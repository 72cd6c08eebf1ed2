"""Multi-step training of the LM head with the Dust estimator and SGD momentum.

Each step runs the estimator (``dust_head_grad``) on the current weights,
optionally sums the weight gradient across data-parallel ranks, and applies
the heavy-ball update (``dust_sgd_momentum``) to the fp32 master weights,
refreshing the bf16 copy the next step reads. Step s draws its noise at draw
indices [s K, (s+1) K) of the seed, so every step has fresh noise and a
resumed run (``first_step``) continues the same stream. Argument marshalling
only: every step runs in the library's kernels.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def train_head(ctx, H: torch.Tensor, W_master: torch.Tensor, targets: torch.Tensor, *,
               steps: int, lr: float, mu: float, K: int, sigma: float, S: int = 0,
               seed: int = 0, token_offset: int = 0, W_lp: Optional[torch.Tensor] = None,
               v: Optional[torch.Tensor] = None, first_step: int = 0,
               allreduce: Optional[Callable[[torch.Tensor], None]] = None) -> dict:
    """``steps`` updates of W_master (V x d fp32, in place).

    W_lp: bf16 copy the estimator reads (H must then be bf16); None runs the
    estimator on W_master itself (fp32 H). v: momentum buffer (zeros if None).
    Returns the per-step mean clean loss of this rank's tokens (before each
    update, on the host) and the momentum buffer."""
    if W_master.dtype != torch.float32:
        raise TypeError("W_master must be fp32")
    W_read = W_lp if W_lp is not None else W_master
    if W_read.dtype != H.dtype:
        raise TypeError("H must have the dtype of the weights the estimator reads")
    v = torch.zeros_like(W_master) if v is None else v
    G = torch.empty_like(W_master)
    loss = torch.empty(H.shape[0], dtype=torch.float32, device=H.device)
    losses = torch.empty(steps, dtype=torch.float32, device=H.device)
    for s in range(steps):
        ctx.head_grad(H, W_read, targets, K=K, sigma=sigma, S=S, seed=seed,
                      token_offset=token_offset, draw_offset=(first_step + s) * K,
                      out={"G": G, "loss": loss}, asynchronous=True)
        if allreduce is not None:
            allreduce(G)
        losses[s] = loss.mean()
        ctx.sgd_momentum(G, v, W_master, lr=lr, mu=mu, W_bf16=W_lp)
    ctx.check()
    return {"losses": losses.cpu(), "v": v}
