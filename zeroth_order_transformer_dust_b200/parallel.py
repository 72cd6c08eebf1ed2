"""Token-sharded estimator across GPUs (one process per GPU).

Tokens are independent units of the estimator ("Dust：无需反向传播的
Transformer零阶预训练", §1: every token is its own population member) and the
weight gradient is a sum over tokens (G_W = sum_t g_t x_t^T), so a batch splits
across ranks by tokens: rank r runs the estimator on its contiguous token
range with token_offset = start, which reproduces exactly the noise a single
run over the whole batch would draw, and one sum all-reduce of the per-rank
G_W (NCCL over NVLink/NVSwitch on GPUs) gives the estimate of the full batch.

The draws split the same way: rank r can run every token with its own
contiguous range of the K draws (draw_offset = its first draw), again the
noise of a single run. Its estimate carries 1/K_r for its K_r draws, so it is
weighted by K_r / K before the same sum all-reduce (draw_shard,
combine_draw_shards).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def token_shard(T_total: int, world: int, rank: int) -> Tuple[int, int]:
    """(first token, token count) of `rank`'s contiguous share of T_total tokens.

    The first T_total % world ranks take one extra token; shares are disjoint
    and cover [0, T_total) in rank order.
    """
    if world < 1 or not 0 <= rank < world or T_total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def sequence_shard(T_total: int, seq_len: int, world: int, rank: int) -> Tuple[int, int]:
    """(first token, token count) of `rank`'s share when the batch must split
    at sequence boundaries: the attention-internals estimator couples the
    tokens of one sequence (noise on a key or value row moves the outputs of
    every later token of its sequence), so ranks take whole sequences of
    seq_len tokens, distributed as token_shard distributes tokens."""
    if seq_len < 1 or T_total % seq_len:
        raise ValueError("T_total must be a positive multiple of seq_len")
    first, count = token_shard(T_total // seq_len, world, rank)
    return first * seq_len, count * seq_len


def draw_shard(K_total: int, world: int, rank: int) -> Tuple[int, int]:
    """(first draw, draw count) of `rank`'s contiguous share of K_total draws,
    distributed as token_shard distributes tokens."""
    return token_shard(K_total, world, rank)


def combine_draw_shards(x: torch.Tensor, K_local: int, K_total: int,
                        group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """In place: the estimate over all K_total draws from this rank's estimate
    over its K_local draws, x <- sum over ranks of (K_local / K_total) x. The
    estimator scales its sum over draws by 1/K, so the weighted sum equals a
    single run over all draws (G_W, or g_t of the same tokens)."""
    if K_total < 1 or not 0 <= K_local <= K_total:
        raise ValueError("bad draw counts")
    x.mul_(K_local / K_total)
    return allreduce_weight_grad(x, group)


def allreduce_weight_grad(G: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Sum the per-rank weight-gradient estimates in place (G_W over all tokens)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(G, op=dist.ReduceOp.SUM, group=group)
    return G


def sharded_head_grad(ctx, H_local: torch.Tensor, W: torch.Tensor, y_local: torch.Tensor,
                      token_offset: int, group: Optional[dist.ProcessGroup] = None, **kw) -> dict:
    """LM-head estimator over this rank's tokens, G_W summed over all ranks.

    H_local / y_local hold this rank's tokens, which start at absolute token
    `token_offset` of the batch (see token_shard). Returns the rank's outputs
    with "G" replaced by the all-reduced estimate.
    """
    out = ctx.head_grad(H_local, W, y_local, token_offset=token_offset, **kw)
    if "G" in out:
        allreduce_weight_grad(out["G"], group)
    return out


def sharded_mlp_grad(ctx, X_local: torch.Tensor, W_up: torch.Tensor, W_down: torch.Tensor,
                     W_head: torch.Tensor, y_local: torch.Tensor, token_offset: int,
                     group: Optional[dist.ProcessGroup] = None, **kw) -> dict:
    """Hidden-MLP estimator over this rank's tokens (split as token_shard
    splits them), G_W summed over all ranks."""
    out = ctx.mlp_grad(X_local, W_up, W_down, W_head, y_local, token_offset=token_offset, **kw)
    if "G" in out:
        allreduce_weight_grad(out["G"], group)
    return out


def sharded_attn_grad(ctx, X_local: torch.Tensor, Q_local: torch.Tensor, K_local: torch.Tensor,
                      V_local: torch.Tensor, E_local: torch.Tensor, token_offset: int,
                      group: Optional[dist.ProcessGroup] = None, **kw) -> dict:
    """Attention-internals estimator over this rank's whole sequences (see
    sequence_shard; token_offset is the rank's first token), G_W summed over
    all ranks."""
    out = ctx.attn_grad(X_local, Q_local, K_local, V_local, E_local, token_offset=token_offset,
                        **kw)
    if "G" in out:
        allreduce_weight_grad(out["G"], group)
    return out
