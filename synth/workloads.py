"""Workload table and seeded input generators.

Recipe (all host-side, numpy PCG64; the workload seed's SeedSequence spawns
one child stream per tensor, in the order H, W, targets for the LM-head
workloads, x, W_up, W_down, W_head, targets, O for the MLP-block workloads and
x, Q, K, V, E for the attention-internals workloads):

* H ~ N(0, 1), then each row divided by its RMS sqrt(mean(h^2)).
* W ~ N(0, 1/d), so logits z = W h are roughly N(0, 1) per entry.
* MLP: x ~ N(0, 1); W_up ~ N(0, 1/d); W_down ~ N(0, 1/d_ff); W_head ~ N(0, 1/d);
  the attention output O ~ N(0, 1) for the output-projection variant.
* Attention internals: the projection input x ~ N(0, 1) (rounded like the
  other float inputs); the cached projections Q, K, V ~ N(0, 1) in fp32, so
  the scores q.k / sqrt(d_h) are about N(0, 1); the error signal at the
  attention output E ~ N(0, 1) in fp32. Sequences of L tokens, H heads of
  width d_h, as in a GPT-2-small block.
* targets: uniform on [0, V) for the tiny fp32 workload, otherwise a
  Zipf(1.1) law truncated to ranks 1..V (rank k -> token id k-1), sampled by
  inverse CDF.
* bf16 workloads round every float input to bf16 (round to nearest even)
  on the host; the returned float32 arrays hold exactly those bf16 values.

The shapes follow the Dust pages' model scale (a 1024-wide head over a
50304-entry vocabulary, populations of 64 to 16k draws); the pages train on
FineWeb, which these synthetic inputs stand in for.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    variant: str        # "head", "mlp" (up-projection), "mlp_down", "attn_out",
                        # or "attn_q" / "attn_k" / "attn_v" (attention internals)
    T: int
    d: int
    V: int
    K: int
    S: int              # <= 0: full vocabulary
    sigma: float
    seed: int
    dtype: str          # "f32" or "bf16"
    targets: str        # "uniform" or "zipf"
    d_ff: int = 0
    seq_len: int = 0    # attention internals: tokens per sequence
    n_heads: int = 0
    head_dim: int = 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def token_draws(self) -> int:
        return self.T * self.K


CONFIGS = {
    # Tiny LM-head estimator, fp32 end to end, full vocabulary.
    "tiny_fp32": Workload("tiny_fp32", "head", T=128, d=64, V=1024, K=16, S=0,
                          sigma=0.05, seed=0, dtype="f32", targets="uniform"),
    # LM head, full vocabulary, bf16 operands.
    "full_bf16": Workload("full_bf16", "head", T=4096, d=512, V=50304, K=64, S=0,
                          sigma=1e-2, seed=1, dtype="bf16", targets="zipf"),
    # LM head, vocabulary-subset draws (S = 256).
    "subset_bf16": Workload("subset_bf16", "head", T=8192, d=1024, V=50304, K=1024,
                            S=256, sigma=1e-2, seed=2, dtype="bf16", targets="zipf"),
    # Hidden MLP up-projection.
    "mlp_bf16": Workload("mlp_bf16", "mlp", T=8192, d=768, V=50304, K=256, S=0,
                         sigma=1e-2, seed=3, dtype="bf16", targets="zipf", d_ff=3072),
    # Hidden MLP down-projection (noise on W_down's output), same shapes.
    "mlp_down_bf16": Workload("mlp_down_bf16", "mlp_down", T=8192, d=768, V=50304, K=256, S=0,
                              sigma=1e-2, seed=3, dtype="bf16", targets="zipf", d_ff=3072),
    # Attention output projection writing into the MLP block's input, same shapes.
    "attn_out_bf16": Workload("attn_out_bf16", "attn_out", T=8192, d=768, V=50304, K=256, S=0,
                              sigma=1e-2, seed=3, dtype="bf16", targets="zipf", d_ff=3072),
    # Attention internals: noise on the query, key or value projection's
    # output of a 12-head, 768-wide causal attention over 8 sequences of 1024.
    "attn_q_bf16": Workload("attn_q_bf16", "attn_q", T=8192, d=768, V=1, K=256, S=0,
                            sigma=1e-2, seed=5, dtype="bf16", targets="none", seq_len=1024,
                            n_heads=12, head_dim=64),
    "attn_k_bf16": Workload("attn_k_bf16", "attn_k", T=8192, d=768, V=1, K=256, S=0,
                            sigma=1e-2, seed=5, dtype="bf16", targets="none", seq_len=1024,
                            n_heads=12, head_dim=64),
    "attn_v_bf16": Workload("attn_v_bf16", "attn_v", T=8192, d=768, V=1, K=256, S=0,
                            sigma=1e-2, seed=5, dtype="bf16", targets="none", seq_len=1024,
                            n_heads=12, head_dim=64),
    # The subset estimator at a 128256-entry vocabulary (a Llama-3-size head):
    # the shared-memory kernel with a cluster of 8 CTAs per token.
    "subset_v128k_bf16": Workload("subset_v128k_bf16", "head", T=8192, d=1024, V=128256,
                                  K=1024, S=512, sigma=1e-2, seed=6, dtype="bf16",
                                  targets="zipf"),
    # Subset draws of S = 1024 entries: eight 128-slot blocks a draw in the
    # shared-memory kernel (16 warps per SM).
    "subset_s1024_bf16": Workload("subset_s1024_bf16", "head", T=8192, d=1024, V=50304,
                                  K=1024, S=1024, sigma=1e-2, seed=7, dtype="bf16",
                                  targets="zipf"),
    # LM head at 243M-model head scale, subset draws (S = 512), 16k draws.
    "large_subset_bf16": Workload("large_subset_bf16", "head", T=16384, d=1024, V=50304,
                                  K=16384, S=512, sigma=5e-3, seed=4, dtype="bf16",
                                  targets="zipf"),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((bits >> 16) & 1)
    out = ((bits + bias) & 0xFFFF0000).astype(np.uint32)
    return out.view(np.float32).reshape(x.shape)


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x.astype(np.float32)
    return bf16_round(x32) if dtype == "bf16" else x32


def zipf_targets(rng: np.random.Generator, n: int, V: int, s: float = 1.1) -> np.ndarray:
    """Truncated Zipf(s) over ranks 1..V by inverse CDF; returns ids rank-1."""
    ranks = np.arange(1, V + 1, dtype=np.float64)
    pmf = ranks ** (-s)
    cdf = np.cumsum(pmf)
    cdf /= cdf[-1]
    u = rng.random(n)
    idx = np.searchsorted(cdf, u, side="right")
    return np.minimum(idx, V - 1).astype(np.int32)


def _targets(rng, wl: Workload) -> np.ndarray:
    if wl.targets == "uniform":
        return rng.integers(0, wl.V, size=wl.T, dtype=np.int64).astype(np.int32)
    return zipf_targets(rng, wl.T, wl.V)


def _streams(seed: int, n: int):
    """Independent child generators, one per input tensor, so that the size of
    one tensor never shifts the values of another (a workload cut to its first
    T tokens keeps the same weights and the same first T rows and targets)."""
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def make_head_inputs(wl: Workload) -> dict:
    """H (T x d), W (V x d), targets (T,) for an LM-head workload."""
    rH, rW, ry = _streams(wl.seed, 3)
    H = rH.standard_normal((wl.T, wl.d))
    H /= np.sqrt(np.mean(H * H, axis=1, keepdims=True))
    W = rW.standard_normal((wl.V, wl.d)) * (1.0 / np.sqrt(wl.d))
    y = _targets(ry, wl)
    return {"H": _cast(H, wl.dtype), "W": _cast(W, wl.dtype), "targets": y}


def make_mlp_inputs(wl: Workload) -> dict:
    """x (T x d), W_up (d_ff x d), W_down (d x d_ff), W_head (V x d), targets, and
    O (T x d ~ N(0, 1)), the attention output the output-projection variant
    takes as its layer input (its own sixth stream, so the others are unchanged)."""
    rX, rU, rD, rHd, ry, rO = _streams(wl.seed, 6)
    X = rX.standard_normal((wl.T, wl.d))
    W_up = rU.standard_normal((wl.d_ff, wl.d)) * (1.0 / np.sqrt(wl.d))
    W_down = rD.standard_normal((wl.d, wl.d_ff)) * (1.0 / np.sqrt(wl.d_ff))
    W_head = rHd.standard_normal((wl.V, wl.d)) * (1.0 / np.sqrt(wl.d))
    y = _targets(ry, wl)
    O = rO.standard_normal((wl.T, wl.d))
    return {"X": _cast(X, wl.dtype), "W_up": _cast(W_up, wl.dtype),
            "W_down": _cast(W_down, wl.dtype), "W_head": _cast(W_head, wl.dtype),
            "targets": y, "O": _cast(O, wl.dtype)}


def make_attn_inputs(wl: Workload) -> dict:
    """x (T x d), the cached projections Q, K, V (T x D, fp32) and the error
    signal E at the attention output (T x D, fp32), D = n_heads head_dim."""
    rX, rQ, rK, rV, rE = _streams(wl.seed, 5)
    D = wl.n_heads * wl.head_dim
    X = rX.standard_normal((wl.T, wl.d))
    out = {"X": _cast(X, wl.dtype)}
    for name, r in (("Q", rQ), ("K", rK), ("V", rV), ("E", rE)):
        out[name] = r.standard_normal((wl.T, D)).astype(np.float32)
    return out
