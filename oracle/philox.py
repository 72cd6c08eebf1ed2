"""Counter-based noise for the oracle: Philox4x32-10 and Box-Muller.

The Dust pages say only that the noise is Gaussian, drawn independently per
token and per draw ("Dust：无需反向传播的Transformer零阶预训练", §1,
激活空间扰动). The generator is this build's reading, implemented here from
its published definition, independently of the CUDA path:

Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
as 1, 2, 3", SC'11): a 4 x 32-bit counter and a 2 x 32-bit key; ten rounds,
each multiplying counter words 0 and 2 by 0xD2511F53 and 0xCD9E8D57 into
64-bit products and recombining hi/lo halves with XORs of the other words and
the key; between rounds the key is bumped by (0x9E3779B9, 0xBB67AE85).

Counter layout (this build's reading; the pages are silent):
  key  = (seed & 0xffffffff, seed >> 32)
  ctr1 = token index (t + token_offset), ctr2 = draw index (i + draw_offset),
  ctr3 = tag | (stream_id << 8)
  A slot k (vocabulary index, subset slot or hidden channel) takes output
  word ((k >> 5) & 3) of the counter with ctr0 = ((k >> 7) << 5) | (k & 31).

Gaussians (Box-Muller on 24-bit uniforms): words (w0, w1) give
(R cos 2 pi u2, R sin 2 pi u2) for output words 0 and 1, words (w2, w3) the
same for output words 2 and 3, with u1 = ((wa >> 8) + 1) 2^-24 in (0, 1],
u2 = (wb >> 8) 2^-24 in [0, 1), R = sqrt(-2 ln u1). |eps| <= sqrt(48 ln 2).
"""
from __future__ import annotations

import math

import numpy as np

MASK32 = np.uint64(0xFFFFFFFF)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_S32 = np.uint64(32)

TAG_HEAD = 0           # noise on the LM-head logits
TAG_SUBSET_OFFSET = 1  # the per-draw subset offset b
TAG_MLP_UP = 2         # noise on the MLP up-projection output
TAG_MLP_DOWN = 3       # noise on the MLP down-projection output
TAG_ATTN_OUT = 4       # noise on the attention output projection's output
TAG_ATTN_Q = 5         # noise on the query projection's output
TAG_ATTN_K = 6         # noise on the key projection's output
TAG_ATTN_V = 7         # noise on the value projection's output


def _u32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.uint64) & MASK32


def philox4x32_10(ctr, key):
    """Philox4x32-10 of counter (c0, c1, c2, c3) under key (k0, k1).

    Arguments broadcast; each is an integer array holding 32-bit values.
    Returns four uint64 arrays holding the 32-bit output words.
    """
    c0, c1, c2, c3 = (_u32(c) for c in ctr)
    k0, k1 = (_u32(k) for k in key)
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + _W0) & MASK32
            k1 = (k1 + _W1) & MASK32
        prod0 = _M0 * c0          # < 2^64: exact in uint64
        prod1 = _M1 * c2
        hi0, lo0 = prod0 >> _S32, prod0 & MASK32
        hi1, lo1 = prod1 >> _S32, prod1 & MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def seed_key(seed: int):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.uint64(seed & 0xFFFFFFFF), np.uint64(seed >> 32)


def box_muller(wa, wb):
    """Two N(0,1) values from two 32-bit words (fp64)."""
    wa = np.asarray(wa, dtype=np.uint64)
    wb = np.asarray(wb, dtype=np.uint64)
    u1 = ((wa >> np.uint64(8)) + np.uint64(1)).astype(np.float64) * 2.0 ** -24
    u2 = (wb >> np.uint64(8)).astype(np.float64) * 2.0 ** -24
    radius = np.sqrt(-2.0 * np.log(u1))
    theta = 2.0 * math.pi * u2
    return radius * np.cos(theta), radius * np.sin(theta)


def slot_counter_word(k):
    """Counter word 0 and output word index that carry slot k."""
    k = np.asarray(k, dtype=np.int64)
    ctr0 = ((k >> 7) << 5) | (k & 31)
    word = (k >> 5) & 3
    return ctr0, word


def _ctr3(tag: int, stream_id: int) -> int:
    return (int(tag) & 0xFF) | ((int(stream_id) & 0xFFFFFF) << 8)


def gaussians(seed: int, t_abs, i_abs, slots, tag: int, stream_id: int = 0) -> np.ndarray:
    """eps(seed, t, i, k) for the given slots.

    ``t_abs`` and ``i_abs`` are absolute token and draw indices (offsets already
    added) and must broadcast against each other; ``slots`` is a 1-D array of
    slot indices. The result has shape broadcast(t_abs, i_abs).shape + (n,).
    """
    slots = np.asarray(slots, dtype=np.int64)
    ctr0, word = slot_counter_word(slots)
    t = np.asarray(t_abs, dtype=np.uint64)[..., None]
    i = np.asarray(i_abs, dtype=np.uint64)[..., None]
    k0, k1 = seed_key(seed)
    w = philox4x32_10((ctr0.astype(np.uint64), t, i, np.uint64(_ctr3(tag, stream_id))), (k0, k1))
    n0, n1 = box_muller(w[0], w[1])
    n2, n3 = box_muller(w[2], w[3])
    out = np.where(word == 0, n0, np.where(word == 1, n1, np.where(word == 2, n2, n3)))
    return out


def subset_offset(seed: int, t_abs, i_abs, V: int, stream_id: int = 0) -> np.ndarray:
    """The per-(token, draw) subset offset b = floor(w0 * V / 2^32)."""
    k0, k1 = seed_key(seed)
    t = np.asarray(t_abs, dtype=np.uint64)
    i = np.asarray(i_abs, dtype=np.uint64)
    w = philox4x32_10((np.uint64(0), t, i, np.uint64(_ctr3(TAG_SUBSET_OFFSET, stream_id))), (k0, k1))
    return ((w[0] * np.uint64(V)) >> _S32).astype(np.int64)


def default_subset_a(V: int) -> int:
    """Smallest integer >= V (sqrt(5) - 1) / 2 that is coprime to V."""
    a = int(math.ceil(V * ((math.sqrt(5.0) - 1.0) / 2.0)))
    a = max(a, 1)
    while math.gcd(a, V) != 1:
        a += 1
    return a
