"""Token sharding through the CUDA path, on one device: the estimator run on
two shards of a batch (token_offset = the shard's first token; whole
sequences for the attention internals) reproduces the run over the whole
batch — every token's loss, rewards and g row, and G_W as the sum of the
shards' G_W. This is the decomposition the multi-rank path relies on
(tokens are independent units of the estimator and G_W is a sum over
tokens), here as two sequential calls; the all-reduce itself is tested with
gloo ranks on the CPU.

Tolerances: the shards and the whole run compute each token's row with the
same arithmetic, but fp32 sums whose order depends on the tiling of the batch
(the reward's partial sums over vocabulary tiles, G_W's sum over tokens) may
round differently, so values agree to a few fp32 ulps of their size rather
than bit for bit.
"""
import numpy as np
import pytest
import torch

import synth
import zeroth_order_transformer_dust_b200 as dust
from _util import np64, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


def _compare(whole, parts, spans, keys):
    for k in keys:
        stacked = np.concatenate([p[k] for p in parts], axis=0)
        assert stacked.shape == whole[k].shape
        scale = max(np.abs(whole[k]).max(), 1e-30)
        assert np.abs(stacked - whole[k]).max() <= 1e-5 * scale, k
    G = sum(p["G"] for p in parts)
    assert rel_fro(G, whole["G"]) < 1e-5
    assert sum(n for _, n in spans) == whole["g"].shape[0]


@pytest.mark.parametrize("S,dtype", [(50, "bf16"), (0, "bf16"), (50, "f32")])
def test_head_shards(ctx, S, dtype):
    wl = synth.Workload("shard_head", "head", T=40, d=64, V=1000, K=48, S=S, sigma=1e-2, seed=17,
                        dtype=dtype, targets="zipf")
    inp = synth.make_head_inputs(wl)
    W = to_dev(inp["W"], dtype)
    kw = dict(K=wl.K, sigma=wl.sigma, S=S, seed=wl.seed, want_rewards=True, want_g=True)

    def run(t0, n):
        out = ctx.head_grad(to_dev(inp["H"][t0:t0 + n], dtype), W,
                            to_dev(inp["targets"][t0:t0 + n], "i32"), token_offset=t0, **kw)
        torch.cuda.synchronize()
        return {k: np64(v) for k, v in out.items()}

    spans = [(0, 27), (27, 13)]
    _compare(run(0, wl.T), [run(t0, n) for t0, n in spans], spans, ("loss", "rewards", "g"))


def test_mlp_shards(ctx):
    wl = synth.Workload("shard_mlp", "mlp", T=24, d=64, d_ff=256, V=1000, K=16, S=0, sigma=1e-2,
                        seed=19, dtype="bf16", targets="zipf")
    inp = synth.make_mlp_inputs(wl)
    Ws = [to_dev(inp[k], "bf16") for k in ("W_up", "W_down", "W_head")]

    def run(t0, n):
        out = ctx.mlp_grad(to_dev(inp["X"][t0:t0 + n], "bf16"), *Ws,
                           to_dev(inp["targets"][t0:t0 + n], "i32"), K=wl.K, sigma=wl.sigma,
                           seed=wl.seed, token_offset=t0, want_rewards=True, want_g=True)
        torch.cuda.synchronize()
        return {k: np64(v) for k, v in out.items()}

    spans = [(0, 16), (16, 8)]
    _compare(run(0, wl.T), [run(t0, n) for t0, n in spans], spans, ("loss", "rewards", "g"))


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_attention_shards_by_whole_sequences(ctx, which):
    wl = synth.CONFIGS["attn_q_bf16"].with_(T=120, d=48, seq_len=40, n_heads=2, head_dim=64,
                                            K=40)
    x = synth.make_attn_inputs(wl)

    def run(t0, n):
        sl = slice(t0, t0 + n)
        dev = [to_dev(x[k][sl], "f32") for k in ("Q", "K", "V", "E")]
        out = ctx.attn_grad(to_dev(x["X"][sl], "bf16"), *dev, seq_len=wl.seq_len,
                            n_heads=wl.n_heads, which=which, K=wl.K, sigma=wl.sigma,
                            seed=wl.seed, token_offset=t0, want_rewards=True, want_g=True)
        torch.cuda.synchronize()
        return {k: np64(v) for k, v in out.items()}

    spans = [(0, 80), (80, 40)]
    _compare(run(0, wl.T), [run(t0, n) for t0, n in spans], spans, ("rewards", "g"))


@pytest.mark.parametrize("S,dtype", [(50, "bf16"), (0, "bf16"), (50, "f32")])
def test_head_draw_shards(ctx, S, dtype):
    """Draw sharding: two calls over every token with disjoint draw ranges
    (draw_offset = the range's first draw) give the whole run's rewards as
    their columns, and its g and G_W once each is weighted by its share of
    the draws (parallel.combine_draw_shards, here without a process group)."""
    from zeroth_order_transformer_dust_b200.parallel import combine_draw_shards, draw_shard
    wl = synth.Workload("shard_draws", "head", T=24, d=64, V=1000, K=45, S=S, sigma=1e-2,
                        seed=19, dtype=dtype, targets="zipf")
    inp = synth.make_head_inputs(wl)
    H, W, y = to_dev(inp["H"], dtype), to_dev(inp["W"], dtype), to_dev(inp["targets"], "i32")
    kw = dict(sigma=wl.sigma, S=S, seed=wl.seed, want_rewards=True, want_g=True)
    whole = ctx.head_grad(H, W, y, K=wl.K, **kw)
    G = torch.zeros_like(whole["G"])
    g = torch.zeros_like(whole["g"])
    for rank in range(2):
        i0, k = draw_shard(wl.K, 2, rank)
        part = ctx.head_grad(H, W, y, K=k, draw_offset=i0, **kw)
        torch.cuda.synchronize()
        assert torch.equal(part["rewards"], whole["rewards"][:, i0:i0 + k])
        G += combine_draw_shards(part["G"], k, wl.K)
        g += combine_draw_shards(part["g"], k, wl.K)
    torch.cuda.synchronize()
    assert rel_fro(np64(g), np64(whole["g"])) < 1e-5
    assert rel_fro(np64(G), np64(whole["G"])) < (2e-3 if dtype == "bf16" else 1e-5)
