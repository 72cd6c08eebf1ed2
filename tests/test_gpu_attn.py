"""Attention-internals estimator on the GPU against the oracle ("Dust：无需反向传播
的Transformer零阶预训练", §1: the attention internals' reward comes from the
change of the attention output; only the attention output is recomputed).

Tolerances. The kernels evaluate the per-head rewards in closed forms of the
clean attention in fp32 (sums over at most L rows of terms of relative
precision ~2^-23), so the rewards are compared within 2e-5 absolute plus
1e-5 of their size (they reach ~0.7 here, against ~0.03 for the LM head);
g within 1e-4 relative Frobenius; G within 1e-5 (fp32 input) or 2e-3 (bf16
input) relative Frobenius, the bars of the other variants.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import zeroth_order_transformer_dust_b200 as dust
from _util import np64, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


def _run(ctx, wl, which, **kw):
    x = synth.make_attn_inputs(wl)
    dev = {k: to_dev(v, "f32") for k, v in x.items() if k != "X"}
    X = to_dev(x["X"], wl.dtype)
    out = ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=wl.seq_len,
                        n_heads=wl.n_heads, which=which, K=wl.K, sigma=wl.sigma, seed=wl.seed,
                        want_rewards=True, want_g=True, **kw)
    torch.cuda.synchronize()
    return x, {k: np64(v) for k, v in out.items()}


def _oracle(wl, x, which, **kw):
    prm = oracle.Params(T=wl.T, d=wl.d, V=1, K=wl.K, sigma=wl.sigma, seed=wl.seed, **kw)
    return oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], wl.seq_len, wl.n_heads,
                            which, prm)


def _check(got, ref, dtype):
    dr = np.abs(got["rewards"] - ref["rewards"])
    assert np.all(dr <= 2e-5 + 1e-5 * np.abs(ref["rewards"])), dr.max()
    assert rel_fro(got["g"], ref["g"]) < 1e-4
    assert rel_fro(got["G"], ref["G"]) < (2e-3 if dtype == "bf16" else 1e-5)


BASE = synth.CONFIGS["attn_q_bf16"].with_(T=80, d=96, seq_len=40, n_heads=3, head_dim=64, K=300)


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_parity_two_sequences(ctx, which):
    # 40-token sequences (a 64-row tile plus nothing, and ragged), 300 draws
    # (two rounds of 256 threads, the second ragged), three 64-wide heads
    x, got = _run(ctx, BASE, which)
    _check(got, _oracle(BASE, x, which), "bf16")


@pytest.mark.parametrize("head_dim,which", [(32, "q"), (32, "k"), (128, "k"), (128, "v")])
def test_parity_other_head_widths(ctx, head_dim, which):
    wl = BASE.with_(T=66, seq_len=33, n_heads=2, head_dim=head_dim, K=70, d=40, dtype="f32")
    x, got = _run(ctx, wl, which)
    _check(got, _oracle(wl, x, which), "f32")


def test_wide_heads_two_rounds(ctx):
    # 128-wide heads on the tensor cores (two K blocks per operand) with two
    # rounds of draws
    wl = BASE.with_(T=70, seq_len=35, n_heads=2, head_dim=128, K=300, d=24)
    x, got = _run(ctx, wl, "q")
    _check(got, _oracle(wl, x, "q"), "bf16")


@pytest.mark.parametrize("which", ["q", "k"])
def test_large_sigma(ctx, which):
    # sigma = 0.5: the score changes reach far beyond 1/16, so the exact expm1
    # path of the epilogues runs as well as the series
    wl = BASE.with_(T=40, seq_len=20, n_heads=2, K=64, d=16, sigma=0.5)
    x, got = _run(ctx, wl, which)
    _check(got, _oracle(wl, x, which), "bf16")


def test_long_sequence_tiles(ctx):
    # 150 keys per row at the end: three 64-row tiles, the last ragged
    wl = BASE.with_(T=150, seq_len=150, n_heads=1, K=20, d=24)
    for which in ("q", "k"):
        x, got = _run(ctx, wl, which)
        _check(got, _oracle(wl, x, which), "bf16")


@pytest.mark.parametrize("which", ["q", "k"])
def test_cuda_core_path(ctx, which, monkeypatch):
    # the CUDA-core form of the query and key draws (the tensor-core form is
    # the default for head widths 64 and 128)
    monkeypatch.setenv("DUST_ATTN_TC", "0")
    x, got = _run(ctx, BASE, which)
    _check(got, _oracle(BASE, x, which), "bf16")


def test_tensor_core_range_is_reported(ctx, monkeypatch):
    # fp16 operands hold |x| < 32768: a larger key is reported, not wrapped
    wl = BASE.with_(T=20, seq_len=10, n_heads=2, K=8, d=8)
    x = synth.make_attn_inputs(wl)
    dev = {k: to_dev(v, "f32") for k, v in x.items() if k != "X"}
    X = to_dev(x["X"], "bf16")
    dev["K"][3, 5] = 1e6
    with pytest.raises(dust.DustError, match="fp16 range"):
        ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=10, n_heads=2,
                      which="q", K=8, sigma=1e-2)
    # the context stays usable, and the CUDA-core path takes the same input
    monkeypatch.setenv("DUST_ATTN_TC", "0")
    ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=10, n_heads=2, which="q",
                  K=8, sigma=1e-2)
    torch.cuda.synchronize()


def test_offsets_and_stream(ctx):
    wl = BASE.with_(T=24, seq_len=12, n_heads=2, K=40, d=16)
    x, got = _run(ctx, wl, "k", token_offset=1000, draw_offset=77, stream_id=5)
    ref = _oracle(wl, x, "k", token_offset=1000, draw_offset=77, stream_id=5)
    _check(got, ref, "bf16")


def test_one_token_sequences(ctx):
    wl = BASE.with_(T=12, seq_len=1, n_heads=2, K=16, d=8)
    for which in ("q", "k", "v"):
        x, got = _run(ctx, wl, which)
        ref = _oracle(wl, x, which)
        _check(got, ref, "bf16")
        if which != "v":
            assert np.abs(got["rewards"]).max() < 1e-6     # a one-key softmax cannot move


def test_sigma_zero_is_exactly_zero(ctx):
    wl = BASE.with_(T=20, seq_len=10, n_heads=2, K=8, d=8, sigma=0.0)
    for which in ("q", "k", "v"):
        _, got = _run(ctx, wl, which)
        assert not got["rewards"].any() and not got["g"].any() and not got["G"].any()


def test_rejects_bad_shapes(ctx):
    wl = BASE.with_(T=20, seq_len=10, n_heads=2, K=8, d=8)
    x = synth.make_attn_inputs(wl)
    dev = {k: to_dev(v, "f32") for k, v in x.items() if k != "X"}
    X = to_dev(x["X"], "bf16")
    with pytest.raises(dust.DustError):     # T not a multiple of seq_len
        ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=7, n_heads=2,
                      which="q", K=8, sigma=1e-2)
    with pytest.raises(dust.DustError):     # head_dim 16
        ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=10, n_heads=8,
                      which="q", K=8, sigma=1e-2)
    with pytest.raises(ValueError):
        ctx.attn_grad(X, dev["Q"], dev["K"], dev["V"], dev["E"], seq_len=10, n_heads=2,
                      which="o", K=8, sigma=1e-2)


@pytest.mark.parametrize("name", ["attn_q_bf16", "attn_k_bf16", "attn_v_bf16"])
def test_full_size_sampled_tokens(ctx, name):
    # the benchmark workload (8 sequences of 1024, 12 heads of 64, K = 256) in
    # the launch configuration bench.py times; the oracle recomputes the
    # perturbed attention for sampled tokens and the first draws
    wl = synth.CONFIGS[name]
    which = wl.variant[-1]
    x, got = _run(ctx, wl, which)
    L, H = wl.seq_len, wl.n_heads
    draws = np.arange(3)
    tag = oracle.attn.WHICH_TAG[which]
    for s in (0, 1023, 4100, 8191):
        b, pos = divmod(s, L)
        rows = slice(b * L, (b + 1) * L)
        Ob, _ = oracle.attention_seq(x["Q"][rows], x["K"][rows], x["V"][rows], H)
        eps = oracle.gaussians(wl.seed, s, draws, np.arange(H * wl.head_dim), tag)
        r, _ = oracle.attn_draws(x["Q"][rows], x["K"][rows], x["V"][rows], Ob, x["E"][rows], H,
                                 pos, which, eps, np.float32(wl.sigma).item())
        dr = np.abs(got["rewards"][s, :3] - r)
        assert np.all(dr <= 2e-5 + 1e-5 * np.abs(r)), (s, dr)
    assert np.all(np.isfinite(got["G"])) and np.all(np.isfinite(got["g"]))
