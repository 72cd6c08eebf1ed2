"""MLP-block estimators on the GPU (up-projection, down-projection and the
attention output projection) vs the exact fp64 oracle on the same bf16
inputs: small shapes, calls long enough (T K > 131072 rows) that the
perturbed pass runs in several token chunks with a ragged last one, token
slices of the d=768, d_ff=3072, V=50304 workload, and the full workload in
the benchmark's launch configuration on sampled token rows."""
import numpy as np
import pytest
import torch

import oracle
import synth
import zeroth_order_transformer_dust_b200 as dust
from _util import TOL_G, TOL_GW_BF16, TOL_LOSS, np64, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


def _run(ctx, inp, wl, t0=0, T=None, **kw):
    sl = slice(t0, t0 + (T or wl.T))
    X = inp["X"][sl]
    y = inp["targets"][sl]
    out = ctx.mlp_grad(to_dev(X, "bf16"), to_dev(inp["W_up"], "bf16"), to_dev(inp["W_down"], "bf16"),
                       to_dev(inp["W_head"], "bf16"), to_dev(y, "i32"), K=wl.K, sigma=wl.sigma,
                       seed=wl.seed, token_offset=t0, want_rewards=True, want_g=True, **kw)
    torch.cuda.synchronize()
    got = {k: np64(v) for k, v in out.items()}
    prm = oracle.Params(T=X.shape[0], d=wl.d, V=wl.V, d_ff=wl.d_ff, K=wl.K, sigma=wl.sigma,
                        seed=wl.seed, token_offset=t0, **{k: v for k, v in kw.items() if k == "stream_id"})
    ref = oracle.mlp_grad(X, inp["W_up"], inp["W_down"], inp["W_head"], y, prm)
    return got, ref


def _check(got, ref):
    assert np.abs(got["loss"] - ref["loss"]).max() < TOL_LOSS
    assert np.abs(got["rewards"] - ref["rewards"]).max() < TOL_LOSS
    assert rel_fro(got["g"], ref["g"]) < TOL_G
    assert rel_fro(got["G"], ref["G"]) < TOL_GW_BF16


# sigma 0.05 is the largest the one-plane GEMMs with their first-order
# corrections take; above it both planes are contracted
@pytest.mark.parametrize("kw", [dict(), dict(T=1, K=1), dict(d=33, d_ff=200, V=517), dict(K=130),
                                dict(sigma=0.1), dict(sigma=0.05, K=64), dict(sigma=0.06, K=64)])
def test_small_mlp(ctx, kw):
    base = dict(T=24, d=64, d_ff=256, V=1000, K=16, sigma=1e-2)
    base.update(kw)
    wl = synth.Workload("mlp_small", "mlp", S=0, seed=11, dtype="bf16", targets="zipf", **base)
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run(ctx, inp, wl)
    _check(got, ref)


def test_mlp_sigma_zero(ctx):
    wl = synth.Workload("mlp_small", "mlp", T=8, d=32, d_ff=128, V=300, K=4, S=0, sigma=0.0,
                        seed=2, dtype="bf16", targets="zipf")
    inp = synth.make_mlp_inputs(wl)
    got, _ = _run(ctx, inp, wl)
    assert np.all(got["rewards"] == 0) and np.all(got["g"] == 0) and np.all(got["G"] == 0)


def test_mlp_workload_slice(ctx):
    wl = synth.CONFIGS["mlp_bf16"]
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run(ctx, inp, wl, t0=5000, T=3)
    _check(got, ref)


# ---- down-projection variant ----------------------------------------------

def _run_down(ctx, inp, wl, t0=0, T=None):
    sl = slice(t0, t0 + (T or wl.T))
    X = inp["X"][sl]
    y = inp["targets"][sl]
    out = ctx.mlp_grad(to_dev(X, "bf16"), to_dev(inp["W_up"], "bf16"), to_dev(inp["W_down"], "bf16"),
                       to_dev(inp["W_head"], "bf16"), to_dev(y, "i32"), K=wl.K, sigma=wl.sigma,
                       seed=wl.seed, token_offset=t0, want_rewards=True, want_g=True, layer="down")
    torch.cuda.synchronize()
    got = {k: np64(v) for k, v in out.items()}
    prm = oracle.Params(T=X.shape[0], d=wl.d, V=wl.V, d_ff=wl.d_ff, K=wl.K, sigma=wl.sigma,
                        seed=wl.seed, token_offset=t0)
    ref = oracle.mlp_down_grad(X, inp["W_up"], inp["W_down"], inp["W_head"], y, prm)
    return got, ref


def _check_down(got, ref):
    _check(got, ref)
    # the weight gradient itself is an fp32 contraction: against g_gpu^T a in fp64
    assert rel_fro(got["G"], got["g"].T @ ref["a"]) < 1e-5


@pytest.mark.parametrize("kw", [dict(), dict(T=1, K=1), dict(d=33, d_ff=200, V=517), dict(K=130),
                                dict(sigma=0.1), dict(sigma=0.05, K=64)])
def test_small_mlp_down(ctx, kw):
    base = dict(T=24, d=64, d_ff=256, V=1000, K=16, sigma=1e-2)
    base.update(kw)
    wl = synth.Workload("mlp_small", "mlp", S=0, seed=12, dtype="bf16", targets="zipf", **base)
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run_down(ctx, inp, wl)
    assert got["G"].shape == (wl.d, wl.d_ff) and got["g"].shape == (wl.T, wl.d)
    _check_down(got, ref)


def test_mlp_down_sigma_zero(ctx):
    wl = synth.Workload("mlp_small", "mlp", T=8, d=32, d_ff=128, V=300, K=4, S=0, sigma=0.0,
                        seed=2, dtype="bf16", targets="zipf")
    inp = synth.make_mlp_inputs(wl)
    got, _ = _run_down(ctx, inp, wl)
    assert np.all(got["rewards"] == 0) and np.all(got["g"] == 0) and np.all(got["G"] == 0)


def test_mlp_down_workload_slice(ctx):
    wl = synth.CONFIGS["mlp_bf16"]
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run_down(ctx, inp, wl, t0=5000, T=3)
    _check_down(got, ref)


# ---- attention output-projection variant ------------------------------------

def _run_attn(ctx, inp, wl, t0=0, T=None):
    sl = slice(t0, t0 + (T or wl.T))
    X, O, y = inp["X"][sl], inp["O"][sl], inp["targets"][sl]
    out = ctx.mlp_grad(to_dev(X, "bf16"), to_dev(inp["W_up"], "bf16"), to_dev(inp["W_down"], "bf16"),
                       to_dev(inp["W_head"], "bf16"), to_dev(y, "i32"), K=wl.K, sigma=wl.sigma,
                       seed=wl.seed, token_offset=t0, want_rewards=True, want_g=True,
                       layer="attn_out", O=to_dev(O, "bf16"))
    torch.cuda.synchronize()
    got = {k: np64(v) for k, v in out.items()}
    prm = oracle.Params(T=X.shape[0], d=wl.d, V=wl.V, d_ff=wl.d_ff, K=wl.K, sigma=wl.sigma,
                        seed=wl.seed, token_offset=t0)
    ref = oracle.attn_out_grad(X, O, inp["W_up"], inp["W_down"], inp["W_head"], y, prm)
    return got, ref


@pytest.mark.parametrize("kw", [dict(), dict(T=1, K=1), dict(d=40, d_ff=200, V=517), dict(K=130),
                                dict(sigma=0.1), dict(sigma=0.05, K=64)])
def test_small_attn_out(ctx, kw):
    base = dict(T=24, d=64, d_ff=256, V=1000, K=16, sigma=1e-2)
    base.update(kw)
    wl = synth.Workload("attn_small", "attn_out", S=0, seed=13, dtype="bf16", targets="zipf", **base)
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run_attn(ctx, inp, wl)
    assert got["G"].shape == (wl.d, wl.d) and got["g"].shape == (wl.T, wl.d)
    _check(got, ref)


def test_attn_out_sigma_zero(ctx):
    wl = synth.Workload("attn_small", "attn_out", T=8, d=32, d_ff=128, V=300, K=4, S=0, sigma=0.0,
                        seed=2, dtype="bf16", targets="zipf")
    inp = synth.make_mlp_inputs(wl)
    got, _ = _run_attn(ctx, inp, wl)
    assert np.all(got["rewards"] == 0) and np.all(got["g"] == 0) and np.all(got["G"] == 0)


def test_attn_out_workload_slice(ctx):
    wl = synth.CONFIGS["attn_out_bf16"]
    inp = synth.make_mlp_inputs(wl)
    got, ref = _run_attn(ctx, inp, wl, t0=5000, T=3)
    _check(got, ref)


def test_attn_out_rejects_bad_O(ctx):
    wl = synth.Workload("attn_small", "attn_out", T=8, d=32, d_ff=128, V=300, K=4, S=0,
                        sigma=1e-2, seed=2, dtype="bf16", targets="zipf")
    inp = synth.make_mlp_inputs(wl)
    args = [to_dev(inp[k], "bf16") for k in ("X", "W_up", "W_down", "W_head")]
    O = torch.zeros(8, 12, dtype=torch.bfloat16, device="cuda")     # d_o not a multiple of 8
    with pytest.raises(dust.DustError):
        ctx.mlp_grad(*args, to_dev(inp["targets"], "i32"), K=4, sigma=1e-2, layer="attn_out", O=O)


# ---- several token chunks in one call ----------------------------------------
# The perturbed pass takes floor(131072 / K) tokens (all K draws each) per
# chunk. These calls run three chunks, the last one ragged, so the chunk
# offsets into u, the logits, the targets and the reward rows are all used.

_RUNNERS = {"up": (_run, _check), "down": (_run_down, _check_down), "attn_out": (_run_attn, _check)}


def _chunk_workload(layer, T, K):
    variant = "attn_out" if layer == "attn_out" else "mlp"
    return synth.Workload("mlp_chunks", variant, T=T, d=32, d_ff=64, V=300, K=K, S=0,
                          sigma=1e-2, seed=21, dtype="bf16", targets="zipf")


@pytest.mark.parametrize("layer", ["up", "down", "attn_out"])
@pytest.mark.parametrize("T,K", [(5, 50000), (7, 40000)])
def test_mlp_block_multi_chunk(ctx, layer, T, K):
    per_chunk = 131072 // K
    assert T > 2 * per_chunk and T % per_chunk != 0     # three chunks, the last one ragged
    wl = _chunk_workload(layer, T, K)
    run, check = _RUNNERS[layer]
    got, ref = run(ctx, synth.make_mlp_inputs(wl), wl)
    check(got, ref)


@pytest.mark.parametrize("layer", ["up", "down", "attn_out"])
def test_mlp_block_multi_chunk_token_offset(ctx, layer):
    """A token shard (token_offset 11) whose call also spans three chunks."""
    wl = _chunk_workload(layer, 32, 50000)
    run, check = _RUNNERS[layer]
    got, ref = run(ctx, synth.make_mlp_inputs(wl), wl, t0=11, T=5)
    check(got, ref)


# ---- the full workloads, sampled rows ----------------------------------------

def _full_size(ctx, layer):
    wl = synth.CONFIGS["attn_out_bf16" if layer == "attn_out" else
                       ("mlp_down_bf16" if layer == "down" else "mlp_bf16")]
    inp = synth.make_mlp_inputs(wl)
    dev = {k: to_dev(inp[k], "bf16") for k in ("X", "W_up", "W_down", "W_head")}
    kw = dict(O=to_dev(inp["O"], "bf16")) if layer == "attn_out" else {}
    out = ctx.mlp_grad(dev["X"], dev["W_up"], dev["W_down"], dev["W_head"],
                       to_dev(inp["targets"], "i32"), K=wl.K, sigma=wl.sigma, seed=wl.seed,
                       want_rewards=True, want_g=True, layer=layer, **kw)
    torch.cuda.synchronize()
    return wl, inp, dev, out


@pytest.mark.parametrize("layer", ["up", "down", "attn_out"])
def test_mlp_block_full_size_sampled_rows(ctx, layer):
    """The whole T=8192, K=256 call (16 chunks of 512 tokens, as the benchmark
    runs it); token rows from chunks 0, 7 and 15 against the oracle, and G
    against sum_t g_t x_t^T rebuilt in fp64 from the returned g."""
    wl, inp, dev, out = _full_size(ctx, layer)
    assert (131072 // wl.K) == 512 and wl.T == 16 * 512
    for t in (1, 7 * 512 + 100, 16 * 512 - 1):
        prm = oracle.Params(T=1, d=wl.d, V=wl.V, d_ff=wl.d_ff, K=wl.K, sigma=wl.sigma,
                            seed=wl.seed, token_offset=t)
        args = (inp["X"][t:t + 1],)
        if layer == "attn_out":
            args += (inp["O"][t:t + 1],)
        fn = {"up": oracle.mlp_grad, "down": oracle.mlp_down_grad,
              "attn_out": oracle.attn_out_grad}[layer]
        ref = fn(*args, inp["W_up"], inp["W_down"], inp["W_head"], inp["targets"][t:t + 1], prm)
        assert abs(out["loss"][t].item() - ref["loss"][0]) < TOL_LOSS
        assert np.abs(np64(out["rewards"][t]) - ref["rewards"][0]).max() < TOL_LOSS
        assert rel_fro(np64(out["g"][t]), ref["g"][0]) < TOL_G
    # G = sum_t g_t z_t^T over all tokens, z the layer input: x (up), GELU(u) (down), o (attn_out)
    g = out["g"].double()
    if layer == "up":
        Z = dev["X"].double()
    elif layer == "attn_out":
        Z = to_dev(inp["O"], "bf16").double()
    else:
        u = dev["X"].double() @ dev["W_up"].double().T
        Z = 0.5 * u * (1.0 + torch.erf(u / np.sqrt(2.0)))
    rows = torch.randint(0, g.shape[1], (48,), generator=torch.Generator().manual_seed(1)).cuda()
    ref_rows = (g[:, rows].T @ Z).cpu().numpy()
    tol = 1e-5 if layer == "down" else TOL_GW_BF16
    assert rel_fro(np64(out["G"][rows]), ref_rows) < tol
