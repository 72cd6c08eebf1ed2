"""MLP up-projection estimator on the GPU vs the fp64 oracle (bf16 rounding
points mirrored), on small shapes and on token slices of the d=768,
d_ff=3072, V=50304 workload."""
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


@pytest.mark.parametrize("kw", [dict(), dict(T=1, K=1), dict(d=33, d_ff=200, V=517), dict(K=130),
                                dict(sigma=0.1)])
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
                                dict(sigma=0.1)])
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
                                dict(sigma=0.1)])
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
