"""cos(K) report of the LM-head estimator ("Dust：无需反向传播的Transformer零阶预训练",
§2 梯度对齐): the law fit on CPU, and the nested draw-block estimates on the
GPU against the oracle's estimates and exact gradient."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from _util import to_dev
from zeroth_order_transformer_dust_b200.alignment import fit_cos_law


def test_fit_recovers_an_exact_law():
    ks = [64, 256, 1024, 4096, 16384]
    for c_max, c in ((0.97, 900.0), (0.5, 20.0), (1.0, 50304.0)):
        cos = [c_max / math.sqrt(1 + c / k) for k in ks]
        f = fit_cos_law(ks, cos)
        assert abs(f["c_max"] - c_max) < 1e-9 * max(1.0, c_max)
        assert abs(f["c"] - c) < 1e-6 * c
        assert f["rmse"] < 1e-12
    # c_max = 1 exactly: the constrained fit recovers c too
    cos = [1.0 / math.sqrt(1 + 4.9e6 / k) for k in ks]
    f = fit_cos_law(ks, cos)
    assert abs(f["c_at_cmax1"] - 4.9e6) < 1e-6 * 4.9e6 and f["rmse_at_cmax1"] < 1e-12


def test_fit_reports_misfit():
    ks = [64, 256, 1024, 4096]
    cos = [0.2, 0.6, 0.3, 0.7]           # no law of this form fits these
    f = fit_cos_law(ks, cos)
    assert f["rmse"] is None or f["rmse"] > 0.05


def _exact(H, W, y):
    z = H @ W.T
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    p[np.arange(len(y)), y] -= 1.0
    return p


@pytest.mark.gpu
@pytest.mark.parametrize("S", [0, 64])
def test_nested_blocks_match_the_oracle(cuda_ok, S):
    import zeroth_order_transformer_dust_b200 as dust
    from zeroth_order_transformer_dust_b200.alignment import cosine_vs_k

    wl = synth.CONFIGS["tiny_fp32"].with_(T=48, K=96, S=S)
    inp = synth.make_head_inputs(wl)
    H, W, y = inp["H"], inp["W"], inp["targets"]
    ks = [16, 40, 96]
    ctx = dust.Context(0)
    got = cosine_vs_k(ctx, to_dev(H, "f32"), to_dev(W, "f32"), to_dev(y, "i32"), ks=ks,
                      sigma=wl.sigma, S=S, seed=wl.seed, token_chunk=20)
    torch.cuda.synchronize()
    gx = _exact(H.astype(np.float64), W.astype(np.float64), y)
    Gx = gx.T @ H
    for j, k in enumerate(ks):
        prm = oracle.Params(T=wl.T, d=wl.d, V=wl.V, K=k, S=S, sigma=wl.sigma, seed=wl.seed)
        ref = oracle.head_grad(H, W, y, prm)
        g = ref["g"]
        cos_g = float((g * gx).sum() / np.sqrt((g * g).sum() * (gx * gx).sum()))
        G = ref["G"]
        cos_G = float((G * Gx).sum() / np.sqrt((G * G).sum() * (Gx * Gx).sum()))
        assert got["K"][j] == k
        assert abs(got["cos_g"][j] - cos_g) < 1e-4
        assert abs(got["cos_G"][j] - cos_G) < 1e-4
