"""Gradient alignment of the LM-head estimator against the exact gradient.

The pages ("Dust：无需反向传播的Transformer零阶预训练", §2 梯度对齐) report that
the cosine between the estimate and the true gradient follows
cos(K) = c_max / sqrt(1 + c/K) in the number of draws K. This module measures
that curve for one workload: it runs the estimator in draw blocks
[K_{j-1}, K_j) (``draw_offset`` keeps the noise of one K_max-draw run), sums
the blocks into nested estimates for every K in the list, and compares each
with the closed form dL/dz = softmax(z) - onehot(y).

This is analysis around the estimator, not a step of it: the estimates come
from the library's kernels; the exact gradient and the cosines are formed here
with plain torch on the device.
"""
from __future__ import annotations

import math

import torch


def _exact_grad_rows(H, W, y, t0, t1):
    z = H[t0:t1].float() @ W.float().t()
    g = torch.softmax(z, dim=1)
    g[torch.arange(t1 - t0, device=g.device), y[t0:t1].long()] -= 1.0
    return g


def fit_cos_law(ks, cos):
    """Least-squares fit of cos(K) = c_max / sqrt(1 + c/K).

    1/cos^2 = 1/c_max^2 + (c/c_max^2)/K is linear in 1/K; the fit is taken
    there and its RMSE is reported on cos itself."""
    n = len(ks)
    xs = [1.0 / k for k in ks]
    ys = [1.0 / (c * c) for c in cos]
    mx, my = sum(xs) / n, sum(ys) / n
    sxx = sum((x - mx) ** 2 for x in xs)
    slope = sum((x - mx) * (v - my) for x, v in zip(xs, ys)) / sxx if sxx > 0 else 0.0
    icept = my - slope * mx
    # with c_max held at 1: 1/cos^2 - 1 = c/K, least squares in 1/K through 0
    c1 = sum(x * (v - 1.0) for x, v in zip(xs, ys)) / sum(x * x for x in xs)
    pred1 = [1.0 / math.sqrt(max(1e-300, 1.0 + c1 / k)) for k in ks]
    rmse1 = math.sqrt(sum((p - v) ** 2 for p, v in zip(pred1, cos)) / n)
    out = {"c_max": None, "c": None, "rmse": None, "c_at_cmax1": c1, "rmse_at_cmax1": rmse1}
    if icept <= 0:   # c >> K over the whole range: only c_max^2 / c is identified
        return out
    c_max = 1.0 / math.sqrt(icept)
    c = slope / icept
    pred = [c_max / math.sqrt(max(1e-300, 1.0 + c / k)) for k in ks]
    out.update(c_max=c_max, c=c, rmse=math.sqrt(sum((p - v) ** 2 for p, v in zip(pred, cos)) / n))
    return out


@torch.no_grad()
def cosine_vs_k(ctx, H, W, y, *, ks, sigma, S=0, seed=0, token_chunk=2048):
    """Cosine of the estimate g (T x V, flattened) and of G_W (V x d) with the
    exact gradients, for every K in ``ks`` (ascending). Returns a dict with
    the per-K cosines, the mean per-token cosine and the cos(K) fit."""
    ks = sorted(int(k) for k in ks)
    T, V = H.shape[0], W.shape[0]
    dev = H.device
    acc = torch.zeros(T, V, dtype=torch.float32, device=dev)
    blk = torch.empty(T, V, dtype=torch.float32, device=dev)
    # exact G_W = sum_t grad_t h_t^T, and its norm
    G_true = torch.zeros(W.shape[0], H.shape[1], dtype=torch.float32, device=dev)
    for t0 in range(0, T, token_chunk):
        t1 = min(T, t0 + token_chunk)
        G_true += _exact_grad_rows(H, W, y, t0, t1).t() @ H[t0:t1].float()
    res = {"K": [], "cos_g": [], "cos_g_token_mean": [], "cos_G": []}
    done = 0
    for k in ks:
        n = k - done
        out = ctx.head_grad(H, W, y, K=n, sigma=sigma, S=S, seed=seed, draw_offset=done,
                            want_G=False, want_loss=False, out={"g": blk})
        # g of a K-draw run is the mean over its draws: sum the blocks by weight
        acc.add_(out["g"], alpha=float(n))
        done = k
        dot = nrm_e = nrm_x = 0.0
        tok_cos = 0.0
        G_est = torch.zeros_like(G_true)
        for t0 in range(0, T, token_chunk):
            t1 = min(T, t0 + token_chunk)
            ge = acc[t0:t1] / float(k)
            gx = _exact_grad_rows(H, W, y, t0, t1)
            d = (ge * gx).sum(dim=1, dtype=torch.float64)
            ne = (ge * ge).sum(dim=1, dtype=torch.float64)
            nx = (gx * gx).sum(dim=1, dtype=torch.float64)
            dot += float(d.sum())
            nrm_e += float(ne.sum())
            nrm_x += float(nx.sum())
            tok_cos += float((d / torch.sqrt(ne * nx).clamp_min(1e-300)).sum())
            G_est += ge.t() @ H[t0:t1].float()
        res["K"].append(k)
        res["cos_g"].append(dot / math.sqrt(max(nrm_e * nrm_x, 1e-300)))
        res["cos_g_token_mean"].append(tok_cos / T)
        res["cos_G"].append(float(torch.nn.functional.cosine_similarity(
            G_est.flatten().double(), G_true.flatten().double(), dim=0)))
    res["fit_g"] = fit_cos_law(res["K"], res["cos_g"])
    res["fit_G"] = fit_cos_law(res["K"], res["cos_G"])
    return res
