"""Pins of the attention-internals oracle ("Dust：无需反向传播的Transformer零阶
预训练", §1: the attention internals' reward comes from the change of the
attention output; only the attention output is recomputed per draw).

The oracle is checked against things other than itself:
* the causal attention against PyTorch's scaled_dot_product_attention (fp64);
* sigma = 0 gives exactly zero rewards and estimates;
* locality: noise on q_s moves o_s only, noise on k_s or v_s moves o_t for
  t >= s of the same sequence only (bit for bit elsewhere);
* the small-sigma limit r / sigma -> -eps . grad, with grad the autograd
  gradient of sum_t <o_t, e_t> with respect to the perturbed row (fp64);
* values: the reward is exactly linear in the noise, r = -sigma sum_t a_ts
  <eps, e_t> with the clean probabilities, at any sigma;
* one-token sequences: q and k noise cannot move a softmax over one key;
* convergence of g to the autograd gradient as K grows;
* G = sum_s g_s x_s^T as an explicit loop;
* the per-head closed forms the draw kernels evaluate (query, key, value)
  agree with the recompute to rounding at small and large sigma.
"""

import numpy as np
import pytest
import torch

import oracle
import synth


def _inputs(T=12, L=6, H=2, dh=4, d=5, seed=11):
    wl = synth.CONFIGS["attn_q_bf16"].with_(T=T, d=d, seq_len=L, n_heads=H, head_dim=dh,
                                            seed=seed, dtype="f32")
    return synth.make_attn_inputs(wl)


def _torch_objective_grad(Q, K, V, E, L, H, which):
    """Autograd gradient of sum_t <o_t, e_t> with respect to Q, K or V (fp64)."""
    T, D = Q.shape
    n, dh = T // L, D // H
    t = {k: torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=(k == which))
         for k, x in (("q", Q), ("k", K), ("v", V))}

    def heads(x):
        return x.reshape(n, L, H, dh).transpose(1, 2)

    o = torch.nn.functional.scaled_dot_product_attention(
        heads(t["q"]), heads(t["k"]), heads(t["v"]), is_causal=True)
    o = o.transpose(1, 2).reshape(T, D)
    (o * torch.tensor(np.asarray(E, np.float64))).sum().backward()
    return t[which].grad.numpy(), o.detach().numpy()


def test_attention_matches_torch_sdpa():
    x = _inputs(T=24, L=8, H=3, dh=4)
    O, A = oracle.attention(x["Q"], x["K"], x["V"], 8, 3)
    _, o_ref = _torch_objective_grad(x["Q"], x["K"], x["V"], x["E"], 8, 3, "q")
    assert np.abs(O - o_ref).max() < 1e-13
    assert np.allclose(A.sum(axis=-1), 1.0, atol=1e-14)
    assert np.all(A[..., np.triu_indices(8, 1)[0], np.triu_indices(8, 1)[1]] == 0.0)


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_sigma_zero_gives_exact_zeros(which):
    x = _inputs()
    prm = oracle.Params(T=12, d=5, V=1, K=8, sigma=0.0, seed=3)
    out = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 6, 2, which, prm)
    assert not out["rewards"].any() and not out["g"].any() and not out["G"].any()


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_locality_of_the_perturbation(which):
    x = _inputs(T=8, L=8)
    O, _ = oracle.attention(x["Q"], x["K"], x["V"], 8, 2)
    rng = np.random.default_rng(0)
    for pos in (0, 3, 7):
        delta = 0.3 * rng.standard_normal((4, x["Q"].shape[1]))
        O1 = oracle.perturbed_outputs(x["Q"], x["K"], x["V"], 2, pos, which, delta)
        moved = np.any(O1 != O[None], axis=(0, 2))
        expect = np.zeros(8, dtype=bool)
        if which == "q":
            expect[pos] = True
        else:
            expect[pos:] = True
        if which in ("q", "k") and pos == 0:
            expect[0] = False          # row 0's softmax has one entry: always 1
        assert np.array_equal(moved, expect), (pos, moved)


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_small_sigma_limit_is_the_autograd_directional_derivative(which):
    x = _inputs(T=12, L=6, H=2, dh=4)
    L, H = 6, 2
    grad, _ = _torch_objective_grad(x["Q"], x["K"], x["V"], x["E"], L, H, which)
    O, _ = oracle.attention(x["Q"], x["K"], x["V"], L, H)
    sig = 1e-6
    eps = np.random.default_rng(1).standard_normal((5, 8))
    for s in (0, 4, 7, 11):
        b, pos = divmod(s, L)
        rows = slice(b * L, (b + 1) * L)
        r, _ = oracle.attn_draws(x["Q"][rows], x["K"][rows], x["V"][rows], O[rows],
                                 x["E"][rows], H, pos, which, eps, sig)
        lin = -(eps @ grad[s])
        scale = np.abs(eps).max() * np.abs(grad[s]).sum() + 1e-30
        assert np.abs(r / sig - lin).max() < 1e-4 * scale, (s, r / sig, lin)


def test_value_noise_reward_is_exactly_linear():
    x = _inputs(T=12, L=6, H=2, dh=4)
    L, H, dh = 6, 2, 4
    O, A = oracle.attention(x["Q"], x["K"], x["V"], L, H)
    eps = np.random.default_rng(2).standard_normal((3, 8))
    for sig in (0.5, 3.0):
        for s in (1, 6, 11):
            b, pos = divmod(s, L)
            rows = slice(b * L, (b + 1) * L)
            r, _ = oracle.attn_draws(x["Q"][rows], x["K"][rows], x["V"][rows], O[rows],
                                     x["E"][rows], H, pos, "v", eps, sig)
            want = np.zeros(3)
            for h in range(H):
                cols = slice(h * dh, (h + 1) * dh)
                for t in range(pos, L):
                    want -= sig * A[b, h, t, pos] * (eps[:, cols] @ x["E"][b * L + t, cols])
            assert np.allclose(r, want, rtol=1e-12, atol=1e-12)


def test_one_token_sequences():
    x = _inputs(T=5, L=1, H=2, dh=4)
    prm = oracle.Params(T=5, d=5, V=1, K=16, sigma=0.7, seed=9)
    for which in ("q", "k"):
        out = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 1, 2, which, prm)
        assert not out["rewards"].any()
    out = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 1, 2, "v", prm)
    eps = np.stack([oracle.gaussians(9, s, np.arange(16), np.arange(8), oracle.TAG_ATTN_V)
                    for s in range(5)])
    want = -prm.sigma32 * np.einsum("sid,sd->si", eps, x["E"].astype(np.float64))
    assert np.allclose(out["rewards"], want, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_estimate_converges_to_the_gradient(which):
    # one head of width 4 over a 3-token sequence, K = 6000 draws, small sigma:
    # E|g - grad|^2 = |grad|^2 (D + 1) / K, so cos(g, grad) is about 0.9996
    x = _inputs(T=3, L=3, H=1, dh=4, d=3, seed=21)
    grad, _ = _torch_objective_grad(x["Q"], x["K"], x["V"], x["E"], 3, 1, which)
    prm = oracle.Params(T=3, d=3, V=1, K=6000, sigma=1e-4, seed=5)
    out = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 3, 1, which, prm,
                           draw_chunk=2000)
    g = out["g"]
    for s in range(3):
        if np.linalg.norm(grad[s]) < 1e-9:
            continue                     # k_0 moves nothing under a causal mask
        cos = g[s] @ grad[s] / (np.linalg.norm(g[s]) * np.linalg.norm(grad[s]))
        assert cos > 0.99, (s, cos)
        ratio = np.linalg.norm(g[s]) / np.linalg.norm(grad[s])
        assert abs(ratio - 1.0) < 0.05, (s, ratio)


def test_weight_gradient_is_the_outer_product_sum():
    x = _inputs(T=12, L=6, H=2, dh=4, d=5)
    prm = oracle.Params(T=12, d=5, V=1, K=6, sigma=0.1, seed=4)
    out = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 6, 2, "k", prm)
    G = np.zeros((8, 5))
    for s in range(12):
        G += np.outer(out["g"][s], x["X"][s].astype(np.float64))
    assert np.abs(G - out["G"]).max() < 1e-12


def test_sequences_are_independent_and_offsets_compose():
    # two sequences in one call equal the second sequence alone at token offset L
    x = _inputs(T=12, L=6, H=2, dh=4, d=5)
    prm = oracle.Params(T=12, d=5, V=1, K=5, sigma=0.05, seed=8)
    both = oracle.attn_grad(x["X"], x["Q"], x["K"], x["V"], x["E"], 6, 2, "q", prm)
    prm2 = oracle.Params(T=6, d=5, V=1, K=5, sigma=0.05, seed=8, token_offset=6)
    second = oracle.attn_grad(x["X"][6:], x["Q"][6:], x["K"][6:], x["V"][6:], x["E"][6:], 6, 2,
                              "q", prm2)
    assert np.array_equal(both["rewards"][6:], second["rewards"])


def test_closed_forms_of_the_kernels_equal_the_recompute():
    # The draw kernels never recompute a perturbed softmax: per head they use
    #   query: r_h = -sum_tau a expm1(d_tau) (<v_tau, e_s> - gbar_s)
    #                 / (1 + sum_tau a expm1(d_tau)),  d_tau = sigma eps.k_tau / sqrt(d_h)
    #   key:   r_h = -sum_{t>=s} u_t / (1 + u_t) (<v_s, e_t> - gbar_t),
    #          u_t = a_t,s expm1(sigma eps.q_t / sqrt(d_h))
    #   value: r_h = -sigma eps . sum_{t>=s} a_t,s e_t
    # with a the clean probabilities and gbar_t = <o_t, e_t> per head. These
    # are exact rewrites, so they match the oracle's recompute to rounding at
    # any sigma.
    L, H, dh = 7, 2, 4
    x = _inputs(T=L, L=L, H=H, dh=dh)
    Q, K, V, E = (x[k].astype(np.float64) for k in ("Q", "K", "V", "E"))
    O, A = oracle.attention(Q, K, V, L, H)
    c = 1.0 / np.sqrt(dh)
    eps = np.random.default_rng(3).standard_normal((5, H * dh))
    for sig in (0.01, 0.7):
        for s in (0, 3, 6):
            for which in ("q", "k", "v"):
                r_ref, _ = oracle.attn_draws(Q, K, V, O, E, H, s, which, eps, sig)
                r = np.zeros(len(eps))
                for h in range(H):
                    cols = slice(h * dh, (h + 1) * dh)
                    a = A[0, h]
                    gbar = (O[:, cols] * E[:, cols]).sum(axis=1)
                    x_h = sig * eps[:, cols]
                    if which == "q":
                        em = np.expm1(c * x_h @ K[: s + 1, cols].T)          # (n, s+1)
                        gam = V[: s + 1, cols] @ E[s, cols]
                        D = em @ a[s, : s + 1]
                        N = em @ (a[s, : s + 1] * (gam - gbar[s]))
                        r += -N / (1 + D)
                    elif which == "k":
                        u = a[s:, s][None, :] * np.expm1(c * x_h @ Q[s:, cols].T)
                        beta = E[s:, cols] @ V[s, cols] - gbar[s:]
                        r += -(u / (1 + u)) @ beta
                    else:
                        w = a[s:, s] @ E[s:, cols]
                        r += -(x_h @ w)
                assert np.allclose(r, r_ref, rtol=1e-10, atol=1e-13), (which, s, sig)
