"""LM-head estimator on the GPU vs the fp64 oracle, element by element.

Small cases span several tiles and ragged tails; the large workloads are
checked on token slices (token_offset reproduces the exact noise of the
full run) and, at full size in the launch configuration the benchmark uses,
on sampled token rows plus the outer-product identity for G_W.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import zeroth_order_transformer_dust_b200 as dust
from _util import TOL_G, TOL_GW_BF16, TOL_GW_F32, TOL_LOSS, np64, rel_fro, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


def _inputs(wl, T=None, t0=0):
    inp = synth.make_head_inputs(wl)
    sl = slice(t0, t0 + (T or wl.T))
    return inp["H"][sl], inp["W"], inp["targets"][sl]


def _gpu(ctx, H, W, y, wl, **kw):
    out = ctx.head_grad(to_dev(H, wl.dtype), to_dev(W, wl.dtype), to_dev(y, "i32"), K=wl.K,
                        sigma=wl.sigma, S=wl.S, seed=wl.seed, want_rewards=True, want_g=True, **kw)
    torch.cuda.synchronize()
    return {k: np64(v) for k, v in out.items()}


def _oracle(H, W, y, wl, **kw):
    prm = oracle.Params(T=H.shape[0], d=H.shape[1], V=W.shape[0], K=wl.K, S=wl.S, sigma=wl.sigma,
                        seed=wl.seed, **kw)
    return oracle.head_grad(H, W, y, prm)


def _compare(got, ref, gw_tol):
    assert np.abs(got["loss"] - ref["loss"]).max() < TOL_LOSS
    assert np.abs(got["rewards"] - ref["rewards"]).max() < TOL_LOSS
    assert rel_fro(got["g"], ref["g"]) < TOL_G
    assert rel_fro(got["G"], ref["G"]) < gw_tol


def test_tiny_fp32_full_vocab(ctx):
    wl = synth.CONFIGS["tiny_fp32"]
    H, W, y = _inputs(wl)
    _compare(_gpu(ctx, H, W, y, wl), _oracle(H, W, y, wl), TOL_GW_F32)


def test_full_vocab_bf16_slice(ctx):
    wl = synth.CONFIGS["full_bf16"]
    t0, n = 1000, 6
    H, W, y = _inputs(wl, n, t0)
    got = _gpu(ctx, H, W, y, wl, token_offset=t0)
    _compare(got, _oracle(H, W, y, wl, token_offset=t0), TOL_GW_BF16)


def test_subset_bf16_slice(ctx):
    wl = synth.CONFIGS["subset_bf16"]
    t0, n = 4321, 8
    H, W, y = _inputs(wl, n, t0)
    got = _gpu(ctx, H, W, y, wl, token_offset=t0)
    _compare(got, _oracle(H, W, y, wl, token_offset=t0), TOL_GW_BF16)


def test_large_subset_slice(ctx):
    wl = synth.CONFIGS["large_subset_bf16"]
    t0, n = 16381, 3
    H, W, y = _inputs(wl, n, t0)
    got = _gpu(ctx, H, W, y, wl, token_offset=t0)
    _compare(got, _oracle(H, W, y, wl, token_offset=t0), TOL_GW_BF16)


def _small(T=37, d=40, V=1000, K=9, S=0, sigma=0.02, seed=5, dtype="bf16"):
    wl = synth.Workload("small", "head", T=T, d=d, V=V, K=K, S=S, sigma=sigma, seed=seed,
                        dtype=dtype, targets="zipf")
    return wl


@pytest.mark.parametrize("kw", [
    dict(), dict(S=100), dict(S=1000), dict(S=1), dict(S=129, K=33), dict(T=1), dict(K=1),
    dict(K=1, S=3), dict(V=257, S=256), dict(V=5, S=2, d=3), dict(d=1), dict(sigma=0.2),
    dict(sigma=0.2, S=300), dict(dtype="f32"), dict(dtype="f32", S=77), dict(V=4099, S=640, K=40),
    # fixed-point accumulation with a reduced scale (16384 < K <= 65536), and the
    # fp32-atomic fallback (K > 65536)
    dict(T=3, K=20000, S=32), dict(T=2, K=70000, S=64, V=700),
    # vocabularies beyond one or two CTAs' shared memory: clusters of 4 to 8
    # CTAs (windows crossing into the next CTA's slice and wrapping past V)
    dict(V=70001, S=300, K=256, T=4), dict(V=128256, S=512, K=256, T=4, d=24),
    dict(V=200003, S=512, K=256, T=4, d=16), dict(V=200003, S=77, K=300, T=3, d=16, dtype="f32"),
    # fp32 accumulators (K > 65536) with the target in another CTA's slice
    dict(V=70001, S=64, K=70000, T=1, d=16),
    # full vocabulary: ragged slabs at several V, more tokens than CTAs
    dict(V=4099, K=20), dict(V=20000, K=33, T=5, d=16), dict(V=100000, K=9, T=3, d=16),
    dict(T=200, K=5, V=1000), dict(T=300, K=2, V=3000, dtype="f32"),
    dict(V=120000, K=8, T=3, d=16),
    # the per-token draw list (K <= 512, S <= 256) with clusters of two CTAs
    # and several tokens per cluster
    dict(V=50304, S=256, K=512, T=160, d=16),
    # five to eight 128-slot blocks a draw (S up to 1024): exact and ragged S,
    # windows crossing slices of a two-CTA cluster, the library expm1 (large
    # sigma) and fp32 accumulators (K > 65536) at ragged S
    dict(V=50304, S=1024, K=64, T=5, d=16), dict(V=50304, S=777, K=100, T=4, d=16),
    dict(V=3000, S=640, K=50), dict(V=3000, S=1000, K=33, sigma=0.2), dict(V=9000, S=900, K=40, T=6),
    dict(T=2, K=70000, S=700, V=2000, d=8), dict(V=100003, S=1023, K=40, T=3, d=16),
    # windows that cover the whole vocabulary (S = V; the target always in
    # the window), and eight blocks with fp32 accumulators
    dict(V=1000, S=1000, K=20), dict(V=1024, S=1024, K=16, T=9), dict(T=1, K=66000, S=1024, V=2048, d=8),
    # beyond 1024 entries a draw: the L2-fed kernel
    dict(V=5000, S=1500, K=30), dict(V=50304, S=2048, K=20, T=3, d=16),
    # the draw list at three and four blocks a draw in clusters of 3 to 8
    # CTAs (up to 256 draws a CTA), with several tokens per cluster
    dict(V=128256, S=512, K=1024, T=3, d=16), dict(V=70001, S=400, K=1024, T=3, d=16),
    dict(V=100003, S=257, K=300, T=40, d=16), dict(V=128256, S=511, K=2048, T=2, d=16),
    # cluster sizes other than powers of two (3 to 8 CTAs, whichever covers the
    # most SMs): clusters of 3 with the draw list, and vocabularies whose
    # smallest fitting cluster has 4, 5 or 6 CTAs
    dict(V=60000, S=512, K=700, T=5, d=16), dict(V=90001, S=129, K=100, T=7, d=16),
    dict(V=120001, S=384, K=600, T=3, d=16), dict(V=150001, S=300, K=500, T=4, d=16),
])
def test_edge_shapes(ctx, kw):
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    got = _gpu(ctx, H, W, y, wl)
    ref = _oracle(H, W, y, wl)
    _compare(got, ref, TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16)


# More full-vocabulary shapes: K = 2, 3, 4 and odd K, single tokens with many
# draws, exact and ragged 128-slot blocks, the largest vocabularies here, sigma
# that needs the exact expm1 and sigma that does not, fp32 inputs, and more
# tokens than CTAs.
@pytest.mark.parametrize("kw", [
    dict(K=2), dict(K=3), dict(K=4, T=3), dict(K=33, V=3000), dict(T=1, K=64, V=50304, d=16),
    dict(V=128, K=7), dict(V=129, K=7), dict(V=2, K=5), dict(V=122000, K=6, T=3, d=16),
    dict(V=124000, K=6, T=2, d=16), dict(sigma=0.2, K=35), dict(dtype="f32", K=10, V=2049),
    dict(T=97, K=3, V=50304, d=16),
    # sigma small enough for the series degrees (the reward pass's hardware
    # exponential): degree 4 at 1e-2, degree 3 at 5e-3
    dict(sigma=0.01, K=20, V=3000), dict(sigma=0.005, K=20, V=4099, T=9),
    dict(sigma=0.01, dtype="f32", K=16, V=1024), dict(sigma=0.0104, K=64, V=50304, T=2, d=16),
])
def test_full_vocab_more_shapes(ctx, kw):
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    _compare(_gpu(ctx, H, W, y, wl), _oracle(H, W, y, wl),
             TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16)


@pytest.mark.parametrize("kw", [dict(), dict(K=1), dict(V=4099, K=20), dict(T=200, K=5, V=1000),
                                dict(T=2, K=64, V=50304, d=16, sigma=0.01), dict(sigma=0.2),
                                dict(T=40, K=7, V=20000, d=16, sigma=0.005)])
def test_full_vocab_two_passes(cuda_ok, monkeypatch, kw):
    """The reward pass and the g pass (DUST_FULL_KERNEL=2), which run where no
    one-pass plan fits, against the oracle."""
    monkeypatch.setenv("DUST_FULL_KERNEL", "2")
    c = dust.Context(0)
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    _compare(_gpu(c, H, W, y, wl), _oracle(H, W, y, wl), TOL_GW_BF16)


def test_full_vocab_runs_in_one_pass(ctx):
    """The full_bf16 shapes take the one-pass kernel (its stage name), with
    more tokens than clusters; sampled rows against the oracle."""
    wl = synth.CONFIGS["full_bf16"]
    t0, n = 3000, 40
    H, W, y = _inputs(wl, n, t0)
    ctx.set_stage_timing(True)
    try:
        got = _gpu(ctx, H, W, y, wl, token_offset=t0)
        stages = ctx.stage_times()
    finally:
        ctx.set_stage_timing(False)
    assert "full_draws" in stages and "reward" not in stages
    for t in (0, 17, 39):
        ref = _oracle(H[t:t + 1], W, y[t:t + 1], wl, token_offset=t0 + t)
        assert abs(got["loss"][t] - ref["loss"][0]) < TOL_LOSS
        assert np.abs(got["rewards"][t] - ref["rewards"][0]).max() < TOL_LOSS
        assert rel_fro(got["g"][t], ref["g"][0]) < TOL_G


def test_full_vocab_split_over_two_streams(cuda_ok, monkeypatch):
    """On full_bf16 shapes the two passes take the last tokens on the SMs the
    one-pass clusters leave empty (three more launches than the one-pass
    kernel alone, DUST_FULL_SPLIT=0); every row, g and G_W agree with the
    unsplit call, and rows on both sides of the split with the oracle."""
    wl = synth.CONFIGS["full_bf16"]
    t0, n = 1234, 600
    H, W, y = _inputs(wl, n, t0)
    split = dust.Context(0)
    monkeypatch.setenv("DUST_FULL_SPLIT", "0")
    whole = dust.Context(0)
    l0 = split.kernel_launches
    a = _gpu(split, H, W, y, wl, token_offset=t0)
    la = split.kernel_launches - l0
    l0 = whole.kernel_launches
    b = _gpu(whole, H, W, y, wl, token_offset=t0)
    lb = whole.kernel_launches - l0
    assert la == lb + 3
    np.testing.assert_array_equal(a["loss"], b["loss"])
    assert np.abs(a["rewards"] - b["rewards"]).max() < TOL_LOSS
    assert rel_fro(a["g"], b["g"]) < TOL_G
    assert rel_fro(a["G"], b["G"]) < TOL_GW_BF16
    for t in (0, 300, 540, 570, 599):
        ref = _oracle(H[t:t + 1], W, y[t:t + 1], wl, token_offset=t0 + t)
        assert np.abs(a["rewards"][t] - ref["rewards"][0]).max() < TOL_LOSS
        assert rel_fro(a["g"][t], ref["g"][0]) < TOL_G


@pytest.mark.parametrize("kw", [dict(T=300, d=64, K=4, dtype="f32"), dict(T=300, d=32, K=3, sigma=0.2)])
def test_full_vocab_split_shapes(cuda_ok, monkeypatch, kw):
    """The split on other V = 50304 shapes: fp32 inputs (an fp32 g operand) and
    a sigma beyond the expm1 series' range, every row against the oracle; then
    G_W again without rewards or g requested (the two passes' rewards go to
    scratch), equal to the first."""
    wl = _small(V=50304, **kw)
    H, W, y = _inputs(wl)
    c = dust.Context(0)
    monkeypatch.setenv("DUST_FULL_SPLIT", "0")
    whole = dust.Context(0)
    l0 = c.kernel_launches
    got = _gpu(c, H, W, y, wl)
    launches = c.kernel_launches - l0
    _gpu(whole, H, W, y, wl)
    assert launches == whole.kernel_launches + 3
    _compare(got, _oracle(H, W, y, wl), TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16)
    out = c.head_grad(to_dev(H, wl.dtype), to_dev(W, wl.dtype), to_dev(y, "i32"), K=wl.K,
                      sigma=wl.sigma, seed=wl.seed)
    torch.cuda.synchronize()
    assert c.kernel_launches - l0 == 2 * launches
    assert rel_fro(np64(out["G"]), got["G"]) < 1e-6


@pytest.mark.parametrize("kw", [dict(S=100), dict(S=1000), dict(V=4099, S=640, K=40),
                                dict(V=50304, S=512, K=64, T=3, d=16), dict(T=2, K=70000, S=64, V=700),
                                dict(V=20000, S=300, K=33, sigma=0.2, T=4, d=16)])
def test_l2_fed_subset_kernel(cuda_ok, monkeypatch, kw):
    """The L2-fed subset kernel (DUST_SUBSET_KERNEL=1), which runs beyond the
    shared-memory kernel's reach (S > 1024 or larger V), on shapes the
    shared-memory kernel would otherwise take."""
    monkeypatch.setenv("DUST_SUBSET_KERNEL", "1")
    c = dust.Context(0)
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    _compare(_gpu(c, H, W, y, wl), _oracle(H, W, y, wl), TOL_GW_BF16)


@pytest.mark.parametrize("kw", [dict(), dict(S=129, K=33), dict(V=4099, S=640, K=40),
                                dict(T=200, K=5, V=1000), dict(T=300, K=3, V=3001, S=50)])
def test_single_cta_tensor_core_path(cuda_ok, monkeypatch, kw):
    """The GEMMs in single-CTA mode (one 128 x 256 tile per SM, fewer operand
    stages) give the same estimator as the CTA-pair default, on ragged rows
    and columns."""
    monkeypatch.setenv("DUST_TC_PAIR", "0")
    c = dust.Context(0)
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    _compare(_gpu(c, H, W, y, wl), _oracle(H, W, y, wl), TOL_GW_BF16)


@pytest.mark.parametrize("c", [2.0 ** 20, 2.0 ** -26])
@pytest.mark.parametrize("S", [0, 100])
def test_gw_with_h_outside_the_fp16_range(ctx, c, S):
    """The G_W GEMM reads H as fp16 with a power-of-two scale taken from its
    largest magnitude: H scaled by 2^20 (beyond the fp16 maximum) or 2^-26
    (below its normal range), with W scaled by the inverse so the logits stay
    the same, gives the oracle's G_W."""
    wl = _small(T=37, d=40, V=1000, K=9, S=S)
    H, W, y = _inputs(wl)
    H, W = H * c, W / c
    got = _gpu(ctx, H, W, y, wl)
    ref = _oracle(H, W, y, wl)
    _compare(got, ref, TOL_GW_BF16)


@pytest.mark.parametrize("kw", [dict(), dict(S=129, K=33), dict(V=4099, K=20), dict(T=200, K=5, V=1000)])
def test_cuda_core_gemms(cuda_ok, monkeypatch, kw):
    """With the tensor cores off every GEMM runs on CUDA cores, G_W on the
    fp16 g operand and the fp16 copy of H included."""
    monkeypatch.setenv("DUST_DISABLE_TC", "1")
    c = dust.Context(0)
    wl = _small(**kw)
    H, W, y = _inputs(wl)
    _compare(_gpu(c, H, W, y, wl), _oracle(H, W, y, wl), TOL_GW_BF16)


def _host(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    t = t.to(torch.int32) if dtype == "i32" else t.to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    return t.pin_memory()


@pytest.mark.parametrize("wl", [synth.CONFIGS["tiny_fp32"], _small(S=100, K=40),
                                _small(dtype="f32", S=77), _small(T=3, K=20000, S=32)],
                         ids=["tiny_fp32", "subset_bf16", "subset_f32", "subset_bf16_k20000"])
def test_host_entry_matches_the_oracle(ctx, wl):
    """dust_head_grad_host (inputs and outputs in pinned host memory, the copies
    inside the call): all four outputs against the oracle."""
    H, W, y = _inputs(wl)
    out = ctx.head_grad_host(_host(H, wl.dtype), _host(W, wl.dtype), _host(y, "i32"), K=wl.K,
                             sigma=wl.sigma, S=wl.S, seed=wl.seed, want_rewards=True, want_g=True)
    assert all(not v.is_cuda for v in out.values())
    got = {k: v.double().numpy() for k, v in out.items()}
    _compare(got, _oracle(H, W, y, wl), TOL_GW_F32 if wl.dtype == "f32" else TOL_GW_BF16)
    # and the same bits as the device-buffer entry point on the same inputs
    dev = _gpu(ctx, H, W, y, wl)
    np.testing.assert_array_equal(got["rewards"], dev["rewards"])
    np.testing.assert_array_equal(got["loss"], dev["loss"])


def test_host_entry_reports_a_bad_target(ctx):
    wl = _small(S=50)
    H, W, y = _inputs(wl)
    y = y.copy()
    y[5] = -1
    with pytest.raises(dust.DustError) as ei:
        ctx.head_grad_host(_host(H, wl.dtype), _host(W, wl.dtype), _host(y, "i32"), K=wl.K,
                           sigma=wl.sigma, S=wl.S, seed=wl.seed)
    assert ei.value.status == 4


def test_single_entry_vocabulary(ctx):
    # V = 1: the loss is exactly 0 and every reward vanishes (up to rounding)
    for S in (0, 1):
        wl = _small(V=1, S=S, K=3)
        H, W, y = _inputs(wl)
        got = _gpu(ctx, H, W, y, wl)
        assert np.abs(got["loss"]).max() < TOL_LOSS
        assert np.abs(got["rewards"]).max() < TOL_LOSS


def test_sigma_zero_is_exactly_zero(ctx):
    for S in (0, 50):
        wl = _small(sigma=0.0, S=S)
        H, W, y = _inputs(wl)
        got = _gpu(ctx, H, W, y, wl)
        assert np.all(got["rewards"] == 0) and np.all(got["g"] == 0) and np.all(got["G"] == 0)


def test_options_stream_id_stride_literal(ctx):
    wl = _small(S=64, K=12)
    H, W, y = _inputs(wl)
    for kw, okw in ((dict(stream_id=9), dict(stream_id=9)), (dict(subset_a=7), dict(subset_a=7)),
                    (dict(literal_target_scale=True), dict(literal_target_scale=True))):
        got = _gpu(ctx, H, W, y, wl, **kw)
        ref = _oracle(H, W, y, wl, **okw)
        _compare(got, ref, TOL_GW_BF16)


def test_token_slices_and_draw_splits_compose(ctx):
    wl = _small(T=50, S=200, K=24)
    H, W, y = _inputs(wl)
    full = _gpu(ctx, H, W, y, wl)
    part = _gpu(ctx, H[17:29], W, y[17:29], wl, token_offset=17)
    np.testing.assert_array_equal(part["rewards"], full["rewards"][17:29])
    np.testing.assert_allclose(part["g"], full["g"][17:29], rtol=0, atol=1e-6)
    # draws [0, 10) + [10, 24): rewards concatenate, K*g sums
    a = _gpu(ctx, H, W, y, wl.with_(K=10))
    b = _gpu(ctx, H, W, y, wl.with_(K=14), draw_offset=10)
    np.testing.assert_array_equal(np.concatenate([a["rewards"], b["rewards"]], axis=1), full["rewards"])
    np.testing.assert_allclose(10 * a["g"] + 14 * b["g"], 24 * full["g"], rtol=0, atol=1e-4)


def test_bad_target_is_reported(ctx):
    wl = _small()
    H, W, y = _inputs(wl)
    y = y.copy()
    y[3] = wl.V
    with pytest.raises(dust.DustError) as ei:
        _gpu(ctx, H, W, y, wl)
    assert ei.value.status == 4
    # the context stays usable
    y[3] = 0
    _gpu(ctx, H, W, y, wl)


def test_deterministic_rewards(ctx):
    wl = _small(S=100, K=64)
    H, W, y = _inputs(wl)
    a = _gpu(ctx, H, W, y, wl)
    b = _gpu(ctx, H, W, y, wl)
    np.testing.assert_array_equal(a["rewards"], b["rewards"])
    np.testing.assert_array_equal(a["loss"], b["loss"])
    assert rel_fro(a["g"], b["g"]) < 1e-6


@pytest.mark.parametrize("name,rows", [("full_bf16", (0, 2049, 4095)),
                                       ("subset_bf16", (1, 8191)),
                                       ("large_subset_bf16", (0, 9999))])
def test_full_size_sampled_rows(ctx, name, rows):
    """Full-size call (the benchmark's launch configuration); sampled token rows vs the oracle,
    and G_W against sum_t g_t h_t^T rebuilt in fp64 from the returned g on sampled rows."""
    wl = synth.CONFIGS[name]
    inp = synth.make_head_inputs(wl)
    H, W, y = inp["H"], inp["W"], inp["targets"]
    Hd, Wd, yd = to_dev(H, wl.dtype), to_dev(W, wl.dtype), to_dev(y, "i32")
    out = ctx.head_grad(Hd, Wd, yd, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                        want_rewards=True, want_g=True)
    torch.cuda.synchronize()
    for t in rows:
        ref = _oracle(H[t:t + 1], W, y[t:t + 1], wl, token_offset=t)
        assert abs(out["loss"][t].item() - ref["loss"][0]) < TOL_LOSS
        assert np.abs(np64(out["rewards"][t]) - ref["rewards"][0]).max() < TOL_LOSS
        assert rel_fro(np64(out["g"][t]), ref["g"][0]) < TOL_G
    vs = torch.randint(0, wl.V, (64,), generator=torch.Generator().manual_seed(0))
    g_cols = out["g"][:, vs.cuda()].double()
    ref_rows = (g_cols.T @ Hd.double()).cpu().numpy()
    assert rel_fro(np64(out["G"][vs.cuda()]), ref_rows) < TOL_GW_BF16
