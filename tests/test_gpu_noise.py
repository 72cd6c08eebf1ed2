"""GPU noise vs the oracle: Philox words bit-exact, Gaussians within 2e-6."""
import numpy as np
import pytest
import torch

import oracle
import zeroth_order_transformer_dust_b200 as dust
from _util import TOL_GAUSS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx(cuda_ok):
    return dust.Context(0)


def test_philox_words_bit_exact(ctx):
    rng = np.random.default_rng(0)
    for seed in (0, 1, 0xFFFFFFFFFFFFFFFF, int(rng.integers(0, 2 ** 63))):
        ctr = rng.integers(0, 2 ** 32, size=(1 << 16, 4), dtype=np.uint64)
        ctr[:4] = [[0, 0, 0, 0], [0xFFFFFFFF] * 4, [1, 2, 3, 4], [0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344]]
        t = torch.from_numpy(ctr.astype(np.uint32).view(np.int32)).cuda()
        got = ctx.debug_philox(seed, t).cpu().numpy().view(np.uint32).astype(np.uint64)
        key = (seed & 0xFFFFFFFF, seed >> 32)
        ref = oracle.philox4x32_10((ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3]), key)
        assert np.array_equal(got, np.stack(ref, axis=1))


@pytest.mark.parametrize("table", [False, True])
@pytest.mark.parametrize("tag,stream", [(oracle.TAG_HEAD, 0), (oracle.TAG_MLP_UP, 0), (oracle.TAG_HEAD, 77)])
def test_gaussians_match_oracle(ctx, tag, stream, table):
    nt, ni, ns = 64, 96, 50304 // 24 + 5      # ragged slot count
    seed, t0, i0 = 1234567, 1000, 5000
    got = ctx.debug_gauss(nt, ni, ns, tag=tag, seed=seed, token_offset=t0, draw_offset=i0,
                          stream_id=stream, table=table).cpu().numpy().astype(np.float64)
    ref = oracle.gaussians(seed, np.arange(nt)[:, None] + t0, np.arange(ni)[None, :] + i0,
                           np.arange(ns), tag, stream)
    err = np.abs(got - ref).max()
    assert err < TOL_GAUSS, err


@pytest.mark.parametrize("table", [False, True])
def test_gaussian_extremes_match_oracle(ctx, table):
    # many draws so that the tails (|eps| > 4.5) are exercised
    nt, ni, ns = 8, 4096, 512
    got = ctx.debug_gauss(nt, ni, ns, seed=99, table=table).cpu().numpy().astype(np.float64)
    ref = oracle.gaussians(99, np.arange(nt)[:, None], np.arange(ni)[None, :], np.arange(ns), 0)
    assert np.abs(ref).max() > 4.5
    assert np.abs(got - ref).max() < TOL_GAUSS
