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


def test_packed_table_step_equals_the_scalar_one_bit_for_bit(ctx):
    """The draw kernels run the table-driven Box-Muller step in packed fp32x2
    form (two pairs per instruction); the scalar form that the exhaustive
    radius and angle checks below cover must give the same bits."""
    for seed, tag, t0 in ((3, oracle.TAG_HEAD, 0), (0xFFFFFFFFFFFF, oracle.TAG_HEAD, 123456),
                          (77, oracle.TAG_MLP_UP, 9)):
        a = ctx.debug_gauss(128, 256, 1024, tag=tag, seed=seed, token_offset=t0, table=True)
        b = ctx.debug_gauss(128, 256, 1024, tag=tag, seed=seed, token_offset=t0, table=True,
                            scalar=True)
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("table", [False, True])
def test_gaussian_extremes_match_oracle(ctx, table):
    # many draws so that the tails (|eps| > 4.5) are exercised
    nt, ni, ns = 8, 4096, 512
    got = ctx.debug_gauss(nt, ni, ns, seed=99, table=table).cpu().numpy().astype(np.float64)
    ref = oracle.gaussians(99, np.arange(nt)[:, None], np.arange(ni)[None, :], np.arange(ns), 0)
    assert np.abs(ref).max() > 4.5
    assert np.abs(got - ref).max() < TOL_GAUSS


# Exhaustive checks of the two one-dimensional pieces of the Box-Muller
# transform over all 2^24 inputs each. A Gaussian is the rounded product
# fl(A~ B~) of a radius factor A~ = A + dA and an angle factor B~ = B + dB, so
# for one radius input and any angle input
#   |eps error| <= |dA| |B~| + A |dB| + 2^-24 |A~| |B~|   (round to nearest)
#              <= |dA| b + A max|dB| + 2^-24 (A + |dA|) b,  b = max|B~|,
# and the maximum of that over the 2^24 radius inputs bounds the error of every
# pair of words. The polynomial step multiplies the radius R (A = R,
# B = cos or sin); the table step multiplies rho = R / sqrt(2 ln 2) into a
# table that carries sqrt(2 ln 2) (A = rho, B = sqrt(2 ln 2) cos or sin).
# The bound holding is the 2e-6 bar for every pair of words.
R_MAX = float(np.sqrt(-2.0 * np.log(2.0 ** -24)))
KAPPA = float(np.sqrt(2.0 * np.log(2.0)))
KAPPA_F32 = np.float32(1.17741)          # the library's rounded sqrt(2 ln 2)


def _radius_ref():
    j = np.arange(1, (1 << 24) + 1, dtype=np.float64)
    return np.sqrt(-2.0 * np.log(j * 2.0 ** -24))


def _angle_ref():
    theta = np.arange(1 << 24, dtype=np.float64) * (np.pi * 2.0 ** -23)
    return np.cos(theta), np.sin(theta)


@pytest.fixture(scope="module")
def radius_err(ctx):
    """{table: (|dA| per radius input, A)}"""
    ref = _radius_ref()
    out = {}
    got = ctx.debug_bm_radius(1.0).cpu().numpy().astype(np.float64)
    out[False] = (np.abs(got - ref), ref)
    got = ctx.debug_bm_radius(table=True).cpu().numpy().astype(np.float64)
    out[True] = (np.abs(got - ref / KAPPA), ref / KAPPA)
    return out


@pytest.fixture(scope="module")
def angle_err(ctx):
    c, s = _angle_ref()
    out = {}
    for table in (False, True):
        scale = KAPPA if table else 1.0
        got = ctx.debug_bm_angle(table).cpu().numpy().astype(np.float64)
        out[table] = max(np.abs(got[:, 0] - scale * c).max(), np.abs(got[:, 1] - scale * s).max())
    return out


@pytest.mark.parametrize("table", [False, True])
def test_radius_all_inputs(radius_err, table):
    # a few 1e-7 everywhere (in units of R), including u1 -> 1 where the
    # radius -> 0
    err = radius_err[table][0] * (KAPPA if table else 1.0)
    assert err.max() < 9e-7, err.max()
    assert err[-(1 << 18):].max() < 2e-7      # the series branch, v < 2^-6


def test_radius_scales_with_sigma(ctx):
    # the polynomial step's radius is fl(fl(sigma sqrt(2 ln 2)) rho): bit for
    # bit the float32 products of rho
    rho = ctx.debug_bm_radius(table=True).cpu().numpy()
    for sigma in (1.0, 5e-3, 1e-2, 0.37):
        got = ctx.debug_bm_radius(sigma).cpu().numpy()
        want = (np.float32(sigma) * KAPPA_F32) * rho
        assert want.dtype == np.float32 and np.array_equal(got, want)
    assert not ctx.debug_bm_radius(0.0).any()         # sigma = 0: exact zeros


@pytest.mark.parametrize("table", [False, True])
def test_angle_all_inputs(angle_err, table):
    assert angle_err[table] < (2.5e-7 if table else 2e-7), angle_err[table]


@pytest.mark.parametrize("table", [False, True])
def test_gaussian_bound_over_all_words(radius_err, angle_err, table):
    d_a, a = radius_err[table]
    d_b = angle_err[table]
    b = (KAPPA if table else 1.0) + d_b              # largest |angle factor|
    per_radius = d_a * b + a * d_b + 2.0 ** -24 * (a + d_a) * b
    bound = per_radius.max() * (1 + 1e-6)
    assert bound < TOL_GAUSS, bound
