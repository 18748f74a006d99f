"""Pins for the oracle's parameters: generator, D, S and the Lloyd-Max codebook.

Each check compares the oracle with something other than itself: a published
generator output, a second rounding implementation, closed forms, a general
purpose numerical integrator, or Max's (1960) Gaussian quantizer tables.
"""

import math

import numpy as np
import pytest
from scipy import integrate, stats
from scipy.special import gammaln

from oracle import params as op

# --------------------------------------------------------------------------
# SplitMix64
# --------------------------------------------------------------------------
M64 = (1 << 64) - 1


def _sequential_splitmix64(state, n):
    """The generator as published: state += gamma; finalize(state)."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & M64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_first_output():
    # SplitMix64 from state 0: first output 0xE220A8397B1DCDAF.
    assert int(op.splitmix64(0, [0])[0]) == 0xE220A8397B1DCDAF


@pytest.mark.parametrize("seed", [0, 1, 12345, (1 << 63) + 7])
def test_splitmix64_counter_form_equals_sequential(seed):
    want = _sequential_splitmix64(seed, 50)
    got = [int(v) for v in op.splitmix64(seed, np.arange(50))]
    assert got == want


def test_stream_offsets_do_not_overlap():
    c0 = op.stream_counters(op.STREAM_D, 4096)
    c1 = op.stream_counters(op.STREAM_S, 2 * 4096 * 4096)
    assert int(c0.max()) < int(c1.min())


# --------------------------------------------------------------------------
# binary16 rounding: the oracle's formula against numpy's own conversion
# --------------------------------------------------------------------------
def test_round_to_binary16_matches_numpy_cast():
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.standard_normal(200000) * 3,
        rng.standard_normal(20000) * 1e-5,          # subnormal range
        np.ldexp(1.0 + (2 * np.arange(1, 400) + 1) * 2.0 ** -11, 0),   # exact ties at 1.x
        np.ldexp(1.0 + 2.0 ** -11 + 2.0 ** -40, 0) * np.ones(1),       # just above a tie
        -np.ldexp(3.0, -20) * np.ones(1),           # subnormal tie region
        np.array([0.0, -0.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26]),
    ])
    ours = op.round_to_binary16(v)
    theirs = v.astype(np.float16).astype(np.float64)
    assert np.array_equal(ours, theirs)


# --------------------------------------------------------------------------
# D and S
# --------------------------------------------------------------------------
def test_rademacher_values_and_balance():
    D = op.rademacher_diagonal(1 << 16, seed=0)
    assert set(np.unique(D)) == {-1, 1}
    # mean of 65536 fair signs: SE = 1/256
    assert abs(D.mean()) < 4.0 / 256
    assert not np.array_equal(D, op.rademacher_diagonal(1 << 16, seed=1))


def test_gaussian_projection_is_binary16_gaussian():
    S = op.gaussian_projection(512, 512, seed=0)
    assert np.array_equal(S, S.astype(np.float16).astype(np.float64))
    x = S.ravel()
    n = x.size
    assert abs(x.mean()) < 4 / math.sqrt(n)
    assert abs(x.var() - 1.0) < 4 * math.sqrt(2.0 / n)
    kurt = np.mean(x ** 4) / x.var() ** 2
    assert abs(kurt - 3.0) < 4 * math.sqrt(24.0 / n)
    assert stats.kstest(x[:20000], "norm").pvalue > 1e-3


# --------------------------------------------------------------------------
# Coordinate law and codebook
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [16, 128, 1024])
def test_coordinate_density_integrates_to_one(d):
    val, _ = integrate.quad(lambda x: op.coordinate_density(x, d), -1, 1, limit=400, points=[0.0])
    assert abs(val - 1.0) < 1e-10


@pytest.mark.parametrize("d", [16, 128, 1024])
def test_density_second_moment_is_one_over_d(d):
    # A coordinate of a uniform unit vector has E[X^2] = 1/d exactly.
    val, _ = integrate.quad(lambda x: x * x * op.coordinate_density(x, d), -1, 1, limit=400, points=[0.0])
    assert abs(val * d - 1.0) < 1e-9


@pytest.mark.parametrize("d", [16, 128, 1024, 4096])
@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_lloyd_max_centroid_and_midpoint_conditions(d, B):
    c, t, _ = op.lloyd_max(d, B)
    L = 1 << B
    assert c.shape == (L,) and t.shape == (L - 1,)
    assert np.all(np.diff(c) > 0)
    assert np.allclose(c, -c[::-1], rtol=0, atol=1e-15)
    # midpoint condition
    assert np.max(np.abs(t - 0.5 * (c[:-1] + c[1:]))) < 1e-12
    # centroid condition, with an independent adaptive integrator
    edges = np.concatenate([[-1.0], t, [1.0]])
    f = lambda x: op.coordinate_density(x, d)  # noqa: E731
    s = 1.0 / math.sqrt(d)
    for k in range(L):
        lo, hi = max(edges[k], -40 * s), min(edges[k + 1], 40 * s)
        mass, _ = integrate.quad(f, lo, hi, epsabs=0, epsrel=1e-13, limit=400)
        mom, _ = integrate.quad(lambda x: x * f(x), lo, hi, epsabs=0, epsrel=1e-13, limit=400)
        assert abs(mom / mass - c[k]) < 1e-9


@pytest.mark.parametrize("d", [16, 128, 1024, 4096])
def test_one_bit_centroid_closed_form(d):
    # E[X | X > 0] = 2 * integral_0^1 x f_d = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c, _, _ = op.lloyd_max(d, 1)
    want = math.exp(gammaln(d / 2) - gammaln((d + 1) / 2)) / math.sqrt(math.pi)
    # relative 1e-10: the incomplete-beta evaluation is good to ~3e-12 at d = 4096
    assert abs(c[1] - want) < 1e-10 * want
    assert c[0] == -c[1]


# Max (1960), "Quantizing for minimum distortion", optimum quantizers for a
# unit-variance Gaussian: positive output levels and mean squared error.
MAX_LEVELS = {
    1: [0.7979],
    2: [0.4528, 1.510],
    3: [0.2451, 0.7560, 1.344, 2.152],
    4: [0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733],
}
MAX_MSE = {1: 0.3634, 2: 0.1175, 3: 0.03454, 4: 0.009497}


@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_large_d_limit_is_max_gaussian_quantizer(B):
    # The coordinate law tends to N(0, 1/d); at d = 4096 the scaled
    # codebook must sit on Max's Gaussian table (4 printed digits).
    d = 4096
    c, _, _ = op.lloyd_max(d, B)
    got = c[1 << (B - 1):] * math.sqrt(d)
    want = np.array(MAX_LEVELS[B])
    assert np.all(np.abs(got - want) < 1.5e-3 * np.maximum(want, 1.0))
    D = op.mse_distortion(d, c)
    assert abs(D - MAX_MSE[B]) < 2e-3 * MAX_MSE[B] + 1e-5


@pytest.mark.parametrize("d", [16, 128, 1024, 4096])
def test_distortion_within_pages_shannon_factor(d):
    # 0h-n0 explainer, section on the Shannon bound: distortion / (d 2^-2b) <= e,
    # in units where the unit vector's total energy is 1 (D* = 4^-B).
    prev = None
    for B in (1, 2, 3, 4):
        c, _, _ = op.lloyd_max(d, B)
        D = op.mse_distortion(d, c)
        assert 0 < D * 4 ** B <= math.e
        if prev is not None:
            assert 3.0 <= prev / D <= 4.5
        prev = D


def test_params_object_rounds_to_fp32_and_is_symmetric():
    P = op.Params(128, 3, 128, seed=0)
    assert P.centroids.dtype == np.float64
    assert np.array_equal(P.centroids, P.centroids.astype(np.float32).astype(np.float64))
    assert np.array_equal(P.centroids, -P.centroids[::-1])
    assert np.array_equal(P.thresholds, -P.thresholds[::-1])
    assert P.thresholds[P.L // 2 - 1] == 0.0
    assert P.R.shape == (128, 128) and P.S.shape == (128, 128)
