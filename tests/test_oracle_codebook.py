"""Pins for the oracle's Lloyd-Max codebook.

"Google TurboQuant: 6x KV-cache compression", section "Stage 1: PolarQuant":
Lloyd-Max solves continuous k-means on the known coordinate law and returns
MSE-minimising boundaries and centroids per bit width. The checks below use
closed forms (d = 3 makes the law uniform; b = 1 gives +-E|T|), a brute-force
minimisation with an independent integrator, the textbook Gaussian limit, and
invariants (symmetry, MSE falling with bits).
"""

import numpy as np
import pytest
from scipy import integrate, optimize, special, stats

from oracle import codebook


def _density(d):
    k = (d - 3) / 2.0
    z = integrate.quad(lambda t: (1 - t * t) ** k, -1, 1, epsabs=1e-14, epsrel=1e-13)[0]
    return lambda t: (1 - t * t) ** k / z


def _mse_by_quad(d, c):
    """Nearest-centroid MSE with scipy quad on the raw density (independent of the oracle's integrals)."""
    f = _density(d)
    c = np.sort(np.asarray(c, dtype=np.float64))
    edges = np.concatenate(([-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]))
    tot = 0.0
    for i, ci in enumerate(c):
        tot += integrate.quad(lambda t: (t - ci) ** 2 * f(t), edges[i], edges[i + 1],
                              epsabs=1e-15, epsrel=1e-12)[0]
    return tot


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_uniform_closed_form(bits):
    # d = 3: (1-t^2)^0 is uniform on [-1, 1]; optimal L-level quantizer is the
    # uniform grid with cell width 2/L, per-coordinate MSE = (2/L)^2/12, d*MSE = 4^-b.
    L = 1 << bits
    c, beta = codebook.lloyd_max(3, bits)
    assert np.allclose(c, -1.0 + (2 * np.arange(L) + 1) / L, atol=1e-12)
    assert 3 * codebook.mse(3, c, beta) == pytest.approx(4.0 ** -bits, abs=1e-12)


@pytest.mark.parametrize("d", [3, 4, 5, 16, 128, 1536])
def test_one_bit_closed_form(d):
    # b = 1: centroids +-E|T| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)).
    c, beta = codebook.lloyd_max(d, 1)
    want = np.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / np.sqrt(np.pi)
    assert c[1] == pytest.approx(want, rel=1e-12)
    assert c[0] == -c[1] and beta[0] == 0.0


def test_one_bit_d128_value():
    c, _ = codebook.lloyd_max(128, 1)
    assert c[1] == pytest.approx(0.0706616, abs=5e-8)


@pytest.mark.parametrize("d,bits", [(3, 1), (4, 1), (5, 1), (3, 2), (4, 2), (5, 2)])
def test_brute_force_minimum(d, bits):
    """Grid + local search over symmetric codebooks reaches the Lloyd-Max optimum."""
    c, _ = codebook.lloyd_max(d, bits)
    if bits == 1:
        grid = np.linspace(0.01, 0.99, 99)
        vals = [_mse_by_quad(d, [-a, a]) for a in grid]
        a0 = grid[int(np.argmin(vals))]
        res = optimize.minimize_scalar(lambda a: _mse_by_quad(d, [-a, a]),
                                       bounds=(a0 - 0.01, a0 + 0.01), method="bounded",
                                       options={"xatol": 1e-10})
        best = np.array([-res.x, res.x])
    else:
        grid = np.linspace(0.02, 0.98, 25)
        vals = {(a, b): _mse_by_quad(d, [-b, -a, a, b]) for a in grid for b in grid if b > a}
        a0, b0 = min(vals, key=vals.get)
        res = optimize.minimize(lambda p: _mse_by_quad(d, [-p[1], -p[0], p[0], p[1]]),
                                x0=[a0, b0], method="Nelder-Mead",
                                options={"xatol": 1e-9, "fatol": 1e-15, "maxiter": 4000})
        best = np.array([-res.x[1], -res.x[0], res.x[0], res.x[1]])
    assert np.allclose(best, c, atol=2e-5)
    assert _mse_by_quad(d, c) <= _mse_by_quad(d, best) + 1e-13


@pytest.mark.parametrize("d,bits", [(16, 2), (128, 3), (128, 4), (1536, 2)])
def test_centroid_condition_independent_integrator(d, bits):
    """Each centroid is the conditional mean of its cell (quad on the raw density)."""
    f = _density(d)
    c, beta = codebook.lloyd_max(d, bits)
    lim = min(1.0, 40.0 / np.sqrt(d))
    edges = np.concatenate(([-lim], beta, [lim]))
    for i in range(len(c)):
        lo, hi = edges[i], edges[i + 1]
        num = integrate.quad(lambda t: t * f(t), lo, hi, epsabs=1e-16, epsrel=1e-12, limit=200)[0]
        den = integrate.quad(f, lo, hi, epsabs=1e-16, epsrel=1e-12, limit=200)[0]
        assert c[i] == pytest.approx(num / den, rel=1e-9, abs=1e-13)
    assert np.allclose(beta, 0.5 * (c[:-1] + c[1:]), atol=0)


@pytest.mark.parametrize("d", [5, 128, 1536])
def test_symmetry_and_mse_falls_with_bits(d):
    prev = np.inf
    for bits in range(1, 5):
        c, beta = codebook.lloyd_max(d, bits)
        assert np.array_equal(c, -c[::-1])
        assert np.all(np.diff(c) > 0)
        m = codebook.mse(d, c, beta)
        assert m < prev
        prev = m


def _gaussian_lloyd(bits, iters=20000):
    """Independent Lloyd-Max for N(0,1) using scipy.stats.norm (textbook limit)."""
    L = 1 << bits
    c = stats.norm.ppf((np.arange(L) + 0.5) / L)
    for _ in range(iters):
        e = np.concatenate(([-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]))
        new = (stats.norm.pdf(e[:-1]) - stats.norm.pdf(e[1:])) / (stats.norm.cdf(e[1:]) - stats.norm.cdf(e[:-1]))
        if np.max(np.abs(new - c)) < 1e-14:
            c = new
            break
        c = new
    return c


# Max (1960), "Quantizing for minimum distortion", table of optimum output levels
# for a unit-variance Gaussian (positive half, 4 significant digits).
MAX_1960 = {
    1: [0.7979],
    2: [0.4528, 1.510],
    3: [0.2451, 0.7560, 1.344, 2.152],
    4: [0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733],
}


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_large_d_limit_is_gaussian_lloyd_max(bits):
    g = _gaussian_lloyd(bits)
    L = 1 << bits
    assert np.allclose(g[L // 2:], MAX_1960[bits], rtol=6e-4, atol=0)
    c, _ = codebook.lloyd_max(1536, bits)
    # sqrt(d) T -> N(0,1) with O(1/d) corrections: a few 1e-3 at d = 1536
    assert np.allclose(c * np.sqrt(1536), g, rtol=5e-3)


def test_reference_probe_mse_values():
    # d * MSE values of an earlier independent probe (a sanity reference only).
    want = {(128, 1): 0.360889, (128, 2): 0.116000, (128, 3): 0.033966, (128, 4): 0.009315,
            (1536, 2): 0.117358, (1536, 4): 0.009485}
    for (d, b), v in want.items():
        c, beta = codebook.lloyd_max(d, b)
        assert d * codebook.mse(d, c, beta) == pytest.approx(v, abs=1.5e-6)
    c, _ = codebook.lloyd_max(128, 3)
    assert np.allclose(c[4:] * np.sqrt(128), [0.24442, 0.75333, 1.33660, 2.13147], atol=1e-5)


def test_mse_formula_matches_quad():
    for d, bits in [(4, 2), (128, 3)]:
        c, beta = codebook.lloyd_max(d, bits)
        assert codebook.mse(d, c, beta) == pytest.approx(_mse_by_quad(d, c), rel=1e-9)
