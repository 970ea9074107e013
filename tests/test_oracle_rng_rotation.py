"""Pins for the oracle's random stream and rotation.

The rotation is the orthogonal factor of a QR decomposition of a Gaussian
matrix ("Google TurboQuant: 6x KV-cache compression", section "Stage 1:
PolarQuant"). These tests tie the oracle to facts outside itself: the
published SplitMix64 test vector, the normal law, orthogonality, the QR
factorisation of G, and the exact sphere-coordinate law of a Haar rotation.
"""

import numpy as np
import pytest
from scipy import stats

from oracle import codebook, rng, rotation


def test_splitmix64_published_vector():
    # First outputs of SplitMix64 seeded with 0 (reference implementation by
    # Steele/Lea/Flood, as distributed with xoshiro): e220a8397b1dcdaf, 6e789e6aa1b965f4, 06c45d188009454f.
    got = [int(v) for v in rng.splitmix64(0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_splitmix64_counter_slices():
    full = rng.splitmix64(12345, 100)
    assert np.array_equal(full[40:70], rng.splitmix64(12345, 30, start=40))


def test_uniforms_in_unit_interval_and_53_bit():
    u = rng.uniforms(7, 100_000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert np.all((u * 2.0**53) == np.floor(u * 2.0**53))
    assert stats.kstest(u, "uniform").pvalue > 1e-4


def test_gaussians_are_standard_normal():
    g = rng.gaussians(3, 200_000)
    assert abs(g.mean()) < 4.0 / np.sqrt(len(g))
    assert abs(g.var() - 1.0) < 4.0 * np.sqrt(2.0 / len(g))
    assert stats.kstest(g, "norm").pvalue > 1e-4
    # cos/sin outputs of one pair are independent: correlation ~ 0
    assert abs(np.corrcoef(g[0::2], g[1::2])[0, 1]) < 4.0 / np.sqrt(len(g) / 2)


def test_gaussians_box_muller_first_pair_by_hand():
    a, b = rng.uniforms(99, 2)
    r = np.sqrt(-2.0 * np.log(1.0 - a))
    g = rng.gaussians(99, 2)
    assert g[0] == pytest.approx(r * np.cos(2 * np.pi * b), rel=0, abs=1e-15)
    assert g[1] == pytest.approx(r * np.sin(2 * np.pi * b), rel=0, abs=1e-15)


@pytest.mark.parametrize("d", [8, 32, 128])
def test_rotation_orthogonal_and_is_q_of_g(d):
    Pi, S = rotation.rotation(d, seed=5, m=d)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) <= 1e-13
    G = rng.gaussians(5, d * d).reshape(d, d)
    R = Pi.T @ G                      # G = Pi R with R upper triangular, diag(R) > 0
    assert np.max(np.abs(np.tril(R, -1))) <= 1e-12 * np.max(np.abs(R))
    assert np.all(np.diag(R) > 0)
    # S continues the same stream after G
    assert np.array_equal(S, rng.gaussians(5, d * d + d * d)[d * d:].reshape(d, d))


def test_rotation_preserves_norms():
    Pi, _ = rotation.rotation(128, seed=1)
    x = np.random.default_rng(1).standard_normal((64, 128)) * 3.0
    y = x @ Pi.T
    rel = np.abs(np.linalg.norm(y, axis=1) / np.linalg.norm(x, axis=1) - 1.0)
    assert rel.max() <= 1e-14


def test_rotation_is_haar_first_column_law():
    # For a Haar rotation, Pi e_1 is a uniform point on the sphere, so each of
    # its coordinates follows the sphere-coordinate law (1-t^2)^((d-3)/2).
    d = 16
    cols = np.array([rotation.rotation(d, seed=s)[0][:, 0] for s in range(600)])
    t = cols.ravel()
    assert stats.kstest(t, lambda v: codebook.cdf(v, d)).pvalue > 1e-4
    # and the sign fix does not bias the diagonal: E[Pi_11] = 0
    assert abs(cols[:, 0].mean()) < 4.0 / np.sqrt(d * 600)


def test_rotated_spiky_vector_spreads_out():
    # A rotation spreads a one-hot / outlier-heavy direction over all coordinates
    # with the known marginal law (the point of random preconditioning).
    d = 128
    Pi, _ = rotation.rotation(d, seed=2)
    x = np.zeros(d)
    x[3] = 10.0
    x[77] = -7.0
    y = Pi @ (x / np.linalg.norm(x))
    assert stats.kstest(y, lambda v: codebook.cdf(v, d)).pvalue > 1e-3
