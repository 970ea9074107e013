"""Pins of the recursive polar transform and its angle codebooks (oracle/polar.py), against facts
outside the oracle: exact inversion, the norm as the last radius, closed forms (the uniform
level-1 law and its grid codebook with MSE step^2/12; the level-2 law sin^2), the simulated
law of each level's angles for rotated Gaussian vectors (KS tests), independence of the
levels, and the Lloyd-Max fixed point checked by Monte Carlo conditional means."""

import numpy as np
import pytest
from scipy import stats

from oracle import polar, rotation


@pytest.mark.parametrize("d", [2, 8, 128, 1024])
def test_inverse_recovers_the_vector_and_the_last_radius_is_the_norm(d):
    x = np.random.default_rng(d).standard_normal((50, d)) * 3.0
    ang, r = polar.transform(x)
    assert len(ang) == polar.n_levels(d) and ang[-1].shape == (50, 1)
    assert np.allclose(r, np.linalg.norm(x, axis=1), rtol=1e-14, atol=0)
    assert np.max(np.abs(polar.inverse(ang, r) - x)) <= 1e-12 * np.max(np.abs(x))
    # level-1 angles span (-pi, pi], deeper ones [0, pi/2]
    assert np.all(np.abs(ang[0]) <= np.pi)
    for a in ang[1:]:
        assert np.all((a >= 0) & (a <= np.pi / 2))


def test_rejects_a_dimension_that_is_not_a_power_of_two():
    with pytest.raises(ValueError):
        polar.n_levels(96)


@pytest.mark.parametrize("level", [1, 2, 3, 5])
def test_each_level_follows_its_law_for_a_uniform_direction(level):
    # the laws are stated for a uniform direction (what the random rotation produces over the
    # rotation's draw); a normalised Gaussian row is one, and is what is sampled here
    d = 64
    g = np.random.default_rng(level).standard_normal((4000, d))
    ang, _ = polar.transform(g / np.linalg.norm(g, axis=1, keepdims=True))
    sample = ang[level - 1].ravel()[:20000]
    p = stats.kstest(sample, lambda t: polar.cdf(t, level)).pvalue
    assert p > 1e-3, p


def test_level_laws_closed_forms():
    t = np.linspace(-np.pi, np.pi, 9)
    assert np.allclose(polar.cdf(t, 1), (t + np.pi) / (2 * np.pi))
    p = np.linspace(0, np.pi / 2, 9)
    assert np.allclose(polar.cdf(p, 2), np.sin(p) ** 2, atol=1e-15)   # two 2-D blocks: Beta(1, 1) in sin^2
    for level in (2, 3, 4, 6):   # a density on [0, pi/2], symmetric about pi/4
        from scipy import integrate
        assert abs(integrate.quad(lambda q: polar.pdf(q, level), 0, np.pi / 2)[0] - 1) < 1e-10
        assert np.allclose(polar.pdf(p, level), polar.pdf(np.pi / 2 - p, level))


def test_levels_are_independent():
    g = np.random.default_rng(7).standard_normal((20000, 8))
    ang, _ = polar.transform(g)
    r = np.corrcoef(np.stack([ang[0][:, 0], ang[0][:, 1], ang[1][:, 0], ang[2][:, 0]]))
    assert np.max(np.abs(r - np.eye(4))) < 0.03


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_level_one_codebook_is_the_uniform_grid(bits):
    c, b = polar.lloyd_max(1, bits)
    L = 1 << bits
    step = 2 * np.pi / L
    assert np.allclose(c, -np.pi + step * (np.arange(L) + 0.5))
    assert np.allclose(b, -np.pi + step * np.arange(1, L))
    # its MSE on the uniform law is step^2 / 12 (Monte Carlo)
    t = np.random.default_rng(bits).uniform(-np.pi, np.pi, 200000)
    mse = np.mean((t - c[polar.quantize(t, b)]) ** 2)
    assert abs(mse / (step ** 2 / 12) - 1) < 0.02


@pytest.mark.parametrize("level,bits", [(2, 2), (3, 3), (5, 2)])
def test_deeper_codebooks_are_lloyd_max_fixed_points(level, bits):
    c, b = polar.lloyd_max(level, bits)
    assert np.all(np.diff(c) > 0) and np.allclose(b, 0.5 * (c[:-1] + c[1:]))
    assert np.allclose(c + c[::-1], np.pi / 2)   # symmetric about pi/4
    # each centroid is the mean of the angles in its cell, checked on simulated angles
    d = 2 ** (level + 1)
    g = np.random.default_rng(level * 10 + bits).standard_normal((400000 // d * 2, d))
    ang, _ = polar.transform(g)
    a = ang[level - 1].ravel()
    cell = polar.quantize(a, b)
    for i in range(len(c)):
        sel = a[cell == i]
        assert abs(sel.mean() - c[i]) < 4 * sel.std() / np.sqrt(len(sel)) + 1e-4, (i, sel.mean(), c[i])


def test_encode_decode_distortion_falls_with_bits_and_vanishes_at_high_precision():
    d = 64
    Pi = rotation.rotation(d, 3, 0)[0]
    x = np.random.default_rng(4).standard_normal((300, d))
    errs = []
    for bits in (1, 2, 3):
        books = polar.codebooks(d, bits)
        e = polar.encode(x, Pi, books)
        xh = polar.decode(e["idx"], e["n_exact"], Pi, books)
        errs.append(np.mean(np.sum((xh - x) ** 2, 1) / np.sum(x ** 2, 1)))
    assert errs[0] > errs[1] > errs[2]
    books = polar.codebooks(d, 8)
    e = polar.encode(x, Pi, books)
    xh = polar.decode(e["idx"], e["n_exact"], Pi, books)
    assert np.mean(np.sum((xh - x) ** 2, 1) / np.sum(x ** 2, 1)) < 1e-3
    assert polar.bits_per_vector(d, [4, 2, 2, 2, 2, 2]) == 32 * 4 + 31 * 2


@pytest.mark.parametrize("d,bits", [(8, 2), (128, [4, 2, 2, 2, 2, 2, 2])])
def test_score_up_the_tree_equals_the_dot_product_with_the_reconstruction(d, bits):
    Pi = rotation.rotation(d, 5, 0)[0]
    rs = np.random.default_rng(d)
    x = rs.standard_normal((40, d)) * 2.0
    q = rs.standard_normal(d)
    books = polar.codebooks(d, bits)
    e = polar.encode(x, Pi, books)
    xh = polar.decode(e["idx"], e["n_exact"], Pi, books)
    got = polar.score(q, e["idx"], e["n_exact"], Pi, books)
    assert np.allclose(got, xh @ q, rtol=1e-12, atol=1e-12 * np.abs(xh @ q).max())


def _read_golden(name):
    import os
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            key, *rest = line.split()
            vals[key] = rest
    return vals


def test_pack_hand_worked_example():
    g = _read_golden("polar_pack_d8.txt")
    d = int(g["d"][0])
    bits = [int(v) for v in g["bits"]]
    idx = [np.array([[int(v) for v in g[f"level{lv}"]]]) for lv in (1, 2, 3)]
    want = np.array([[int(v, 16) for v in g["bytes"]]], dtype=np.uint8)
    assert polar.row_bytes(d, bits) == 16
    assert np.array_equal(polar.pack(idx, d, bits), want)
    got = polar.unpack(want, d, bits)
    assert all(np.array_equal(a, b) for a, b in zip(got, idx))


@pytest.mark.parametrize("d,bits", [(128, [4, 2, 2, 2, 2, 2, 2]), (32, 3), (64, [1, 4, 3, 2, 1, 1]), (256, 2)])
def test_pack_round_trip_and_zero_pad(d, bits):
    nl = polar.n_levels(d)
    bl = [bits] * nl if np.isscalar(bits) else bits
    rs = np.random.default_rng(d)
    idx = [rs.integers(0, 1 << bl[lv], size=(9, d >> (lv + 1))) for lv in range(nl)]
    codes = polar.pack(idx, d, bits)
    assert codes.shape == (9, polar.row_bytes(d, bits)) and codes.shape[1] % 16 == 0
    assert all(np.array_equal(a, b) for a, b in zip(polar.unpack(codes, d, bits), idx))
    total = polar.bits_per_vector(d, bits)
    tail = np.unpackbits(codes, axis=1, bitorder="little")[:, total:]
    assert not tail.any()
