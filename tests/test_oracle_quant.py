"""Pins for the oracle's encode, pack and QJL stages.

Encode follows "Google TurboQuant: 6x KV-cache compression" (ebisuda.net),
sections "Stage 1: PolarQuant" and "Stage 2: QJL residual correction". The
pins: a hand-derived packing example, round trips, the tie and zero-vector
readings, the expected distortion (d * MSE of the codebook), the exact bias of
a 1-bit MSE stage under a Haar rotation, and the unbiasedness and exact
variance of the QJL estimator.
"""

import os

import numpy as np
import pytest
from scipy import special

from oracle import codebook, quant, rotation

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            key, *rest = line.split()
            vals[key] = rest
    return vals


def test_pack_hand_worked_example():
    g = _read_golden("pack_d32_b3.txt")
    d, bits = int(g["d"][0]), int(g["bits"][0])
    idx = np.array([[int(v) for v in g["indices"]]])
    want = np.array([[int(v, 16) for v in g["bytes"]]], dtype=np.uint8)
    assert np.array_equal(quant.pack(idx, bits), want)
    assert np.array_equal(quant.unpack(want, d, bits), idx)


@pytest.mark.parametrize("d,bits", [(32, 1), (32, 3), (128, 2), (128, 3), (128, 4), (1536, 2), (5, 3)])
def test_pack_round_trip_and_pad_bits(d, bits):
    rs = np.random.default_rng(d * 10 + bits)
    idx = rs.integers(0, 1 << bits, size=(17, d))
    codes = quant.pack(idx, bits)
    assert codes.shape == (17, (d * bits + 7) // 8)
    assert np.array_equal(quant.unpack(codes, d, bits), idx)
    tail = d * bits % 8
    if tail:
        assert np.all(codes[:, -1] >> tail == 0)


def test_bucketize_tie_goes_to_lower_cell():
    c, beta = codebook.lloyd_max(128, 3)
    y = np.array([beta[0], np.nextafter(beta[0], 1.0), beta[3], -1.0, 1.0, 0.0])
    assert list(quant.bucketize(y, beta)) == [0, 1, 3, 0, 7, 3]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_zero_vector(bits):
    Pi, _ = rotation.rotation(128, 0)
    c, beta = codebook.lloyd_max(128, bits)
    e = quant.encode_mse(np.zeros((2, 128)), Pi, c, beta)
    assert np.all(e["idx"] == (1 << (bits - 1)) - 1)
    assert np.all(e["n_stored"] == 0)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_empirical_distortion_matches_codebook_mse(bits):
    # Rotated coordinates follow the sphere law, so the mean relative error
    # ||x - x_hat||^2 / ||x||^2 over many vectors estimates d * MSE(d, b).
    d = 128
    Pi, _ = rotation.rotation(d, 0)
    c, beta = codebook.lloyd_max(d, bits)
    x = np.random.default_rng(bits).standard_normal((4096, d))
    e = quant.encode_mse(x, Pi, c, beta)
    xh = quant.reconstruct_mse(e["idx"], e["n_exact"], Pi, c)
    dist = np.sum((x - xh) ** 2, 1) / np.sum(x * x, 1)
    se = dist.std(ddof=1) / np.sqrt(len(dist))
    assert abs(dist.mean() - d * codebook.mse(d, c, beta)) < 4 * se


def test_stored_norm_rounding():
    x = np.random.default_rng(0).standard_normal((1000, 128)) * 5
    Pi, _ = rotation.rotation(128, 0)
    c, beta = codebook.lloyd_max(128, 2)
    for dt, eps in (("f32", 2.0 ** -24), ("f16", 2.0 ** -11)):
        e = quant.encode_mse(x, Pi, c, beta, dt)
        assert np.all(np.abs(e["n_stored"].astype(np.float64) / e["n_exact"] - 1) <= eps)


def test_one_bit_mse_inner_product_bias_is_exact():
    # With b = 1 and a Haar rotation, E_Pi <q, x_hat> = d c1^2 <q, x> where
    # c1 = Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2)): the MSE stage shrinks inner
    # products (-> 2/pi for large d), the bias the QJL stage is there to remove.
    d, trials = 16, 4000
    rs = np.random.default_rng(11)
    x = rs.standard_normal(d)
    q = rs.standard_normal(d)
    c, beta = codebook.lloyd_max(d, 1)
    vals = []
    for s in range(trials):
        Pi, _ = rotation.rotation(d, 1000 + s)
        e = quant.encode_mse(x[None], Pi, c, beta)
        vals.append(float(quant.reconstruct_mse(e["idx"], e["n_exact"], Pi, c)[0] @ q))
    vals = np.array(vals)
    c1 = np.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / np.sqrt(np.pi)
    assert c1 == pytest.approx(c[1], rel=1e-12)
    se = vals.std(ddof=1) / np.sqrt(trials)
    assert abs(vals.mean() - d * c1 * c1 * (x @ q)) < 4 * se
    assert abs(vals.mean() - x @ q) > 8 * se          # it is biased


def test_qjl_term_unbiased_and_exact_variance():
    # For s ~ N(0, I): E[<s,q> sign(<s,r>)] = sqrt(2/pi) <q, r>/||r|| and
    # Var = ||q||^2 - (2/pi) <q, r_hat>^2, so the m-row estimate
    # ||r|| sqrt(pi/2)/m <S q, sign(S r)> has mean <q, r> and variance
    # (pi/2) ||r||^2 / m (||q||^2 - (2/pi) <q, r_hat>^2).
    d, m, trials = 24, 16, 20000
    rs = np.random.default_rng(3)
    q = rs.standard_normal(d)
    r = rs.standard_normal(d) * 0.3 + 0.5 * q
    rn = np.linalg.norm(r)
    est = np.empty(trials)
    for t in range(trials):
        S = rs.standard_normal((m, d))
        sigma = (S @ r >= 0).astype(np.int64)
        est[t] = quant.qjl_estimate(q, S @ q, sigma[None], np.array([rn]), m)[0]
    var = np.pi / 2 * rn ** 2 / m * (q @ q - 2 / np.pi * (q @ r / rn) ** 2)
    assert abs(est.mean() - q @ r) < 4 * np.sqrt(var / trials)
    assert est.var(ddof=1) == pytest.approx(var, rel=4 * np.sqrt(2.0 / trials))


def test_prod_estimator_unbiased_over_seeds():
    # Full two-stage encode (1-bit MSE + 1-bit QJL) per seed: the mean over
    # seeds of the prod score equals <q, x> (the MSE bias is corrected).
    from oracle import ops
    d, m, trials = 16, 16, 3000
    rs = np.random.default_rng(5)
    x = rs.standard_normal(d)
    q = rs.standard_normal(d)
    c, beta = codebook.lloyd_max(d, 1)
    vals = np.empty(trials)
    for s in range(trials):
        Pi, S = rotation.rotation(d, 5000 + s, m)
        e = quant.encode_prod(x[None], Pi, S, c, beta, "f32")
        vals[s] = ops.score_prod(q, e["idx"], e["n_exact"], e["sigma"], e["r_exact"], Pi, S, c)[0]
    se = vals.std(ddof=1) / np.sqrt(trials)
    assert abs(vals.mean() - x @ q) < 4 * se


def test_prod_residual_and_signs():
    d, m = 128, 128
    Pi, S = rotation.rotation(d, 2, m)
    c, beta = codebook.lloyd_max(d, 2)
    x = np.random.default_rng(2).standard_normal((512, d))
    e = quant.encode_prod(x, Pi, S, c, beta)
    xh = quant.reconstruct_mse(e["idx"], e["n_exact"], Pi, c)
    assert np.allclose(e["r_exact"], np.linalg.norm(x - xh, axis=1), rtol=1e-13)
    assert np.array_equal(e["sigma"], ((x - xh) @ S.T >= 0).astype(np.int64))
    # ||r||^2 / ||x||^2 averages d * MSE(d, 2)
    rel = (e["r_exact"] / e["n_exact"]) ** 2
    assert abs(rel.mean() - d * codebook.mse(d, c, beta)) < 4 * rel.std(ddof=1) / np.sqrt(len(rel))
    # sign(0) = +1: a zero projection row gives sigma = 1
    S0 = S.copy()
    S0[7] = 0.0
    e0 = quant.encode_prod(x[:4], Pi, S0, c, beta)
    assert np.all(e0["sigma"][:, 7] == 1)


def test_dequantize_prod_is_unbiased_vector_estimate():
    # E_S[x_tilde] = x for fixed Pi: average of QJL back-projections over S draws.
    d, m, trials = 16, 16, 6000
    rs = np.random.default_rng(8)
    x = rs.standard_normal(d)
    Pi, _ = rotation.rotation(d, 3)
    c, beta = codebook.lloyd_max(d, 1)
    acc = np.zeros(d)
    acc2 = np.zeros(d)
    for t in range(trials):
        S = rs.standard_normal((m, d))
        e = quant.encode_prod(x[None], Pi, S, c, beta, "f32")
        xt = quant.dequantize(e["idx"], e["n_exact"], Pi, c, e["sigma"], e["r_exact"], S)[0]
        acc += xt
        acc2 += xt * xt
    mean = acc / trials
    se = np.sqrt((acc2 / trials - mean ** 2) / trials)
    assert np.all(np.abs(mean - x) < 4.5 * se)
