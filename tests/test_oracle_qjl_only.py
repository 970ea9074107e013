"""Pins of the oracle's QJL-only (1-bit) path: a sign sketch of the whole vector plus its norm.

"TurboQuant: redefining AI efficiency" (hakusoku.com), section "QJL: zero-overhead 1-bit
compression"; "TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net), section
"QJL". Checked against facts outside the oracle: the closed-form mean and variance of the
sign estimator for Gaussian projections, the unbiasedness of the back-projection, the sign
convention at zero, and the prod path's definition with an empty MSE stage.
"""

import numpy as np
import pytest

from oracle import codebook, ops, quant, rotation


def test_qjl_only_score_unbiased_with_exact_variance_over_projections():
    # For s ~ N(0, I): E[<s, q> sign(<s, x>)] = sqrt(2/pi) <q, x> / ||x|| and the second moment
    # is ||q||^2, so with m rows the estimate ||x|| sqrt(pi/2)/m <S q, 2 sigma - 1> has mean <q, x>
    # and variance (pi/2) ||x||^2 / m (||q||^2 - (2/pi) <q, x/||x||>^2).
    d, m, trials = 20, 24, 20000
    rs = np.random.default_rng(11)
    x = rs.standard_normal(d)
    q = rs.standard_normal(d) + 0.7 * x
    nx = np.linalg.norm(x)
    est = np.empty(trials)
    for t in range(trials):
        S = rs.standard_normal((m, d))
        e = quant.encode_qjl(x[None], S, "f32")
        est[t] = ops.score_qjl(q, e["sigma"], e["n_exact"], S)[0]
    var = np.pi / 2 * nx ** 2 / m * (q @ q - 2 / np.pi * (q @ x / nx) ** 2)
    assert abs(est.mean() - q @ x) < 4 * np.sqrt(var / trials)
    assert est.var(ddof=1) == pytest.approx(var, rel=4 * np.sqrt(2.0 / trials))


def test_qjl_only_dequantize_is_unbiased_vector_estimate():
    d, m, trials = 12, 16, 8000
    rs = np.random.default_rng(12)
    x = rs.standard_normal(d)
    acc, acc2 = np.zeros(d), np.zeros(d)
    for _ in range(trials):
        S = rs.standard_normal((m, d))
        e = quant.encode_qjl(x[None], S, "f32")
        xt = quant.dequantize_qjl(e["sigma"], e["n_exact"], S)[0]
        acc += xt
        acc2 += xt * xt
    mean = acc / trials
    se = np.sqrt((acc2 / trials - mean ** 2) / trials)
    assert np.all(np.abs(mean - x) < 4.5 * se)


def test_qjl_only_signs_norm_and_zero_vector():
    d, m = 64, 96
    _, S = rotation.rotation(d, 4, m)
    x = np.random.default_rng(4).standard_normal((50, d)) * 3.0
    x[7] = 0.0
    e = quant.encode_qjl(x, S, "f16")
    # sign bit j is the sign of projection j, with sign(0) = +1
    assert np.array_equal(e["sigma"], ((x @ S.T) >= 0).astype(np.int64))
    assert np.all(e["sigma"][7] == 1)
    assert np.allclose(e["n_exact"], np.linalg.norm(x, axis=1), rtol=1e-14)
    assert e["n_stored"].dtype == np.float16 and e["n_stored"][7] == 0
    q = np.random.default_rng(5).standard_normal(d)
    assert ops.score_qjl(q, e["sigma"][7:8], e["n_stored"][7:8], S)[0] == 0.0
    # signs depend only on the directions of the projection rows
    e2 = quant.encode_qjl(x, 2.0 * S, "f16")
    assert np.array_equal(e2["sigma"], e["sigma"])


def test_qjl_only_equals_prod_with_an_empty_mse_stage():
    # With zero MSE bits the prod reconstruction is 0 (a one-cell Lloyd-Max quantizer of a
    # symmetric law sits at its mean 0), so the residual is x itself, its norm is ||x||, and
    # the prod estimator and decode reduce to the QJL-only ones.
    d, m = 32, 64
    Pi, S = rotation.rotation(d, 6, m)
    x = np.random.default_rng(6).standard_normal((40, d))
    c0, beta0 = np.zeros(1), np.zeros(0)
    p = quant.encode_prod(x, Pi, S, c0, beta0, "f32")
    e = quant.encode_qjl(x, S, "f32")
    assert np.array_equal(p["sigma"], e["sigma"])
    assert np.allclose(p["r_exact"], e["n_exact"], rtol=1e-14)
    q = np.random.default_rng(7).standard_normal(d)
    s_prod = ops.score_prod(q, p["idx"], p["n_exact"], p["sigma"], p["r_exact"], Pi, S, c0)
    s_qjl = ops.score_qjl(q, e["sigma"], e["n_exact"], S)
    assert np.allclose(s_prod, s_qjl, rtol=1e-12, atol=1e-12)
    xt_prod = quant.dequantize(p["idx"], p["n_exact"], Pi, c0, p["sigma"], p["r_exact"], S)
    assert np.allclose(xt_prod, quant.dequantize_qjl(e["sigma"], e["n_exact"], S), rtol=1e-12, atol=1e-12)
    # a one-cell Lloyd-Max codebook of the symmetric coordinate law is its mean, {0}
    cz, bz = codebook.lloyd_max(d, 0)
    assert cz.shape == (1,) and abs(cz[0]) < 1e-15 and bz.shape == (0,)


def test_qjl_only_score_equals_inner_product_with_dequantized_vector():
    d, m = 48, 64
    _, S = rotation.rotation(d, 8, m)
    x = np.random.default_rng(8).standard_normal((30, d))
    q = np.random.default_rng(9).standard_normal(d)
    e = quant.encode_qjl(x, S, "f16")
    s = ops.score_qjl(q, e["sigma"], e["n_stored"], S)
    xt = quant.dequantize_qjl(e["sigma"], e["n_stored"], S)
    assert np.allclose(s, xt @ q, rtol=1e-12, atol=1e-12)


def _qjl_cache(B, Hkv, L, d, m, seed):
    _, S = rotation.rotation(d, seed, m)
    x = np.random.default_rng(seed).standard_normal((B * Hkv * L, d)) * 1.5
    e = quant.encode_qjl(x, S, "f16")
    return {"sigma": e["sigma"].reshape(B, Hkv, L, m), "n": e["n_stored"].reshape(B, Hkv, L), "S": S}


def _prod_cache(B, Hkv, L, d, seed):
    Pi, S = rotation.rotation(d, seed, d)
    c, beta = codebook.lloyd_max(d, 2)
    x = np.random.default_rng(seed).standard_normal((B * Hkv * L, d))
    e = quant.encode_prod(x, Pi, S, c, beta, "f16")
    return {"idx": e["idx"].reshape(B, Hkv, L, d), "n": e["n_stored"].reshape(B, Hkv, L), "Pi": Pi, "c": c,
            "sigma": e["sigma"].reshape(B, Hkv, L, d), "rnorm": e["rnorm_stored"].reshape(B, Hkv, L), "S": S}


@pytest.mark.parametrize("k_kind,v_kind", [("qjl", "qjl"), ("qjl", "prod"), ("prod", "qjl")])
def test_attention_two_routes_agree_with_qjl_only_caches(k_kind, v_kind):
    B, Hkv, G, L, d = 2, 2, 2, 300, 32
    kq = _qjl_cache(B, Hkv, L, d, 64, 20) if k_kind == "qjl" else _prod_cache(B, Hkv, L, d, 20)
    vq = _qjl_cache(B, Hkv, L, d, 96, 21) if v_kind == "qjl" else _prod_cache(B, Hkv, L, d, 21)
    q = np.random.default_rng(22).standard_normal((B, Hkv * G, d))
    lens = [300, 171]
    a = ops.decode_attention(q, kq, vq, lens, 1 / np.sqrt(d))
    b = ops.decode_attention_streaming(q, kq, vq, lens, 1 / np.sqrt(d), chunk=64)
    assert np.allclose(a, b, rtol=1e-11, atol=1e-12)
