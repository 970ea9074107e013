"""Pins for the oracle's scores, decode attention and top-k search.

Attention is the textbook softmax(q K^T / sqrt(d_k)) V ("TurboQuant /
PolarQuant / QJL technical deep dive" (gemilab.net), section "Scaled
dot-product attention"). Scores are the inner-product estimates the
attention and the search consume. The pins compare two independent routes
(explicit dequantize vs rotated-domain lookup / chunked log-sum-exp), check a
library softmax, the degenerate cases (uniform and one-hot attention), the
grouped-query mapping, and brute-force top-k.
"""

import numpy as np
import pytest
from scipy import special

from oracle import codebook, ops, quant, rotation


def _cache(B, Hkv, L, d, bits, seed, prod, scale_rows=None):
    rs = np.random.default_rng(seed)
    x = rs.standard_normal((B, Hkv, L, d))
    if scale_rows is not None:
        x = x * scale_rows
    m = d if prod else 0
    Pi, S = rotation.rotation(d, seed, m)
    c, beta = codebook.lloyd_max(d, bits - 1 if prod else bits)
    flat = x.reshape(-1, d)
    if prod:
        e = quant.encode_prod(flat, Pi, S, c, beta, "f16")
        out = {"idx": e["idx"].reshape(B, Hkv, L, d), "n": e["n_stored"].reshape(B, Hkv, L),
               "sigma": e["sigma"].reshape(B, Hkv, L, m), "rnorm": e["rnorm_stored"].reshape(B, Hkv, L),
               "Pi": Pi, "S": S, "c": c}
    else:
        e = quant.encode_mse(flat, Pi, c, beta, "f16")
        out = {"idx": e["idx"].reshape(B, Hkv, L, d), "n": e["n_stored"].reshape(B, Hkv, L),
               "Pi": Pi, "c": c}
    return x, out


def test_score_lookup_route_equals_explicit_inner_product():
    d = 64
    x, k = _cache(1, 1, 300, d, 3, 1, prod=False)
    q = np.random.default_rng(9).standard_normal(d)
    s = ops.score_mse(q, k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"])
    xh = quant.dequantize(k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"])
    assert np.allclose(s, xh @ q, rtol=1e-12, atol=1e-12)


def test_prod_score_equals_inner_product_with_dequantized_vector():
    d = 64
    x, k = _cache(1, 1, 300, d, 3, 2, prod=True)
    q = np.random.default_rng(9).standard_normal(d)
    s = ops.score_prod(q, k["idx"][0, 0], k["n"][0, 0], k["sigma"][0, 0], k["rnorm"][0, 0],
                       k["Pi"], k["S"], k["c"])
    xt = quant.dequantize(k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"], k["sigma"][0, 0],
                          k["rnorm"][0, 0], k["S"])
    assert np.allclose(s, xt @ q, rtol=1e-12, atol=1e-12)


def test_softmax_attention_matches_library_softmax():
    rs = np.random.default_rng(0)
    K, V, q = rs.standard_normal((50, 8)), rs.standard_normal((50, 8)), rs.standard_normal(8)
    o = ops.softmax_attention(q, K, V, 0.3)
    assert np.allclose(o, special.softmax(0.3 * K @ q) @ V, rtol=1e-13)


@pytest.mark.parametrize("prod_k,prod_v", [(False, False), (True, True), (True, False)])
def test_attention_two_routes_agree(prod_k, prod_v):
    B, Hkv, Hq, L, d = 2, 2, 4, 2500, 32
    _, k = _cache(B, Hkv, L, d, 3, 4, prod_k)
    _, v = _cache(B, Hkv, L, d, 3 if prod_v else 4, 5, prod_v)
    q = np.random.default_rng(6).standard_normal((B, Hq, d)) * 2
    lens = np.array([L, 1777])
    o1 = ops.decode_attention(q, k, v, lens, 1 / np.sqrt(d))
    o2 = ops.decode_attention_streaming(q, k, v, lens, 1 / np.sqrt(d), chunk=333)
    assert np.allclose(o1, o2, rtol=1e-11, atol=1e-12)


def test_attention_uniform_and_one_hot_limits():
    B, Hkv, Hq, L, d = 1, 1, 2, 40, 32
    _, k = _cache(B, Hkv, L, d, 3, 7, False)
    _, v = _cache(B, Hkv, L, d, 3, 8, False)
    vhat = quant.dequantize(v["idx"][0, 0], v["n"][0, 0], v["Pi"], v["c"])
    # zero query: all logits equal -> mean of the dequantized values
    o = ops.decode_attention(np.zeros((B, Hq, d)), k, v, [L], 1.0)
    assert np.allclose(o[0, 0], vhat.mean(0), rtol=1e-12)
    # a query aligned with one dequantized key and a huge scale -> that key's value
    khat = quant.dequantize(k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"])
    j = int(np.argmax(np.linalg.norm(khat, axis=1)))
    q = np.tile(khat[j] / np.linalg.norm(khat[j]), (B, Hq, 1))
    o = ops.decode_attention(q, k, v, [L], 1e4)
    assert np.allclose(o[0, 1], vhat[j], rtol=1e-9)


def test_gqa_head_mapping():
    B, Hkv, Hq, L, d = 1, 2, 4, 30, 32
    _, k = _cache(B, Hkv, L, d, 3, 10, False)
    _, v = _cache(B, Hkv, L, d, 3, 11, False)
    q = np.random.default_rng(12).standard_normal((B, Hq, d))
    o = ops.decode_attention(q, k, v, [L], 0.2)
    for h in range(Hq):
        hk = h // 2
        K = quant.dequantize(k["idx"][0, hk], k["n"][0, hk], k["Pi"], k["c"])
        V = quant.dequantize(v["idx"][0, hk], v["n"][0, hk], v["Pi"], v["c"])
        assert np.allclose(o[0, h], special.softmax(0.2 * K @ q[0, h]) @ V, rtol=1e-12)


def test_topk_brute_force_and_ties():
    rs = np.random.default_rng(1)
    s = np.round(rs.standard_normal((5, 200)), 1)       # many exact ties
    idx, val = ops.topk(s, 10)
    for r in range(5):
        pairs = sorted(((-s[r, i], i) for i in range(200)))[:10]
        assert list(idx[r]) == [i for _, i in pairs]
        assert np.array_equal(val[r], s[r, idx[r]])


def test_search_scores_match_per_query_scores():
    d = 64
    _, k = _cache(1, 1, 500, d, 2, 13, False)
    Q = np.random.default_rng(14).standard_normal((7, d))
    S = ops.search_scores(Q, k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"])
    for i in range(7):
        assert np.allclose(S[i], ops.score_mse(Q[i], k["idx"][0, 0], k["n"][0, 0], k["Pi"], k["c"]),
                           rtol=1e-12, atol=1e-12)
