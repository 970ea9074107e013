"""GPU parity of scores, decode attention, append and search against the oracle.

Kernel parity: the GPU reads caches filled with the ORACLE's codes (packed by
the oracle and uploaded), so both sides score identical codes. End-to-end
parity (GPU encode -> GPU attention vs oracle encode -> oracle attention) is
checked separately with the same tolerance."""

import numpy as np
import pytest
import torch

from gpu_util import ATTN_RTOL, OracleHandle, check_codes, check_norms, score_tolerance, to_np64
from oracle import ops, quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    m = build_lib()
    return m


NORM_NP = {0: "f32", 1: "f16"}


def oracle_cache(tq, h, oh, x):
    """Oracle-encoded cache for x [B, Hkv, L, d] (np fp64) uploaded into a GPU Cache; returns (cache, odict)."""
    B, Hkv, L, d = x.shape
    e = oh.encode(x.reshape(-1, d), NORM_NP[h.norm_dtype])
    cache = tq.Cache(h, B, Hkv, L)
    cache.codes.copy_(torch.from_numpy(quant.pack(e["idx"], oh.bits).reshape(B, Hkv, L, -1)))
    cache.norms.copy_(torch.from_numpy(e["n_stored"].reshape(B, Hkv, L)))
    od = {"idx": e["idx"].reshape(B, Hkv, L, d), "n": e["n_stored"].reshape(B, Hkv, L), "Pi": oh.Pi, "c": oh.c}
    if oh.m:
        cache.signs.copy_(torch.from_numpy(quant.pack(e["sigma"], 1).reshape(B, Hkv, L, -1)))
        cache.rnorms.copy_(torch.from_numpy(e["rnorm_stored"].reshape(B, Hkv, L)))
        od.update({"sigma": e["sigma"].reshape(B, Hkv, L, oh.m), "rnorm": e["rnorm_stored"].reshape(B, Hkv, L),
                   "S": oh.S})
    return cache, od


def _kv(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("bits,m,G", [(3, 0, 4), (3, 128, 4), (4, 0, 1), (2, 0, 8), (2, 64, 2)])
def test_score_on_oracle_codes(tq, bits, m, G):
    B, Hkv, L, d = 2, 2, 1000, 128
    Hq = Hkv * G
    h = tq.Handle(d, bits, 3, qjl_m=m)
    oh = OracleHandle(d, h.bits_mse, 3, m)
    x = _kv((B, Hkv, L, d), 1, 2.0)
    cache, od = oracle_cache(tq, h, oh, x)
    q = torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(5))
    lens = torch.tensor([L, 617], dtype=torch.int32)
    logits = tq.score(h, q.cuda(), cache, lens.cuda())
    got = logits.cpu().numpy()
    qn = q.double().numpy()
    for b in range(B):
        for hq in range(Hq):
            hk = hq // G
            Lb = int(lens[b])
            if m:
                ref = ops.score_prod(qn[b, hq], od["idx"][b, hk, :Lb], od["n"][b, hk, :Lb], od["sigma"][b, hk, :Lb],
                                     od["rnorm"][b, hk, :Lb], oh.Pi, oh.S, oh.c)
            else:
                ref = ops.score_mse(qn[b, hq], od["idx"][b, hk, :Lb], od["n"][b, hk, :Lb], oh.Pi, oh.c)
            tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), od["n"][b, hk, :Lb].astype(np.float64), d)
            assert np.all(np.abs(got[b, hq, :Lb] - ref) <= tol)
            assert np.all(got[b, hq, Lb:] == 0)  # untouched tail


def _attn_case(tq, kb, km, vb, vm, G, lens, L, B=2, Hkv=2, d=128, q_dtype=torch.float32):
    Hq = Hkv * G
    hk = tq.Handle(d, kb, 10, qjl_m=km)
    hv = tq.Handle(d, vb, 11, qjl_m=vm)
    ohk, ohv = OracleHandle(d, hk.bits_mse, 10, km), OracleHandle(d, hv.bits_mse, 11, vm)
    kc, kod = oracle_cache(tq, hk, ohk, _kv((B, Hkv, L, d), 12, 1.5))
    vc, vod = oracle_cache(tq, hv, ohv, _kv((B, Hkv, L, d), 13))
    q = (torch.randn(B, Hq, d, generator=torch.Generator().manual_seed(14)) * 2).to(q_dtype)
    lens_t = torch.tensor(lens, dtype=torch.int32)
    scale = 1.0 / np.sqrt(d)
    o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t.cuda(), scale).cpu().numpy()
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, l) for l in lens], scale)
    for b in range(B):
        for h in range(Hq):
            if lens[b] == 0:
                assert np.all(o[b, h] == 0)
                continue
            err = np.linalg.norm(o[b, h] - ref[b, h])
            assert err <= ATTN_RTOL * np.linalg.norm(ref[b, h]), (b, h, err)
    return o


@pytest.mark.parametrize("kb,km,vb,vm,G", [(3, 128, 3, 128, 4), (4, 0, 4, 0, 4), (3, 0, 2, 0, 1),
                                            (2, 0, 3, 128, 8), (4, 0, 3, 64, 2)])
def test_attention_on_oracle_codes(tq, kb, km, vb, vm, G):
    _attn_case(tq, kb, km, vb, vm, G, lens=[1000, 333], L=1000)


def test_attention_edge_lengths(tq):
    _attn_case(tq, 3, 128, 3, 128, 4, lens=[1, 0], L=300)
    _attn_case(tq, 4, 0, 4, 0, 4, lens=[129, 128], L=129)
    _attn_case(tq, 4, 0, 4, 0, 4, lens=[2000, 1999], L=2000, q_dtype=torch.bfloat16)


def test_attention_end_to_end(tq):
    """GPU encode -> GPU attention (prod 2+1 K and V). The parity gate is the attention over
    the GPU's own codes against the oracle on those codes (1e-3); the end-to-end error against
    the oracle's own encode is reported: the encode may put a coordinate or sign on the other
    side of a boundary where the rotated value lies within 1e-5 of it, and a flipped key index
    moves that key's logit by a whole centroid step."""
    B, Hkv, G, L, d = 1, 2, 4, 3000, 128
    hk, hv = tq.Handle(d, 3, 20, qjl_m=128), tq.Handle(d, 3, 21, qjl_m=128)
    ohk, ohv = OracleHandle(d, 2, 20, 128), OracleHandle(d, 2, 21, 128)
    k = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    v = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    kc.fill(k.cuda())
    vc.fill(v.cuda())
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(3))
    lens = torch.tensor([L], dtype=torch.int32).cuda()
    o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens, 1 / np.sqrt(d)).cpu().numpy()

    def gpu_codes(cache, oh):
        return {"idx": quant.unpack(cache.codes.cpu().numpy().reshape(-1, 32), d, 2).reshape(B, Hkv, L, d),
                "n": to_np64(cache.norms.cpu()), "Pi": oh.Pi, "c": oh.c,
                "sigma": quant.unpack(cache.signs.cpu().numpy().reshape(-1, 16), d, 1).reshape(B, Hkv, L, d),
                "rnorm": to_np64(cache.rnorms.cpu()), "S": oh.S}

    ref_gpu = ops.decode_attention(q.double().numpy(), gpu_codes(kc, ohk), gpu_codes(vc, ohv), [L], 1 / np.sqrt(d))
    _, kod = oracle_cache(tq, hk, ohk, to_np64(k))
    _, vod = oracle_cache(tq, hv, ohv, to_np64(v))
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [L], 1 / np.sqrt(d))
    e2e = []
    for h in range(Hkv * G):
        assert np.linalg.norm(o[0, h] - ref_gpu[0, h]) <= ATTN_RTOL * np.linalg.norm(ref_gpu[0, h])
        e2e.append(np.linalg.norm(o[0, h] - ref[0, h]) / np.linalg.norm(ref[0, h]))
    print(f"end-to-end relative error vs the oracle's own encode: max {max(e2e):.2e}")
    assert max(e2e) < 2e-2


@pytest.mark.parametrize("m", [0, 128])
def test_append_matches_encode_and_capacity(tq, m):
    B, Hkv, L_cap, d = 3, 2, 40, 128
    h = tq.Handle(d, 3, 7, qjl_m=m)
    oh = OracleHandle(d, h.bits_mse, 7, m)
    cache = tq.Cache(h, B, Hkv, L_cap)
    cache.codes.zero_()
    cache.norms.zero_()
    lens = torch.tensor([0, 5, L_cap - 2], dtype=torch.int32).cuda()
    toks = []
    for t in range(3):
        x = torch.randn(B, Hkv, d, generator=torch.Generator().manual_seed(100 + t)).to(torch.bfloat16)
        toks.append(x)
        cache.append(x.cuda(), lens, advance=True)
    st = h.status()
    assert st == tq.TQ_ECAPACITY                # third append overflowed sequence 2
    assert h.status() == tq.TQ_OK               # the error word was cleared
    assert lens.cpu().tolist() == [3, 8, L_cap]
    codes = cache.codes.cpu().numpy()
    norms = cache.norms.cpu().numpy()
    start = [0, 5, L_cap - 2]
    for t in range(3):
        exp = oh.encode(to_np64(toks[t]).reshape(-1, d), "f16" if m else "f32")
        for b in range(B):
            pos = start[b] + t
            if pos >= L_cap:
                continue
            for hh in range(Hkv):
                r = b * Hkv + hh
                sub = {k: (v[r:r + 1] if isinstance(v, np.ndarray) and v.ndim >= 1 and len(v) == B * Hkv else v)
                       for k, v in exp.items()}
                check_codes(codes[b, hh, pos][None], sub, oh)
                check_norms(norms[b, hh, pos:pos + 1], exp["n_stored"][r:r + 1])
    # append with advance = 0 writes the slot but leaves len unchanged
    x = torch.randn(B, Hkv, d).to(torch.bfloat16).cuda()
    cache.append(x, lens, advance=False)
    assert lens.cpu().tolist() == [3, 8, L_cap]


@pytest.mark.parametrize("bits,d,n,k", [(2, 256, 20000, 10), (4, 256, 9000, 10), (3, 128, 5000, 64),
                                        (2, 1536, 3000, 10), (4, 128, 70, 1), (2, 128, 33, 33)])
def test_search_on_oracle_codes(tq, bits, d, n, k):
    h = tq.Handle(d, bits, 8)
    oh = OracleHandle(d, bits, 8)
    db = np.random.default_rng(1).standard_normal((n, d))
    db /= np.linalg.norm(db, axis=1, keepdims=True)
    e = oh.encode(db, "f32")
    codes = torch.from_numpy(quant.pack(e["idx"], bits)).cuda()
    norms = torch.from_numpy(e["n_stored"]).cuda()
    nq = 77
    Q = np.random.default_rng(2).standard_normal((nq, d))
    idx, sc = h.search_topk(torch.from_numpy(Q).float().cuda(), codes, norms, k)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    S = ops.search_scores(Q.astype(np.float32).astype(np.float64), e["idx"], e["n_stored"], oh.Pi, oh.c)
    ri, rs = ops.topk(S, k)
    for i in range(nq):
        tol = score_tolerance(S[i], np.linalg.norm(Q[i]), 1.0, d)
        assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0
        kth = rs[i, -1]
        assert np.all(S[i, idx[i]] >= kth - tol[idx[i]])
        assert np.all(np.abs(sc[i] - S[i, idx[i]]) <= tol[idx[i]])
        assert np.all(np.diff(sc[i]) <= 0)


@pytest.mark.parametrize("B,Hkv,L,lens", [(1, 2, 5000, [4999]), (2, 3, 2048, [2048, 1]), (3, 1, 800, [0, 800, 129])])
def test_attention_tensor_core_path_matches_simt_and_oracle(tq, B, Hkv, L, lens):
    """3-bit prod K/V at d=128, 4 query heads per KV head: the int8 tensor-core kernel, the
    SIMT kernel (TQ_SIMT=1) and the oracle agree (caches hold the oracle's codes)."""
    import os
    G, d = 4, 128
    hk = tq.Handle(d, 3, 30, qjl_m=128)
    hv = tq.Handle(d, 3, 31, qjl_m=128)
    ohk, ohv = OracleHandle(d, 2, 30, 128), OracleHandle(d, 2, 31, 128)
    rs = np.random.default_rng(B * 100 + L)
    std = np.exp(0.5 * rs.standard_normal((1, Hkv, 1, d)))
    kc, kod = oracle_cache(tq, hk, ohk, rs.standard_normal((B, Hkv, L, d)) * std)
    vc, vod = oracle_cache(tq, hv, ohv, rs.standard_normal((B, Hkv, L, d)) * std)
    q = torch.from_numpy(rs.standard_normal((B, Hkv * G, d))).float()
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    scale = 1 / np.sqrt(d)
    o_fast = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    os.environ["TQ_SIMT"] = "1"
    try:
        o_simt = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    finally:
        del os.environ["TQ_SIMT"]
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, x) for x in lens], scale)
    for b in range(B):
        for h in range(Hkv * G):
            if lens[b] == 0:
                assert np.all(o_fast[b, h] == 0) and np.all(o_simt[b, h] == 0)
                continue
            nr = np.linalg.norm(ref[b, h])
            assert np.linalg.norm(o_fast[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
            assert np.linalg.norm(o_simt[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
    assert hk.status() == tq.TQ_OK


@pytest.mark.parametrize("B,Hkv,L,lens", [(3, 2, 8192, [8192, 5003, 1]), (1, 8, 2048, [0])])
def test_score_tensor_core_path_matches_simt_and_oracle(tq, B, Hkv, L, lens):
    """prod 2+1 keys at d=128, 4 query heads per KV head: the int8 tensor-core score kernel
    (many 256-key blocks and chunks per head, ragged lengths, an empty sequence), the SIMT
    kernel (TQ_SIMT=1) and the oracle agree."""
    import os
    G, d = 4, 128
    h = tq.Handle(d, 3, 21, qjl_m=128)
    oh = OracleHandle(d, 2, 21, 128)
    rs = np.random.default_rng(L + B)
    std = np.exp(0.5 * rs.standard_normal((1, Hkv, 1, d)))
    cache, od = oracle_cache(tq, h, oh, rs.standard_normal((B, Hkv, L, d)) * std)
    q = torch.from_numpy(rs.standard_normal((B, Hkv * G, d))).float()
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    fast = tq.score(h, q.cuda(), cache, lens_t).cpu().numpy()
    os.environ["TQ_SIMT"] = "1"
    try:
        simt = tq.score(h, q.cuda(), cache, lens_t).cpu().numpy()
    finally:
        del os.environ["TQ_SIMT"]
    qn = q.double().numpy()
    for b in range(B):
        Lb = lens[b]
        for hq in range(Hkv * G):
            hk = hq // G
            assert np.all(fast[b, hq, Lb:] == 0)
            if Lb == 0:
                continue
            ref = ops.score_prod(qn[b, hq], od["idx"][b, hk, :Lb], od["n"][b, hk, :Lb], od["sigma"][b, hk, :Lb],
                                 od["rnorm"][b, hk, :Lb], oh.Pi, oh.S, oh.c)
            tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), od["n"][b, hk, :Lb].astype(np.float64), d)
            assert np.all(np.abs(fast[b, hq, :Lb] - ref) <= tol), (b, hq)
            assert np.all(np.abs(simt[b, hq, :Lb] - ref) <= tol), (b, hq)
    assert h.status() == tq.TQ_OK


@pytest.mark.parametrize("B,Hkv,L,lens", [(2, 2, 5000, [5000, 2001]), (2, 1, 600, [1, 0])])
def test_attention_mse4_tensor_core_path_matches_simt_and_oracle(tq, B, Hkv, L, lens):
    """4-bit MSE K/V with fp16 norms at d=128, 4 query heads per KV head: the int8 tensor-core
    kernel (codebook in Walsh-plane form), the SIMT kernel (TQ_SIMT=1) and the oracle agree."""
    import os
    G, d = 4, 128
    hk = tq.Handle(d, 4, 40, norm_dtype=tq.TQ_F16)
    hv = tq.Handle(d, 4, 41, norm_dtype=tq.TQ_F16)
    ohk, ohv = OracleHandle(d, 4, 40, 0), OracleHandle(d, 4, 41, 0)
    rs = np.random.default_rng(L + 7 * B)
    scl = rs.uniform(0.5, 2.0, size=(B, Hkv, 1, 1))
    kc, kod = oracle_cache(tq, hk, ohk, rs.standard_normal((B, Hkv, L, d)) * scl)
    vc, vod = oracle_cache(tq, hv, ohv, rs.standard_normal((B, Hkv, L, d)) * scl[:, ::-1])
    q = torch.from_numpy(rs.standard_normal((B, Hkv * G, d)) * 2).float()
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    scale = 1 / np.sqrt(d)
    o_fast = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    os.environ["TQ_SIMT"] = "1"
    try:
        o_simt = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    finally:
        del os.environ["TQ_SIMT"]
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, x) for x in lens], scale)
    for b in range(B):
        for h in range(Hkv * G):
            if lens[b] == 0:
                assert np.all(o_fast[b, h] == 0) and np.all(o_simt[b, h] == 0)
                continue
            nr = np.linalg.norm(ref[b, h])
            assert np.linalg.norm(o_fast[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
            assert np.linalg.norm(o_simt[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
    assert hk.status() == tq.TQ_OK


@pytest.mark.parametrize("d,n,nq,k", [(512, 50000, 40, 32), (1536, 9000, 17, 1), (128, 700, 3, 10),
                                     (640, 3000, 16, 10), (1024, 300, 64, 5), (256, 100, 5, 7)])
def test_search_tensor_core_path_matches_simt_and_oracle(tq, d, n, nq, k):
    """2-bit codes: the tcgen05 search (several 256-vector tiles and chunks, one to twelve
    K-chunks of 128 coordinates, a database shorter than one tile, partial query tiles, k = 1
    and 32) and the SIMT kernel (TQ_SIMT=1) against the oracle.
    Exact duplicate database rows score identically on either path, so the lower index
    must be returned first."""
    import os
    h = tq.Handle(d, 2, 9)
    oh = OracleHandle(d, 2, 9)
    rs = np.random.default_rng(d + n)
    db = rs.standard_normal((n, d))
    db /= np.linalg.norm(db, axis=1, keepdims=True)
    Q = rs.standard_normal((nq, d))
    # plant exact duplicates of the best vector of query 0 at higher indices
    best = int(np.argmax(db @ Q[0]))
    for j in (n - 1, n // 2 + 3):
        if j != best:
            db[j] = db[best]
    e = oh.encode(db, "f32")
    codes = torch.from_numpy(quant.pack(e["idx"], 2)).cuda()
    norms = torch.from_numpy(e["n_stored"]).cuda()
    qg = torch.from_numpy(Q).float().cuda()
    fast = [x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k)]
    os.environ["TQ_SIMT"] = "1"
    try:
        simt = [x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k)]
    finally:
        del os.environ["TQ_SIMT"]
    S = ops.search_scores(Q.astype(np.float32).astype(np.float64), e["idx"], e["n_stored"], oh.Pi, oh.c)
    ri, rsc = ops.topk(S, k)
    for idx, sc in (fast, simt):
        for i in range(nq):
            tol = score_tolerance(S[i], np.linalg.norm(Q[i]), 1.0, d)
            assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0
            assert np.all(S[i, idx[i]] >= rsc[i, -1] - tol[idx[i]])
            assert np.all(np.abs(sc[i] - S[i, idx[i]]) <= tol[idx[i]])
            assert np.all(np.diff(sc[i]) <= 0)
            for a in range(k - 1):   # equal scores: lower index first
                if sc[i, a] == sc[i, a + 1]:
                    assert idx[i, a] < idx[i, a + 1]
    assert h.status() == tq.TQ_OK


@pytest.mark.parametrize("d,n,nq,k", [(1536, 6000, 9, 10), (320, 3000, 13, 32), (128, 200, 4, 1), (512, 20000, 70, 10)])
def test_search_4bit_tensor_core_path_matches_simt_and_oracle(tq, d, n, nq, k):
    """4-bit codes: the tcgen05 search (one to twelve K-chunks, a half last K-chunk at d = 320,
    a database shorter than one 256-vector tile, partial query tiles, k = 1 and 32) and the
    SIMT kernel (TQ_SIMT=1) against the oracle; planted duplicates of a best vector must come
    back lower index first."""
    import os
    h = tq.Handle(d, 4, 11)
    oh = OracleHandle(d, 4, 11)
    rs = np.random.default_rng(d * 7 + n)
    db = rs.standard_normal((n, d))
    db /= np.linalg.norm(db, axis=1, keepdims=True)
    Q = rs.standard_normal((nq, d))
    best = int(np.argmax(db @ Q[0]))
    for j in (n - 1, n // 3 + 1):
        if j != best:
            db[j] = db[best]
    e = oh.encode(db, "f32")
    codes = torch.from_numpy(quant.pack(e["idx"], 4)).cuda()
    norms = torch.from_numpy(e["n_stored"]).cuda()
    qg = torch.from_numpy(Q).float().cuda()
    fast = [x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k)]
    os.environ["TQ_SIMT"] = "1"
    try:
        simt = [x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k)]
    finally:
        del os.environ["TQ_SIMT"]
    S = ops.search_scores(Q.astype(np.float32).astype(np.float64), e["idx"], e["n_stored"], oh.Pi, oh.c)
    ri, rsc = ops.topk(S, k)
    for idx, sc in (fast, simt):
        for i in range(nq):
            tol = score_tolerance(S[i], np.linalg.norm(Q[i]), 1.0, d)
            assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0
            assert np.all(S[i, idx[i]] >= rsc[i, -1] - tol[idx[i]])
            assert np.all(np.abs(sc[i] - S[i, idx[i]]) <= tol[idx[i]])
            assert np.all(np.diff(sc[i]) <= 0)
            for a in range(k - 1):   # equal scores: lower index first
                if sc[i, a] == sc[i, a + 1]:
                    assert idx[i, a] < idx[i, a + 1]
    assert h.status() == tq.TQ_OK
