"""Oracle parity at the split shapes the full-size workloads run.

The int8 tensor-core kernels stream each context chunk (or database chunk) through a
ring of TMA stages. At the small shapes of the other parity tests a chunk holds one or
two blocks, so the ring never wraps. Here every kernel runs chunks of several blocks:

* attn_prod2_kernel at the exact decode-step workload (1 sequence, 8 KV / 32 query
  heads, context 32768: 37 chunks of 896 tokens, each staged whole as 4 key and 4 value
  blocks with one barrier each), plus a ragged length and forced 512-token chunks;
* attn_mse4_kernel with 896-token chunks (4 + 4 blocks on its 4-stage ring);
* score_prod2_kernel with 4-, 5- and 10-block chunks on its 5-stage ring (TQ_SPLITK);
* search_tc_kernel with 3 to 12 tiles of 256 vectors per chunk.

Caches hold the oracle's codes ("Google TurboQuant: 6x KV-cache compression", "Stage 1"
and "Stage 2"; "TurboQuant / PolarQuant / QJL technical deep dive", "Scaled dot-product
attention"; "TurboQuant: redefining AI efficiency", "Impact on high-dimensional vector
search"). Tolerances as in the other parity tests.
"""

import contextlib
import os

import numpy as np
import pytest
import torch

import workloads
from gpu_util import (ATTN_RTOL, OracleHandle, check_codes, check_norms, check_signs, max_rel_score_error,
                      score_tolerance, to_np64)
from oracle import ops, quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


@contextlib.contextmanager
def splitk(n):
    """Forces the kernels' chunk length (tokens or vectors) through TQ_SPLITK."""
    old = os.environ.get("TQ_SPLITK")
    os.environ["TQ_SPLITK"] = str(n)
    try:
        yield
    finally:
        if old is None:
            del os.environ["TQ_SPLITK"]
        else:
            os.environ["TQ_SPLITK"] = old


NORM_NP = {0: "f32", 1: "f16"}


def oracle_cache(tq, h, oh, x):
    """Cache of handle h filled with the oracle's codes of x [B, Hkv, L, d]; returns (cache, dict, encode)."""
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
    return cache, od, e


def _check_attention(o, ref, lens):
    worst = 0.0
    for b in range(o.shape[0]):
        for h in range(o.shape[1]):
            if lens[b] == 0:
                assert np.all(o[b, h] == 0)
                continue
            nr = np.linalg.norm(ref[b, h])
            err = np.linalg.norm(o[b, h] - ref[b, h])
            worst = max(worst, err / nr)
            assert err <= ATTN_RTOL * nr, (b, h, err / nr)
    return worst


@pytest.fixture(scope="module")
def decode_workload(tq):
    """The decode-step workload (prod 2+1 bits, m = 128, fp16 norms; bf16 K/V with lognormal
    channel scales and 2 outlier channels per head; seeds 2, 3 for K, V and 4 for the
    queries; handle seeds 0 and 1), as oracle codes in GPU caches."""
    B, Hkv, Hq, L, d = 1, 8, 32, 32768, 128
    hk, hv = tq.Handle(d, 3, 0, qjl_m=128), tq.Handle(d, 3, 1, qjl_m=128)
    ohk, ohv = OracleHandle(d, 2, 0, 128), OracleHandle(d, 2, 1, 128)
    K = workloads.outlier_kv(B, Hkv, L, d, seed=2)
    V = workloads.outlier_kv(B, Hkv, L, d, seed=3)
    kc, kod, _ = oracle_cache(tq, hk, ohk, to_np64(K))
    vc, vod, _ = oracle_cache(tq, hv, ohv, to_np64(V))
    q = workloads.queries((B, Hq, d), 4)
    return dict(hk=hk, hv=hv, ohk=ohk, ohv=ohv, K=K, V=V, kc=kc, vc=vc, kod=kod, vod=vod, q=q, L=L)


@pytest.mark.parametrize("length,force", [(32768, None), (30001, None), (32768, 512)])
def test_attn_prod2_decode_workload_matches_oracle(tq, decode_workload, length, force):
    """attn_prod2_kernel at the decode-step workload's own split (896-token chunks of 3.5
    blocks: 4 key and 4 value blocks per chunk, a partial last block), at a ragged length
    and with forced 512-token chunks."""
    w = decode_workload
    lens = torch.tensor([length], dtype=torch.int32).cuda()
    scale = 1.0 / np.sqrt(128)
    ctx = splitk(force) if force else contextlib.nullcontext()
    with ctx:
        o = tq.attn_decode(w["hk"], w["hv"], w["q"].cuda(), w["kc"], w["vc"], lens, scale).cpu().numpy()
    assert w["hk"].status() == tq.TQ_OK
    ref = ops.decode_attention(w["q"].double().numpy(), w["kod"], w["vod"], [length], scale)
    worst = _check_attention(o, ref, [length])
    print(f"decode workload, len {length}, chunk {force or 896}: max relative attention error {worst:.2e}")


def test_decode_step_decode_workload_matches_oracle(tq, decode_workload):
    """tq_decode_step at the decode-step workload: the appended token (slot 32767) against the
    oracle's encode of the workload's token, and the output against the oracle's attention over
    the oracle's codes of all 32768 tokens (the new token included)."""
    w = decode_workload
    B, Hkv, Hq, L, d = 1, 8, 32, w["L"], 128
    hk, hv, kc, vc = w["hk"], w["hv"], w["kc"], w["vc"]
    k_new = w["K"][:, :, L - 1].contiguous().cuda()
    v_new = w["V"][:, :, L - 1].contiguous().cuda()
    lens = torch.tensor([L - 1], dtype=torch.int32).cuda()
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    # the caches already hold the oracle's codes of token L - 1: overwrite that slot with garbage first
    for c in (kc, vc):
        c.codes[:, :, L - 1].fill_(0xA5)
        c.signs[:, :, L - 1].fill_(0x5A)
    tq.tq_decode_step(hk.ptr, hv.ptr, w["q"].cuda(), k_new, v_new, B, Hq, Hkv, kc.struct, vc.struct, lens, scale,
                      out, ws)
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    assert lens.cpu().tolist() == [L]
    for c, oh, X in ((kc, w["ohk"], w["K"]), (vc, w["ohv"], w["V"])):
        exp = oh.encode(to_np64(X[:, :, L - 1]).reshape(-1, d), "f16")
        _, bad, frac = check_codes(c.codes[:, :, L - 1].cpu().numpy().reshape(Hkv, -1), exp, oh)
        check_norms(c.norms[:, :, L - 1].cpu().numpy(), exp["n_stored"])
        sfrac = check_signs(c.signs[:, :, L - 1].cpu().numpy().reshape(Hkv, -1), exp, bad)
        print(f"appended token: index mismatch fraction {frac:.2e}, sign mismatch fraction {sfrac:.2e}")
        assert frac == 0.0, "an index of the appended token fell inside the boundary band"
    ref = ops.decode_attention(w["q"].double().numpy(), w["kod"], w["vod"], [L], scale)
    worst = _check_attention(out.cpu().numpy(), ref, [L])
    print(f"decode step at the decode workload: max relative attention error {worst:.2e}")


@pytest.mark.parametrize("lens,force", [([10240, 10239, 9000, 5121], None), ([2048, 1, 0, 1500], 640)])
def test_attn_mse4_multiblock_chunks_match_oracle(tq, lens, force):
    """attn_mse4_kernel with 896-token chunks (4 key + 4 value jobs through its 4-stage ring):
    4 sequences x 8 KV heads x 10240 tokens (the split policy gives 12 chunks of 896, the last
    one partial), ragged and empty lengths; and forced 640-token chunks."""
    B, Hkv, G, d = 4, 8, 4, 128
    L = max(max(lens), 128)
    L = (L + 7) // 8 * 8
    hk = tq.Handle(d, 4, 40, norm_dtype=tq.TQ_F16)
    hv = tq.Handle(d, 4, 41, norm_dtype=tq.TQ_F16)
    ohk, ohv = OracleHandle(d, 4, 40, 0), OracleHandle(d, 4, 41, 0)
    K = workloads.scaled_kv(B, Hkv, L, d, seed=5)
    V = workloads.scaled_kv(B, Hkv, L, d, seed=6)
    kc, kod, _ = oracle_cache(tq, hk, ohk, to_np64(K))
    vc, vod, _ = oracle_cache(tq, hv, ohv, to_np64(V))
    q = workloads.queries((B, Hkv * G, d), 7)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    scale = 1.0 / np.sqrt(d)
    ctx = splitk(force) if force else contextlib.nullcontext()
    with ctx:
        o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    assert hk.status() == tq.TQ_OK
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, x) for x in lens], scale)
    worst = _check_attention(o, ref, lens)
    print(f"4-bit attention, chunk {force or 896}: max relative attention error {worst:.2e}")


@pytest.mark.parametrize("force,lens", [(2560, [8192, 6001]), (1280, [8192, 2561]), (1024, [8192, 7937])])
def test_score_prod2_ring_wraps(tq, force, lens):
    """score_prod2_kernel with chunks of 10, 5 and 4 blocks of 256 keys (its TMA ring has 5
    stages, 3 blocks in flight), ragged lengths; the untouched tail stays zero."""
    B, Hkv, G, L, d = 2, 8, 4, 8192, 128
    h = tq.Handle(d, 3, 21, qjl_m=128)
    oh = OracleHandle(d, 2, 21, 128)
    X = workloads.outlier_kv(B, Hkv, L, d, seed=31)
    cache, od, _ = oracle_cache(tq, h, oh, to_np64(X))
    q = workloads.queries((B, Hkv * G, d), 32)
    with splitk(force):
        got = tq.score(h, q.cuda(), cache, torch.tensor(lens, dtype=torch.int32).cuda()).cpu().numpy()
    assert h.status() == tq.TQ_OK
    qn = q.double().numpy()
    worst = 0.0
    for b in range(B):
        Lb = lens[b]
        for hq in range(Hkv * G):
            hk = hq // G
            ref = ops.score_prod(qn[b, hq], od["idx"][b, hk, :Lb], od["n"][b, hk, :Lb], od["sigma"][b, hk, :Lb],
                                 od["rnorm"][b, hk, :Lb], oh.Pi, oh.S, oh.c)
            n = od["n"][b, hk, :Lb].astype(np.float64)
            tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), n, d)
            assert np.all(np.abs(got[b, hq, :Lb] - ref) <= tol), (b, hq)
            assert np.all(got[b, hq, Lb:] == 0)
            worst = max(worst, max_rel_score_error(got[b, hq, :Lb], ref, np.linalg.norm(qn[b, hq]), n, d))
    print(f"score chunk {force}: max relative score error above the floor {worst:.2e}")


def _search_case(tq, bits, d, n, nq, k, seed, sample=None):
    h = tq.Handle(d, bits, seed)
    oh = OracleHandle(d, bits, seed)
    rs = np.random.default_rng(seed)
    db = rs.standard_normal((n, d))
    db /= np.linalg.norm(db, axis=1, keepdims=True)
    Q = rs.standard_normal((nq, d))
    e = oh.encode(db, "f32")
    codes = torch.from_numpy(quant.pack(e["idx"], bits)).cuda()
    norms = torch.from_numpy(e["n_stored"]).cuda()
    idx, sc = (x.cpu().numpy() for x in h.search_topk(torch.from_numpy(Q).float().cuda(), codes, norms, k))
    assert h.status() == tq.TQ_OK
    rows = np.arange(nq) if sample is None else np.asarray(sample)
    S = ops.search_scores(Q[rows].astype(np.float32).astype(np.float64), e["idx"], e["n_stored"], oh.Pi, oh.c)
    _, rsc = ops.topk(S, k)
    for r, i in enumerate(rows):
        tol = score_tolerance(S[r], np.linalg.norm(Q[i]), 1.0, d)
        assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0 and idx[i].max() < n
        assert np.all(S[r, idx[i]] >= rsc[r, -1] - tol[idx[i]]), i
        assert np.all(np.abs(sc[i] - S[r, idx[i]]) <= tol[idx[i]]), i
        assert np.all(np.diff(sc[i]) <= 0)


@pytest.mark.parametrize("bits", [2, 4])
def test_search_multiblock_chunks_natural_split(tq, bits):
    """1024 queries over 50,000 vectors at d = 256: the search's own split gives 8 query tiles
    x 33 chunks of 1536 vectors (6 tiles of 256) and a shorter last chunk; 64 sampled queries
    are checked against the oracle."""
    _search_case(tq, bits, 256, 50000, 1024, 10, seed=60 + bits, sample=np.arange(0, 1024, 16))


@pytest.mark.parametrize("bits,force", [(2, 1152), (4, 768), (2, 3000)])
def test_search_multiblock_chunks_forced(tq, bits, force):
    """A partial query tile (19 queries) with forced chunks of 3 to 12 tiles (TQ_SPLITK), a
    ragged last chunk, k = 32."""
    with splitk(force):
        _search_case(tq, bits, 512, 7001, 19, 32, seed=70 + bits)
