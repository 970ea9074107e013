"""Oracle parity at the full sizes of the bench's workloads, on sampled outputs.

The caches and databases here are full size (the 4-bit decode workload: 4 sequences x 8
KV heads x 131072 tokens; the 3-bit big-cache decode workload: 64 x 8 x 16640; the streaming score workload: 64 x 8 heads at 16385 keys in
16640 slots; the search workload: 1,000,000 vectors at d = 1536, 1024 queries), so the
kernels run in exactly the launch configuration the bench times. An fp64 encode of that
many vectors would take minutes, so the packed rows are uniformly random bytes (every bit
pattern is a valid row) with norms of Gaussian vectors; the oracle then computes a sample
of the outputs one by one from the same rows. ("TurboQuant / PolarQuant / QJL technical
deep dive", "Scaled dot-product attention"; "Google TurboQuant: 6x KV-cache compression",
"Stage 2"; "TurboQuant: redefining AI efficiency", "Impact on high-dimensional vector
search".)
"""

import numpy as np
import pytest
import torch

import workloads
from gpu_util import ATTN_RTOL, OracleHandle, max_rel_score_error, score_tolerance, unpack_fast
from oracle import ops

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


def test_attn_mse4_full_size_sampled(tq):
    """4-bit MSE K and V (fp16 norms), 4 x 8 KV heads x 131072 tokens, 32 query heads: the
    attention of every query head of three sampled (sequence, KV head) units and two ragged
    lengths against the oracle."""
    B, Hkv, G, L, d = 4, 8, 4, 131072, 128
    lens = [L, L - 1, 100003, L]
    hk = tq.Handle(d, 4, 0, norm_dtype=tq.TQ_F16)
    hv = tq.Handle(d, 4, 1, norm_dtype=tq.TQ_F16)
    ohk, ohv = OracleHandle(d, 4, 0), OracleHandle(d, 4, 1)
    scl = np.random.default_rng(5).uniform(0.5, 2.0, size=(B, Hkv, 1))
    rows, norms = {}, {}
    for name, seed in (("k", 50), ("v", 51)):
        rows[name] = workloads.random_rows((B, Hkv, L), 64, seed)
        norms[name] = workloads.random_norms((B, Hkv, L), d, seed + 100, scale=scl)
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    for c, name in ((kc, "k"), (vc, "v")):
        c.codes.copy_(torch.from_numpy(rows[name]))
        c.norms.copy_(torch.from_numpy(norms[name]))
    q = workloads.queries((B, Hkv * G, d), 7)
    o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, torch.tensor(lens, dtype=torch.int32).cuda(),
                       1.0 / np.sqrt(d)).cpu().numpy()
    assert hk.status() == tq.TQ_OK
    del kc, vc
    worst = 0.0
    for b, h in ((0, 0), (1, 5), (2, 2), (3, 7)):
        Lb = lens[b]
        kod = {"idx": unpack_fast(rows["k"][b, h, :Lb], d, 4)[None, None], "n": norms["k"][b, h, :Lb][None, None],
               "Pi": ohk.Pi, "c": ohk.c}
        vod = {"idx": unpack_fast(rows["v"][b, h, :Lb], d, 4)[None, None], "n": norms["v"][b, h, :Lb][None, None],
               "Pi": ohv.Pi, "c": ohv.c}
        qq = q[b:b + 1, h * G:(h + 1) * G].double().numpy()
        ref = ops.decode_attention(qq, kod, vod, [Lb], 1.0 / np.sqrt(d))
        for g in range(G):
            nr = np.linalg.norm(ref[0, g])
            err = np.linalg.norm(o[b, h * G + g] - ref[0, g])
            worst = max(worst, err / nr)
            assert err <= ATTN_RTOL * nr, (b, h, g, err / nr)
    print(f"4-bit attention, full size: max relative error over the sampled heads {worst:.2e}")


def test_score_prod2_full_size_sampled(tq):
    """prod 2+1 keys (m = 128, fp16 norms), 64 sequences x 8 KV heads in 16640 slots, 32
    query heads, lengths around 16385 (one append into the 16384-token prefill): sampled
    query heads against the oracle, and the untouched tail."""
    B, Hkv, G, Lcap, d = 64, 8, 4, 16640, 128
    lens = [16385 - (b % 5) * 997 for b in range(B)]
    h = tq.Handle(d, 3, 0, qjl_m=128)
    oh = OracleHandle(d, 2, 0, 128)
    codes = workloads.random_rows((B, Hkv, Lcap), 32, 60)
    signs = workloads.random_rows((B, Hkv, Lcap), 16, 61)
    n = workloads.random_norms((B, Hkv, Lcap), d, 62)
    rn = (n.astype(np.float64) * np.random.default_rng(63).uniform(0.2, 0.5, size=(B, Hkv, Lcap))).astype(np.float16)
    cache = tq.Cache(h, B, Hkv, Lcap)
    cache.codes.copy_(torch.from_numpy(codes))
    cache.signs.copy_(torch.from_numpy(signs))
    cache.norms.copy_(torch.from_numpy(n))
    cache.rnorms.copy_(torch.from_numpy(rn))
    q = workloads.queries((B, Hkv * G, d), 64)
    got = tq.score(h, q.cuda(), cache, torch.tensor(lens, dtype=torch.int32).cuda()).cpu().numpy()
    assert h.status() == tq.TQ_OK
    del cache
    qn = q.double().numpy()
    worst = 0.0
    for b, hq in ((0, 0), (1, 13), (17, 31), (42, 6), (63, 20)):
        hk, Lb = hq // G, lens[b]
        idx = unpack_fast(codes[b, hk, :Lb], d, 2)
        sig = unpack_fast(signs[b, hk, :Lb], 128, 1)
        ref = ops.score_prod(qn[b, hq], idx, n[b, hk, :Lb], sig, rn[b, hk, :Lb], oh.Pi, oh.S, oh.c)
        nn = n[b, hk, :Lb].astype(np.float64)
        tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), nn, d)
        assert np.all(np.abs(got[b, hq, :Lb] - ref) <= tol), (b, hq)
        assert np.all(got[b, hq, Lb:] == 0)
        worst = max(worst, max_rel_score_error(got[b, hq, :Lb], ref, np.linalg.norm(qn[b, hq]), nn, d))
    print(f"score, full size: max relative score error above the floor {worst:.2e}")


def test_attn_prod3_big_cache_full_size_sampled(tq):
    """3-bit prod K and V (m = 128, fp16 norms), 64 sequences x 8 KV heads in 16640 slots (the
    872 MB cache of the big-cache decode row, which takes the two-kernel path: scores, then
    values), ragged lengths: every query head of five sampled (sequence, KV head) units against
    the oracle's attention over the same rows."""
    B, Hkv, G, Lcap, d = 64, 8, 4, 16640, 128
    lens = [16385 - (b % 7) * 1501 for b in range(B)]
    hk, hv = tq.Handle(d, 3, 0, qjl_m=128), tq.Handle(d, 3, 1, qjl_m=128)
    ohk, ohv = OracleHandle(d, 2, 0, 128), OracleHandle(d, 2, 1, 128)
    rows = {}
    caches = []
    for name, h, seed in (("k", hk, 80), ("v", hv, 90)):
        codes = workloads.random_rows((B, Hkv, Lcap), 32, seed)
        signs = workloads.random_rows((B, Hkv, Lcap), 16, seed + 1)
        n = workloads.random_norms((B, Hkv, Lcap), d, seed + 2)
        rn = (n.astype(np.float64) * np.random.default_rng(seed + 3).uniform(0.2, 0.5, size=(B, Hkv, Lcap))).astype(
            np.float16)
        c = tq.Cache(h, B, Hkv, Lcap)
        c.codes.copy_(torch.from_numpy(codes))
        c.signs.copy_(torch.from_numpy(signs))
        c.norms.copy_(torch.from_numpy(n))
        c.rnorms.copy_(torch.from_numpy(rn))
        rows[name] = (codes, signs, n, rn)
        caches.append(c)
    q = workloads.queries((B, Hkv * G, d), 85)
    o = tq.attn_decode(hk, hv, q.cuda(), caches[0], caches[1], torch.tensor(lens, dtype=torch.int32).cuda(),
                       1.0 / np.sqrt(d)).cpu().numpy()
    assert hk.status() == tq.TQ_OK
    del caches
    worst = 0.0
    for b, h in ((0, 0), (1, 5), (20, 3), (41, 7), (63, 2)):
        Lb = lens[b]
        od = []
        for name, oh in (("k", ohk), ("v", ohv)):
            codes, signs, n, rn = rows[name]
            od.append({"idx": unpack_fast(codes[b, h, :Lb], d, 2)[None, None], "n": n[b, h, :Lb][None, None],
                       "sigma": unpack_fast(signs[b, h, :Lb], 128, 1)[None, None],
                       "rnorm": rn[b, h, :Lb][None, None], "Pi": oh.Pi, "S": oh.S, "c": oh.c})
        qq = q[b:b + 1, h * G:(h + 1) * G].double().numpy()
        ref = ops.decode_attention(qq, od[0], od[1], [Lb], 1.0 / np.sqrt(d))
        for g in range(G):
            nr = np.linalg.norm(ref[0, g])
            err = np.linalg.norm(o[b, h * G + g] - ref[0, g])
            worst = max(worst, err / nr)
            assert err <= ATTN_RTOL * nr, (b, h, g, err / nr)
    print(f"3-bit attention over the 872 MB cache, full size: max relative error over the sampled heads {worst:.2e}")


@pytest.mark.parametrize("bits", [2, 4])
def test_search_full_size_sampled(tq, bits):
    """1,000,000 packed vectors at d = 1536 with unit norms, 1024 queries, top-10: the top-k
    lists of 6 sampled queries against the oracle's scores of the whole database."""
    n, d, nq, k = 1_000_000, 1536, 1024, 10
    h = tq.Handle(d, bits, 0)
    oh = OracleHandle(d, bits, 0)
    codes = workloads.random_rows((n,), d * bits // 8, 80 + bits)
    norms = np.ones(n, dtype=np.float32)
    Q = workloads.queries((nq, d), 9).numpy()
    Q /= np.linalg.norm(Q, axis=1, keepdims=True)
    idx, sc = (x.cpu().numpy() for x in h.search_topk(torch.from_numpy(Q).cuda(), torch.from_numpy(codes).cuda(),
                                                       torch.from_numpy(norms).cuda(), k))
    assert h.status() == tq.TQ_OK
    sample = [0, 1, 333, 512, 1000, 1023]
    Qs = Q[sample].astype(np.float64)
    S = np.empty((len(sample), n))
    blk = 1 << 14
    for i in range(0, n, blk):
        j = min(n, i + blk)
        S[:, i:j] = ops.search_scores(Qs, unpack_fast(codes[i:j], d, bits), norms[i:j], oh.Pi, oh.c)
    _, rsc = ops.topk(S, k)
    for r, i in enumerate(sample):
        tol = score_tolerance(S[r], np.linalg.norm(Qs[r]), 1.0, d)
        assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0 and idx[i].max() < n
        assert np.all(S[r, idx[i]] >= rsc[r, -1] - tol[idx[i]]), i
        assert np.all(np.abs(sc[i] - S[r, idx[i]]) <= tol[idx[i]]), i
        assert np.all(np.diff(sc[i]) <= 0)
