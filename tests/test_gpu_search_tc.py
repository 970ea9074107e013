"""GPU parity of the tcgen05 search (search_tc_kernel: int8 MMAs into tensor memory, 128
queries x 256 vectors per tile, any 1- to 4-bit codebook through byte-permute tables)
against the oracle ("TurboQuant: redefining AI efficiency", "Impact on high-dimensional
vector search": s = ||x|| <Pi q, c[idx]>, ranked by score, equal scores lower index first).

Shapes cover every code width, several K-chunks per tile (d = 128 .. 1536), a last K-chunk of
64 coordinates (d = 192, 320, 704: code rows only 8-byte aligned), ragged database tiles and
chunks, a ragged second query tile (nq = 130 and 300), forced chunk lengths (TQ_SPLITK), k = 1
and 32, fp16 norms and planted exact duplicates. The SIMT kernel (TQ_SIMT=1) is checked on the
same data. Rule: every returned index scores (oracle) within the tolerance of the k-th best, the
returned scores match the oracle's within the score tolerance, scores are non-increasing and
equal scores come lower index first."""

import contextlib
import os

import numpy as np
import pytest
import torch

from gpu_util import OracleHandle, max_rel_score_error, score_tolerance
from oracle import ops, quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


@contextlib.contextmanager
def env(**kv):
    old = {k: os.environ.get(k) for k in kv}
    os.environ.update({k: str(v) for k, v in kv.items()})
    try:
        yield
    finally:
        for k, v in old.items():
            if v is None:
                del os.environ[k]
            else:
                os.environ[k] = v


def _data(bits, d, n, nq, seed, norm_dtype):
    oh = OracleHandle(d, bits, seed)
    rs = np.random.default_rng(seed)
    db = rs.standard_normal((n, d)) * np.exp(0.3 * rs.standard_normal((n, 1)))
    Q = rs.standard_normal((nq, d))
    best = int(np.argmax(db @ Q[0]))
    for j in (n - 1, n // 2 + 3):   # exact duplicates of query 0's best vector at higher indices
        if j != best:
            db[j] = db[best]
    e = oh.encode(db, norm_dtype)
    return oh, Q, e


def _check(idx, sc, S, Q, e, k, d, n, rows):
    worst = 0.0
    _, rsc = ops.topk(S, k)
    nn = e["n_stored"].astype(np.float64)
    for r, i in enumerate(rows):
        tol = score_tolerance(S[r], np.linalg.norm(Q[i]), nn, d)
        assert len(set(idx[i].tolist())) == k and idx[i].min() >= 0 and idx[i].max() < n, i
        assert np.all(S[r, idx[i]] >= rsc[r, -1] - tol[idx[i]]), i
        assert np.all(np.abs(sc[i] - S[r, idx[i]]) <= tol[idx[i]]), i
        assert np.all(np.diff(sc[i]) <= 0), i
        for a in range(k - 1):
            if sc[i, a] == sc[i, a + 1]:
                assert idx[i, a] < idx[i, a + 1], i
        worst = max(worst, max_rel_score_error(sc[i], S[r, idx[i]], np.linalg.norm(Q[i]), nn[idx[i]], d))
    return worst


def _run(tq, bits, d, n, nq, k, seed, norm_dtype="f32", sample=None, force=None):
    nd = {"f32": tq.TQ_F32, "f16": tq.TQ_F16}[norm_dtype]
    h = tq.Handle(d, bits, seed, norm_dtype=nd)
    oh, Q, e = _data(bits, d, n, nq, seed, norm_dtype)
    codes = torch.from_numpy(quant.pack(e["idx"], bits)).cuda()
    norms = torch.from_numpy(e["n_stored"]).cuda()
    qg = torch.from_numpy(Q).float().cuda()
    if force:
        with env(TQ_SPLITK=force):
            idx, sc = (x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k))
    else:
        idx, sc = (x.cpu().numpy() for x in h.search_topk(qg, codes, norms, k))
    assert h.status() == tq.TQ_OK
    rows = np.arange(nq) if sample is None else np.asarray(sample)
    S = ops.search_scores(Q[rows].astype(np.float32).astype(np.float64), e["idx"], e["n_stored"], oh.Pi, oh.c)
    worst = _check(idx, sc, S, Q, e, k, d, n, rows)
    print(f"search_tc bits={bits} d={d} n={n} nq={nq} k={k}: max relative score error above the floor {worst:.2e}")
    return h, codes, norms, qg, (idx, sc), (S, Q, e, rows)


@pytest.mark.parametrize("bits,d,n,nq,k", [
    (2, 1536, 5000, 130, 10),    # 12 K-chunks, ragged last tile, a ragged second query tile
    (4, 1536, 3001, 9, 32),      # k = 32, one partial query tile
    (3, 384, 4099, 300, 10),     # 3-bit (fields straddle bytes), three query tiles
    (1, 256, 2000, 40, 1),       # 1-bit, k = 1
    (4, 128, 100, 5, 7),         # one K-chunk, a database shorter than one tile
    (2, 512, 20000, 257, 16),    # many tiles per chunk, 257 queries
    (1, 192, 3000, 33, 10),      # d % 128 = 64: a half last K-chunk, 24-byte rows
    (3, 320, 2500, 70, 10),      # 120-byte rows
    (4, 704, 1000, 129, 32),     # 352-byte rows, 129 queries
])
def test_search_tc_matches_oracle(tq, bits, d, n, nq, k):
    _run(tq, bits, d, n, nq, k, seed=bits * 100 + d + nq)


@pytest.mark.parametrize("bits,force", [(2, 256), (4, 768), (3, 1280)])
def test_search_tc_forced_chunks_and_f16_norms(tq, bits, force):
    """Forced chunk lengths (TQ_SPLITK: one to five 256-vector tiles per CTA, so the merge sees
    up to 28 chunks), fp16 norms, k = 32."""
    _run(tq, bits, 256, 7001, 19, 32, seed=70 + bits, norm_dtype="f16", force=force)


def test_search_tc_agrees_with_simt(tq):
    """2- and 4-bit codes at d = 1536: the tcgen05 kernel and the SIMT kernel (TQ_SIMT=1) both
    return valid top-k lists for the oracle."""
    for bits in (2, 4):
        h, codes, norms, qg, _, (S, Q, e, rows) = _run(tq, bits, 1536, 4000, 20, 10, seed=500 + bits)
        with env(TQ_SIMT=1):
            idx, sc = (x.cpu().numpy() for x in h.search_topk(qg, codes, norms, 10))
        assert h.status() == tq.TQ_OK
        _check(idx, sc, S, Q, e, 10, 1536, 4000, rows)


def test_search_tc_full_query_tiles_sampled(tq):
    """1024 queries (8 query tiles of 128) over 60,000 vectors at d = 768: the natural split
    (whole waves of one CTA per SM); 64 sampled queries against the oracle."""
    _run(tq, 2, 768, 60000, 1024, 10, seed=901, sample=np.arange(0, 1024, 16))


def test_search_tc_bound_pass_changes_nothing(tq):
    """From 131,072 vectors on, a bound pass over the first 32,768 seeds each query's score bound
    with their exact k-th best; the full pass then skips vectors below it. The result must equal
    the search without the bound pass (TQ_SEARCH_SAMPLE=0) exactly, and be valid for the oracle."""
    h, codes, norms, qg, (idx, sc), (S, Q, e, rows) = _run(tq, 2, 256, 140000, 200, 10, seed=77,
                                                            sample=np.arange(0, 200, 8))
    with env(TQ_SEARCH_SAMPLE=0):
        idx0, sc0 = (x.cpu().numpy() for x in h.search_topk(qg, codes, norms, 10))
    assert h.status() == tq.TQ_OK
    assert np.array_equal(idx, idx0) and np.array_equal(sc, sc0)
