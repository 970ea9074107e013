"""GPU parity of the recursive polar transform ("PolarQuant explainer", sections 1 and 3;
"TurboQuant: redefining AI efficiency", "PolarQuant") against the oracle (oracle/polar.py):
encode (per-level angle indices, packed rows, norms), append into a cache, and scores
over caches holding the oracle's rows.

Index rule: a GPU index may differ from the oracle's only by one cell (or across the
-pi / pi seam of level 1), and only where the oracle's point lies within 1e-5 of the
boundary ray between the two cells: radius * |angle - boundary| < 1e-5, the same band on
the coordinate scale as the MSE path's rule for rotated coordinates."""

import numpy as np
import pytest
import torch

from gpu_util import check_norms, max_rel_score_error, score_tolerance, to_np64
from oracle import polar, rotation

pytestmark = pytest.mark.gpu

BAND = 1e-5


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


def _oracle(d, bits, seed):
    Pi, _ = rotation.rotation(d, seed)
    return Pi, polar.codebooks(d, bits)


def _radii(y):
    """Radius of every pair at every level (list over levels of [n, d / 2^l])."""
    out, r = [], np.asarray(y, dtype=np.float64)
    while r.shape[1] > 1:
        r = np.hypot(r[:, 0::2], r[:, 1::2])
        out.append(r)
    return out


def check_polar_codes(codes, e, books, d, bits):
    """GPU rows against the oracle encode e; returns the fraction of exempt indices."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, codes.shape[-1])
    gidx = polar.unpack(codes, d, bits)
    radii = _radii(e["y"])
    total = exempt = 0
    exempt_bits = np.zeros((codes.shape[0], codes.shape[1] * 8), dtype=bool)
    lb = [bits] * len(books) if np.isscalar(bits) else bits
    pos = 0
    for lv, (g, w) in enumerate(zip(gidx, e["idx"])):
        c, bnd = books[lv]
        L = len(c)
        mism = g != w
        total += g.size
        if mism.any():
            r, i = np.nonzero(mism)
            a, b = g[r, i], w[r, i]
            seam = (lv == 0) & (np.minimum(a, b) == 0) & (np.maximum(a, b) == L - 1)
            on_origin = radii[lv][r, i] == 0   # a zero pair lies on every boundary ray
            assert np.all((np.abs(a - b) == 1) | seam | on_origin), f"level {lv + 1}: index differs by more than one cell"
            beta = np.where(seam, np.pi, bnd[np.clip(np.minimum(a, b), 0, L - 2)])
            ang = e["angles"][lv][r, i]
            dist = radii[lv][r, i] * np.abs(np.where(seam, np.pi - np.abs(ang), ang - beta))
            assert np.all(dist < BAND), f"level {lv + 1}: mismatch {dist.max():.3g} away from a boundary"
            exempt += len(r)
            for rr, ii in zip(r, i):
                exempt_bits[rr, pos + ii * lb[lv]: pos + (ii + 1) * lb[lv]] = True
        pos += (d >> (lv + 1)) * lb[lv]
    want = polar.pack(e["idx"], d, bits)
    diff = np.unpackbits(want ^ codes, axis=1, bitorder="little").astype(bool)
    assert not np.any(diff & ~exempt_bits), "packed bits differ outside an exempt index (or in the pad)"
    return exempt / total


@pytest.mark.parametrize("d,b1,bu,n,dtype", [(128, 4, 2, 3000, torch.bfloat16), (64, 3, 3, 700, torch.float32),
                                             (256, 2, 1, 300, torch.float16), (32, 4, 4, 65, torch.float32)])
def test_polar_encode_matches_oracle(tq, d, b1, bu, n, dtype):
    h = tq.PolarHandle(d, b1, bu, seed=d + b1)
    bits = h.level_bits()
    assert h.codes_B == polar.row_bytes(d, bits)
    x = torch.randn(n, d, generator=torch.Generator().manual_seed(n)) * 2
    x[3] = 0   # zero vector: every angle atan2(0, 0) = 0
    x = x.to(dtype)
    out = h.encode(x.cuda())
    Pi, books = _oracle(d, bits, d + b1)
    e = polar.encode(to_np64(x), Pi, books)
    frac = check_polar_codes(out["codes"].cpu().numpy(), e, books, d, bits)
    check_norms(out["norms"].cpu().numpy(), e["n_exact"].astype(np.float32))
    print(f"polar encode d={d} bits={b1}/{bu}: exempt index fraction {frac:.2e}")
    assert h.status() == tq.TQ_OK


def test_polar_handle_tables_match_oracle(tq):
    h = tq.PolarHandle(128, 4, 2, seed=3)
    assert (h.levels, h.bits_level1, h.bits_upper) == (7, 4, 2)
    for lv in range(1, 8):
        c, b = h.codebook(lv)
        co, bo = polar.lloyd_max(lv, 4 if lv == 1 else 2)
        assert np.allclose(c, co, atol=2e-10) and np.allclose(b, bo, atol=2e-10)
    Pi, _ = h.rotation()
    assert np.abs(Pi - rotation.rotation(128, 3)[0]).max() < 1e-12


def test_polar_append_matches_oracle_and_capacity(tq):
    B, Hkv, L_cap, d = 3, 2, 33, 128
    h = tq.PolarHandle(d, 4, 2, seed=9)
    bits = h.level_bits()
    Pi, books = _oracle(d, bits, 9)
    cache = tq.Cache(h, B, Hkv, L_cap)
    cache.codes.zero_()
    lens = torch.tensor([0, 7, L_cap - 1], dtype=torch.int32).cuda()
    toks = []
    for t in range(2):
        x = torch.randn(B, Hkv, d, generator=torch.Generator().manual_seed(50 + t)).to(torch.bfloat16)
        toks.append(x)
        cache.append(x.cuda(), lens, advance=True)
    assert h.status() == tq.TQ_ECAPACITY     # the second append found sequence 2 full
    assert lens.cpu().tolist() == [2, 9, L_cap]
    codes = cache.codes.cpu().numpy()
    for t in range(2):
        e = polar.encode(to_np64(toks[t]).reshape(-1, d), Pi, books)
        for b, start in enumerate([0, 7, L_cap - 1]):
            if start + t >= L_cap:
                continue
            for hh in range(Hkv):
                r = b * Hkv + hh
                sub = {"idx": [a[r:r + 1] for a in e["idx"]], "angles": [a[r:r + 1] for a in e["angles"]],
                       "y": e["y"][r:r + 1]}
                check_polar_codes(codes[b, hh, start + t][None], sub, books, d, bits)


@pytest.mark.parametrize("d,b1,bu,G", [(128, 4, 2, 4), (64, 3, 2, 1), (256, 2, 2, 8), (128, 4, 4, 3)])
def test_polar_scores_match_oracle(tq, d, b1, bu, G):
    B, Hkv, L = 2, 2, 900
    h = tq.PolarHandle(d, b1, bu, seed=5)
    bits = h.level_bits()
    Pi, books = _oracle(d, bits, 5)
    rs = np.random.default_rng(d + G)
    x = rs.standard_normal((B * Hkv * L, d)) * np.exp(0.5 * rs.standard_normal(d))
    e = polar.encode(x, Pi, books)
    n32 = e["n_exact"].astype(np.float32)
    cache = tq.Cache(h, B, Hkv, L)
    cache.codes.copy_(torch.from_numpy(polar.pack(e["idx"], d, bits).reshape(B, Hkv, L, -1)))
    cache.norms.copy_(torch.from_numpy(n32.reshape(B, Hkv, L)))
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(6))
    lens = [L, 411]
    got = tq.score(h, q.cuda(), cache, torch.tensor(lens, dtype=torch.int32).cuda()).cpu().numpy()
    qn = q.double().numpy()
    worst = 0.0
    for b in range(B):
        for hq in range(Hkv * G):
            hk, Lb = hq // G, lens[b]
            rows = slice((b * Hkv + hk) * L, (b * Hkv + hk) * L + Lb)
            ref = polar.score(qn[b, hq], [a[rows] for a in e["idx"]], n32[rows], Pi, books)
            nn = n32[rows].astype(np.float64)
            tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), nn, d)
            assert np.all(np.abs(got[b, hq, :Lb] - ref) <= tol), (b, hq)
            assert np.all(got[b, hq, Lb:] == 0)
            worst = max(worst, max_rel_score_error(got[b, hq, :Lb], ref, np.linalg.norm(qn[b, hq]), nn, d))
    print(f"polar scores d={d} bits={b1}/{bu} G={G}: max relative error above the floor {worst:.2e}")
    assert h.status() == tq.TQ_OK


def test_polar_handles_are_rejected_where_unsupported(tq):
    h = tq.PolarHandle(128, 4, 2)
    with pytest.raises(tq.TQError) as ei:
        tq.tq_get_codebook(h.ptr, 2)
    assert ei.value.status == tq.TQ_EINVAL
    q = torch.zeros(1, 4, 128, device="cuda")
    cache = tq.Cache(h, 1, 1, 16)
    with pytest.raises(tq.TQError) as ei:
        tq.attn_decode(h, h, q, cache, cache, torch.ones(1, dtype=torch.int32, device="cuda"), 0.1,
                       workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == tq.TQ_EUNSUPPORTED
