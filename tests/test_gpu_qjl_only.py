"""GPU parity of QJL-only rows (1 bit per projection: the sign sketch of the whole vector
plus its norm, no MSE codes) against the oracle ("TurboQuant: redefining AI efficiency",
"QJL: zero-overhead 1-bit compression"; "TurboQuant / PolarQuant / QJL technical deep
dive", "QJL"): encode (signs within the boundary band, norms within 1 ulp), scores, decode
attention with QJL-only keys and/or values, append and the fused decode step.
Caches for the score and attention tests hold the oracle's rows."""

import numpy as np
import pytest
import torch

from gpu_util import (ATTN_RTOL, OracleHandle, check_norms, check_signs, max_rel_score_error, score_tolerance,
                      to_np64)
from oracle import ops, quant, rotation

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


def _qjl_rows(d, m, seed, x, norm_dtype="f16"):
    _, S = rotation.rotation(d, seed, m)
    return quant.encode_qjl(np.asarray(x, dtype=np.float64).reshape(-1, d), S, norm_dtype), S


def qjl_cache(tq, h, x, seed):
    """Cache of QJL-only handle h holding the oracle's rows of x [B, Hkv, L, d]."""
    B, Hkv, L, d = x.shape
    e, S = _qjl_rows(d, h.m, seed, x, "f16" if h.norm_dtype == tq.TQ_F16 else "f32")
    cache = tq.Cache(h, B, Hkv, L)
    assert cache.codes is None and cache.rnorms is None
    cache.signs.copy_(torch.from_numpy(quant.pack(e["sigma"], 1).reshape(B, Hkv, L, -1)))
    cache.norms.copy_(torch.from_numpy(e["n_stored"].reshape(B, Hkv, L)))
    return cache, {"sigma": e["sigma"].reshape(B, Hkv, L, h.m), "n": e["n_stored"].reshape(B, Hkv, L), "S": S}


def prod_cache(tq, h, oh, x):
    B, Hkv, L, d = x.shape
    e = oh.encode(x.reshape(-1, d), "f16")
    cache = tq.Cache(h, B, Hkv, L)
    cache.codes.copy_(torch.from_numpy(quant.pack(e["idx"], oh.bits).reshape(B, Hkv, L, -1)))
    cache.norms.copy_(torch.from_numpy(e["n_stored"].reshape(B, Hkv, L)))
    cache.signs.copy_(torch.from_numpy(quant.pack(e["sigma"], 1).reshape(B, Hkv, L, -1)))
    cache.rnorms.copy_(torch.from_numpy(e["rnorm_stored"].reshape(B, Hkv, L)))
    return cache, {"idx": e["idx"].reshape(B, Hkv, L, d), "n": e["n_stored"].reshape(B, Hkv, L), "Pi": oh.Pi,
                   "c": oh.c, "sigma": e["sigma"].reshape(B, Hkv, L, oh.m),
                   "rnorm": e["rnorm_stored"].reshape(B, Hkv, L), "S": oh.S}


def test_qjl_only_handle_layout(tq):
    h = tq.Handle(128, 1, 3, qjl_m=128)
    assert (h.bits_mse, h.m, h.codes_B, h.signs_B, h.qjl_only) == (0, 128, 0, 16, True)
    assert h.norm_dtype == tq.TQ_F16
    c, b = h.codebook()
    assert list(c) == [0.0] and len(b) == 0
    Pi, S = h.rotation()
    Pio, So = rotation.rotation(128, 3, 128)
    assert np.max(np.abs(S - So)) < 1e-12


@pytest.mark.parametrize("d,m,n,dtype", [(128, 128, 3000, torch.bfloat16), (128, 256, 37, torch.float32),
                                         (64, 64, 1500, torch.float16), (64, 96, 5, torch.float32)])
def test_qjl_only_encode_matches_oracle(tq, d, m, n, dtype):
    """Signs of S x (a mismatch only where |(S x)_j| < 1e-5 ||x||) and the fp16 norm (1 ulp);
    row 1 is the zero vector (all sign bits set, norm 0)."""
    h = tq.Handle(d, 1, 5, qjl_m=m)
    x = torch.randn(n, d, generator=torch.Generator().manual_seed(d + m + n)) * 3
    x[min(1, n - 1)] = 0
    x = x.to(dtype)
    out = h.encode(x.cuda())
    assert out["codes"] is None and out["rnorms"] is None
    e, _ = _qjl_rows(d, m, 5, to_np64(x))
    check_norms(out["norms"].cpu().numpy(), e["n_stored"])
    frac = check_signs(out["signs"].cpu().numpy(), e, np.zeros(0, dtype=np.int64))
    assert np.all(np.unpackbits(out["signs"][min(1, n - 1)].cpu().numpy()) == 1)
    print(f"QJL-only encode d={d} m={m} n={n}: sign mismatch fraction {frac:.2e}")
    assert h.status() == tq.TQ_OK


@pytest.mark.parametrize("G,m", [(4, 128), (2, 64)])
def test_qjl_only_scores_match_oracle(tq, G, m):
    B, Hkv, L, d = 2, 2, 1500, 128
    h = tq.Handle(d, 1, 7, qjl_m=m)
    x = np.random.default_rng(7).standard_normal((B, Hkv, L, d)) * 2
    cache, od = qjl_cache(tq, h, x, 7)
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(8))
    lens = [L, 777]
    got = tq.score(h, q.cuda(), cache, torch.tensor(lens, dtype=torch.int32).cuda()).cpu().numpy()
    qn = q.double().numpy()
    worst = 0.0
    for b in range(B):
        for hq in range(Hkv * G):
            hk, Lb = hq // G, lens[b]
            ref = ops.score_qjl(qn[b, hq], od["sigma"][b, hk, :Lb], od["n"][b, hk, :Lb], od["S"])
            n = od["n"][b, hk, :Lb].astype(np.float64)
            tol = score_tolerance(ref, np.linalg.norm(qn[b, hq]), n, d)
            assert np.all(np.abs(got[b, hq, :Lb] - ref) <= tol), (b, hq)
            assert np.all(got[b, hq, Lb:] == 0)
            worst = max(worst, max_rel_score_error(got[b, hq, :Lb], ref, np.linalg.norm(qn[b, hq]), n, d))
    print(f"QJL-only scores (m={m}): max relative error above the floor {worst:.2e}")
    assert h.status() == tq.TQ_OK


@pytest.mark.parametrize("k_kind,v_kind,G", [("qjl", "prod", 4), ("prod", "qjl", 4), ("qjl", "qjl", 2)])
def test_qjl_only_attention_matches_oracle(tq, k_kind, v_kind, G):
    B, Hkv, L, d = 2, 2, 1200, 128
    xk = np.random.default_rng(11).standard_normal((B, Hkv, L, d)) * 1.5
    xv = np.random.default_rng(12).standard_normal((B, Hkv, L, d))
    if k_kind == "qjl":
        hk = tq.Handle(d, 1, 13, qjl_m=128)
        kc, kod = qjl_cache(tq, hk, xk, 13)
    else:
        hk = tq.Handle(d, 3, 13, qjl_m=128)
        kc, kod = prod_cache(tq, hk, OracleHandle(d, 2, 13, 128), xk)
    if v_kind == "qjl":
        hv = tq.Handle(d, 1, 14, qjl_m=128)
        vc, vod = qjl_cache(tq, hv, xv, 14)
    else:
        hv = tq.Handle(d, 3, 14, qjl_m=128)
        vc, vod = prod_cache(tq, hv, OracleHandle(d, 2, 14, 128), xv)
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(15)) * 2
    lens = [L, 301]
    o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, torch.tensor(lens, dtype=torch.int32).cuda(),
                       1 / np.sqrt(d)).cpu().numpy()
    ref = ops.decode_attention(q.double().numpy(), kod, vod, lens, 1 / np.sqrt(d))
    for b in range(B):
        for h in range(Hkv * G):
            nr = np.linalg.norm(ref[b, h])
            assert np.linalg.norm(o[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK


def test_qjl_only_decode_step_equals_separate_calls_and_append_matches_oracle(tq):
    """QJL-only keys with prod-3 values: tq_decode_step against tq_append + tq_append +
    tq_attn_decode (bit for bit), and the appended key row against the oracle."""
    B, Hkv, G, L_cap, d = 2, 4, 4, 2048, 128
    hk = tq.Handle(d, 1, 21, qjl_m=128)
    hv = tq.Handle(d, 3, 22, qjl_m=128)
    g = torch.Generator().manual_seed(23)
    K = torch.randn(B, Hkv, L_cap, d, generator=g).to(torch.bfloat16).cuda()
    V = torch.randn(B, Hkv, L_cap, d, generator=g).to(torch.bfloat16).cuda()
    q = torch.randn(B, Hkv * G, d, generator=g).cuda()
    k_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    v_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    pairs = []
    for _ in range(2):
        kc, vc = tq.Cache(hk, B, Hkv, L_cap), tq.Cache(hv, B, Hkv, L_cap)
        kc.fill(K)
        vc.fill(V)
        pairs.append((kc, vc))
    L0 = [1999, 1024]
    scale = 1 / np.sqrt(d)
    (kc1, vc1), (kc2, vc2) = pairs
    lens1 = torch.tensor(L0, dtype=torch.int32).cuda()
    lens2 = lens1.clone()
    kc1.append(k_new.cuda(), lens1, advance=False)
    vc1.append(v_new, lens1, advance=True)
    o1 = tq.attn_decode(hk, hv, q, kc1, vc1, lens1, scale)
    o2 = torch.empty_like(o1)
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hkv * G, Hkv, L_cap), dtype=torch.uint8,
                     device="cuda")
    tq.tq_decode_step(hk.ptr, hv.ptr, q, k_new.cuda(), v_new, B, Hkv * G, Hkv, kc2.struct, vc2.struct, lens2, scale,
                      o2, ws)
    torch.cuda.synchronize()
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    assert lens1.cpu().tolist() == lens2.cpu().tolist() == [x + 1 for x in L0]
    assert torch.equal(kc1.signs, kc2.signs) and torch.equal(kc1.norms, kc2.norms)
    assert torch.equal(vc1.codes, vc2.codes) and torch.equal(vc1.signs, vc2.signs)
    assert torch.equal(o1, o2)
    e, _ = _qjl_rows(d, 128, 21, to_np64(k_new))
    for b in range(B):
        rows = slice(b * Hkv, (b + 1) * Hkv)
        sub = {"z": e["z"][rows], "sigma": e["sigma"][rows], "n_exact": e["n_exact"][rows]}
        check_signs(kc1.signs[b, :, L0[b]].cpu().numpy(), sub, np.zeros(0, dtype=np.int64))
        check_norms(kc1.norms[b, :, L0[b]].cpu().numpy(), e["n_stored"][rows])
