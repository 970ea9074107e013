"""tq_decode_step (append K and V at slot len[b], attend over len[b] + 1 tokens, advance
len) against the same work done by separate calls, and against the oracle. With Hkv in
{2, 4, 8} the step's appends are column-sliced over a cluster of Hkv CTAs; their rows must
be bit-identical to the per-vector append of tq_append
("Google TurboQuant: 6x KV-cache compression", "Stage 1" / "Stage 2"; "TurboQuant /
PolarQuant / QJL technical deep dive", "Scaled dot-product attention")."""

import numpy as np
import pytest
import torch

from gpu_util import ATTN_RTOL, OracleHandle, to_np64
from oracle import ops, quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    m = build_lib()
    assert torch.cuda.is_available()
    return m


def _setup(tq, bits, m, B, Hkv, G, L_cap, L0, seed, norm_dtype=None):
    d = 128
    hk = tq.Handle(d, bits, seed, qjl_m=m, norm_dtype=norm_dtype)
    hv = tq.Handle(d, bits, seed + 1, qjl_m=m, norm_dtype=norm_dtype)
    g = torch.Generator().manual_seed(seed)
    K = (torch.randn(B, Hkv, L_cap, d, generator=g) * 1.5).to(torch.bfloat16).cuda()
    V = torch.randn(B, Hkv, L_cap, d, generator=g).to(torch.bfloat16).cuda()
    caches = []
    for _ in range(2):
        kc, vc = tq.Cache(hk, B, Hkv, L_cap), tq.Cache(hv, B, Hkv, L_cap)
        kc.fill(K)
        vc.fill(V)
        caches.append((kc, vc))
    q = torch.randn(B, Hkv * G, d, generator=g).cuda()
    k_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v_new = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    return hk, hv, caches, q, k_new, v_new


def _step(tq, hk, hv, q, k_new, v_new, kc, vc, lens, scale):
    B, Hq, d = q.shape
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, kc.Hkv, kc.L_cap), dtype=torch.uint8,
                     device="cuda")
    tq.tq_decode_step(hk.ptr, hv.ptr, q, k_new, v_new, B, Hq, kc.Hkv, kc.struct, vc.struct, lens, scale, out, ws)
    return out


@pytest.mark.parametrize("bits,m,B,Hkv,G,L_cap,L0,f16", [
    (3, 128, 2, 8, 4, 4096, [4000, 0], False),      # int8 tensor-core attention, an empty sequence
    (3, 128, 3, 4, 4, 2048, [2047, 1500, 2048], False),  # last slot, middle, a full sequence
    (3, 0, 2, 2, 4, 1024, [700, 1023], False),      # MSE-only K/V: the SIMT attention kernel
    (4, 0, 1, 2, 2, 512, [3], False),
    (4, 0, 2, 2, 4, 3072, [3000, 1024], True),       # 4-bit MSE, fp16 norms: the Walsh-plane kernel
    (1, 128, 2, 4, 2, 512, [100, 511], False),       # QJL-only K/V (no MSE bits)
    (3, 128, 1, 1, 4, 640, [639], False),            # Hkv = 1: the per-vector append (no column slices)
    (2, 64, 1, 16, 2, 256, [200], False),            # Hkv = 16: above the cluster size, per-vector append
])
def test_decode_step_equals_separate_calls(tq, bits, m, B, Hkv, G, L_cap, L0, f16):
    hk, hv, caches, q, k_new, v_new = _setup(tq, bits, m, B, Hkv, G, L_cap, L0, seed=bits * 10 + B,
                                             norm_dtype=tq.TQ_F16 if f16 else None)
    scale = 1.0 / np.sqrt(128)
    (kc1, vc1), (kc2, vc2) = caches
    lens1 = torch.tensor(L0, dtype=torch.int32).cuda()
    lens2 = lens1.clone()
    # separate calls
    kc1.append(k_new, lens1, advance=False)
    vc1.append(v_new, lens1, advance=True)
    o1 = tq.attn_decode(hk, hv, q, kc1, vc1, lens1, scale)
    s1 = (hk.status(), hv.status())
    # one decode step
    o2 = _step(tq, hk, hv, q, k_new, v_new, kc2, vc2, lens2, scale)
    s2 = (hk.status(), hv.status())
    torch.cuda.synchronize()
    full = any(x >= L_cap for x in L0)
    assert s1 == s2 and (s1[0] == tq.TQ_ECAPACITY) == full
    assert lens1.cpu().tolist() == lens2.cpu().tolist() == [min(x + 1, L_cap) for x in L0]
    for a, b in [(kc1, kc2), (vc1, vc2)]:
        for name in ("codes", "norms", "signs", "rnorms"):   # QJL-only rows have no codes or rnorms
            x, y = getattr(a, name), getattr(b, name)
            assert (x is None) == (y is None) and (x is None or torch.equal(x, y)), name
    assert torch.equal(o1, o2)


def test_decode_step_matches_oracle(tq):
    """One step on a 3-bit prod cache; the output against the oracle's textbook attention
    over the step's own codes (the appended token included)."""
    B, Hkv, G, L_cap, L0 = 2, 2, 4, 1024, [600, 1023]
    hk, hv, caches, q, k_new, v_new = _setup(tq, 3, 128, B, Hkv, G, L_cap, L0, seed=5)
    kc, vc = caches[0]
    lens = torch.tensor(L0, dtype=torch.int32).cuda()
    scale = 1.0 / np.sqrt(128)
    out = _step(tq, hk, hv, q, k_new, v_new, kc, vc, lens, scale).cpu().numpy()
    assert hk.status() == tq.TQ_OK
    n = [x + 1 for x in L0]
    ohk, ohv = OracleHandle(128, 2, 5, 128), OracleHandle(128, 2, 6, 128)

    def od(cache, oh):
        codes = cache.codes.cpu().numpy()
        return {"idx": quant.unpack(codes.reshape(-1, codes.shape[-1]), 128, 2).reshape(B, Hkv, L_cap, 128),
                "n": to_np64(cache.norms.cpu()), "Pi": oh.Pi, "c": oh.c,
                "sigma": quant.unpack(cache.signs.cpu().numpy().reshape(-1, 16), 128, 1).reshape(B, Hkv, L_cap, 128),
                "rnorm": to_np64(cache.rnorms.cpu()), "S": oh.S}

    ref = ops.decode_attention(q.double().cpu().numpy(), od(kc, ohk), od(vc, ohv), n, scale)
    for b in range(B):
        for h in range(Hkv * G):
            nr = np.linalg.norm(ref[b, h])
            assert np.linalg.norm(out[b, h] - ref[b, h]) <= ATTN_RTOL * nr, (b, h)
