"""Guard bands around every output and workspace buffer of the hot calls (the substitute for a
memory checker, which is not available on this machine): each buffer sits between two 256-byte
bands filled with a known pattern, and after the call every band must be unchanged. Also the
resume property of a handle: it is fully described by (d, bits, m, seed, norm dtype), so a
handle rebuilt from those parameters has the same rotation, projection and codebook bytes and
decodes an existing cache to the same results."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

BAND = 256
PATTERN = 0xA5


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


class Guarded:
    """A device buffer with guard bands: `view(dtype, shape)` is the interior the call may write."""

    def __init__(self, nbytes):
        self.n = (int(nbytes) + 15) // 16 * 16
        self.raw = torch.full((BAND + self.n + BAND,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        count = int(np.prod(shape)) if len(shape) else 1
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        assert nbytes <= self.n
        return self.raw[BAND:BAND + nbytes].view(dtype).view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.raw[:BAND].cpu().numpy()
        tail = self.raw[BAND + self.n:].cpu().numpy()
        assert np.all(head == PATTERN) and np.all(tail == PATTERN), f"{what}: a guard band was written"


def _rows(tq, h, lead):
    """Guarded packed storage for vectors of leading shape `lead` (None where the handle has none)."""
    n = int(np.prod(lead))
    out = {"codes": None, "signs": None, "rnorms": None}
    g = {}
    if h.codes_B:
        g["codes"] = Guarded(n * h.codes_B)
        out["codes"] = g["codes"].view(torch.uint8, tuple(lead) + (h.codes_B,))
    g["norms"] = Guarded(n * (2 if h.norm_dtype == tq.TQ_F16 else 4))
    out["norms"] = g["norms"].view(h.norm_torch_dtype(), tuple(lead))
    if h.m:
        g["signs"] = Guarded(n * h.signs_B)
        out["signs"] = g["signs"].view(torch.uint8, tuple(lead) + (h.signs_B,))
        if h.bits_mse:
            g["rnorms"] = Guarded(n * 2)
            out["rnorms"] = g["rnorms"].view(torch.float16, tuple(lead))
    return out, g


def _check_all(guards, what):
    for name, gb in guards.items():
        gb.check(f"{what}: {name}")


@pytest.mark.parametrize("kind", ["mse3", "prod3", "qjl1", "mse4f16", "polar"])
def test_encode_append_score_attention_stay_inside_their_buffers(tq, kind):
    d, B, Hkv, G, L = 128, 2, 2, 4, 1104   # L + 8 slots: a multiple of 8, as the tensor-core kernels need
    if kind == "polar":
        hk = tq.PolarHandle(d, 4, 2, seed=1)
    elif kind == "mse3":
        hk = tq.Handle(d, 3, 1)
    elif kind == "prod3":
        hk = tq.Handle(d, 3, 1, qjl_m=128)
    elif kind == "qjl1":
        hk = tq.Handle(d, 1, 1, qjl_m=128)
    else:
        hk = tq.Handle(d, 4, 1, norm_dtype=tq.TQ_F16)
    x = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16).cuda()
    # encode of 2 * 2 * 1104 rows (tensor-core encode where the handle has it), then of 37 rows
    for n in (B * Hkv * L, 37):
        rows, guards = _rows(tq, hk, (n,))
        tq.tq_encode(hk.ptr, x.reshape(-1, d)[:n], n, rows["codes"], rows["signs"], rows["norms"], rows["rnorms"])
        _check_all(guards, f"{kind} encode {n}")
    # a cache in guarded buffers: fill, append (advance), score
    rows, guards = _rows(tq, hk, (B, Hkv, L + 8))
    cache = tq.Cache(hk, B, Hkv, L + 8)
    cache.codes, cache.signs, cache.norms, cache.rnorms = rows["codes"], rows["signs"], rows["norms"], rows["rnorms"]
    cache.struct = tq.make_cache(cache.codes, cache.signs, cache.norms, cache.rnorms, L + 8)
    tmp = hk.encode(x)
    for name in ("codes", "signs", "norms", "rnorms"):
        if tmp[name] is not None:
            getattr(cache, name)[:, :, :L].copy_(tmp[name])
    lens = torch.tensor([L, L - 300], dtype=torch.int32, device="cuda")
    cache.append(torch.randn(B, Hkv, d, device="cuda").to(torch.bfloat16), lens, advance=True)
    _check_all(guards, f"{kind} append")
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(8)).cuda()
    lg = Guarded(B * Hkv * G * (L + 8) * 4)
    wg = Guarded(tq.tq_score_workspace_bytes(hk.ptr, B, Hkv * G))
    logits = lg.view(torch.float32, (B, Hkv * G, L + 8))
    tq.score(hk, q, cache, lens, logits=logits, workspace=wg.view(torch.uint8, (wg.n,)))
    lg.check(f"{kind} score logits")
    wg.check(f"{kind} score workspace")
    assert hk.status() == tq.TQ_OK
    if kind == "polar":
        return
    # decode attention (K and V both of this kind) and the fused decode step
    og = Guarded(B * Hkv * G * d * 4)
    ws_bytes = tq.tq_attn_workspace_bytes(hk.ptr, hk.ptr, B, Hkv * G, Hkv, L + 8)
    awg = Guarded(ws_bytes)
    out = og.view(torch.float32, (B, Hkv * G, d))
    tq.attn_decode(hk, hk, q, cache, cache, lens, 0.1, out=out, workspace=awg.view(torch.uint8, (awg.n,)))
    og.check(f"{kind} attention output")
    awg.check(f"{kind} attention workspace")
    knew = torch.randn(B, Hkv, d, device="cuda").to(torch.bfloat16)
    tq.tq_decode_step(hk.ptr, hk.ptr, q, knew, knew, B, Hkv * G, Hkv, cache.struct, cache.struct, lens, 0.1, out,
                      awg.view(torch.uint8, (awg.n,)))
    og.check(f"{kind} decode-step output")
    awg.check(f"{kind} decode-step workspace")
    _check_all(guards, f"{kind} decode-step cache")
    assert hk.status() == tq.TQ_OK


@pytest.mark.parametrize("bits,d", [(2, 1536), (4, 512), (3, 256)])
def test_search_stays_inside_its_buffers(tq, bits, d):
    h = tq.Handle(d, bits, 2)
    n, nq, k = 5000, 21, 10
    db = torch.randn(n, d, generator=torch.Generator().manual_seed(9)).cuda()
    enc = h.encode(db)
    q = torch.randn(nq, d, generator=torch.Generator().manual_seed(10)).cuda()
    ig, sg = Guarded(nq * k * 8), Guarded(nq * k * 4)
    wg = Guarded(tq.tq_search_workspace_bytes(h.ptr, nq, n, k))
    idx, score = ig.view(torch.int64, (nq, k)), sg.view(torch.float32, (nq, k))
    tq.tq_search_topk(h.ptr, q, nq, enc["codes"], enc["norms"], n, k, idx, score, wg.view(torch.uint8, (wg.n,)))
    for gb, name in ((ig, "idx"), (sg, "score"), (wg, "workspace")):
        gb.check(f"search {bits}-bit {name}")
    assert h.status() == tq.TQ_OK


def test_noalloc_attention_stays_inside_its_output(tq):
    hk, hv = tq.Handle(128, 3, 0, qjl_m=128), tq.Handle(128, 3, 1, qjl_m=128)
    B, Hkv, L = 1, 2, 700
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    x = torch.randn(B, Hkv, L, 128, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16).cuda()
    kc.fill(x)
    vc.fill(x)
    q = torch.randn(B, 8, 128, device="cuda")
    og = Guarded(B * 8 * 128 * 4)
    tq.tq_attn_decode_noalloc(hk.ptr, hv.ptr, q, B, 8, Hkv, kc.struct, vc.struct,
                              torch.tensor([L], dtype=torch.int32, device="cuda"), 0.1, og.view(torch.float32, (B, 8, 128)))
    og.check("no-alloc attention output")


@pytest.mark.parametrize("bits,m,nd", [(3, 128, None), (4, 0, 1), (1, 128, None)])
def test_a_handle_rebuilt_from_its_parameters_decodes_the_same_cache(tq, bits, m, nd):
    """Resume: the cache is plain bytes plus lengths; a new handle with the same (d, bits, m,
    seed, norm dtype) has identical Pi, S and codebook and gives bit-identical attention."""
    d, B, Hkv, L = 128, 1, 2, 900
    kw = dict(qjl_m=m, norm_dtype=nd)
    h1, v1 = tq.Handle(d, bits, 5, **kw), tq.Handle(d, 3, 6, qjl_m=128)
    kc, vc = tq.Cache(h1, B, Hkv, L), tq.Cache(v1, B, Hkv, L)
    x = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(12)).to(torch.bfloat16).cuda()
    kc.fill(x)
    vc.fill(x)
    q = torch.randn(B, 4 * Hkv, d, generator=torch.Generator().manual_seed(13)).cuda()
    lens = torch.tensor([L - 5], dtype=torch.int32, device="cuda")
    o1 = tq.attn_decode(h1, v1, q, kc, vc, lens, 0.1)
    Pi1, S1 = h1.rotation()
    c1, b1 = h1.codebook()
    h1.close()
    h2, v2 = tq.Handle(d, bits, 5, **kw), tq.Handle(d, 3, 6, qjl_m=128)
    Pi2, S2 = h2.rotation()
    c2, b2 = h2.codebook()
    assert Pi1.tobytes() == Pi2.tobytes() and c1.tobytes() == c2.tobytes() and b1.tobytes() == b2.tobytes()
    if m:
        assert S1.tobytes() == S2.tobytes()
    o2 = tq.attn_decode(h2, v2, q, kc, vc, lens, 0.1)
    assert torch.equal(o1, o2)
