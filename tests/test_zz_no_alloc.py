"""GPU test of tq_attn_decode_noalloc, the decode-attention entry point that allocates nothing.

Who needs it: code that may not allocate device memory while it runs -- a
plugin inside an inference engine that only receives its input and output
buffers, or a serving loop whose allocator is frozen after start-up. Instead of
a caller workspace, the call uses a fixed 4 MiB scratch array compiled into
libtq.so. This file is collected last on purpose: it must pass when run alone
in a fresh process and after every other test (the array keeps whatever the
previous call left in it).
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


def _caches(tq, bits_k, m_k, bits_v, m_v, B, Hkv, L, seed):
    d = 128
    hk = tq.Handle(d, bits_k, seed, qjl_m=m_k)
    hv = tq.Handle(d, bits_v, seed + 1, qjl_m=m_v)
    g = torch.Generator().manual_seed(seed)
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    kc.fill(torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16).cuda())
    vc.fill(torch.randn(B, Hkv, L, d, generator=g).to(torch.bfloat16).cuda())
    return hk, hv, kc, vc


def _both(tq, hk, hv, kc, vc, q, lens):
    """(output of tq_attn_decode with a caller workspace, output of tq_attn_decode_noalloc)."""
    B, Hq, d = q.shape
    scale = 1.0 / np.sqrt(d)
    ref = tq.attn_decode(hk, hv, q, kc, vc, lens, scale)
    out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
    tq.tq_attn_decode_noalloc(hk.ptr, hv.ptr, q, B, Hq, kc.Hkv, kc.struct, vc.struct, lens, scale, out)
    torch.cuda.synchronize()
    return ref.cpu().numpy(), out.cpu().numpy()


def _close(ref, got):
    # the same kernels with the same split run on both paths (the split depends on the shape only),
    # so the outputs must agree bit for bit; a stale or misplaced partial would show here
    assert np.array_equal(ref, got)


def test_noalloc_matches_workspace_entry_point_twice(tq):
    # first call: prod 2+1 K and V, GQA 4:1, ragged lengths
    hk, hv, kc, vc = _caches(tq, 3, 128, 3, 128, B=2, Hkv=2, L=1500, seed=40)
    q1 = torch.randn(2, 8, 128, generator=torch.Generator().manual_seed(1)).cuda()
    lens1 = torch.tensor([1500, 777], dtype=torch.int32, device="cuda")
    ref1, got1 = _both(tq, hk, hv, kc, vc, q1, lens1)
    _close(ref1, got1)
    # second call in a row, other shapes and formats: the scratch holds the first call's data
    hk2, hv2, kc2, vc2 = _caches(tq, 4, 0, 4, 0, B=1, Hkv=4, L=900, seed=50)
    q2 = torch.randn(1, 8, 128, generator=torch.Generator().manual_seed(2)).cuda()
    lens2 = torch.tensor([900], dtype=torch.int32, device="cuda")
    ref2, got2 = _both(tq, hk2, hv2, kc2, vc2, q2, lens2)
    _close(ref2, got2)
    assert hk.status() == tq.TQ_OK and hk2.status() == tq.TQ_OK


def test_noalloc_empty_batch_is_a_no_op(tq):
    # B == 0: TQ_OK without touching anything, like tq_attn_decode (whose caches may then be NULL)
    hk = tq.Handle(128, 3, 0, qjl_m=128)
    hv = tq.Handle(128, 3, 1, qjl_m=128)
    status = tq._lib.lib.tq_attn_decode_noalloc(hk.ptr, hv.ptr, None, tq.TQ_F32, 0, 8, 2, None, None, None,
                                                ctypes.c_float(0.1), None, None)
    assert status == tq.TQ_OK


def test_noalloc_rejects_shapes_beyond_its_scratch(tq):
    hk = tq.Handle(128, 3, 0, qjl_m=128)
    hv = tq.Handle(128, 3, 1, qjl_m=128)
    B, Hq, Hkv, L_cap = 64, 64, 8, 1 << 20
    assert tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L_cap) > (4 << 20)
    cache = tq._lib.tq_cache(256, 256, 256, 256, L_cap)   # never dereferenced: the size check comes first
    status = tq._lib.lib.tq_attn_decode_noalloc(hk.ptr, hv.ptr, ctypes.c_void_p(256), tq.TQ_F32, B, Hq, Hkv,
                                                ctypes.byref(cache), ctypes.byref(cache), ctypes.c_void_p(256),
                                                ctypes.c_float(0.1), ctypes.c_void_p(256), None)
    assert status == tq.TQ_EINVAL
    assert "4194304-byte array" in tq.tq_last_error()
