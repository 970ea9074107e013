"""The tcgen05 3-bit decode attention (attn_prod2_tc_kernel, selected by TQ_ATTN_TC=1) against
the oracle.

Keys and values are prod 2+1 caches (2-bit codes, 128 QJL signs, fp16 norms) at d = 128
with 4 query heads per KV head ("TurboQuant / PolarQuant / QJL technical deep dive",
"Scaled dot-product attention"; "Google TurboQuant: 6x KV-cache compression", "Stage 1"
and "Stage 2"). The kernel is persistent (one CTA per SM walking items of (sequence, KV
head, chunk)), so the cases here give CTAs several items, empty items (a sequence of
length 0, chunks past a short sequence's end), partial 128-token tiles, and chunks of
up to 16 tiles; each is compared element by element with the oracle at the attention
tolerance, and with the mma.sync kernel (the default), whose integer arithmetic it shares.
"""

import contextlib
import os

import numpy as np
import pytest
import torch

import workloads
from gpu_util import ATTN_RTOL, OracleHandle, to_np64
from oracle import ops
from test_gpu_splitk import _check_attention, oracle_cache, splitk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    return build_lib()


@contextlib.contextmanager
def tc_kernel():
    """Selects the tcgen05 attention kernel for the calls inside."""
    os.environ["TQ_ATTN_TC"] = "1"
    try:
        yield
    finally:
        del os.environ["TQ_ATTN_TC"]


def _case(tq, B, Hkv, lens, seed):
    d, G = 128, 4
    L = (max(max(lens), 128) + 7) // 8 * 8
    hk, hv = tq.Handle(d, 3, seed, qjl_m=128), tq.Handle(d, 3, seed + 1, qjl_m=128)
    ohk, ohv = OracleHandle(d, 2, seed, 128), OracleHandle(d, 2, seed + 1, 128)
    K = workloads.outlier_kv(B, Hkv, L, d, seed=seed + 2)
    V = workloads.outlier_kv(B, Hkv, L, d, seed=seed + 3)
    kc, kod, _ = oracle_cache(tq, hk, ohk, to_np64(K))
    vc, vod, _ = oracle_cache(tq, hv, ohv, to_np64(V))
    q = workloads.queries((B, Hkv * G, d), seed + 4)
    return hk, hv, kc, vc, kod, vod, q


# (B, Hkv, lens, forced chunk): items = B * Hkv * nsplit; with 148 SMs the cases with more
# items than SMs run several items per CTA.
CASES = [
    (1, 8, [32768], None),                 # the decode-step workload: 8 x 18 chunks of 1920 tokens (15 tiles)
    (3, 8, [4096, 0, 1001], 512),          # 192 items: empty sequence, partial tiles, two items per CTA
    (2, 2, [300, 129], None),              # one item per (sequence, head), partial tiles of 44 and 1 tokens
    (5, 8, [2048, 2047, 17, 1536, 640], 256),   # 320 items, mostly empty past the short sequences' ends
]


@pytest.mark.parametrize("B,Hkv,lens,force", CASES)
def test_attn_tc_matches_oracle(tq, B, Hkv, lens, force):
    hk, hv, kc, vc, kod, vod, q = _case(tq, B, Hkv, lens, seed=80 + B)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    scale = 1.0 / np.sqrt(128)
    ctx = splitk(force) if force else contextlib.nullcontext()
    with ctx:
        o_mma = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
        with tc_kernel():
            o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, x) for x in lens], scale)
    worst = _check_attention(o, ref, lens)
    worst_mma = _check_attention(o_mma, ref, lens)
    # the two kernels share the integer arithmetic; only the weight steps' last bits differ
    diff = 0.0
    for b in range(B):
        for h in range(Hkv * 4):
            if lens[b]:
                nr = np.linalg.norm(ref[b, h])
                diff = max(diff, np.linalg.norm(o[b, h] - o_mma[b, h]) / nr)
    assert diff <= ATTN_RTOL / 4, diff
    print(f"tcgen05 attention B={B} Hkv={Hkv} chunk {force or 'policy'}: max relative error {worst:.2e} "
          f"(mma.sync kernel {worst_mma:.2e}, between the two {diff:.2e})")


def test_attn_tc_decode_step_new_token_in_a_middle_tile(tq):
    """tq_decode_step with the appended slot in the middle of a chunk and of a tile (the
    kernel reads that token's rows from global memory after waiting for the append): equal
    to tq_attn_decode over the cache the step leaves behind."""
    B, Hkv, Hq, d = 2, 8, 32, 128
    lens0 = [3000, 701]
    hk, hv, kc, vc, kod, vod, q = _case(tq, B, Hkv, [x + 1 for x in lens0], seed=90)
    k_new = workloads.outlier_kv(B, Hkv, 1, d, seed=95)[:, :, 0].contiguous().cuda()
    v_new = workloads.outlier_kv(B, Hkv, 1, d, seed=96)[:, :, 0].contiguous().cuda()
    lens = torch.tensor(lens0, dtype=torch.int32).cuda()
    L = kc.codes.shape[2]
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8, device="cuda")
    scale = 1.0 / np.sqrt(d)
    with splitk(1024), tc_kernel():
        tq.tq_decode_step(hk.ptr, hv.ptr, q.cuda(), k_new, v_new, B, Hq, Hkv, kc.struct, vc.struct, lens, scale,
                          out, ws)
        torch.cuda.synchronize()
        assert lens.cpu().tolist() == [x + 1 for x in lens0]
        again = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens, scale)
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    assert torch.equal(out, again)
