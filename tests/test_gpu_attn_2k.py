"""The two-kernel 3-bit decode attention against the oracle: score_prod2_kernel<true> writes
every key's score (22-bit queries, the fused kernel's logits), value_prod2_kernel turns each
chunk's scores into 16-bit weights and runs the value pass ("TurboQuant / PolarQuant / QJL
technical deep dive", "Scaled dot-product attention"; "Google TurboQuant: 6x KV-cache
compression", "Stage 2"). The library uses it for caches of 256 MB and more; TQ_ATTN_2K=1
forces it here at sizes the oracle finishes quickly. The cases reach value chunks of one to
eight 256-token blocks (the 4-stage ring wraps), ragged and empty sequences, and the decode
step, whose score kernel reads the appended key again after waiting for the append.
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
def two_kernels(on=True):
    """TQ_ATTN_2K=1 (or 0) for the calls inside, workspace sizing included."""
    old = os.environ.get("TQ_ATTN_2K")
    os.environ["TQ_ATTN_2K"] = "1" if on else "0"
    try:
        yield
    finally:
        if old is None:
            del os.environ["TQ_ATTN_2K"]
        else:
            os.environ["TQ_ATTN_2K"] = old


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


# (B, Hkv, lens, forced value chunk)
CASES = [
    (2, 8, [4096, 1000], None),          # the split policy: one-block value chunks, a ragged sequence
    (3, 8, [3000, 0, 1025], 512),        # two-block chunks, an empty sequence, a one-token last block
    (1, 8, [32768], 2048),               # the decode workload's shape, eight-block chunks (the ring wraps)
    (1, 8, [30001], 1280),               # five-block chunks, a ragged last chunk
]


@pytest.mark.parametrize("B,Hkv,lens,force", CASES)
def test_attn_2k_matches_oracle(tq, B, Hkv, lens, force):
    hk, hv, kc, vc, kod, vod, q = _case(tq, B, Hkv, lens, seed=60 + B)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    scale = 1.0 / np.sqrt(128)
    ctx = splitk(force) if force else contextlib.nullcontext()
    with ctx:
        with two_kernels(True):
            o = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
        with two_kernels(False):
            o_fused = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale).cpu().numpy()
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    ref = ops.decode_attention(q.double().numpy(), kod, vod, [max(1, x) for x in lens], scale)
    worst = _check_attention(o, ref, lens)
    # the same integer arithmetic as the fused kernel; only the weight steps' last bits differ
    diff = 0.0
    for b in range(B):
        for h in range(Hkv * 4):
            if lens[b]:
                diff = max(diff, np.linalg.norm(o[b, h] - o_fused[b, h]) / np.linalg.norm(ref[b, h]))
    assert diff <= ATTN_RTOL / 4, diff
    print(f"two-kernel attention B={B} chunk {force or 'policy'}: max relative error {worst:.2e} "
          f"(against the fused kernel {diff:.2e})")


def test_attn_2k_decode_step_rereads_the_appended_key(tq):
    """tq_decode_step on the two-kernel path with the appended slot inside a key block whose copy
    was issued before the append finished (the slots hold garbage bytes before the step): equal
    to tq_attn_decode over the cache the step leaves behind."""
    B, Hkv, Hq, d = 2, 8, 32, 128
    lens0 = [3000, 701]
    hk, hv, kc, vc, kod, vod, q = _case(tq, B, Hkv, [x + 1 for x in lens0], seed=70)
    k_new = workloads.outlier_kv(B, Hkv, 1, d, seed=75)[:, :, 0].contiguous().cuda()
    v_new = workloads.outlier_kv(B, Hkv, 1, d, seed=76)[:, :, 0].contiguous().cuda()
    for c in (kc, vc):
        for b, l0 in enumerate(lens0):
            c.codes[b, :, l0].fill_(0xA5)
            c.signs[b, :, l0].fill_(0x5A)
    lens = torch.tensor(lens0, dtype=torch.int32).cuda()
    L = kc.codes.shape[2]
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(d)
    with two_kernels(True):
        ws = torch.empty(tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L), dtype=torch.uint8,
                         device="cuda")
        tq.tq_decode_step(hk.ptr, hv.ptr, q.cuda(), k_new, v_new, B, Hq, Hkv, kc.struct, vc.struct, lens, scale,
                          out, ws)
        torch.cuda.synchronize()
        assert lens.cpu().tolist() == [x + 1 for x in lens0]
        again = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens, scale)
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    assert torch.equal(out, again)


def test_attn_2k_needs_the_scores_buffer(tq):
    """The two-kernel form runs only when the workspace holds its scores buffer: with the
    minimum workspace (the size asked for when the form is off) the call runs the single-kernel
    attention and returns exactly its result; with tq_attn_workspace_bytes' size it runs the
    two kernels (a result that differs in the last bits, within the tolerance)."""
    B, Hkv, Hq, d = 2, 8, 32, 128
    lens = [2000, 1500]
    hk, hv, kc, vc, kod, vod, q = _case(tq, B, Hkv, lens, seed=40)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()
    L = kc.codes.shape[2]
    scale = 1.0 / np.sqrt(d)
    with two_kernels(False):
        n_min = tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L)
        o_single = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale)
    with two_kernels(True):
        n_two = tq.tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, Hkv, L)
        assert n_two >= n_min + B * Hq * L * 4
        ws_min = torch.empty(n_min, dtype=torch.uint8, device="cuda")
        o_min = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale, workspace=ws_min)
        o_two = tq.attn_decode(hk, hv, q.cuda(), kc, vc, lens_t, scale)
    assert hk.status() == tq.TQ_OK and hv.status() == tq.TQ_OK
    assert torch.equal(o_min, o_single)
    ref = ops.decode_attention(q.double().numpy(), kod, vod, lens, scale)
    _check_attention(o_two.cpu().numpy(), ref, lens)
