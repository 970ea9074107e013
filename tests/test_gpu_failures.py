"""Device-side failure detection without a GPU fault: a bounded wait that runs out is
recorded in the handle's error word and read back as TQ_ETIMEOUT, after which the CUDA
context keeps working (the same path every kernel takes when a copy or a release never
completes). Capacity overflow of an append is covered in test_gpu_score_attn.py."""

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    m = build_lib()
    assert torch.cuda.is_available()
    return m


def test_bounded_wait_timeout_is_reported_and_the_context_survives(tq):
    h = tq.Handle(128, 2, 0)
    assert h.status() == tq.TQ_OK
    tq.tq_selftest_wait_timeout(h.ptr, 64)          # at most 64 polls, a few ms
    assert tq.tq_last_status(h.ptr) == tq.TQ_ETIMEOUT
    assert h.status() == tq.TQ_OK                   # read once, then cleared
    # the context is intact: an encode afterwards runs and matches its own re-run
    x = torch.randn(300, 128, generator=torch.Generator().manual_seed(0)).cuda()
    a = h.encode(x)
    b = h.encode(x)
    torch.cuda.synchronize()
    assert torch.equal(a["codes"], b["codes"]) and torch.equal(a["norms"], b["norms"])
    assert h.status() == tq.TQ_OK
    # and the timeout is per handle: another handle's word is untouched
    h2 = tq.Handle(128, 2, 1)
    tq.tq_selftest_wait_timeout(h.ptr, 1)
    assert h2.status() == tq.TQ_OK and h.status() == tq.TQ_ETIMEOUT


def test_selftest_rejects_a_bad_limit(tq):
    h = tq.Handle(128, 2, 0)
    for bad in (0, -1, (1 << 16) + 1):
        with pytest.raises(tq.TQError) as e:
            tq.tq_selftest_wait_timeout(h.ptr, bad)
        assert e.value.status == tq.TQ_EINVAL


def _env(name, value):
    import contextlib
    import os

    @contextlib.contextmanager
    def cm():
        old = os.environ.get(name)
        os.environ[name] = value
        try:
            yield
        finally:
            if old is None:
                del os.environ[name]
            else:
                os.environ[name] = old
    return cm()


def test_check_mode_reports_out_of_range_lengths(tq):
    """TQ_CHECK=1: a device length outside 0 .. L_cap is reported (TQ_EINVAL from the error word)
    instead of being clamped silently; valid lengths report nothing, and without TQ_CHECK the
    same bad length is clamped as before."""
    B, Hkv, G, L, d = 3, 2, 4, 256, 128
    hk, hv = tq.Handle(d, 3, 0, qjl_m=128), tq.Handle(d, 3, 1, qjl_m=128)
    kc, vc = tq.Cache(hk, B, Hkv, L), tq.Cache(hv, B, Hkv, L)
    x = torch.randn(B, Hkv, L, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    kc.fill(x)
    vc.fill(x)
    q = torch.randn(B, Hkv * G, d, generator=torch.Generator().manual_seed(2)).cuda()
    good = torch.tensor([L, 0, 100], dtype=torch.int32, device="cuda")
    bad = torch.tensor([L + 1, -3, 100], dtype=torch.int32, device="cuda")
    with _env("TQ_CHECK", "1"):
        tq.attn_decode(hk, hv, q, kc, vc, good, 0.1)
        tq.score(hk, q, kc, good)
        assert hk.status() == tq.TQ_OK
        tq.attn_decode(hk, hv, q, kc, vc, bad, 0.1)
        assert hk.status() == tq.TQ_EINVAL
        assert "TQ_CHECK" in tq.tq_last_error()
        tq.score(hk, q, kc, bad)
        assert hk.status() == tq.TQ_EINVAL
        kc.append(x[:, :, 0].contiguous(), bad, advance=False)
        assert hk.status() == tq.TQ_EINVAL
    tq.attn_decode(hk, hv, q, kc, vc, bad, 0.1)
    assert hk.status() == tq.TQ_OK


def test_injected_timeout_is_reported_by_hot_calls(tq):
    """TQ_FAULT=timeout: a hot call records the error a timed-out wait records (no wait runs);
    tq_last_status returns TQ_ETIMEOUT once and the handle keeps working."""
    h = tq.Handle(128, 3, 0)
    x = torch.randn(64, 128, generator=torch.Generator().manual_seed(3)).cuda()
    with _env("TQ_FAULT", "timeout"):
        h.encode(x)
    assert h.status() == tq.TQ_ETIMEOUT
    a = h.encode(x)
    assert h.status() == tq.TQ_OK
    b = h.encode(x)
    torch.cuda.synchronize()
    assert torch.equal(a["codes"], b["codes"])
