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
