"""GPU parity of the handle constants, encode (MSE and prod), pack and append
against the oracle ("Google TurboQuant: 6x KV-cache compression", sections
"Stage 1: PolarQuant" and "Stage 2: QJL residual correction")."""

import numpy as np
import pytest
import torch

from gpu_util import OracleHandle, check_codes, check_norms, check_signs, to_np64
from oracle import quant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq():
    from conftest import build_lib
    m = build_lib()
    assert torch.cuda.is_available()
    return m


NORM_NP = {0: "f32", 1: "f16"}


def _encode_and_check(tq, x_cpu, d, bits, seed, m=0, norm_dtype=None):
    h = tq.Handle(d, bits, seed, qjl_m=m, norm_dtype=norm_dtype)
    oh = OracleHandle(d, h.bits_mse, seed, m)
    out = h.encode(x_cpu.cuda())
    torch.cuda.synchronize()
    exp = oh.encode(to_np64(x_cpu), NORM_NP[h.norm_dtype])
    gidx, bad, frac = check_codes(out["codes"].cpu().numpy().reshape(-1, h.codes_B), exp, oh)
    check_norms(out["norms"].cpu().numpy().reshape(-1), exp["n_stored"])
    sfrac = None
    if m:
        sfrac = check_signs(out["signs"].cpu().numpy().reshape(-1, h.signs_B), exp, bad)
        keep = np.ones(len(exp["idx"]), bool)
        keep[bad] = False
        check_norms(out["rnorms"].cpu().numpy().reshape(-1)[keep], exp["rnorm_stored"][keep])
    assert h.status() == tq.TQ_OK
    return frac, sfrac


def test_handle_constants_match_oracle(tq):
    for d, bits, m, seed in [(128, 3, 0, 0), (128, 3, 128, 2), (1536, 2, 0, 0), (64, 4, 0, 5)]:
        h = tq.Handle(d, bits, seed, qjl_m=m)
        oh = OracleHandle(d, h.bits_mse, seed, m)
        Pi, S = h.rotation()
        c, b = h.codebook()
        assert np.abs(Pi - oh.Pi).max() <= 1e-12
        assert np.abs(c - oh.c).max() <= 1e-12 and np.abs(b - oh.beta).max() <= 1e-12
        if m:
            assert np.abs(S - oh.S).max() <= 1e-12
        assert h.codes_B == d * h.bits_mse // 8 and h.signs_B == m // 8


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
def test_encode_mse_d128(tq, bits, dtype):
    x = torch.randn(1001, 128, generator=torch.Generator().manual_seed(bits)).to(dtype)
    frac, _ = _encode_and_check(tq, x, 128, bits, seed=bits)
    assert frac < 1e-3


@pytest.mark.parametrize("d,bits", [(32, 3), (96, 2), (256, 4), (1536, 2), (1536, 4)])
def test_encode_mse_other_dims(tq, d, bits):
    x = torch.randn(257, d, generator=torch.Generator().manual_seed(d))
    frac, _ = _encode_and_check(tq, x, d, bits, seed=11)
    assert frac < 1e-3


def test_encode_fp16_norms(tq):
    x = torch.randn(700, 128, generator=torch.Generator().manual_seed(4)) * 7
    _encode_and_check(tq, x, 128, 3, seed=4, norm_dtype=tq.TQ_F16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bits,m", [(3, 128), (2, 128), (4, 64), (3, 256)])
def test_encode_prod(tq, dtype, bits, m):
    x = torch.randn(777, 128, generator=torch.Generator().manual_seed(bits + m)).to(dtype)
    frac, sfrac = _encode_and_check(tq, x, 128, bits, seed=2, m=m)
    assert frac < 1e-3 and sfrac < 1e-3


def test_encode_edge_rows(tq):
    """Zero vectors, one-hot rows, huge and tiny scales, n = 1 and n = 65 (ragged tile)."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(65, 128, generator=g)
    x[0] = 0
    x[1] = 0
    x[1, 17] = 3.0
    x[2] *= 1e4
    x[3] *= 1e-4
    _encode_and_check(tq, x, 128, 3, seed=1)
    _encode_and_check(tq, x, 128, 3, seed=1, m=128)
    _encode_and_check(tq, x[:1].clone(), 128, 2, seed=1)
    h = tq.Handle(128, 3, 1)
    out = h.encode(torch.zeros(0, 128, device="cuda"))     # n = 0 is a no-op
    assert out["codes"].shape == (0, 48)


def test_pack_indices_bit_exact(tq):
    for d, bits in [(128, 1), (128, 2), (128, 3), (128, 4), (1536, 2), (32, 3)]:
        h = tq.Handle(d, bits, 0)
        idx = np.random.default_rng(bits).integers(0, 1 << bits, size=(300, d)).astype(np.uint8)
        got = h.pack_indices(torch.from_numpy(idx).cuda()).cpu().numpy()
        assert np.array_equal(got, quant.pack(idx, bits))


def test_config1_encode_full(tq):
    """MSE-only d=128, b=3, 4096 fp32 N(0,1) keys (seed 0): parity and empirical distortion."""
    import workloads as synth
    x = synth.mse_keys()
    frac, _ = _encode_and_check(tq, x, 128, 3, seed=0)
    assert frac < 1e-4


# ---- tensor-core encode (d = 128, bf16 / f16 input, >= 1024 rows): persistent CTAs over
# 128-vector tiles, taken in turn by 4 (MSE) or 2 (prod) epilogue groups. 170,365 rows =
# 1330 full tiles + a ragged tile of 125: on a 148-SM B200 every CTA runs 9 or 10 tiles, so
# every group and every pipeline stage is reused at least twice.

TC_ROWS = 148 * 128 * 9 - 128 * 2 + 125


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_encode_tc_mse(tq, bits, dtype):
    x = torch.randn(TC_ROWS, 128, generator=torch.Generator().manual_seed(40 + bits)).to(dtype)
    frac, _ = _encode_and_check(tq, x, 128, bits, seed=bits)
    assert frac < 1e-4


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_encode_tc_prod(tq, bits, dtype):
    x = torch.randn(TC_ROWS, 128, generator=torch.Generator().manual_seed(50 + bits)).to(dtype)
    frac, sfrac = _encode_and_check(tq, x, 128, bits, seed=2, m=128)
    assert frac < 1e-4 and sfrac < 1e-4


def test_encode_tc_prod_fp32_norms(tq):
    """prod with fp32 norms: the two epilogue groups share one staged x tile (the fp64 norm
    pass reads it), in tile order."""
    x = torch.randn(TC_ROWS, 128, generator=torch.Generator().manual_seed(61)).to(torch.bfloat16)
    frac, sfrac = _encode_and_check(tq, x, 128, 3, seed=3, m=128, norm_dtype=tq.TQ_F32)
    assert frac < 1e-4 and sfrac < 1e-4


def test_encode_tc_edge_rows(tq):
    """Zero, one-hot and extreme-scale rows inside a tensor-core batch, fp32 and fp16 norms."""
    g = torch.Generator().manual_seed(6)
    x = torch.randn(3000, 128, generator=g)
    x[5] = 0
    x[130] = 0
    x[131, 3] = 2.0
    x[1000] *= 1e3
    x[2999] *= 1e-3
    xb = x.to(torch.bfloat16)
    _encode_and_check(tq, xb, 128, 3, seed=1)
    _encode_and_check(tq, xb, 128, 3, seed=1, m=128)
    _encode_and_check(tq, xb, 128, 2, seed=1, m=128, norm_dtype=tq.TQ_F32)
    _encode_and_check(tq, x.to(torch.float16), 128, 4, seed=1, norm_dtype=tq.TQ_F16)
    _encode_and_check(tq, xb, 128, 2, seed=1, norm_dtype=tq.TQ_F16)
    _encode_and_check(tq, x.to(torch.float16), 128, 1, seed=1, m=0)


def test_encode_tc_matches_simt(tq, monkeypatch):
    """The tensor-core and SIMT kernels agree on codes and signs away from decision
    boundaries (both are checked against the oracle above; here against each other)."""
    x = torch.randn(4096 + 61, 128, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16).cuda()
    h = tq.Handle(128, 3, 2, qjl_m=128)
    a = h.encode(x)
    monkeypatch.setenv("TQ_SIMT", "1")
    b = h.encode(x)
    torch.cuda.synchronize()
    same_codes = (a["codes"] == b["codes"]).all(dim=1).float().mean().item()
    same_signs = (a["signs"] == b["signs"]).all(dim=1).float().mean().item()
    assert same_codes > 0.999 and same_signs > 0.999
    # fp16 norms: the tensor-core path takes ||(Pi_hi + Pi_lo) x||, within 1 ulp of ||x||
    ulp = (a["norms"].float() - b["norms"].float()).abs() / torch.finfo(torch.float16).eps / b["norms"].float().abs()
    assert ulp.max().item() <= 1.0


@pytest.mark.parametrize("d,bits,n,dtype", [
    (1536, 2, 3000, torch.float32),    # 6 passes of 256 coordinates, a ragged last tile
    (1536, 4, 1200, torch.bfloat16),   # bf16 input: the x_l contraction is skipped
    (512, 3, 2000, torch.float16),     # 3-bit fields straddle words
    (256, 1, 40000, torch.float32),    # one pass; more tiles than SMs (several per CTA)
    (768, 2, 300, torch.float32),      # a single, partial tile
])
def test_encode_large_d_tensor_core_path(tq, d, bits, n, dtype):
    """The tcgen05 encode of large vectors (MSE, d % 256 = 0): indices within the boundary band of
    the oracle's, norms within an ulp; zero rows and huge / tiny scales included; and the same
    rows as the SIMT kernel (TQ_SIMT=1) outside that band."""
    import os
    g = torch.Generator().manual_seed(d + bits)
    x = torch.randn(n, d, generator=g) * torch.exp(0.5 * torch.randn(n, 1, generator=g))
    x[0] = 0
    x[min(5, n - 1)] *= 1e4
    x[min(9, n - 1)] *= 1e-4
    x = x.to(dtype)
    frac, _ = _encode_and_check(tq, x, d, bits, seed=d)
    print(f"large-d encode d={d} bits={bits} n={n} {dtype}: index mismatch fraction {frac:.2e}")
    assert frac < 1e-3
    h = tq.Handle(d, bits, d)
    fast = h.encode(x.cuda())
    os.environ["TQ_SIMT"] = "1"
    try:
        simt = h.encode(x.cuda())
    finally:
        del os.environ["TQ_SIMT"]
    from gpu_util import unpack_fast
    a = unpack_fast(fast["codes"].cpu().numpy().reshape(n, -1), d, bits)
    b = unpack_fast(simt["codes"].cpu().numpy().reshape(n, -1), d, bits)
    differ = (a != b).mean()
    # the two kernels round y differently by ~1e-7: only coordinates at a decision boundary differ
    assert differ < 1e-4, differ
    assert torch.equal(fast["norms"], simt["norms"]) or torch.allclose(fast["norms"], simt["norms"], rtol=2e-7)
