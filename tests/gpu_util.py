"""Helpers for the GPU parity tests: oracle-side expectations and the tolerance rules.

Expected values always come from the oracle on the seeded inputs (never from
the CUDA path). GPU outputs are decoded here with plain bit arithmetic and
compared against those expectations:

* indices: a GPU index may differ from the oracle's only by one cell, and only
  where the oracle's rotated coordinate lies within 1e-5 of the boundary
  between the two cells (the fraction is returned);
* packed bytes: bit-exact except inside the fields of such exempt coordinates;
* norms: within 1 ulp of the stored dtype;
* signs: a mismatch only where |z_oracle| < 1e-5 * ||x|| (vectors with an index
  mismatch excluded);
* scores: |s - s_ref| <= 1e-3 (|s_ref| + ||q|| ||x|| / sqrt(d));
* attention: ||o - o_ref|| <= 1e-3 ||o_ref|| per (sequence, query head).
"""

import numpy as np
import torch

from oracle import codebook, quant, rotation

BOUNDARY_BAND = 1e-5
SCORE_RTOL = 1e-3
ATTN_RTOL = 1e-3


class OracleHandle:
    """The oracle's own Pi, S and codebook for (d, bits, seed, m); bits = MSE bits."""

    def __init__(self, d, bits_mse, seed, m=0):
        self.d, self.bits, self.m, self.seed = d, bits_mse, m, seed
        self.Pi, self.S = rotation.rotation(d, seed, m)
        self.c, self.beta = codebook.lloyd_max(d, bits_mse)

    def encode(self, x, norm_dtype):
        x = np.asarray(x, dtype=np.float64).reshape(-1, self.d)
        if self.m:
            return quant.encode_prod(x, self.Pi, self.S, self.c, self.beta, norm_dtype)
        return quant.encode_mse(x, self.Pi, self.c, self.beta, norm_dtype)


def to_np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def unpack_bits(codes, d, bits):
    """GPU bytes [n, B] -> indices [n, d] (LSB-first contiguous layout, decoded in the test)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n = codes.shape[0]
    bitstream = np.unpackbits(codes, axis=1, bitorder="little")[:, : d * bits].reshape(n, d, bits)
    return (bitstream.astype(np.int64) << np.arange(bits)).sum(axis=2)


def check_codes(gpu_codes, exp, oh):
    """Checks GPU code bytes against the oracle encode `exp`; returns (gpu_idx, bad_rows, fraction)."""
    gpu_codes = np.asarray(gpu_codes, dtype=np.uint8).reshape(-1, gpu_codes.shape[-1])
    n, d, b = gpu_codes.shape[0], oh.d, oh.bits
    gidx = unpack_bits(gpu_codes, d, b)
    eidx = exp["idx"]
    mism = gidx != eidx
    frac = float(mism.mean())
    if mism.any():
        r, j = np.nonzero(mism)
        g, e = gidx[r, j], eidx[r, j]
        assert np.all(np.abs(g - e) == 1), "index differs by more than one cell"
        beta = oh.beta[np.minimum(g, e)]
        dist = np.abs(exp["y"][r, j] - beta)
        assert np.all(dist < BOUNDARY_BAND), f"index mismatch {dist.max():.3g} away from a boundary"
    # bytes: bit-exact outside exempt fields (pad bits included)
    want = quant.pack(eidx, b)
    assert want.shape == gpu_codes.shape
    diff = np.unpackbits(want ^ gpu_codes, axis=1, bitorder="little")
    rr, pos = np.nonzero(diff)
    if len(rr):
        jj = pos // b
        assert np.all(jj < d), "pad bits differ"
        assert np.all(mism[rr, jj]), "packed bits differ outside an exempt index"
    return gidx, np.unique(np.nonzero(mism)[0]), frac


def check_norms(gpu_norms, exp_stored):
    g = np.asarray(gpu_norms).reshape(-1)
    e = np.asarray(exp_stored).reshape(-1)
    assert g.dtype == e.dtype
    both_inf = np.isinf(e) & (g == e)          # a norm above the fp16 range saturates on both sides
    g, e = g[~both_inf], e[~both_inf]
    ulp = np.spacing(np.abs(e)).astype(np.float64)
    err = np.abs(g.astype(np.float64) - e.astype(np.float64))
    assert np.all(err <= ulp * (1 + 1e-6)), f"norm off by {np.max(err / np.maximum(ulp, 1e-300)):.2f} ulp"


def check_signs(gpu_signs, exp, bad_rows):
    m = exp["z"].shape[1]
    gs = np.unpackbits(np.asarray(gpu_signs, dtype=np.uint8).reshape(len(exp["z"]), -1), axis=1,
                       bitorder="little")[:, :m].astype(np.int64)
    mism = gs != exp["sigma"]
    if len(bad_rows):
        mism[bad_rows] = False
    frac = float(mism.mean())
    if mism.any():
        r, j = np.nonzero(mism)
        band = BOUNDARY_BAND * exp["n_exact"][r]
        assert np.all(np.abs(exp["z"][r, j]) < band), "sign mismatch away from zero"
    return frac


def score_tolerance(s_ref, qnorm, n, d):
    return SCORE_RTOL * (np.abs(s_ref) + qnorm * np.abs(n) / np.sqrt(d))


def max_rel_score_error(got, ref, qnorm, n, d):
    """Largest purely relative score error |s - s_ref| / |s_ref| over the scores above the
    tolerance floor (|s_ref| >= ||q|| ||x|| / sqrt(d), the size of a typical inner product);
    reported by the tests next to the pass/fail rule of score_tolerance."""
    ref = np.asarray(ref, dtype=np.float64)
    floor = qnorm * np.abs(np.asarray(n, dtype=np.float64)) / np.sqrt(d)
    sel = np.abs(ref) >= floor
    if not np.any(sel):
        return 0.0
    return float(np.max(np.abs(np.asarray(got, dtype=np.float64)[sel] - ref[sel]) / np.abs(ref[sel])))


def unpack_fast(codes, d, bits):
    """The LSB-first layout decoded with byte shifts for widths that divide 8 (1, 2, 4):
    index j sits in byte (j*b) // 8 at bit (j*b) % 8. Same result as oracle.quant.unpack
    (checked on the CPU), fast enough for million-row tables; other widths use unpack."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    if bits not in (1, 2, 4):
        return quant.unpack(codes, d, bits)
    per = 8 // bits
    shifts = (np.arange(per, dtype=np.uint8) * bits)
    lead = codes.shape[:-1]
    out = (codes[..., None] >> shifts) & np.uint8((1 << bits) - 1)
    return out.reshape(lead + (codes.shape[-1] * per,))[..., :d]
