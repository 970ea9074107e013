"""The arithmetic the int8 tensor-core kernels rely on, pinned on the CPU against the oracle's
codebooks and its LSB-first packer ("Google TurboQuant: 6x KV-cache compression", "Stage 1":
Lloyd-Max codebooks of the coordinate law; the cache layout packs index j at bits
[j b, (j + 1) b) of a vector's little-endian bit stream):

  * a 2-bit Lloyd-Max codebook is symmetric, hence affine in its two index bits:
    c[idx] = c0 + (c1 - c0) b0 + (c2 - c0) b1;
  * a 16-level one has only odd-degree Walsh terms in the +-1 variables of its index bits, so
    c[idx] = c[0] + sum_S w_S beta_S(idx) over the four bits and the four three-bit parities;
  * the word-level extraction of those 0/1 planes from packed code words ((w >> s) & 0x01010101
    and & 0x10101010; for 4-bit nibbles the shifted copies combined by XOR) picks exactly the
    planes of the right coordinates;
  * a value rounded to a 15-bit integer splits exactly into int8 pieces hi * 128 + lo.
"""

import itertools

import numpy as np
import pytest

from oracle import codebook, quant

PLANES4 = [(0,), (1,), (2,), (3,), (0, 1, 2), (0, 1, 3), (0, 2, 3), (1, 2, 3)]


def _bits(idx, k):
    return (idx >> k) & 1


def _beta(idx, plane):
    v = 0
    for k in plane:
        v ^= _bits(idx, k)
    return v


@pytest.mark.parametrize("d", [64, 128, 256, 1536])
def test_two_bit_codebook_is_affine_in_its_index_bits(d):
    c, _ = codebook.lloyd_max(d, 2)
    assert abs(c[3] - c[2] - c[1] + c[0]) <= 1e-15 * np.max(np.abs(c))
    for idx in range(4):
        rec = c[0] + (c[1] - c[0]) * _bits(idx, 0) + (c[2] - c[0]) * _bits(idx, 1)
        assert abs(rec - c[idx]) <= 1e-15 * np.max(np.abs(c))


@pytest.mark.parametrize("d", [64, 128, 256, 1536])
def test_four_bit_codebook_has_only_odd_walsh_terms(d):
    c, _ = codebook.lloyd_max(d, 4)
    cmax = np.max(np.abs(c))
    # Walsh coefficients a_T = 1/16 sum_idx c[idx] prod_{i in T} (2 b_i - 1)
    a = {}
    for T in range(16):
        sgn = [np.prod([2 * _bits(idx, i) - 1 for i in range(4) if T >> i & 1]) for idx in range(16)]
        a[T] = float(np.dot(c, sgn)) / 16.0
        if bin(T).count("1") % 2 == 0:
            assert abs(a[T]) <= 1e-14 * cmax, (T, a[T])
    # the plane form: c[idx] = c[0] + sum_S w_S beta_S(idx), w_S = 2 a_{mask(S)} (from
    # prod (2 b_i - 1) over an odd set = 1 - 2 beta for the four bits and the three-bit parities)
    masks = [sum(1 << i for i in p) for p in PLANES4]
    w = [2.0 * a[m] for m in masks]
    assert abs(a[15]) <= 1e-14 * cmax   # the 4-bit term is even: it vanishes as well
    for idx in range(16):
        rec = c[0] + sum(ws * _beta(idx, p) for ws, p in zip(w, PLANES4))
        assert abs(rec - c[idx]) <= 1e-13 * cmax, (idx, rec, c[idx])


def _plane_words(w, S):
    """The kernels' plane S of every nibble of a 32-bit word (bit 0: low nibble, bit 4: high)."""
    x1, x2, x3 = w >> 1, w >> 2, w >> 3
    return [w, x1, x2, x3, w ^ x1 ^ x2, w ^ x1 ^ x3, w ^ x2 ^ x3, x1 ^ x2 ^ x3][S]


def test_four_bit_plane_extraction_matches_the_packed_layout():
    rs = np.random.default_rng(0)
    idx = rs.integers(0, 16, size=(5, 128))
    words = quant.pack(idx, 4).view("<u4")          # 32 B per vector = 8 words of 8 nibbles
    for v in range(idx.shape[0]):
        for wi, w in enumerate(words[v].tolist()):
            for S, plane in enumerate(PLANES4):
                p = _plane_words(w, S)
                for byte in range(4):
                    coord = 8 * wi + 2 * byte          # byte k of a word holds coordinates 2k (low), 2k + 1
                    lo = (p & (0x01010101)) >> (8 * byte) & 0xFF
                    hi = (p & (0x10101010)) >> (8 * byte) & 0xFF
                    assert lo == _beta(idx[v, coord], plane)
                    assert hi == 16 * _beta(idx[v, coord + 1], plane)


def test_two_bit_plane_extraction_matches_the_packed_layout():
    rs = np.random.default_rng(1)
    idx = rs.integers(0, 4, size=(5, 128))
    words = quant.pack(idx, 2).view("<u4")          # 32 B per vector = 8 words of 16 codes
    for v in range(idx.shape[0]):
        for wi, w in enumerate(words[v].tolist()):
            for s in range(4):
                x = w >> s
                for byte in range(4):
                    # bit s of a byte: code 4 byte-lane + s // 2 of the word's byte, plane s % 2;
                    # bit s + 4: code + 2, same plane
                    code_lo = 16 * wi + 4 * byte + s // 2
                    code_hi = code_lo + 2
                    lo = (x & 0x01010101) >> (8 * byte) & 0xFF
                    hi = (x & 0x10101010) >> (8 * byte) & 0xFF
                    assert lo == _bits(idx[v, code_lo], s % 2)
                    assert hi == 16 * _bits(idx[v, code_hi], s % 2)


def test_fifteen_bit_values_split_exactly_into_int8_pieces():
    # the kernels round a value to xi in [-16256, 16256], then hi = xi / 128 rounded half away
    # from zero and lo = xi - 128 hi
    for xi in range(-16256, 16257):
        hi = (xi + 64) >> 7 if xi >= 0 else -((-xi + 64) >> 7)
        lo = xi - 128 * hi
        assert -127 <= hi <= 127 and -64 <= lo <= 64
        assert 128 * hi + lo == xi


def test_twenty_two_bit_query_values_split_exactly_into_three_int8_pieces():
    # the attention and score kernels round a query value to xi in [-127 * 2^14, 127 * 2^14], then
    # hi = xi / 2^14 and mid = (xi - 2^14 hi) / 2^7, each rounded half away from zero, and
    # lo = xi - 2^14 hi - 2^7 mid; every piece fits an int8 and they rebuild xi exactly
    def split(xi):
        hi = (xi + 8192) >> 14 if xi >= 0 else -((-xi + 8192) >> 14)
        r = xi - hi * 16384
        mid = (r + 64) >> 7 if r >= 0 else -((-r + 64) >> 7)
        return hi, mid, r - 128 * mid
    top = 127 * 16384
    rs = np.random.default_rng(0)
    values = list(range(-20000, 20001)) + [top - k for k in range(20000)] + [-top + k for k in range(20000)]
    values += rs.integers(-top, top + 1, size=50000).tolist()
    for xi in values:
        hi, mid, lo = split(int(xi))
        assert -127 <= hi <= 127 and -64 <= mid <= 64 and -64 <= lo <= 64
        assert hi * 16384 + mid * 128 + lo == xi


def test_sixteen_bit_weights_split_exactly_into_u8_pieces():
    # softmax weights are rounded to w in [0, 65535] and split into hi = w >> 8, lo = w & 255
    for w in range(0, 65536):
        hi, lo = w >> 8, w & 255
        assert 0 <= hi <= 255 and 0 <= lo <= 255 and 256 * hi + lo == w


def test_int32_accumulation_cannot_overflow_at_the_largest_shapes():
    # 3-bit prod attention, key side: 256 code (and 128 sign) positions of |piece| <= 127, the hi
    # sum scaled by 2^14 and added to the mid sum scaled by 2^7 and the lo sum
    assert 256 * 127 * 16384 + 256 * 64 * 128 + 256 * 64 < 2 ** 31
    # value side: 1024 tokens (the largest chunk) of u8 pieces <= 255 times a 0/16 plane value,
    # and the chunk sum of 16-bit weights
    assert 1024 * 255 * 16 < 2 ** 31 and 1024 * 65535 < 2 ** 31
    # the 4-bit kernel's hi sum over 8 planes x 128 coordinates is formed in float (exact below 2^24)
    assert 8 * 128 * 127 < 2 ** 24
    # tcgen05 search at its largest d (65536): acc_hi = sum C_h Q_h and acc_mid = sum (C_h Q_l + C_l Q_h)
    assert 65536 * 127 * 127 < 2 ** 31 and 65536 * (127 * 64 + 64 * 127) < 2 ** 31
    # the x16 family's sums are multiples of 16, so the exact division by 16 loses nothing
    for parts in itertools.product([0, 16, 32, 48], repeat=3):
        assert sum(parts) % 16 == 0


@pytest.mark.parametrize("bits,d", [(1, 128), (2, 128), (2, 1536), (4, 128), (4, 96)])
def test_fast_layout_decoder_of_the_tests_matches_the_oracle_unpack(bits, d):
    from gpu_util import unpack_fast
    rows = np.random.default_rng(bits * 1000 + d).integers(0, 256, size=(300, (d * bits + 7) // 8), dtype=np.uint8)
    assert np.array_equal(unpack_fast(rows, d, bits).astype(np.int64), quant.unpack(rows, d, bits))


def test_search_piece_split_covers_the_15_bit_range():
    """The tcgen05 search rounds centroids and queries to |x| <= 16319 and splits x = 128 h + l
    with h = floor((x + 64) / 128): h and l must fit its int8 operands (|h| <= 127, l in
    [-64, 63]); the dropped l_c l_q term is at most 64 * 64 per coordinate, 1.6e-5 of the
    largest product 16319^2 (max |c| max |q'|)."""
    x = np.arange(-16319, 16320)
    h = np.floor((x + 64) / 128).astype(np.int64)
    assert np.array_equal((x + 64) >> 7, h)   # the kernel's arithmetic shift
    l = x - 128 * h
    assert h.min() == -127 and h.max() == 127 and l.min() == -64 and l.max() == 63
    assert np.array_equal(128 * h + l, x)
    assert 64 * 64 / 16319 ** 2 < 1.6e-5
