"""PolarQuant's recursive polar transform and its angle codebooks (oracle side).

"PolarQuant explainer" (aibr.jp), sections 1 and 3, and "TurboQuant: redefining AI efficiency"
(hakusoku.com), section "PolarQuant": a random preconditioning makes the angles of the polar
representation concentrate; the vector is turned into polar coordinates by a recursive
algorithm, its angles are quantized with codebooks designed from the angles' analytic
distribution (no per-block normalisation), and the reconstruction is used for inner products.

Readings taken (the pages print no formulas; this is the plainest reading, listed in DESIGN):

* Recursion (d a power of two, log2 d levels). Level 1 pairs coordinates (x_2i, x_2i+1) into
  a radius r = hypot(x_2i, x_2i+1) and an angle theta = atan2(x_2i+1, x_2i) in (-pi, pi].
  Level l >= 2 pairs the radii of level l-1 the same way, giving angles psi in [0, pi/2]
  (both radii are non-negative). The last level leaves one radius, ||x||.
* Preconditioning: the random rotation of the MSE path, y = Pi x / ||x||, so y is uniform on
  the unit sphere; the norm is kept per vector, as the TurboQuant path keeps it.
* Angle laws (exact for a uniform direction, because polar angles do not depend on the
  scale and a uniform direction is a normalised Gaussian vector): level-1 angles are uniform
  on (-pi, pi]; a level-l angle splits two blocks of k = 2^(l-1) coordinates, and
  sin^2(psi) = R_b^2 / (R_a^2 + R_b^2) ~ Beta(k/2, k/2), i.e. density
  f(psi) = 2 / B(k/2, k/2) (sin psi cos psi)^(k-1) on [0, pi/2]. All angles are independent.
* Codebooks: Lloyd-Max (continuous k-means) on each level's law with a bit width per level
  given by the caller; level 1 is the uniform law, so its codebook is the uniform grid.
  Indices ascending; boundaries are midpoints; an angle equal to a boundary goes to the
  lower cell.
* Reconstruction: the quantized angles (centroids) through the inverse recursion with a unit
  top radius, then x_hat = ||x|| Pi^T y_hat.

Test infrastructure only; see the package docstring.
"""

import functools

import numpy as np
from scipy import integrate, special


def n_levels(d: int) -> int:
    if d < 2 or d & (d - 1):
        raise ValueError(f"d = {d}: the pairwise recursion needs a power of two >= 2")
    return d.bit_length() - 1


def transform(x):
    """Rows [n, d] -> (angles: list over levels of [n, d / 2^l] arrays, radius [n])."""
    r = np.asarray(x, dtype=np.float64)
    angles = []
    for _ in range(n_levels(r.shape[1])):
        a, b = r[:, 0::2], r[:, 1::2]
        angles.append(np.arctan2(b, a))
        r = np.hypot(a, b)
    return angles, r[:, 0]


def inverse(angles, radius):
    """Inverse of `transform`: from the top radius down through the levels."""
    r = np.asarray(radius, dtype=np.float64)[:, None]
    for ang in reversed(angles):
        out = np.empty((r.shape[0], 2 * r.shape[1]))
        out[:, 0::2] = r * np.cos(ang)
        out[:, 1::2] = r * np.sin(ang)
        r = out
    return r


# ---------------------------------------------------------------- angle laws

def _k(level: int) -> int:
    return 1 << (level - 1)


def cdf(p, level: int):
    """P(angle <= p) at `level` for a uniform direction."""
    p = np.asarray(p, dtype=np.float64)
    if level == 1:
        return np.clip((p + np.pi) / (2 * np.pi), 0.0, 1.0)
    k = _k(level)
    s = np.sin(np.clip(p, 0.0, np.pi / 2)) ** 2
    return special.betainc(k / 2, k / 2, s)


def pdf(p, level: int):
    p = np.asarray(p, dtype=np.float64)
    if level == 1:
        return np.where((p > -np.pi) & (p <= np.pi), 1.0 / (2 * np.pi), 0.0)
    k = _k(level)
    inside = (p >= 0) & (p <= np.pi / 2)
    sc = np.sin(np.clip(p, 0, np.pi / 2)) * np.cos(np.clip(p, 0, np.pi / 2))
    return np.where(inside, 2.0 / special.beta(k / 2, k / 2) * sc ** (k - 1), 0.0)


def support(level: int):
    return (-np.pi, np.pi) if level == 1 else (0.0, np.pi / 2)


def _cell_mass(lo, hi, level):
    return cdf(hi, level) - cdf(lo, level)


@functools.lru_cache(maxsize=None)
def _moment_table(level: int, n: int = 2_000_001):
    """psi and int_0^psi t f(t) dt on a uniform grid of [0, pi/2] (cumulative trapezoid rule;
    the integrand is smooth, so the error is about h^2 = 6e-13 relative)."""
    grid = np.linspace(0.0, np.pi / 2, n)
    return grid, integrate.cumulative_trapezoid(grid * pdf(grid, level), grid, initial=0.0)


def _cell_moment(lo, hi, level):
    """E[angle ; lo < angle <= hi]."""
    if level == 1:
        return (hi * hi - lo * lo) / (4 * np.pi)
    grid, m = _moment_table(level)
    return np.interp(hi, grid, m) - np.interp(lo, grid, m)


def lloyd_max(level: int, bits: int, tol: float = 1e-13, max_iter: int = 20_000):
    """(centroids [2^bits], boundaries [2^bits - 1]) of the level's angle law, fp64, ascending."""
    L = 1 << bits
    lo, hi = support(level)
    if level == 1:
        # the uniform law: the fixed point of the Lloyd iteration is the uniform grid
        edges = lo + (hi - lo) * np.arange(L + 1) / L
        return 0.5 * (edges[:-1] + edges[1:]), edges[1:-1]
    q = (np.arange(L) + 0.5) / L
    k = _k(level)
    c = np.arcsin(np.sqrt(special.betaincinv(k / 2, k / 2, q)))   # start: the law's quantiles
    for _ in range(max_iter):
        beta = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([lo], beta, [hi]))
        new = _cell_moment(edges[:-1], edges[1:], level) / _cell_mass(edges[:-1], edges[1:], level)
        step = np.max(np.abs(new - c))
        c = new
        if step < tol:
            break
    c = 0.5 * (c + (np.pi / 2 - c[::-1]))   # the law is symmetric about pi/4
    return c, 0.5 * (c[:-1] + c[1:])


def quantize(angles, boundaries):
    """Index of each angle's cell: #{i : beta_i < angle}."""
    return np.searchsorted(np.asarray(boundaries), np.asarray(angles), side="left").astype(np.int64)


# ---------------------------------------------------------------- encode / decode

def codebooks(d: int, bits):
    """Per-level (centroids, boundaries); bits[l-1] is level l's width (a single int: all levels)."""
    nl = n_levels(d)
    bits = [bits] * nl if np.isscalar(bits) else list(bits)
    if len(bits) != nl:
        raise ValueError(f"{len(bits)} bit widths for {nl} levels")
    return [lloyd_max(lv, b) for lv, b in zip(range(1, nl + 1), bits)]


def encode(x, Pi, books):
    """x [n, d] -> dict(idx: per-level index arrays, n_exact: ||x||, y: rotated unit rows)."""
    x = np.asarray(x, dtype=np.float64)
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    y = (x / safe[:, None]) @ np.asarray(Pi).T
    angles, _ = transform(y)
    idx = [quantize(a, b) for a, (_, b) in zip(angles, books)]
    return {"idx": idx, "n_exact": n, "y": y, "angles": angles}


def decode(idx, n, Pi, books):
    """x_hat = ||x|| Pi^T inverse(centroids[idx], 1)."""
    ang = [c[i] for i, (c, _) in zip(idx, books)]
    y_hat = inverse(ang, np.ones(len(n)))
    return np.asarray(n, dtype=np.float64)[:, None] * (y_hat @ np.asarray(Pi))


def score(q, idx, n, Pi, books):
    """<q, x_hat> for each encoded row without reconstructing it: with q' = Pi q, pair i of level 1
    contributes S_i = q'_2i cos(theta_i) + q'_2i+1 sin(theta_i) per unit radius, and each further
    level folds two partial scores as S = S_a cos(psi) + S_b sin(psi); the score is ||x|| times the
    top value. q [d], idx per-level index arrays [n, d / 2^l]."""
    qp = np.asarray(Pi) @ np.asarray(q, dtype=np.float64)
    c0 = books[0][0][idx[0]]
    s = qp[0::2][None, :] * np.cos(c0) + qp[1::2][None, :] * np.sin(c0)
    for lv in range(1, len(idx)):
        psi = books[lv][0][idx[lv]]
        s = s[:, 0::2] * np.cos(psi) + s[:, 1::2] * np.sin(psi)
    return np.asarray(n, dtype=np.float64) * s[:, 0]


def bits_per_vector(d: int, bits) -> int:
    nl = n_levels(d)
    bits = [bits] * nl if np.isscalar(bits) else list(bits)
    return sum((d >> lv) * b for lv, b in zip(range(1, nl + 1), bits))


# ---------------------------------------------------------------- packed layout

def row_bytes(d: int, bits) -> int:
    """Bytes of one packed row: the level fields concatenated, rounded up to 16 bytes."""
    return 16 * ((bits_per_vector(d, bits) + 127) // 128)


def pack(idx, d: int, bits) -> np.ndarray:
    """Packs per-level indices (list over levels of [n, d / 2^l]) into rows of row_bytes(d, bits).

    Reading taken (the pages give no bit layout): level 1's indices first, then level 2's, and
    so on; inside the row's little-endian bitstream every index occupies its level's width,
    least significant bit first, one after the other with no gaps; the pad bits up to the
    16-byte row boundary are zero. This pair of functions is the only place the oracle states
    the layout.
    """
    nl = n_levels(d)
    bits = [bits] * nl if np.isscalar(bits) else list(bits)
    n = np.asarray(idx[0]).shape[0]
    streams = []
    for lv in range(nl):
        a = np.asarray(idx[lv], dtype=np.uint64)
        planes = (a[:, :, None] >> np.arange(bits[lv], dtype=np.uint64)) & np.uint64(1)
        streams.append(planes.reshape(n, -1).astype(np.uint8))
    stream = np.concatenate(streams, axis=1)
    out = np.zeros((n, row_bytes(d, bits)), dtype=np.uint8)
    packed = np.packbits(stream, axis=1, bitorder="little")
    out[:, :packed.shape[1]] = packed
    return out


def unpack(codes, d: int, bits):
    """Inverse of :func:`pack`: rows -> list over levels of [n, d / 2^l] int64 indices."""
    nl = n_levels(d)
    bits = [bits] * nl if np.isscalar(bits) else list(bits)
    codes = np.asarray(codes, dtype=np.uint8)
    stream = np.unpackbits(codes, axis=1, bitorder="little").astype(np.int64)
    out, pos = [], 0
    for lv in range(nl):
        cnt, b = d >> (lv + 1), bits[lv]
        f = stream[:, pos:pos + cnt * b].reshape(-1, cnt, b)
        out.append(np.sum(f << np.arange(b, dtype=np.int64), axis=2))
        pos += cnt * b
    return out
