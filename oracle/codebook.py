"""Lloyd-Max scalar codebook for one rotated unit-vector coordinate (oracle side).

"Google TurboQuant: 6x KV-cache compression" (ebisuda.net), section
"Stage 1: PolarQuant (MSE-optimal compression)": after the random rotation
each coordinate of a unit vector follows a known (Beta) law, close to an
independent N(0, 1/d) in high dimension; because the law is known, an optimal
Lloyd-Max quantizer is applied to each coordinate separately. Lloyd-Max solves
the continuous k-means problem: for a given bit width (e.g. 3 bits = 8 levels)
it finds the bucket boundaries and centroids that minimise the MSE. The
codebook is precomputed per bit width and does not depend on the data.

Readings taken:

* The law is the exact marginal of one coordinate of a uniform point on
  S^(d-1): density f(t) proportional to (1 - t^2)^((d-3)/2) on [-1, 1], i.e.
  (t+1)/2 ~ Beta((d-1)/2, (d-1)/2). The pages do not print the Beta
  parameters; this is the law they describe.
* Lloyd iteration: boundaries are midpoints of adjacent centroids; each
  centroid is the conditional mean of its cell. Cell masses use the
  regularised incomplete Beta function (a library routine); cell first moments
  use the closed form  int_a^b t (1-t^2)^k dt = [(1-a^2)^(k+1) - (1-b^2)^(k+1)] / (2(k+1)).
* Start: the quantiles of f at (i + 1/2) / 2^b. Stop when no centroid moves by
  1e-15 or after 1e5 iterations; then make the codebook exactly odd
  (c_i = -c_{L-1-i}).
* Indices are ascending: c_0 < c_1 < ... < c_{L-1}; boundaries
  beta_i = (c_i + c_{i+1}) / 2, i = 0 .. L-2.

Test infrastructure only; see the package docstring.
"""

import numpy as np
from scipy import special


def _alpha(d: int) -> float:
    return (d - 1) / 2.0


def cdf(t, d: int):
    """P(T <= t) for one coordinate of a uniform unit vector in R^d."""
    a = _alpha(d)
    x = (np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0) + 1.0) / 2.0
    return special.betainc(a, a, x)


def _sf(t, d: int):
    a = _alpha(d)
    x = (np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0) + 1.0) / 2.0
    return special.betaincc(a, a, x)


def cell_mass(lo, hi, d: int):
    """P(lo < T <= hi); the upper tail is taken from the complement for accuracy."""
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    upper = lo >= 0
    return np.where(upper, _sf(lo, d) - _sf(hi, d), cdf(hi, d) - cdf(lo, d))


def cell_moment(lo, hi, d: int):
    """E[T ; lo < T <= hi] from the closed form of int t (1-t^2)^k dt, k = (d-3)/2."""
    k1 = (d - 1) / 2.0                      # k + 1
    log_z = special.betaln(0.5, k1)         # int_{-1}^{1} (1-t^2)^k dt = B(1/2, k+1)

    def g(t):
        t = np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0)
        with np.errstate(divide="ignore"):
            return np.exp(k1 * np.log1p(-t * t) - log_z)

    return (g(lo) - g(hi)) / (2.0 * k1)


def lloyd_max(d: int, bits: int, tol: float = 1e-15, max_iter: int = 100_000):
    """Returns (centroids[2^bits], boundaries[2^bits - 1]) in fp64, ascending."""
    if d < 3:
        raise ValueError("the coordinate law needs d >= 3")
    L = 1 << bits
    a = _alpha(d)
    q = (np.arange(L) + 0.5) / L
    c = 2.0 * special.betaincinv(a, a, q) - 1.0
    for _ in range(max_iter):
        beta = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-1.0], beta, [1.0]))
        mass = cell_mass(edges[:-1], edges[1:], d)
        new = cell_moment(edges[:-1], edges[1:], d) / mass
        step = np.max(np.abs(new - c))
        c = new
        if step < tol:
            break
    c = 0.5 * (c - c[::-1])
    beta = 0.5 * (c[:-1] + c[1:])
    return c, beta


def mse(d: int, centroids, boundaries=None) -> float:
    """Per-coordinate E[(T - c(T))^2] with nearest-centroid cells.

    Uses sum_i int_cell (t - c_i)^2 f = E[T^2] - sum_i (2 c_i m1_i - c_i^2 p_i),
    E[T^2] = 1/d, which holds for any codebook whose cells partition [-1, 1].
    """
    c = np.asarray(centroids, dtype=np.float64)
    if boundaries is None:
        boundaries = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate(([-1.0], np.asarray(boundaries, dtype=np.float64), [1.0]))
    p = cell_mass(edges[:-1], edges[1:], d)
    m1 = cell_moment(edges[:-1], edges[1:], d)
    return 1.0 / d - float(np.sum(2.0 * c * m1 - c * c * p))
