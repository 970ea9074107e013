"""Seeded random stream for the rotation and the QJL matrix (oracle side).

The pages only say that the rotation is the orthogonal factor of a QR
decomposition of a Gaussian matrix ("Google TurboQuant: 6x KV-cache
compression", section "Stage 1: PolarQuant") and that QJL projects with a
random matrix ("TurboQuant / PolarQuant / QJL technical deep dive", section
"QJL"). They name no generator. Reading taken (so that the library and this
oracle can each derive the same matrices from a seed without sharing code):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): state starts at ``seed``; each draw adds the
  golden-ratio increment and returns the variant-13 mix of the new state.
* a uniform in [0, 1) is the top 53 bits of a draw times 2**-53;
* Box-Muller (1958) turns two consecutive uniforms (a, b) into two N(0,1)
  values with u1 = 1 - a in (0, 1] and u2 = b: r = sqrt(-2 ln u1),
  g0 = r cos(2 pi u2), g1 = r sin(2 pi u2), emitted in that order.

Test infrastructure only; see the package docstring.
"""

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, count: int, start: int = 0) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the SplitMix64 stream seeded with ``seed``.

    The generator is counter based: draw i (0-based) mixes ``seed + (i+1)*golden``
    (mod 2**64), so a slice of the stream is computed without running the prefix.
    """
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        z = z ^ (z >> np.uint64(31))
    return z


def uniforms(seed: int, count: int, start: int = 0) -> np.ndarray:
    """Uniforms in [0, 1) from the top 53 bits of each draw."""
    return (splitmix64(seed, count, start) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def gaussians(seed: int, count: int) -> np.ndarray:
    """The first ``count`` standard normals of the Box-Muller stream for ``seed``.

    Pairs are formed from draws (2p, 2p+1); both outputs of a pair are used,
    cosine first. If ``count`` is odd the last sine output is dropped.
    """
    pairs = (count + 1) // 2
    u = uniforms(seed, 2 * pairs)
    u1 = 1.0 - u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    return out[:count]
