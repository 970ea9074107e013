"""Random orthogonal rotation Pi and QJL projection matrix S (oracle side).

"Google TurboQuant: 6x KV-cache compression" (ebisuda.net), section
"Stage 1: PolarQuant (MSE-optimal compression)": every input vector is
rotated by a random orthogonal matrix obtained from the QR decomposition of a
Gaussian matrix, after which each coordinate follows a known Beta-type law.
"TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net), section
"QJL": the residual is projected by a random Gaussian matrix A (k x d).

Readings taken where the pages are silent:

* G (d x d) is filled row-major with the first d*d values of the Gaussian
  stream of :mod:`oracle.rng`; S (m x d) continues the same stream, row-major.
* QR is unique only up to the signs of Q's columns; the sign is fixed so that
  diag(R) > 0, which makes Pi := Q Haar distributed. The rotated vector is
  y = Pi u.

Test infrastructure only; see the package docstring.
"""

import numpy as np

from .rng import gaussians


def rotation(d: int, seed: int, m: int = 0):
    """Returns (Pi, S) in fp64: Pi is d x d orthogonal, S is m x d Gaussian (None if m == 0)."""
    g = gaussians(seed, d * d + m * d)
    G = g[: d * d].reshape(d, d)
    Q, R = np.linalg.qr(G)
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    Pi = Q * s[None, :]          # scale column j by sign(R_jj)  ->  diag(R') > 0
    S = g[d * d:].reshape(m, d) if m > 0 else None
    return Pi, S
