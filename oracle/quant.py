"""Encode, bit-pack, QJL sign sketch and dequantize (oracle side).

Steps, in the order the pages give them:

1. Norm / direction split v = r u, r = ||v|| kept per vector, u = v / r
   ("TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net),
   section "PolarQuant: Cartesian to polar"; "TurboQuant: redefining AI
   efficiency" (hakusoku.com), reader comment on the radius: one scalar per
   vector, left unquantized).
2. Rotate, y = Pi u, and map every coordinate to its Lloyd-Max cell
   ("Google TurboQuant: 6x KV-cache compression" (ebisuda.net), section
   "Stage 1: PolarQuant"); no per-block scale or zero point is stored.
3. Pack the b-bit indices (the deep-dive page's "memory-layout optimisation").
4. Optional 1-bit QJL stage on the residual: project with a Gaussian matrix and
   keep only the sign of each projection, plus the residual norm (ebisuda.net
   section "Stage 2: QJL residual correction"; gemilab.net section "QJL";
   hakusoku.com section "QJL").

Readings taken where the pages are silent:

* Norm: n = ||x||_2 in fp64; it is stored rounded (round-to-nearest-even) to
  the handle's dtype (fp32 or fp16), but quantisation uses the exact n.
* Index: idx_j = #{i : beta_i < y_j}; a coordinate equal to a boundary goes to
  the lower cell. A zero vector has y = 0, so idx = 2^(b-1) - 1 everywhere.
* Reconstruction: x_hat = n Pi^T c[idx], no renormalisation.
* Prod (b total bits): b-1 bits for the MSE stage; residual r = x - x_hat in
  the original domain with the exact n; z = S r; sign bit sigma_j = 1 iff
  z_j >= 0 (sign(0) = +1); rnorm = ||r|| stored as fp16.
* Bit layout (LSB-first contiguous): bit t of idx_j sits at bit j*b + t of the
  vector's little-endian bitstream; rows are ceil(d*b/8) bytes, pad bits 0.
  Signs use the same rule with b = 1. This function pair is the only place the
  oracle states the layout.

Test infrastructure only; see the package docstring.
"""

import numpy as np

_DTYPES = {"f32": np.float32, "f16": np.float16}


def pack(idx, bits: int) -> np.ndarray:
    """Packs indices [n, d] (each < 2^bits) into bytes [n, ceil(d*bits/8)], LSB-first."""
    idx = np.asarray(idx, dtype=np.uint64)
    n, d = idx.shape
    planes = (idx[:, :, None] >> np.arange(bits, dtype=np.uint64)) & np.uint64(1)
    bitstream = planes.reshape(n, d * bits).astype(np.uint8)
    return np.packbits(bitstream, axis=1, bitorder="little")


def unpack(codes, d: int, bits: int) -> np.ndarray:
    """Inverse of :func:`pack`: bytes [n, B] -> indices [n, d] (int64)."""
    codes = np.asarray(codes, dtype=np.uint8)
    n = codes.shape[0]
    bitstream = np.unpackbits(codes, axis=1, bitorder="little")[:, : d * bits]
    planes = bitstream.reshape(n, d, bits).astype(np.int64)
    return np.sum(planes << np.arange(bits, dtype=np.int64), axis=2)


def norms(x) -> np.ndarray:
    """Exact (fp64) Euclidean norm of each row."""
    x = np.asarray(x, dtype=np.float64)
    return np.sqrt(np.sum(x * x, axis=1))


def rotate(x, Pi):
    """Returns (n, y): fp64 norms and rotated unit directions y = Pi u (rows)."""
    x = np.asarray(x, dtype=np.float64)
    n = norms(x)
    safe = np.where(n > 0, n, 1.0)
    u = np.where(n[:, None] > 0, x / safe[:, None], 0.0)
    return n, u @ Pi.T


def bucketize(y, boundaries) -> np.ndarray:
    """idx = #{i : beta_i < y}; ties go to the lower cell."""
    return np.searchsorted(np.asarray(boundaries, dtype=np.float64), y, side="left").astype(np.int64)


def encode_mse(x, Pi, centroids, boundaries, norm_dtype="f32"):
    """MSE stage. Returns dict(idx, n_exact, n_stored, y)."""
    n, y = rotate(x, Pi)
    idx = bucketize(y, boundaries)
    return {"idx": idx, "n_exact": n, "n_stored": n.astype(_DTYPES[norm_dtype]), "y": y}


def reconstruct_mse(idx, n, Pi, centroids):
    """x_hat = n * Pi^T c[idx] for each row (n: fp64 per row)."""
    c = np.asarray(centroids, dtype=np.float64)
    return np.asarray(n, dtype=np.float64)[:, None] * (c[idx] @ Pi)


def encode_prod(x, Pi, S, centroids, boundaries, norm_dtype="f16"):
    """MSE stage with b-1 bits plus the 1-bit QJL sketch of the residual.

    Returns dict(idx, sigma, z, n_exact, n_stored, r_exact, rnorm_stored, y).
    """
    x64 = np.asarray(x, dtype=np.float64)
    e = encode_mse(x64, Pi, centroids, boundaries, norm_dtype)
    x_hat = reconstruct_mse(e["idx"], e["n_exact"], Pi, centroids)
    r = x64 - x_hat
    z = r @ S.T
    sigma = (z >= 0).astype(np.int64)
    rn = norms(r)
    e.update({"sigma": sigma, "z": z, "r_exact": rn, "rnorm_stored": rn.astype(np.float16)})
    return e


QJL_SCALE = np.sqrt(np.pi / 2.0)


def qjl_estimate(q, Sq, sigma, rnorm, m: int):
    """QJL inner-product term  rnorm * sqrt(pi/2)/m * <S q, 2 sigma - 1>  for each row.

    The query stays in full precision while the data side is one sign bit per
    projection ("TurboQuant: redefining AI efficiency" (hakusoku.com), section
    "QJL"); the constant makes the estimate unbiased: for s ~ N(0, I),
    E[<s, q> sign(<s, r>)] = sqrt(2/pi) <q, r> / ||r||.
    """
    pm = 2.0 * np.asarray(sigma, dtype=np.float64) - 1.0
    return np.asarray(rnorm, dtype=np.float64) * QJL_SCALE / m * (pm @ np.asarray(Sq, dtype=np.float64))


def dequantize(idx, n, Pi, centroids, sigma=None, rnorm=None, S=None):
    """Vector estimate: x_hat (MSE) or x_tilde = x_hat + rnorm sqrt(pi/2)/m S^T (2 sigma - 1) (prod).

    Reading taken for the prod decode: the deep-dive page says the decoder
    approximately restores the residual from its 1-bit projection; the plainest
    unbiased restoration is the QJL back-projection above (E_S[x_tilde] = x).
    """
    xh = reconstruct_mse(idx, n, Pi, centroids)
    if sigma is None:
        return xh
    m = S.shape[0]
    pm = 2.0 * np.asarray(sigma, dtype=np.float64) - 1.0
    return xh + (np.asarray(rnorm, dtype=np.float64) * QJL_SCALE / m)[:, None] * (pm @ S)


def encode_qjl(x, S, norm_dtype="f16"):
    """QJL-only encode: one sign bit per Gaussian projection of the whole vector, plus its norm.

    "TurboQuant: redefining AI efficiency" (hakusoku.com), section "QJL: zero-overhead
    1-bit compression": a random Johnson-Lindenstrauss projection keeps only each
    coordinate's sign, with no per-block constants; "TurboQuant / PolarQuant / QJL
    technical deep dive" (gemilab.net), section "QJL".

    Readings taken: the sketch is the prod stage with no MSE bits, i.e. the residual of a
    zero reconstruction, r = x; sigma_j = 1 iff (S x)_j >= 0 (sign(0) = +1, so a zero
    vector has every bit set); the one stored scalar is ||x|| in the handle's norm dtype,
    which plays the role of the residual norm in the estimator. Returns dict(sigma, z,
    n_exact, n_stored).
    """
    x = np.asarray(x, dtype=np.float64)
    z = x @ np.asarray(S, dtype=np.float64).T
    n = norms(x)
    return {"sigma": (z >= 0).astype(np.int64), "z": z, "n_exact": n, "n_stored": n.astype(_DTYPES[norm_dtype])}


def dequantize_qjl(sigma, n, S):
    """Vector estimate of a QJL-only row: x_tilde = n sqrt(pi/2)/m S^T (2 sigma - 1) (unbiased over S)."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    pm = 2.0 * np.asarray(sigma, dtype=np.float64) - 1.0
    return (np.asarray(n, dtype=np.float64) * QJL_SCALE / m)[:, None] * (pm @ S)
