"""Inner-product scores, decode attention and top-k search on packed codes (oracle side).

* Scores: the inner product is what attention and vector search consume
  ("TurboQuant / PolarQuant / QJL technical deep dive" (gemilab.net), section
  "Key insight: direction decides precision"; "TurboQuant: redefining AI
  efficiency" (hakusoku.com), section "QJL": a full-precision query is
  combined with low-precision data). MSE stage: s = n <Pi q, c[idx]>, which is
  <q, x_hat> rewritten with Pi orthogonal. Prod adds the QJL term of
  :func:`oracle.quant.qjl_estimate` with the stored residual norm. QJL-only
  rows (no MSE bits) score with that term alone, the norm in place of the
  residual norm.
* Decode attention: softmax(q K^T / sqrt(d_k)) V over the cached keys and
  values (gemilab.net, sections "Scaled dot-product attention" and "Why the
  KV cache exists"). Reading taken: grouped-query attention maps query head h
  to KV head floor(h / (Hq / Hkv)); K and V use separate handles (their own
  Pi, S and codebook).
* Search: rank database vectors by the estimated inner product (hakusoku.com,
  section "Impact on high-dimensional vector search"). Reading taken: exact
  top-k by a full sort, equal scores ordered by lower index first.

Everything is fp64. Test infrastructure only; see the package docstring.
"""

import numpy as np

from .quant import QJL_SCALE, dequantize, dequantize_qjl, qjl_estimate


def score_mse(q, idx, n_stored, Pi, centroids):
    """Scores of one query q [d] against rows (idx [L, d], n_stored [L]): n <Pi q, c[idx]>."""
    qr = Pi @ np.asarray(q, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    return np.asarray(n_stored, dtype=np.float64) * (c[idx] @ qr)


def score_prod(q, idx, n_stored, sigma, rnorm_stored, Pi, S, centroids):
    """Prod scores: MSE part plus rnorm sqrt(pi/2)/m <S q, 2 sigma - 1>."""
    q = np.asarray(q, dtype=np.float64)
    m = S.shape[0]
    pm = 2.0 * np.asarray(sigma, dtype=np.float64) - 1.0
    qjl = np.asarray(rnorm_stored, dtype=np.float64) * QJL_SCALE / m * (pm @ (S @ q))
    return score_mse(q, idx, n_stored, Pi, centroids) + qjl


def score_qjl(q, sigma, n_stored, S):
    """QJL-only scores (sign sketch of the whole key plus its norm): n sqrt(pi/2)/m <S q, 2 sigma - 1>
    ("TurboQuant: redefining AI efficiency" (hakusoku.com), section "QJL")."""
    q = np.asarray(q, dtype=np.float64)
    return qjl_estimate(q, np.asarray(S) @ q, sigma, n_stored, np.asarray(S).shape[0])


def _scores(q, kq, b, hk, L):
    """Scores of one query against rows 0 .. L-1 of cache (b, hk): MSE, prod or QJL-only."""
    if "idx" not in kq:
        return score_qjl(q, kq["sigma"][b, hk, :L], kq["n"][b, hk, :L], kq["S"])
    if "sigma" in kq:
        return score_prod(q, kq["idx"][b, hk, :L], kq["n"][b, hk, :L], kq["sigma"][b, hk, :L],
                          kq["rnorm"][b, hk, :L], kq["Pi"], kq["S"], kq["c"])
    return score_mse(q, kq["idx"][b, hk, :L], kq["n"][b, hk, :L], kq["Pi"], kq["c"])


def softmax_attention(q, K, V, scale):
    """Textbook softmax(scale * q K^T) V for one query q [d]; K, V are [L, d] (fp64)."""
    logits = scale * (np.asarray(K, dtype=np.float64) @ np.asarray(q, dtype=np.float64))
    logits = logits - np.max(logits)
    p = np.exp(logits)
    return (p / np.sum(p)) @ np.asarray(V, dtype=np.float64)


def decode_attention(q, kq, vq, lens, scale):
    """GQA decode attention over explicitly dequantized caches (the textbook route).

    q: [B, Hq, d]. kq / vq: dicts describing one quantized cache each, with keys
    ``idx`` [B, Hkv, L, d], ``n`` [B, Hkv, L] (stored norms), ``Pi``, ``c`` and,
    for prod caches, ``sigma`` [B, Hkv, L, m], ``rnorm`` [B, Hkv, L], ``S``. A
    QJL-only cache has no ``idx``: ``sigma``, ``n`` and ``S`` only.
    Returns o [B, Hq, d].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kq["n"].shape[1]
    group = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        L = int(lens[b])
        for hk in range(Hkv):
            K = _dequant_rows(kq, b, hk, L)
            V = _dequant_rows(vq, b, hk, L)
            for g in range(group):
                h = hk * group + g
                out[b, h] = softmax_attention(q[b, h], K, V, scale)
    return out


def _dequant_rows(cq, b, hk, L):
    if "idx" not in cq:
        return dequantize_qjl(cq["sigma"][b, hk, :L], cq["n"][b, hk, :L], cq["S"])
    sig = cq.get("sigma")
    return dequantize(cq["idx"][b, hk, :L], cq["n"][b, hk, :L], cq["Pi"], cq["c"],
                      None if sig is None else sig[b, hk, :L],
                      None if sig is None else cq["rnorm"][b, hk, :L],
                      cq.get("S"))


def decode_attention_streaming(q, kq, vq, lens, scale, chunk=1000):
    """Second route to :func:`decode_attention`, restated in the rotated domain.

    Logits come from the score formulas (no key is dequantized); the context is
    cut into chunks, each with its own max and sum, merged by log-sum-exp; the
    value sum is kept as acc = sum_i p_i n_i c[vidx_i] (rotated domain) plus
    acc_s = sum_i p_i rnorm_i (2 sigma_i - 1) (prod), and mapped back once:
    o = (Pi^T acc + sqrt(pi/2)/m S^T acc_s) / sum_i p_i.
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kq["n"].shape[1]
    group = Hq // Hkv
    out = np.zeros((B, Hq, d))
    v_qjl_only = "idx" not in vq
    cv = None if v_qjl_only else np.asarray(vq["c"], dtype=np.float64)
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            hk = h // group
            s_all = _scores(q[b, h], kq, b, hk, L)
            parts = []
            for lo in range(0, L, chunk):
                hi = min(L, lo + chunk)
                lg = scale * s_all[lo:hi]
                mx = np.max(lg)
                p = np.exp(lg - mx)
                w = p * np.asarray(vq["n"][b, hk, lo:hi], dtype=np.float64)
                acc = np.zeros(d) if v_qjl_only else w @ cv[vq["idx"][b, hk, lo:hi]]
                acc_s = None
                if "sigma" in vq:
                    # QJL-only values: the norm is the projected vector's own norm
                    rn = vq["n"] if v_qjl_only else vq["rnorm"]
                    ws = p * np.asarray(rn[b, hk, lo:hi], dtype=np.float64)
                    acc_s = ws @ (2.0 * np.asarray(vq["sigma"][b, hk, lo:hi], dtype=np.float64) - 1.0)
                parts.append((mx, np.sum(p), acc, acc_s))
            M = max(pt[0] for pt in parts)
            den = sum(pt[1] * np.exp(pt[0] - M) for pt in parts)
            acc = sum(pt[2] * np.exp(pt[0] - M) for pt in parts)
            o = np.zeros(d) if v_qjl_only else vq["Pi"].T @ acc
            if "sigma" in vq:
                acc_s = sum(pt[3] * np.exp(pt[0] - M) for pt in parts)
                m = vq["S"].shape[0]
                o = o + QJL_SCALE / m * (vq["S"].T @ acc_s)
            out[b, h] = o / den
    return out


def topk(scores, k: int):
    """Exact top-k of each row of ``scores`` [nq, n]: (idx int64 [nq, k], score [nq, k]).

    Descending by score; equal scores keep the lower index first.
    """
    scores = np.asarray(scores, dtype=np.float64)
    order = np.argsort(-scores, axis=1, kind="stable")[:, :k]
    return order.astype(np.int64), np.take_along_axis(scores, order, axis=1)


def search_scores(Q, idx, n_stored, Pi, centroids):
    """Estimated inner products of queries Q [nq, d] with a database (idx [n, d], n_stored [n])."""
    Qr = np.asarray(Q, dtype=np.float64) @ Pi.T          # rows are Pi q
    c = np.asarray(centroids, dtype=np.float64)
    return (c[idx] @ Qr.T).T * np.asarray(n_stored, dtype=np.float64)[None, :]
