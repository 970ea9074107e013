"""Seeded synthetic inputs for the five workloads (shared by the tests, the bench and the oracle checks).

This module draws inputs only; it holds none of the method's arithmetic.
Every tensor comes from ``torch.Generator('cpu').manual_seed(seed)`` so the
GPU path and the CPU oracle see bit-identical inputs. The pages evaluate on
LLM KV caches and vector-search benchmarks that are not available here; these
recipes stand in for them with the shapes and value laws stated per function.
"""

import torch


def _gen(seed):
    return torch.Generator(device="cpu").manual_seed(int(seed))


def mse_keys(n=4096, d=128, seed=0, dtype=torch.float32):
    """Keys i.i.d. N(0, 1), [n, d] (MSE-only d=128, b=3 workload: n=4096, seed 0)."""
    return torch.randn(n, d, generator=_gen(seed)).to(dtype)


def queries(shape, seed):
    """Queries i.i.d. N(0, 1), fp32."""
    return torch.randn(*shape, generator=_gen(seed))


def outlier_kv(B=1, Hkv=8, L=32768, d=128, seed=2, sigma_log=0.5, outliers=2, factor=10.0):
    """bf16 K or V [B, Hkv, L, d]: per (head, channel) std ~ LogNormal(0, sigma_log),
    `outliers` channels per head (seeded permutation) scaled by `factor`."""
    g = _gen(seed)
    std = torch.exp(sigma_log * torch.randn(Hkv, d, generator=g))
    for h in range(Hkv):
        ch = torch.randperm(d, generator=g)[:outliers]
        std[h, ch] *= factor
    x = torch.randn(B, Hkv, L, d, generator=g) * std[None, :, None, :]
    return x.to(torch.bfloat16)


def scaled_kv(B=4, Hkv=8, L=131072, d=128, seed=5, lo=0.5, hi=2.0):
    """bf16 [B, Hkv, L, d]: N(0, 1) times a per-(sequence, head) scale ~ U(lo, hi)."""
    g = _gen(seed)
    s = lo + (hi - lo) * torch.rand(B, Hkv, generator=g)
    out = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hkv):
            out[b, h] = (torch.randn(L, d, generator=g) * s[b, h]).to(torch.bfloat16)
    return out


def unit_database(n=1_000_000, d=1536, seed=8, block=1 << 16):
    """fp32 [n, d] rows drawn N(0, I) then L2-normalised (search database / queries)."""
    g = _gen(seed)
    out = torch.empty(n, d, dtype=torch.float32)
    for i in range(0, n, block):
        j = min(n, i + block)
        x = torch.randn(j - i, d, generator=g)
        out[i:j] = x / x.norm(dim=1, keepdim=True)
    return out


def stream_prefill(B=64, Hkv=8, L=16384, d=128, seed=10):
    """bf16 prefill [B, Hkv, L, d] of the streaming workload, N(0, 1)."""
    return torch.randn(B, Hkv, L, d, generator=_gen(seed)).to(torch.bfloat16)


def stream_step(t, B=64, Hkv=8, Hq=32, d=128, seed0=11):
    """Step t (1-based) of the streaming workload: new token bf16 [B, Hkv, d] and
    queries fp32 [B, Hq, d], both N(0, 1) from seed seed0 + t."""
    g = _gen(seed0 + t)
    tok = torch.randn(B, Hkv, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g)
    return tok, q


def random_rows(shape, row_bytes, seed):
    """Packed rows [*shape, row_bytes] of uniformly random bytes (numpy uint8). Every bit
    pattern is a valid row of codes or sign bits, so such rows stand in for an encoded cache
    where a test needs full-size caches faster than an fp64 encode can produce them."""
    import numpy as np
    return np.random.default_rng(seed).integers(0, 256, size=tuple(shape) + (row_bytes,), dtype=np.uint8)


def random_norms(shape, d, seed, scale=None, dtype="float16"):
    """Norms [*shape] of Gaussian vectors in R^d: sqrt(chi^2_d) times an optional per-row scale
    (numpy array broadcast to shape), stored in `dtype` (numpy)."""
    import numpy as np
    n = np.sqrt(np.random.default_rng(seed).chisquare(d, size=tuple(shape)))
    if scale is not None:
        n = n * scale
    return n.astype(dtype)
