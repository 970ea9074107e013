"""B200-native TurboQuant-style vector quantization (libtq.so + thin binding).

Encode stores each vector's norm, rotates it by a seeded random orthogonal
matrix, maps every rotated coordinate to a Lloyd-Max codebook index and
bit-packs the indices; prod handles add a 1-bit QJL sign sketch of the
residual and its norm ("Google TurboQuant: 6x KV-cache compression",
sections "Stage 1: PolarQuant" and "Stage 2: QJL residual correction").
Scores, GQA decode attention and top-k search read only the packed codes.

The ``tq_*`` functions mirror the C ABI of ``include/tq.h`` one to one;
:class:`Handle` and :class:`Cache` only allocate PyTorch tensors for them.
Everything runs in the library's CUDA kernels; if libtq.so is missing the
import fails.
"""

from . import _lib
from ._lib import (  # noqa: F401  (the C ABI, same names)
    TQ_BF16, TQ_EINVAL, TQ_ECAPACITY, TQ_ECUDA, TQ_ENOMEM, TQ_ETIMEOUT, TQ_EUNSUPPORTED, TQ_F16, TQ_F32, TQ_OK,
    TQError, make_cache, tq_append, tq_attn_decode, tq_attn_decode_noalloc, tq_decode_step, tq_attn_workspace_bytes, tq_code_bytes, tq_codebook_host,
    tq_create, tq_create_polar, tq_create_prod, tq_destroy, tq_get_polar_codebook, tq_polar_codebook_host,
    tq_polar_info, tq_encode, tq_get_codebook, tq_get_info, tq_get_rotation,
    tq_last_error, tq_last_status, tq_pack_indices, tq_rotation_host, tq_score, tq_score_workspace_bytes,
    tq_search_topk, tq_search_workspace_bytes, tq_selftest_wait_timeout, tq_set_norm_dtype, tq_timer_enable,
    tq_timer_read,
)


def _torch():
    import torch
    return torch


class Handle:
    """Owns one library handle: Pi, S, S Pi^T and the codebook on the current device.

    ``bits`` is the total bits per coordinate; with ``qjl_m > 0`` it splits into
    ``bits - 1`` MSE bits plus one QJL sign per projection. ``bits = 1`` with
    ``qjl_m > 0`` gives QJL-only rows: the signs and the norm, no codes.
    """

    def __init__(self, d, bits, seed=0, qjl_m=0, norm_dtype=None):
        self._h = tq_create_prod(d, bits, qjl_m, seed) if qjl_m else tq_create(d, bits, seed)
        if norm_dtype is not None:
            tq_set_norm_dtype(self._h, norm_dtype)
        self.d, self.bits_mse, self.m, self.norm_dtype = tq_get_info(self._h)
        self.codes_B, self.signs_B = tq_code_bytes(self._h)
        self.seed = seed

    @property
    def prod(self):
        return self.m > 0

    @property
    def qjl_only(self):
        return self.m > 0 and self.bits_mse == 0

    @property
    def ptr(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            tq_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def codebook(self):
        return tq_get_codebook(self._h, self.bits_mse)

    def rotation(self):
        return tq_get_rotation(self._h, self.d, self.m)

    def norm_torch_dtype(self):
        torch = _torch()
        return torch.float16 if self.norm_dtype == TQ_F16 else torch.float32

    def alloc_rows(self, shape, device="cuda"):
        """Empty packed storage for vectors of leading shape ``shape``."""
        torch = _torch()
        shape = tuple(shape) if isinstance(shape, (tuple, list)) else (shape,)
        out = {"codes": None, "norms": torch.empty(shape, dtype=self.norm_torch_dtype(), device=device),
               "signs": None, "rnorms": None}
        if self.codes_B:
            out["codes"] = torch.empty(shape + (self.codes_B,), dtype=torch.uint8, device=device)
        if self.prod:
            out["signs"] = torch.empty(shape + (self.signs_B,), dtype=torch.uint8, device=device)
        if self.prod and not self.qjl_only:
            out["rnorms"] = torch.empty(shape, dtype=torch.float16, device=device)
        return out

    def encode(self, x, out=None, stream=None):
        """Encodes x [..., d] (fp32 / fp16 / bf16, contiguous, on the GPU)."""
        x = x.contiguous()
        lead = tuple(x.shape[:-1])
        n = 1
        for s in lead:
            n *= s
        out = out or self.alloc_rows(lead, x.device)
        tq_encode(self._h, x, n, out["codes"], out["signs"], out["norms"], out["rnorms"], stream)
        return out

    def pack_indices(self, idx, stream=None):
        torch = _torch()
        n = idx.shape[0]
        codes = torch.empty((n, self.codes_B), dtype=torch.uint8, device=idx.device)
        tq_pack_indices(self._h, idx.contiguous(), n, codes, stream)
        return codes

    def status(self, stream=None):
        return tq_last_status(self._h, stream)

    def search_topk(self, q, codes, norms, k, workspace=None, stream=None):
        torch = _torch()
        nq, n = q.shape[0], codes.shape[0]
        idx = torch.empty((nq, k), dtype=torch.int64, device=q.device)
        score = torch.empty((nq, k), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = torch.empty(tq_search_workspace_bytes(self._h, nq, n, k), dtype=torch.uint8,
                                    device=q.device)
        tq_search_topk(self._h, q.contiguous(), nq, codes, norms, n, k, idx, score, workspace, stream)
        return idx, score


class PolarHandle(Handle):
    """Recursive polar transform handle ("PolarQuant explainer", sections 1 and 3): log2(d)
    levels of angles, ``bits_level1`` bits at level 1 and ``bits_upper`` at the others."""

    def __init__(self, d, bits_level1, bits_upper, seed=0, norm_dtype=None):
        self._h = tq_create_polar(d, bits_level1, bits_upper, seed)
        if norm_dtype is not None:
            tq_set_norm_dtype(self._h, norm_dtype)
        self.d, self.bits_mse, self.m, self.norm_dtype = tq_get_info(self._h)
        self.codes_B, self.signs_B = tq_code_bytes(self._h)
        self.levels, self.bits_level1, self.bits_upper = tq_polar_info(self._h)
        self.seed = seed

    def level_bits(self):
        return [self.bits_level1] + [self.bits_upper] * (self.levels - 1)

    def codebook(self, level=1):
        return tq_get_polar_codebook(self._h, level, self.level_bits()[level - 1])


class Cache:
    """A quantized K or V cache [B][Hkv][L_cap] for one handle (tensors + ABI struct)."""

    def __init__(self, handle, B, Hkv, L_cap, device="cuda"):
        self.handle, self.B, self.Hkv, self.L_cap = handle, B, Hkv, L_cap
        rows = handle.alloc_rows((B, Hkv, L_cap), device)
        self.codes, self.signs, self.norms, self.rnorms = rows["codes"], rows["signs"], rows["norms"], rows["rnorms"]
        self.struct = make_cache(self.codes, self.signs, self.norms, self.rnorms, L_cap)

    def fill(self, x, stream=None):
        """Encodes x [B, Hkv, L, d] into slots 0 .. L-1 of every (sequence, head)."""
        B, Hkv, L, d = x.shape
        assert (B, Hkv) == (self.B, self.Hkv) and L <= self.L_cap and d == self.handle.d
        if L == self.L_cap:
            tq_encode(self.handle.ptr, x.contiguous(), B * Hkv * L, self.codes, self.signs, self.norms,
                      self.rnorms, stream)
            return
        tmp = self.handle.encode(x.contiguous(), stream=stream)
        for name in ("codes", "norms", "signs", "rnorms"):
            if tmp[name] is not None:
                getattr(self, name)[:, :, :L].copy_(tmp[name])

    def append(self, x_new, len_, advance=True, stream=None):
        tq_append(self.handle.ptr, x_new.contiguous(), self.B, self.Hkv, self.struct, len_, advance, stream)


def score(hk, q, kcache, len_, logits=None, workspace=None, stream=None):
    """Scores q [B, Hq, d] fp32 against a key cache; logits [B, Hq, L_cap] fp32."""
    torch = _torch()
    B, Hq, _ = q.shape
    if logits is None:
        logits = torch.zeros((B, Hq, kcache.L_cap), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(tq_score_workspace_bytes(hk.ptr, B, Hq), dtype=torch.uint8, device=q.device)
    tq_score(hk.ptr, q.contiguous(), B, Hq, kcache.Hkv, kcache.struct, len_, logits, workspace, stream)
    return logits


def attn_decode(hk, hv, q, kcache, vcache, len_, scale, out=None, workspace=None, stream=None):
    """GQA decode attention of q [B, Hq, d] (fp32 or bf16) over quantized K/V caches -> fp32 [B, Hq, d]."""
    torch = _torch()
    B, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(tq_attn_workspace_bytes(hk.ptr, hv.ptr, B, Hq, kcache.Hkv, kcache.L_cap),
                                dtype=torch.uint8, device=q.device)
    tq_attn_decode(hk.ptr, hv.ptr, q.contiguous(), B, Hq, kcache.Hkv, kcache.struct, vcache.struct, len_, scale,
                   out, workspace, stream)
    return out
