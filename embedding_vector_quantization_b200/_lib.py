"""ctypes binding of libtq.so: one Python function per C entry point, same names.

Argument marshalling only -- every step of the quantization path runs in the
library's CUDA kernels. Tensors are PyTorch tensors used as device memory;
the stream is ``torch.cuda.current_stream()`` unless one is given. A non-zero
status raises :class:`TQError` with the library's message. If libtq.so is
missing, importing this module raises (there is no fallback).
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_EINVAL, TQ_ENOMEM, TQ_ECUDA, TQ_ECAPACITY, TQ_ETIMEOUT, TQ_EUNSUPPORTED = range(7)
TQ_F32, TQ_F16, TQ_BF16 = 0, 1, 2
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_EINVAL", 2: "TQ_ENOMEM", 3: "TQ_ECUDA", 4: "TQ_ECAPACITY",
                5: "TQ_ETIMEOUT", 6: "TQ_EUNSUPPORTED"}


class TQError(RuntimeError):
    def __init__(self, status, func, msg):
        self.status = status
        super().__init__(f"{func} -> {STATUS_NAMES.get(status, status)}: {msg}")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtq.so not found at {LIB_PATH}; build it with "
                      "`python embedding_vector_quantization_b200/build.py` (needs nvcc)")
lib = ctypes.CDLL(LIB_PATH)


class tq_cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("norms", ctypes.c_void_p),
                ("rnorms", ctypes.c_void_p), ("L_cap", ctypes.c_int64)]


_vp, _i, _i64, _u64, _sz, _f = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                ctypes.c_size_t, ctypes.c_float)
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_cp = ctypes.POINTER(tq_cache)

_SIGS = {
    "tq_codebook_host": (_i, [_i, _i, _dp, _dp]),
    "tq_rotation_host": (_i, [_i, _i, _u64, _dp, _dp]),
    "tq_create": (_i, [_i, _i, _u64, ctypes.POINTER(_vp)]),
    "tq_create_prod": (_i, [_i, _i, _i, _u64, ctypes.POINTER(_vp)]),
    "tq_create_polar": (_i, [_i, _i, _i, _u64, ctypes.POINTER(_vp)]),
    "tq_polar_info": (_i, [_vp, _ip, _ip, _ip]),
    "tq_get_polar_codebook": (_i, [_vp, _i, _dp, _dp]),
    "tq_polar_codebook_host": (_i, [_i, _i, _dp, _dp]),
    "tq_set_norm_dtype": (_i, [_vp, _i]),
    "tq_destroy": (None, [_vp]),
    "tq_get_info": (_i, [_vp, _ip, _ip, _ip, _ip]),
    "tq_code_bytes": (_i, [_vp, _ip, _ip]),
    "tq_get_codebook": (_i, [_vp, _dp, _dp]),
    "tq_get_rotation": (_i, [_vp, _dp, _dp]),
    "tq_encode": (_i, [_vp, _vp, _i, _i64, _vp, _vp, _vp, _vp, _vp]),
    "tq_pack_indices": (_i, [_vp, _vp, _i64, _vp, _vp]),
    "tq_append": (_i, [_vp, _vp, _i, _i, _i, _cp, _vp, _i, _vp]),
    "tq_score_workspace_bytes": (_sz, [_vp, _i, _i]),
    "tq_attn_workspace_bytes": (_sz, [_vp, _vp, _i, _i, _i, _i64]),
    "tq_search_workspace_bytes": (_sz, [_vp, _i, _i64, _i]),
    "tq_score": (_i, [_vp, _vp, _i, _i, _i, _cp, _vp, _vp, _vp, _sz, _vp]),
    "tq_attn_decode": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _cp, _cp, _vp, _f, _vp, _vp, _sz, _vp]),
    "tq_attn_decode_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _cp, _cp, _vp, _f, _vp, _vp]),
    "tq_decode_step": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _cp, _cp, _vp, _f, _vp, _vp, _sz, _vp]),
    "tq_search_topk": (_i, [_vp, _vp, _i, _vp, _vp, _i64, _i, _vp, _vp, _vp, _sz, _vp]),
    "tq_timer_enable": (_i, [_i]),
    "tq_timer_read": (_i, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), _ip, _i]),
    "tq_last_status": (_i, [_vp, _vp]),
    "tq_selftest_wait_timeout": (_i, [_vp, _i, _vp]),
    "tq_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def last_error() -> str:
    return (lib.tq_last_error() or b"").decode()


def check(status, func):
    if status != TQ_OK:
        raise TQError(status, func, last_error())


# ------------------------------------------------------------------ marshalling

def _ptr(t):
    """Device (or host) address of a tensor / array, or NULL for None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t):
    import torch
    return {torch.float32: TQ_F32, torch.float16: TQ_F16, torch.bfloat16: TQ_BF16}[t.dtype]


def _dptr(a):
    return a.ctypes.data_as(_dp)


def make_cache(codes, signs, norms, rnorms, L_cap) -> tq_cache:
    return tq_cache(_ptr(codes), _ptr(signs), _ptr(norms), _ptr(rnorms), int(L_cap))


# ------------------------------------------------------------------ entry points (same names)

def tq_codebook_host(d, bits):
    c = np.zeros(1 << bits)
    b = np.zeros((1 << bits) - 1)
    check(lib.tq_codebook_host(d, bits, _dptr(c), _dptr(b)), "tq_codebook_host")
    return c, b


def tq_rotation_host(d, m, seed):
    Pi = np.zeros((d, d))
    S = np.zeros((m, d)) if m else None
    check(lib.tq_rotation_host(d, m, seed, _dptr(Pi), _dptr(S) if m else None), "tq_rotation_host")
    return Pi, S


def tq_create(d, bits, seed):
    h = _vp()
    check(lib.tq_create(d, bits, seed, ctypes.byref(h)), "tq_create")
    return h


def tq_create_prod(d, bits, qjl_m, seed):
    h = _vp()
    check(lib.tq_create_prod(d, bits, qjl_m, seed, ctypes.byref(h)), "tq_create_prod")
    return h


def tq_create_polar(d, bits_level1, bits_upper, seed):
    h = _vp()
    check(lib.tq_create_polar(d, bits_level1, bits_upper, seed, ctypes.byref(h)), "tq_create_polar")
    return h


def tq_polar_info(h):
    n, b1, bu = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    check(lib.tq_polar_info(h, ctypes.byref(n), ctypes.byref(b1), ctypes.byref(bu)), "tq_polar_info")
    return n.value, b1.value, bu.value


def tq_get_polar_codebook(h, level, bits):
    c = np.zeros(1 << bits)
    b = np.zeros((1 << bits) - 1)
    check(lib.tq_get_polar_codebook(h, level, _dptr(c), _dptr(b)), "tq_get_polar_codebook")
    return c, b


def tq_polar_codebook_host(level, bits):
    c = np.zeros(1 << bits)
    b = np.zeros((1 << bits) - 1)
    check(lib.tq_polar_codebook_host(level, bits, _dptr(c), _dptr(b)), "tq_polar_codebook_host")
    return c, b


def tq_set_norm_dtype(h, dtype):
    check(lib.tq_set_norm_dtype(h, dtype), "tq_set_norm_dtype")


def tq_destroy(h):
    lib.tq_destroy(h)


def tq_get_info(h):
    vals = [ctypes.c_int() for _ in range(4)]
    check(lib.tq_get_info(h, *[ctypes.byref(v) for v in vals]), "tq_get_info")
    return tuple(v.value for v in vals)


def tq_code_bytes(h):
    a, b = ctypes.c_int(), ctypes.c_int()
    check(lib.tq_code_bytes(h, ctypes.byref(a), ctypes.byref(b)), "tq_code_bytes")
    return a.value, b.value


def tq_get_codebook(h, bits):
    c = np.zeros(1 << bits)
    b = np.zeros((1 << bits) - 1)
    check(lib.tq_get_codebook(h, _dptr(c), _dptr(b)), "tq_get_codebook")
    return c, b


def tq_get_rotation(h, d, m):
    Pi = np.zeros((d, d))
    S = np.zeros((m, d)) if m else None
    check(lib.tq_get_rotation(h, _dptr(Pi), _dptr(S) if m else None), "tq_get_rotation")
    return Pi, S


def tq_encode(h, x, n, codes, signs, norms, rnorms, stream=None):
    check(lib.tq_encode(h, _ptr(x), _dtype_code(x), n, _ptr(codes), _ptr(signs), _ptr(norms), _ptr(rnorms),
                        _stream(stream)), "tq_encode")


def tq_pack_indices(h, idx, n, codes, stream=None):
    check(lib.tq_pack_indices(h, _ptr(idx), n, _ptr(codes), _stream(stream)), "tq_pack_indices")


def tq_append(h, x_new, B, Hkv, cache, len_, advance, stream=None):
    check(lib.tq_append(h, _ptr(x_new), _dtype_code(x_new), B, Hkv, ctypes.byref(cache), _ptr(len_),
                        int(bool(advance)), _stream(stream)), "tq_append")


def tq_score_workspace_bytes(hk, B, Hq):
    return lib.tq_score_workspace_bytes(hk, B, Hq)


def tq_attn_workspace_bytes(hk, hv, B, Hq, Hkv, L_cap):
    return lib.tq_attn_workspace_bytes(hk, hv, B, Hq, Hkv, L_cap)


def tq_search_workspace_bytes(h, nq, n, k):
    return lib.tq_search_workspace_bytes(h, nq, n, k)


def tq_score(hk, q, B, Hq, Hkv, kcache, len_, logits, workspace, stream=None):
    check(lib.tq_score(hk, _ptr(q), B, Hq, Hkv, ctypes.byref(kcache), _ptr(len_), _ptr(logits), _ptr(workspace),
                       workspace.numel() * workspace.element_size(), _stream(stream)), "tq_score")


def tq_attn_decode(hk, hv, q, B, Hq, Hkv, kcache, vcache, len_, scale, out, workspace, stream=None):
    check(lib.tq_attn_decode(hk, hv, _ptr(q), _dtype_code(q), B, Hq, Hkv, ctypes.byref(kcache),
                             ctypes.byref(vcache), _ptr(len_), float(scale), _ptr(out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)), "tq_attn_decode")


def tq_attn_decode_noalloc(hk, hv, q, B, Hq, Hkv, kcache, vcache, len_, scale, out, stream=None):
    """tq_attn_decode without a workspace (scratch from the library's fixed 4 MiB device array)."""
    check(lib.tq_attn_decode_noalloc(hk, hv, _ptr(q), _dtype_code(q), B, Hq, Hkv, ctypes.byref(kcache),
                                     ctypes.byref(vcache), _ptr(len_), float(scale), _ptr(out), _stream(stream)),
          "tq_attn_decode_noalloc")


def tq_decode_step(hk, hv, q, k_new, v_new, B, Hq, Hkv, kcache, vcache, len_, scale, out, workspace, stream=None):
    """Append k_new / v_new [B, Hkv, d] at slot len[b], attend over len[b] + 1 tokens, advance len."""
    if k_new.dtype != v_new.dtype:
        raise TQError(1, "tq_decode_step", "k_new and v_new must have one dtype")
    check(lib.tq_decode_step(hk, hv, _ptr(q), _dtype_code(q), _ptr(k_new), _ptr(v_new), _dtype_code(k_new), B, Hq,
                             Hkv, ctypes.byref(kcache), ctypes.byref(vcache), _ptr(len_), float(scale), _ptr(out),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
          "tq_decode_step")


def tq_search_topk(h, q, nq, codes, norms, n, k, idx, score, workspace, stream=None):
    check(lib.tq_search_topk(h, _ptr(q), nq, _ptr(codes), _ptr(norms), n, k, _ptr(idx), _ptr(score),
                             _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
          "tq_search_topk")


def tq_timer_enable(on):
    check(lib.tq_timer_enable(int(bool(on))), "tq_timer_enable")


def tq_timer_read(name=None, forget=True):
    """(milliseconds, launches) recorded for kernel `name` (None = all); forget=False keeps graph-captured pairs."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int(0)
    check(lib.tq_timer_read(name.encode() if name else None, ctypes.byref(ms), ctypes.byref(n), int(bool(forget))),
          "tq_timer_read")
    return ms.value, n.value


def tq_selftest_wait_timeout(h, limit, stream=None):
    """Makes one bounded device wait run out on purpose; the handle's next status is TQ_ETIMEOUT."""
    check(lib.tq_selftest_wait_timeout(h, int(limit), _stream(stream)), "tq_selftest_wait_timeout")


def tq_last_status(h, stream=None):
    """Returns the status word (TQ_OK, TQ_ECAPACITY, ...) without raising."""
    return lib.tq_last_status(h, _stream(stream))


def tq_last_error():
    return last_error()
