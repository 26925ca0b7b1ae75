"""ctypes binding of ``libiskv.so`` (declared in ``include/iskv.h``).

Argument marshalling only: every step of the path runs in the library's CUDA kernels. Device
buffers are passed as raw pointers (``int``) or as torch tensors (their ``data_ptr()``); streams as
raw ``cudaStream_t`` values or ``torch.cuda.Stream`` objects. The functions keep the C names and
return the C status code; :func:`check` turns a non-zero code into :class:`IsKVError`.

Importing this module loads the library and fails loudly when it is missing: there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "IsKVError", "iskv_config", "lib", "check", "ISKV_OK", "ISKV_ERR_INVALID_ARG",
    "ISKV_ERR_CAPACITY", "ISKV_ERR_CUDA", "ISKV_ERR_NOT_CONVERGED", "ISKV_ERR_NONFINITE",
    "ISKV_ERR_UNSUPPORTED", "ISKV_ERR_TIMEOUT", "ISKV_BF16", "ISKV_F32", "LIB_PATH",
    "iskv_create", "iskv_destroy", "iskv_append_block", "iskv_decode_attn", "iskv_reconstruct",
    "iskv_get_factors", "iskv_num_tokens", "iskv_storage_bytes", "iskv_schedule",
    "iskv_sync_status", "iskv_strerror", "iskv_reset", "iskv_launch_count", "iskv_fold_stats",
    "iskv_join", "iskv_append_decode",
    "iskv_decode_view", "iskv_decode_attn_noalloc", "ISKV_NOALLOC_SCRATCH_FLOATS",
    "iskv_protect", "iskv_prefill",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libiskv.so")

ISKV_OK = 0
ISKV_ERR_INVALID_ARG = -1
ISKV_ERR_CAPACITY = -2
ISKV_ERR_CUDA = -3
ISKV_ERR_NOT_CONVERGED = -4
ISKV_ERR_NONFINITE = -5
ISKV_ERR_UNSUPPORTED = -6
ISKV_ERR_TIMEOUT = -7
ISKV_BF16 = 0
ISKV_F32 = 1


class iskv_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("n_layers", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("rank_k", ctypes.c_int),
        ("rank_v", ctypes.c_int),
        ("block", ctypes.c_int),
        ("window", ctypes.c_int),
        ("max_tokens", ctypes.c_longlong),
        ("kv_dtype", ctypes.c_int),
        ("rope", ctypes.c_int),
        ("rope_theta", ctypes.c_double),
        ("rotate_history", ctypes.c_int),
        ("lookahead_folds", ctypes.c_int),
        ("fixed_basis", ctypes.c_int),
        ("coord_bf16", ctypes.c_int),
        ("prot_cap", ctypes.c_int),
        ("joint_heads", ctypes.c_int),
    ]


class iskv_protect(ctypes.Structure):
    """Key/value protection of iskv_prefill (mirrors the C struct)."""
    _fields_ = [
        ("chunk", ctypes.c_int),
        ("m", ctypes.c_int),
        ("suffix", ctypes.c_int),
        ("rho", ctypes.c_int),
    ]


ISKV_NOALLOC_SCRATCH_FLOATS = 1 << 20


class iskv_decode_view(ctypes.Structure):
    """Cache description for iskv_decode_attn_noalloc (mirrors the C struct)."""
    _fields_ = [
        ("n_c", ctypes.c_longlong),
        ("t", ctypes.c_longlong),
        ("n_max", ctypes.c_longlong),
        ("batch", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("rank_k", ctypes.c_int),
        ("rank_v", ctypes.c_int),
        ("k_k", ctypes.c_int),
        ("k_v", ctypes.c_int),
        ("ring_rows", ctypes.c_int),
        ("kv_dtype", ctypes.c_int),
        ("coords_k", ctypes.c_void_p),
        ("coords_v", ctypes.c_void_p),
        ("basis_k", ctypes.c_void_p),
        ("basis_v", ctypes.c_void_p),
        ("ring_k", ctypes.c_void_p),
        ("ring_v", ctypes.c_void_p),
        ("rope_cs", ctypes.c_void_p),
    ]


class IsKVError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {iskv_strerror(code)} ({code})" if what else
                         f"{iskv_strerror(code)} ({code})")


_vp = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong

_SIGNATURES = {
    "iskv_create": (_i, [ctypes.POINTER(iskv_config), ctypes.POINTER(_vp)]),
    "iskv_destroy": (_i, [_vp]),
    "iskv_append_block": (_i, [_vp, _i, _vp, _vp, _i, _vp]),
    "iskv_decode_attn": (_i, [_vp, _i, _vp, _vp, _vp]),
    "iskv_reconstruct": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "iskv_get_factors": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, ctypes.POINTER(_i),
                              ctypes.POINTER(_ll), _vp]),
    "iskv_num_tokens": (_i, [_vp, _i, ctypes.POINTER(_ll)]),
    "iskv_storage_bytes": (_i, [_vp, _i, ctypes.POINTER(_ll)]),
    "iskv_schedule": (_i, [_i, _i, _ll, _ll, ctypes.POINTER(_ll), ctypes.POINTER(_ll)]),
    "iskv_sync_status": (_i, [_vp, _vp]),
    "iskv_join": (_i, [_vp, _vp]),
    "iskv_append_decode": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "iskv_strerror": (ctypes.c_char_p, [_i]),
    "iskv_reset": (_i, [_vp, _vp]),
    "iskv_launch_count": (_i, [_vp, ctypes.POINTER(_ll)]),
    "iskv_fold_stats": (_i, [_vp, _vp, ctypes.POINTER(_i), ctypes.POINTER(_ll),
                             ctypes.POINTER(_ll)]),
    "iskv_decode_attn_noalloc": (_i, [ctypes.POINTER(iskv_decode_view), _vp, _vp, _vp]),
    "iskv_prefill": (_i, [_vp, _i, _vp, _vp, _ll, ctypes.POINTER(iskv_protect), _vp]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "'python -m rank_kv_cache_isvd_b200.build' (there is no CPU fallback)")
    so = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(so, name)
        fn.restype = res
        fn.argtypes = args
    return so


lib = _load()


def _ptr(x):
    """Raw device pointer of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:      # pragma: no cover - no torch: legacy default stream
            return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def check(code: int, what: str = "") -> int:
    if code != ISKV_OK:
        raise IsKVError(code, what)
    return code


def iskv_strerror(code: int) -> str:
    return lib.iskv_strerror(code).decode()


def iskv_create(cfg: iskv_config):
    """Returns ``(code, handle)``; ``handle`` is an opaque ``int`` (0 on failure)."""
    h = _vp()
    code = lib.iskv_create(ctypes.byref(cfg), ctypes.byref(h))
    return code, (h.value or 0)


def iskv_destroy(handle) -> int:
    return lib.iskv_destroy(handle)


def iskv_append_block(handle, layer: int, k_rows, v_rows, m: int, stream=None) -> int:
    return lib.iskv_append_block(handle, layer, _ptr(k_rows), _ptr(v_rows), m, _stream(stream))


def iskv_decode_attn(handle, layer: int, q, out, stream=None) -> int:
    return lib.iskv_decode_attn(handle, layer, _ptr(q), _ptr(out), _stream(stream))


def iskv_reconstruct(handle, layer: int, which: int, apply_rope: int, out, stream=None) -> int:
    return lib.iskv_reconstruct(handle, layer, which, apply_rope, _ptr(out), _stream(stream))


def iskv_get_factors(handle, layer: int, seq: int, kv_head: int, which: int, coords=None,
                     basis=None, sigma=None, stream=None):
    """Returns ``(code, k, n_c)``."""
    k = _i(0)
    n = _ll(0)
    code = lib.iskv_get_factors(handle, layer, seq, kv_head, which, _ptr(coords), _ptr(basis),
                                _ptr(sigma), ctypes.byref(k), ctypes.byref(n), _stream(stream))
    return code, k.value, n.value


def iskv_num_tokens(handle, layer: int):
    t = _ll(0)
    code = lib.iskv_num_tokens(handle, layer, ctypes.byref(t))
    return code, t.value


def iskv_storage_bytes(handle, layer: int):
    b = _ll(0)
    code = lib.iskv_storage_bytes(handle, layer, ctypes.byref(b))
    return code, b.value


def iskv_schedule(block: int, window: int, t: int, m: int):
    """Returns ``(code, n_c, folds)``; host only, needs no GPU."""
    n = _ll(0)
    f = _ll(0)
    code = lib.iskv_schedule(block, window, t, m, ctypes.byref(n), ctypes.byref(f))
    return code, n.value, f.value


def iskv_reset(handle, stream=None) -> int:
    return lib.iskv_reset(handle, _stream(stream))


def iskv_launch_count(handle):
    n = _ll(0)
    code = lib.iskv_launch_count(handle, ctypes.byref(n))
    return code, n.value


def iskv_fold_stats(handle, stream=None):
    """Returns ``(code, max_sweeps, total_sweeps, cores)``; synchronises the stream."""
    m = _i(0)
    t = _ll(0)
    c = _ll(0)
    code = lib.iskv_fold_stats(handle, _stream(stream), ctypes.byref(m), ctypes.byref(t),
                               ctypes.byref(c))
    return code, m.value, t.value, c.value


def iskv_decode_attn_noalloc(view: iskv_decode_view, q, out, stream=None) -> int:
    return lib.iskv_decode_attn_noalloc(None if view is None else ctypes.byref(view), _ptr(q),
                                        _ptr(out), _stream(stream))


def iskv_append_decode(handle, layer: int, k_row, v_row, q, out, stream=None) -> int:
    return lib.iskv_append_decode(handle, layer, _ptr(k_row), _ptr(v_row), _ptr(q), _ptr(out),
                                  _stream(stream))


def iskv_join(handle, stream=None) -> int:
    return lib.iskv_join(handle, _stream(stream))


def iskv_sync_status(handle, stream=None) -> int:
    return lib.iskv_sync_status(handle, _stream(stream))


def iskv_prefill(handle, layer: int, k_rows, v_rows, T0: int, protect=None, stream=None) -> int:
    """``protect``: an :class:`iskv_protect` or ``None`` (no protection)."""
    return lib.iskv_prefill(handle, layer, _ptr(k_rows), _ptr(v_rows), T0,
                            None if protect is None else ctypes.byref(protect), _stream(stream))
