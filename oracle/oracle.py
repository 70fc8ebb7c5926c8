"""ctypes front end of the fp64 C oracle (test infrastructure only).

Inputs may be numpy arrays or torch tensors of any float dtype; they are
widened exactly to fp64 (a bf16 value is exactly representable in fp64), so
the oracle sees the same bits as the GPU path.  Outputs are fp64 numpy arrays.

Layouts follow the attention core's convention: q, o, dO and dq are
[B, T, H, D]; k, v, dk and dv are [B, T, Hkv, D] with H a multiple of Hkv
(grouped K/V heads; Hkv = H is multi-head attention); lse and delta are
[B, H, T].
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.POINTER(ctypes.c_double)
        L = ctypes.c_long
        LP = ctypes.POINTER(ctypes.c_long)
        lib.oracle_attn_fwd.argtypes = [P, P, P, L, L, L, L, L, ctypes.c_double,
                                        ctypes.c_double, P, P, LP, L]
        lib.oracle_attn_fwd.restype = None
        lib.oracle_attn_bwd.argtypes = [P, P, P, P, L, L, L, L, L, ctypes.c_double,
                                        ctypes.c_double, P, P, P, P, P, LP, L]
        lib.oracle_attn_bwd.restype = None
        lib.oracle_attn_fwd_gqa.argtypes = [P, P, P, L, L, L, L, L, L, ctypes.c_double,
                                            ctypes.c_double, P, P, LP, L]
        lib.oracle_attn_fwd_gqa.restype = None
        lib.oracle_attn_bwd_gqa.argtypes = [P, P, P, P, L, L, L, L, L, L, ctypes.c_double,
                                            ctypes.c_double, P, P, P, P, P, LP, L]
        lib.oracle_attn_bwd_gqa.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().oracle_num_threads())


def _f64(x):
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _heads(heads):
    if heads is None:
        return None, 0, None
    arr = np.ascontiguousarray(np.asarray(heads, dtype=np.int64))
    return arr, len(arr), arr.ctypes.data_as(ctypes.POINTER(ctypes.c_long))


def default_scale(D: int) -> float:
    """Softmax scale 1/sqrt(head_dim), the FlashAttention default."""
    return 1.0 / math.sqrt(D)


def _kv_heads(q, k, v):
    H, Hkv = q.shape[2], k.shape[2]
    if v.shape != k.shape or Hkv < 1 or H % Hkv:
        raise ValueError("k and v need the same shape and a head count that divides q's")
    return Hkv


def attn_fwd(q, k, v, window, eps=1e-6, scale=None, heads=None):
    """Forward of norm(q), norm(k) attention; returns (o, lse).

    k and v may have fewer heads than q (grouped K/V heads): query head h
    reads K/V head h // (H // Hkv).
    heads: optional list of flat b*H + h query-head indices; only those heads
    are computed (the rest of o and lse is NaN).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, D = q.shape
    Hkv = _kv_heads(q, k, v)
    if scale is None:
        scale = default_scale(D)
    o = np.full((B, T, H, D), np.nan)
    lse = np.full((B, H, T), np.nan)
    harr, nh, hp = _heads(heads)
    _load().oracle_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), B, T, H, Hkv, D, int(window),
                                float(eps), float(scale), _ptr(o), _ptr(lse), hp, nh)
    return o, lse


def attn_bwd(q, k, v, dO, window, eps=1e-6, scale=None, heads=None):
    """Backward; returns dict(dq, dk, dv, lse, delta) as fp64 arrays.

    With grouped K/V heads, dk and dv of a K/V head sum the contributions of
    every query head of its group.
    heads: optional list of flat b*Hkv + hk K/V-head indices (b*H + h when
    Hkv = H); those K/V heads and every query head of their groups are
    computed (the rest is NaN).
    """
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, T, H, D = q.shape
    Hkv = _kv_heads(q, k, v)
    if scale is None:
        scale = default_scale(D)
    dq = np.full((B, T, H, D), np.nan)
    dk = np.full((B, T, Hkv, D), np.nan)
    dv = np.full((B, T, Hkv, D), np.nan)
    lse = np.full((B, H, T), np.nan)
    delta = np.full((B, H, T), np.nan)
    harr, nh, hp = _heads(heads)
    _load().oracle_attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), B, T, H, Hkv, D, int(window),
                                float(eps), float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(lse), _ptr(delta), hp, nh)
    return dict(dq=dq, dk=dk, dv=dv, lse=lse, delta=delta)


def unmasked_pairs(T: int, window: int) -> int:
    """Number of visible (query, key) pairs of one head: sum_i (min(i, w) + 1)."""
    w = T if window < 0 else window
    return sum(min(i, w) + 1 for i in range(T))
