"""ctypes binding of the C oracle core (test infrastructure only).

Every function takes and returns numpy arrays; bf16 values travel as their
uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_u64 = ctypes.c_uint64
_u32 = ctypes.c_uint32
_f32 = ctypes.c_float
_f64 = ctypes.c_double
_p = ctypes.c_void_p


def lib():
    global _LIB
    if _LIB is None:
        # ORACLE_LIB lets the mutation test load a deliberately broken copy
        path = os.environ.get("ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        L.oracle_bf16_rne.restype = ctypes.c_uint16
        L.oracle_bf16_rne.argtypes = [_f32]
        L.oracle_bf16_rne_array.restype = None
        L.oracle_bf16_rne_array.argtypes = [_p, _p, _u64]
        L.oracle_adam_scalars.restype = None
        L.oracle_adam_scalars.argtypes = [_f64, _f64, _f64, _f64, _f64, _f64, _u64, _p]
        L.oracle_update.restype = None
        L.oracle_update.argtypes = [_u64, _u32, _p, _u64, _p, _p, _p, _p, _p,
                                    _f64, _f64, _f64, _f64, _f64, _f64, _f32, _u64, _p, _p]
        L.oracle_reduce.restype = None
        L.oracle_reduce.argtypes = [_u64, _u32, _p, _u64, _p]
        _LIB = L
    return _LIB


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_rne(x):
    """fp32 array -> uint16 bf16 bit patterns (round to nearest even)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_bf16_rne_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(b):
    """uint16 bf16 bit patterns -> fp32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def adam_scalars(adam, t):
    """The nine fp32 constants of step t: grad_scale, b1, b2, eps, 1-b1,
    1-b2, lr/(1-b1^t), 1/sqrt(1-b2^t), 1-lr*weight_decay."""
    out = np.zeros(9, dtype=np.float32)
    lib().oracle_adam_scalars(adam["lr"], adam["beta1"], adam["beta2"],
                              adam["eps"], adam["grad_scale"],
                              adam.get("weight_decay", 0.0), t, _ptr(out))
    return out


def reduce(grads):
    """grads: uint16 [nd, n] -> fp32 [n], the rank-order sum."""
    grads = np.ascontiguousarray(grads, dtype=np.uint16)
    nd, n = grads.shape
    out = np.empty(n, dtype=np.float32)
    lib().oracle_reduce(n, nd, _ptr(grads), n, _ptr(out))
    return out


def update(grads, w, m, v, adam, t, want_params=True, want_reduced=False,
           clip_coef=1.0):
    """The elementwise core on contiguous columns.

    grads: uint16 [nd, n]; w, m, v: fp32 [n], updated IN PLACE.
    adam: dict with lr, beta1, beta2, eps, grad_scale and optional
    weight_decay (AdamW; default 0).  clip_coef: fp32 global-norm factor.
    Returns (params uint16 [n] or None, reduced fp32 [n] or None,
             norm_sq float, nonfinite int).
    """
    grads = np.ascontiguousarray(grads, dtype=np.uint16)
    nd, n = grads.shape
    for a in (w, m, v):
        assert a.dtype == np.float32 and a.flags.c_contiguous and a.size == n
    p = np.empty(n, dtype=np.uint16) if want_params else None
    red = np.empty(n, dtype=np.float32) if want_reduced else None
    norm = np.zeros(1, dtype=np.float64)
    bad = np.zeros(1, dtype=np.int64)
    lib().oracle_update(n, nd, _ptr(grads), n, _ptr(w), _ptr(m), _ptr(v),
                        _ptr(p), _ptr(red), adam["grad_scale"], adam["lr"],
                        adam["beta1"], adam["beta2"], adam["eps"],
                        adam.get("weight_decay", 0.0), float(np.float32(clip_coef)), t,
                        _ptr(norm), _ptr(bad))
    return p, red, float(norm[0]), int(bad[0])
