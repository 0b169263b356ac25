"""CPU oracle of the layered MoE decode step (fp32, plain C, via ctypes).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports this
package, and this package imports nothing from the product.

``ops`` exposes each C function with numpy arguments; ``step`` runs whole
decode steps layer by layer, fetching weights through a source object.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


class Dims(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int), ("n_q_heads", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
        ("expert_ffn", ctypes.c_int), ("shared_ffn", ctypes.c_int),
        ("vocab", ctypes.c_int), ("max_seqs", ctypes.c_int),
        ("kv_capacity", ctypes.c_int), ("rms_eps", ctypes.c_float),
        ("rope_theta", ctypes.c_double),
    ]


def lib():
    """Load (building first if needed) ``liboracle.so``."""
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
    return _lib


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


f32p = lambda a: _p(a, ctypes.c_float)  # noqa: E731
u16p = lambda a: _p(a, ctypes.c_uint16)  # noqa: E731
i32p = lambda a: _p(a, ctypes.c_int)  # noqa: E731


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def set_threads(n: int) -> int:
    return lib().or_set_threads(ctypes.c_int(n))


def bf16_round(x) -> np.ndarray:
    x = _f32(x)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().or_bf16_round(ctypes.c_long(x.size), f32p(x), u16p(out))
    return out


def bf16_to_f32(b) -> np.ndarray:
    b = _u16(b)
    out = np.empty(b.shape, dtype=np.float32)
    lib().or_bf16_to_f32(ctypes.c_long(b.size), u16p(b), f32p(out))
    return out


def rmsnorm(h, g, eps: float) -> np.ndarray:
    h = _f32(h)
    g = _u16(g)
    out = np.empty_like(h)
    lib().or_rmsnorm(ctypes.c_int(h.size), f32p(h), u16p(g), ctypes.c_float(eps), f32p(out))
    return out


def matvec(W, x) -> np.ndarray:
    W = _u16(W)
    x = _f32(x)
    rows, cols = W.shape
    y = np.empty(rows, dtype=np.float32)
    lib().or_matvec(ctypes.c_int(rows), ctypes.c_int(cols), u16p(W), f32p(x), f32p(y))
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    v = _f32(v).copy()
    lib().or_rope(ctypes.c_int(v.size), ctypes.c_int(pos), ctypes.c_double(theta), f32p(v))
    return v


def attend(q, K, V) -> np.ndarray:
    q = _f32(q)
    K = _u16(K)
    V = _u16(V)
    n, hd = K.shape
    out = np.empty(hd, dtype=np.float32)
    lib().or_attend(ctypes.c_int(hd), ctypes.c_int(n), f32p(q), u16p(K), u16p(V), f32p(out))
    return out


def topk_softmax(z, k: int):
    z = _f32(z)
    ids = np.empty(k, dtype=np.int32)
    w = np.empty(k, dtype=np.float32)
    lib().or_topk_softmax(ctypes.c_int(z.size), ctypes.c_int(k), f32p(z), i32p(ids), f32p(w))
    return ids, w


def swiglu(Wg, Wu, Wd, y) -> np.ndarray:
    Wg, Wu, Wd = _u16(Wg), _u16(Wu), _u16(Wd)
    y = _f32(y)
    F, d = Wg.shape
    out = np.empty(d, dtype=np.float32)
    lib().or_swiglu(ctypes.c_int(F), ctypes.c_int(d), u16p(Wg), u16p(Wu), u16p(Wd), f32p(y),
                    f32p(out))
    return out


def argmax(v) -> int:
    v = _f32(v)
    return int(lib().or_argmax(ctypes.c_int(v.size), f32p(v)))


from . import step  # noqa: E402,F401  (re-export)
