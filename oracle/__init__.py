"""ORACLE -- TEST INFRASTRUCTURE ONLY.

ctypes wrapper around ``k3moe_oracle.c``, the plain scalar fp64 CPU
statement of the MXFP4 routed-expert MoE layer (what each function computes
and which source passage it follows is written in the C file).  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package; the CUDA library never does.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(hand-worked cases in ``tests/golden/``, closed forms, invariants, brute force
and an independent PyTorch fp64 restatement).  Real Kimi K3 layer outputs are
not available (the pages print no values and no checkpoint is present), so
parity against the real model is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "k3moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so (gcc, fp64, no FMA contraction, OpenMP over rows)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC",
                                   "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
            os.replace(tmp, _LIB)
    return _LIB


def load(path: str | None = None):
    """Load the oracle library (``path`` lets a test load a variant build)."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    lib.oracle_e2m1.argtypes = [ctypes.c_uint]
    lib.oracle_e2m1.restype = dbl
    lib.oracle_e8m0.argtypes = [ctypes.c_uint]
    lib.oracle_e8m0.restype = dbl
    lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_value.restype = dbl
    lib.oracle_bf16_rne.argtypes = [dbl]
    lib.oracle_bf16_rne.restype = ctypes.c_uint16
    lib.oracle_mxfp4_weight.argtypes = [vp, vp, i64, i64, i64]
    lib.oracle_mxfp4_weight.restype = dbl
    lib.oracle_mxfp4_matvec.argtypes = [vp, vp, i64, i64, vp, vp]
    lib.oracle_bf16_matvec.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_router_logits.argtypes = [vp, i64, vp, vp, i64, i64, vp]
    lib.oracle_softmax.argtypes = [vp, i64, vp]
    lib.oracle_topk.argtypes = [vp, i64, i64, vp]
    lib.oracle_route.argtypes = [vp, i64, vp, vp, i64, i64, i64, vp, vp, vp, vp]
    lib.oracle_route_variant.argtypes = [vp, i64, vp, vp, i64, i64, i64, ctypes.c_int, ctypes.c_int,
                                         vp, vp, vp, vp]
    lib.oracle_rmsnorm.argtypes = [vp, i64, vp, dbl, i64, vp]
    lib.oracle_residual_add.argtypes = [vp, i64, i64, vp, vp]
    lib.oracle_expert_ffn_vec.argtypes = [vp, vp, i64, i64, vp]
    lib.oracle_expert_ffn.argtypes = [vp, i64, vp, i64, i64, vp]
    lib.oracle_shared_ffn.argtypes = [vp, i64, vp, vp, vp, i64, i64, vp]
    lib.oracle_combine.argtypes = [vp, i64, vp, i64, vp, vp, vp, vp, i64, i64, i64, vp]
    lib.oracle_layer.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                 vp, vp, vp]
    for name in ("oracle_mxfp4_matvec", "oracle_bf16_matvec", "oracle_router_logits",
                 "oracle_softmax", "oracle_topk", "oracle_route", "oracle_route_variant",
                 "oracle_rmsnorm", "oracle_residual_add", "oracle_expert_ffn_vec",
                 "oracle_expert_ffn", "oracle_shared_ffn", "oracle_combine", "oracle_layer"):
        getattr(lib, name).restype = None
    if path is None:
        _lib = lib
    return lib


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need a C-contiguous array"
    return a.ctypes.data


def _u8(a):
    return np.ascontiguousarray(a, dtype=np.uint8)


def _bf(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 inputs are passed as uint16 bit patterns"
    return a


class Oracle:
    """Thin typed front end; ``Oracle(lib)`` wraps an alternative build."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def e2m1(self, nib: int) -> float:
        return self.lib.oracle_e2m1(nib)

    def e8m0(self, e: int) -> float:
        return self.lib.oracle_e8m0(e)

    def bf16_value(self, b: int) -> float:
        return self.lib.oracle_bf16_value(b)

    def bf16_rne(self, v) -> np.ndarray:
        v = np.asarray(v, dtype=np.float64)
        f = np.vectorize(lambda z: self.lib.oracle_bf16_rne(float(z)), otypes=[np.uint16])
        return f(v) if v.ndim else np.uint16(self.lib.oracle_bf16_rne(float(v)))

    def mxfp4_weight(self, nib, scale, cols, r, c) -> float:
        nib, scale = _u8(nib), _u8(scale)
        return self.lib.oracle_mxfp4_weight(_p(nib), _p(scale), cols, r, c)

    def mxfp4_matvec(self, nib, scale, rows, cols, v) -> np.ndarray:
        nib, scale = _u8(nib), _u8(scale)
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.empty(rows, dtype=np.float64)
        self.lib.oracle_mxfp4_matvec(_p(nib), _p(scale), rows, cols, _p(v), _p(out))
        return out

    def bf16_matvec(self, w, v) -> np.ndarray:
        w = _bf(w)
        v = np.ascontiguousarray(v, dtype=np.float64)
        out = np.empty(w.shape[0], dtype=np.float64)
        self.lib.oracle_bf16_matvec(_p(w), w.shape[0], w.shape[1], _p(v), _p(out))
        return out

    def router_logits(self, x, w, bias=None) -> np.ndarray:
        x = _bf(x)
        w = np.ascontiguousarray(w, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        T, d = x.shape
        E = w.shape[0]
        out = np.empty((T, E), dtype=np.float64)
        self.lib.oracle_router_logits(_p(x), T, _p(w), _p(b), d, E, _p(out))
        return out

    def softmax(self, l) -> np.ndarray:
        l = np.ascontiguousarray(l, dtype=np.float64)
        out = np.empty_like(l)
        self.lib.oracle_softmax(_p(l), l.size, _p(out))
        return out

    def topk(self, l, k) -> np.ndarray:
        l = np.ascontiguousarray(l, dtype=np.float64)
        out = np.empty(k, dtype=np.int32)
        self.lib.oracle_topk(_p(l), l.size, k, _p(out))
        return out

    def route(self, x, w, bias, k):
        """-> (logits [T,E] f64, probs [T,E] f64, idx [T,k] i32, weight [T,k] f64)"""
        x = _bf(x)
        w = np.ascontiguousarray(w, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        T, d = x.shape
        E = w.shape[0]
        logits = np.empty((T, E), dtype=np.float64)
        probs = np.empty((T, E), dtype=np.float64)
        idx = np.empty((T, k), dtype=np.int32)
        weight = np.empty((T, k), dtype=np.float64)
        self.lib.oracle_route(_p(x), T, _p(w), _p(b), d, E, k, _p(logits), _p(probs), _p(idx),
                              _p(weight))
        return logits, probs, idx, weight

    def route_variant(self, x, w, bias, k, renorm=False, bias_select_only=False):
        """route() with the routing variants: the bias moving only the
        selection, and/or the k weights renormalised over the picks.
        -> (logits [T,E] f64 (unbiased when bias_select_only), probs [T,E],
            idx [T,k] i32, weight [T,k] f64)"""
        x = _bf(x)
        w = np.ascontiguousarray(w, dtype=np.float32)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        T, d = x.shape
        E = w.shape[0]
        logits = np.empty((T, E), dtype=np.float64)
        probs = np.empty((T, E), dtype=np.float64)
        idx = np.empty((T, k), dtype=np.int32)
        weight = np.empty((T, k), dtype=np.float64)
        self.lib.oracle_route_variant(_p(x), T, _p(w), _p(b), d, E, k, int(bool(renorm)),
                                      int(bool(bias_select_only)), _p(logits), _p(probs), _p(idx),
                                      _p(weight))
        return logits, probs, idx, weight

    def rmsnorm(self, h, g, eps) -> np.ndarray:
        """x = RNE_bf16(h * g / sqrt(mean(h^2) + eps)) per token: bf16 bits [T, d]."""
        h, g = _bf(h), _bf(g)
        T, d = h.shape
        out = np.empty((T, d), dtype=np.uint16)
        self.lib.oracle_rmsnorm(_p(h), T, _p(g), float(eps), d, _p(out))
        return out

    def residual_add(self, h, y) -> np.ndarray:
        """h (bf16 bits) + y (fp64), fp64."""
        h = _bf(h)
        T, d = h.shape
        y = np.ascontiguousarray(y, dtype=np.float64)
        out = np.empty((T, d), dtype=np.float64)
        self.lib.oracle_residual_add(_p(h), T, d, _p(y), _p(out))
        return out

    def expert_ffn(self, x, blob, d, ff) -> np.ndarray:
        x = _bf(x)
        blob = _u8(blob)
        T = x.shape[0]
        out = np.empty((T, d), dtype=np.float64)
        self.lib.oracle_expert_ffn(_p(x), T, _p(blob), d, ff, _p(out))
        return out

    def expert_ffn_vec(self, xv, blob, d, ff) -> np.ndarray:
        xv = np.ascontiguousarray(xv, dtype=np.float64)
        blob = _u8(blob)
        out = np.empty(d, dtype=np.float64)
        self.lib.oracle_expert_ffn_vec(_p(xv), _p(blob), d, ff, _p(out))
        return out

    def shared_ffn(self, x, wg, wu, wd) -> np.ndarray:
        x, wg, wu, wd = _bf(x), _bf(wg), _bf(wu), _bf(wd)
        T, d = x.shape
        ffs = wg.shape[0]
        out = np.empty((T, d), dtype=np.float64)
        self.lib.oracle_shared_ffn(_p(x), T, _p(wg), _p(wu), _p(wd), d, ffs, _p(out))
        return out

    def combine(self, x, weight, slot_blobs, shared, d, ff) -> np.ndarray:
        """slot_blobs: list (length T*k) of uint8 blobs, one per (token, slot)."""
        x = _bf(x)
        T = x.shape[0]
        weight = np.ascontiguousarray(weight, dtype=np.float64)
        k = weight.shape[1]
        blobs = [_u8(b) for b in slot_blobs]
        assert len(blobs) == T * k
        ptrs = (ctypes.c_void_p * (T * k))(*[b.ctypes.data for b in blobs])
        if shared is None:
            wg = wu = wd = None
            ffs = 0
        else:
            wg, wu, wd = (_bf(a) for a in shared)
            ffs = wg.shape[0]
        y = np.empty((T, d), dtype=np.float64)
        self.lib.oracle_combine(_p(x), T, _p(weight), k, ctypes.cast(ptrs, ctypes.c_void_p),
                                _p(wg), _p(wu), _p(wd), d, ff, ffs, _p(y))
        return y

    def layer(self, x, w_router, bias, blobs, shared, d, ff, k):
        """blobs: [E, blob_bytes] uint8 (or a list of E blobs).
        -> (y [T,d] f64, idx [T,k] i32, weight [T,k] f64)"""
        x = _bf(x)
        T = x.shape[0]
        w = np.ascontiguousarray(w_router, dtype=np.float32)
        E = w.shape[0]
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        blist = [_u8(blobs[e]) for e in range(E)]
        ptrs = (ctypes.c_void_p * E)(*[a.ctypes.data for a in blist])
        if shared is None:
            wg = wu = wd = None
            ffs = 0
        else:
            wg, wu, wd = (_bf(a) for a in shared)
            ffs = wg.shape[0]
        y = np.empty((T, d), dtype=np.float64)
        idx = np.empty((T, k), dtype=np.int32)
        weight = np.empty((T, k), dtype=np.float64)
        self.lib.oracle_layer(_p(x), T, _p(w), _p(b), ctypes.cast(ptrs, ctypes.c_void_p),
                              _p(wg), _p(wu), _p(wd), d, ff, E, k, ffs, _p(y), _p(idx),
                              _p(weight))
        return y, idx, weight


_default = None


def oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
