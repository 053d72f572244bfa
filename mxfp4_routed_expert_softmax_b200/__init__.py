"""Python binding of libk3moe.so, the B200 (sm_100a) MXFP4 routed-expert MoE
layer.  Argument marshalling only: torch tensors supply device memory and
streams, every step of the layer runs in the library's CUDA kernels.  The
C contract of each call is documented in include/k3moe.h.

The library is loaded at import time; if it has not been built (``python
mxfp4_routed_expert_softmax_b200/build.py``) the import fails loudly -- there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libk3moe.so")

K3MOE_OK = 0
K3MOE_ERR_INVALID_ARGUMENT = 1
K3MOE_ERR_UNSUPPORTED_SHAPE = 2
K3MOE_ERR_WORKSPACE_TOO_SMALL = 3
K3MOE_ERR_CUDA = 4
K3MOE_ERR_DEVICE_TIMEOUT = 5
K3MOE_ERR_DEVICE_CHECK = 6

K3MOE_OUT_FP32 = 1
K3MOE_NO_SHARED = 2
K3MOE_STRICT = 4
K3MOE_RENORM_TOPK = 8
K3MOE_BIAS_SELECT_ONLY = 16
K3MOE_ONE_LAUNCH = 32


class K3moeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {k3moe_status_string(status)} ({status})"
                         + (f" [{k3moe_last_error()}]" if status == K3MOE_ERR_CUDA else ""))
        self.status = status


class k3moe_dims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("ff", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("ff_shared", ctypes.c_int32), ("flags", ctypes.c_uint32)]

    def __repr__(self):
        return (f"k3moe_dims(d={self.d}, ff={self.ff}, n_experts={self.n_experts}, "
                f"top_k={self.top_k}, ff_shared={self.ff_shared}, flags={self.flags})")


def make_dims(d, ff, n_experts, top_k, ff_shared, flags=0) -> k3moe_dims:
    return k3moe_dims(d, ff, n_experts, top_k, ff_shared, flags)


class k3moe_cache_stats(ctypes.Structure):
    _fields_ = [("requests", ctypes.c_uint64), ("hits", ctypes.c_uint64), ("fills", ctypes.c_uint64),
                ("evictions", ctypes.c_uint64)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python mxfp4_routed_expert_softmax_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_dp = ctypes.POINTER(k3moe_dims)
_SIGS = {
    "k3moe_abi_version": ([], ctypes.c_int),
    "k3moe_blob_bytes": ([_dp], _sz),
    "k3moe_workspace_size": ([_dp, _i32], _sz),
    "k3moe_host_staging_bytes": ([_dp, _i32], _sz),
    "k3moe_route": ([_vp, _i32, _vp, _vp, _dp, _vp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "k3moe_expert_ffn": ([_vp, _i32, _vp, _dp, _vp, _vp, _sz, _vp], ctypes.c_int),
    "k3moe_layer": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp, _vp, _vp, _sz, _vp],
                    ctypes.c_int),
    "k3moe_layer_residual": ([_vp, _i32, _vp, ctypes.c_float, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp,
                              _sz, _vp], ctypes.c_int),
    "k3moe_layer_from_host": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp, _sz, _vp],
                              ctypes.c_int),
    "k3moe_layer_timed": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp, _sz, _vp,
                           ctypes.POINTER(_vp), _i32, ctypes.POINTER(_i32)], ctypes.c_int),
    "k3moe_layer_noalloc": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp], ctypes.c_int),
    "k3moe_device_status": ([_vp, _vp], ctypes.c_int),
    "k3moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "k3moe_last_error": ([], ctypes.c_char_p),
    "k3moe_debug_set_fault": ([_i32, ctypes.c_uint64], ctypes.c_int),
    "k3moe_cache_slot_bytes": ([_dp], _sz),
    "k3moe_cache_create": ([_dp, _i32, _vp, _sz, _vp, ctypes.POINTER(_vp)], ctypes.c_int),
    "k3moe_cache_destroy": ([_vp], None),
    "k3moe_cache_fetch": ([_vp, _vp, _i32, _vp, _vp], ctypes.c_int),
    "k3moe_cache_plan": ([_vp, _vp, _i32, _vp, ctypes.POINTER(_i32)], ctypes.c_int),
    "k3moe_cache_get_stats": ([_vp, ctypes.POINTER(k3moe_cache_stats)], ctypes.c_int),
    "k3moe_layer_cached": ([_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dp, _vp, _vp, _vp, _sz, _vp],
                           ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res

if lib.k3moe_abi_version() != 1:
    raise ImportError("libk3moe.so ABI version mismatch")


def _ptr(t):
    """Device (or host) address of a tensor / integer address / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def check(status: int, what: str = "k3moe") -> None:
    if status != K3MOE_OK:
        raise K3moeError(status, what)


def k3moe_status_string(status: int) -> str:
    return lib.k3moe_status_string(status).decode()


def k3moe_last_error() -> str:
    return lib.k3moe_last_error().decode()


def k3moe_blob_bytes(dims: k3moe_dims) -> int:
    return lib.k3moe_blob_bytes(ctypes.byref(dims))


def k3moe_workspace_size(dims: k3moe_dims, T_max: int) -> int:
    return lib.k3moe_workspace_size(ctypes.byref(dims), T_max)


def k3moe_host_staging_bytes(dims: k3moe_dims, T: int) -> int:
    return lib.k3moe_host_staging_bytes(ctypes.byref(dims), T)


def k3moe_route(x, T, w_router, bias, dims, idx, weight, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_route(_ptr(x), T, _ptr(w_router), _ptr(bias), ctypes.byref(dims), _ptr(idx),
                           _ptr(weight), _ptr(ws), ws_bytes, _stream(stream))


def k3moe_expert_ffn(x, T, blob, dims, out, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_expert_ffn(_ptr(x), T, _ptr(blob), ctypes.byref(dims), _ptr(out), _ptr(ws),
                                ws_bytes, _stream(stream))


def k3moe_layer(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims, y,
                idx_out, w_out, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_layer(_ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(expert_blobs),
                           _ptr(shared_wg), _ptr(shared_wu), _ptr(shared_wd), ctypes.byref(dims),
                           _ptr(y), _ptr(idx_out), _ptr(w_out), _ptr(ws), ws_bytes,
                           _stream(stream))


def k3moe_layer_residual(h, T, norm_w, eps, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd,
                         dims, h_out, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_layer_residual(_ptr(h), T, _ptr(norm_w), float(eps), _ptr(w_router), _ptr(bias),
                                    _ptr(expert_blobs), _ptr(shared_wg), _ptr(shared_wu), _ptr(shared_wd),
                                    ctypes.byref(dims), _ptr(h_out), _ptr(ws), ws_bytes, _stream(stream))


def k3moe_layer_noalloc(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims, y,
                        stream=None) -> int:
    return lib.k3moe_layer_noalloc(_ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(expert_blobs),
                                   _ptr(shared_wg), _ptr(shared_wu), _ptr(shared_wd),
                                   ctypes.byref(dims), _ptr(y), _stream(stream))


def k3moe_layer_from_host(x_host, T, w_router, bias, expert_blobs, shared_wg, shared_wu,
                          shared_wd, dims, y_host, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_layer_from_host(_ptr(x_host), T, _ptr(w_router), _ptr(bias),
                                     _ptr(expert_blobs), _ptr(shared_wg), _ptr(shared_wu),
                                     _ptr(shared_wd), ctypes.byref(dims), _ptr(y_host), _ptr(ws),
                                     ws_bytes, _stream(stream))


def k3moe_layer_timed(x, T, w_router, bias, expert_blobs, shared_wg, shared_wu, shared_wd, dims,
                      y, ws, events, ws_bytes=None, stream=None):
    """events: list of torch.cuda.Event(enable_timing=True).  -> (status, n_kernels)"""
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    for ev in events:
        if ev.cuda_event == 0:
            ev.record()  # materialise the event handle on the current device
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    nk = ctypes.c_int32(0)
    st = lib.k3moe_layer_timed(_ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(expert_blobs),
                               _ptr(shared_wg), _ptr(shared_wu), _ptr(shared_wd),
                               ctypes.byref(dims), _ptr(y), _ptr(ws), ws_bytes, _stream(stream),
                               arr, len(events), ctypes.byref(nk))
    return st, nk.value


def k3moe_device_status(ws, stream=None) -> int:
    """ws=None: the built-in scratch of k3moe_layer_noalloc on this device."""
    return lib.k3moe_device_status(_ptr(ws), _stream(stream))


def k3moe_debug_set_fault(mode: int, wait_limit_ns: int = 0) -> int:
    """Failure-path tests only: mode 1 makes the next layer calls' bounded
    device waits run out (no GPU fault); wait_limit_ns bounds every wait
    (0: the default).  Reset with (0, 0)."""
    return lib.k3moe_debug_set_fault(mode, wait_limit_ns)


class ExpertCache:
    """Handle of a k3moe_cache (argument marshalling only; the policy and the
    copies are the library's).  slot_mem: device tensor of at least
    n_slots * k3moe_cache_slot_bytes(dims) bytes; host_blob_ptrs: E host
    addresses (kept alive by the caller)."""

    def __init__(self, dims, n_slots, slot_mem, host_blob_ptrs):
        import numpy as np
        self._ptrs = np.ascontiguousarray(np.asarray(host_blob_ptrs, dtype=np.uint64))
        h = ctypes.c_void_p()
        nbytes = slot_mem.numel() * slot_mem.element_size() if hasattr(slot_mem, "numel") else 0
        check(lib.k3moe_cache_create(ctypes.byref(dims), n_slots, _ptr(slot_mem), nbytes,
                                     self._ptrs.ctypes.data, ctypes.byref(h)), "k3moe_cache_create")
        self.handle = h

    def plan(self, experts):
        import numpy as np
        e = np.ascontiguousarray(np.asarray(experts, dtype=np.int32))
        out = np.empty(max(1, e.size), dtype=np.int32)
        n = ctypes.c_int32(0)
        st = lib.k3moe_cache_plan(self.handle, e.ctypes.data, e.size, out.ctypes.data, ctypes.byref(n))
        return st, out[:n.value].tolist()

    def fetch(self, experts, ptr_table, stream=None) -> int:
        import numpy as np
        e = np.ascontiguousarray(np.asarray(experts, dtype=np.int32))
        return lib.k3moe_cache_fetch(self.handle, e.ctypes.data, e.size, _ptr(ptr_table), _stream(stream))

    def stats(self) -> dict:
        st = k3moe_cache_stats()
        check(lib.k3moe_cache_get_stats(self.handle, ctypes.byref(st)), "k3moe_cache_get_stats")
        return {"requests": st.requests, "hits": st.hits, "fills": st.fills, "evictions": st.evictions}

    def close(self):
        if self.handle:
            lib.k3moe_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        self.close()


def k3moe_cache_slot_bytes(dims: k3moe_dims) -> int:
    return lib.k3moe_cache_slot_bytes(ctypes.byref(dims))


def k3moe_layer_cached(cache, x, T, w_router, bias, ptr_table, shared_wg, shared_wu, shared_wd, dims, y,
                       idx_host, ws, ws_bytes=None, stream=None) -> int:
    ws_bytes = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return lib.k3moe_layer_cached(cache.handle, _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(ptr_table),
                                  _ptr(shared_wg), _ptr(shared_wu), _ptr(shared_wd), ctypes.byref(dims),
                                  _ptr(y), _ptr(idx_host), _ptr(ws), ws_bytes, _stream(stream))


def new_workspace(dims: k3moe_dims, T_max: int, device="cuda", host_staging: bool = False):
    """A zero-filled, 256-byte aligned workspace tensor (uint8) for `dims`."""
    import torch
    n = k3moe_workspace_size(dims, T_max)
    if n == 0:
        raise K3moeError(K3MOE_ERR_UNSUPPORTED_SHAPE, "k3moe_workspace_size")
    if host_staging:
        n += k3moe_host_staging_bytes(dims, T_max)
    return torch.zeros(n, dtype=torch.uint8, device=device)
