"""The C-ABI library builds for sm_100a, loads on a machine without a GPU,
exports every symbol include/k3moe.h declares, and rejects bad arguments
before touching the device."""
import ctypes
import importlib.util
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "k3moe.h")


def _build():
    spec = importlib.util.spec_from_file_location(
        "k3moe_build", os.path.join(ROOT, "mxfp4_routed_expert_softmax_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def m():
    _build()
    import mxfp4_routed_expert_softmax_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(k3moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("k3moe_route", "k3moe_expert_ffn", "k3moe_layer", "k3moe_workspace_size",
                 "k3moe_device_status", "k3moe_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(m):
    lib = ctypes.CDLL(m.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_sizes(m):
    d = m.make_dims(7168, 1536, 896, 16, 1536)
    assert m.k3moe_blob_bytes(d) == 17547264
    assert m.k3moe_workspace_size(d, 8) > 0
    assert m.k3moe_workspace_size(m.make_dims(100, 1536, 896, 16, 1536), 8) == 0
    assert m.k3moe_workspace_size(d, 0) == 0


def test_workspace_grows_with_the_grouped_prefill_region(m):
    """Up to 8 tokens: the decode scratch only; more: plus the grouped prefill
    region (per-token pieces, groups, per-(token, slot) outputs), which grows
    with the pass size and stops growing at the pass limit."""
    d = m.make_dims(7168, 1536, 896, 16, 1536)
    w8 = m.k3moe_workspace_size(d, 8)
    assert m.k3moe_workspace_size(d, 1) == w8
    w9, w512, w4096 = (m.k3moe_workspace_size(d, t) for t in (9, 512, 4096))
    assert w8 < w9 < w512 < w4096
    # outputs per (token, slot) dominate: (k+1)*d fp32 per token
    assert w4096 - w512 > (4096 - 512) * 17 * 7168 * 4
    assert m.k3moe_workspace_size(d, 8192) == m.k3moe_workspace_size(d, 100000)


def test_k3_decode_scratch_fits_the_built_in_buffer(m):
    """k3moe_layer_noalloc serves shapes whose decode scratch fits its 16 MiB
    buffer: the K3 shape must (with and without the shared expert)."""
    for ffs in (1536, 0):
        assert 0 < m.k3moe_workspace_size(m.make_dims(7168, 1536, 896, 16, ffs), 8) <= 16 << 20


BIG = 1 << 30
A16 = 0x10000  # a fake 16-byte aligned address: never dereferenced, calls fail validation first


@pytest.mark.parametrize("dims,want", [
    ((100, 1536, 896, 16, 1536, 0), 2),      # d not a multiple of 64
    ((7168, 1000, 896, 16, 1536, 0), 2),     # ff not a multiple of 64
    ((7168, 1536, 0, 1, 1536, 0), 2),        # no experts
    ((7168, 1536, 2048, 16, 1536, 0), 2),    # too many experts
    ((7168, 1536, 896, 0, 1536, 0), 1),      # k = 0
    ((7168, 1536, 896, 33, 1536, 0), 1),     # k > 32
    ((256, 128, 4, 5, 128, 0), 1),           # k > E
    ((7168, 1536, 896, 16, 100, 0), 2),      # shared width not a multiple of 64
    ((7168, 1536, 896, 16, 1536, 64), 1),    # unknown flag
    ((7168, 8192, 896, 16, 1536, 0), 2),     # down tile does not fit shared memory
])
def test_layer_rejects_bad_dims(m, dims, want):
    d = m.make_dims(*dims)
    st = m.lib.k3moe_layer(A16, 1, A16, None, A16, A16, A16, A16, ctypes.byref(d), A16, None, None,
                           A16 * 16, BIG, None)
    assert st == want


def test_layer_rejects_bad_pointers(m):
    d = m.make_dims(256, 128, 32, 4, 128)
    ws = A16 * 16

    def call(x=A16, T=4, wr=A16, blobs=A16, sg=A16, y=A16, wsp=ws, wsb=BIG, dims=d):
        return m.lib.k3moe_layer(x, T, wr, None, blobs, sg, sg, sg, ctypes.byref(dims), y, None,
                                 None, wsp, wsb, None)

    assert call(x=None) == 1
    assert call(x=A16 + 2) == 1
    assert call(T=0) == 1
    assert call(wr=None) == 1
    assert call(blobs=None) == 1
    assert call(sg=None) == 1
    assert call(y=None) == 1
    assert call(wsp=ws + 16) == 1
    assert call(wsb=16) == 3
    # the shared pointers may be null when the shared expert is switched off
    d2 = m.make_dims(256, 128, 32, 4, 128, m.K3MOE_NO_SHARED)
    assert m.lib.k3moe_layer(A16, 4, A16, None, A16, None, None, None, ctypes.byref(d2), A16, None,
                             None, ws, 16, None) == 3


def test_route_and_expert_ffn_reject(m):
    d = m.make_dims(256, 128, 32, 4, 128)
    assert m.lib.k3moe_route(None, 4, A16, None, ctypes.byref(d), A16, A16, A16 * 16, BIG, None) == 1
    assert m.lib.k3moe_route(A16, 4, A16, None, ctypes.byref(d), A16, A16, A16 * 16, 8, None) == 3
    assert m.lib.k3moe_expert_ffn(A16, 4, A16 + 4, ctypes.byref(d), A16, A16 * 16, BIG, None) == 1
    assert m.lib.k3moe_expert_ffn(A16, 4, A16, ctypes.byref(d), A16, A16 * 16, 8, None) == 3
    assert m.lib.k3moe_layer_from_host(None, 4, A16, None, A16, A16, A16, A16, ctypes.byref(d),
                                       A16, A16 * 16, BIG, None) == 1


def test_layer_residual_rejects(m):
    """The pre-norm entry checks its norm weights and eps, then everything
    k3moe_layer checks, before any launch."""
    d = m.make_dims(256, 128, 32, 4, 128)
    ws = A16 * 16

    def call(h=A16, g=A16, eps=1e-6, wsb=BIG, dims=d):
        return m.lib.k3moe_layer_residual(h, 4, g, eps, A16, None, A16, A16, A16, A16, ctypes.byref(dims), A16,
                                          ws, wsb, None)

    assert call(g=None) == 1
    assert call(g=A16 + 8) == 1
    assert call(eps=-1.0) == 1
    assert call(eps=float("nan")) == 1
    assert call(eps=float("inf")) == 1
    assert call(h=None) == 1
    assert call(wsb=16) == 3
    assert call(dims=m.make_dims(100, 128, 32, 4, 128)) == 2


def test_status_strings(m):
    for s in range(7):
        assert m.k3moe_status_string(s) not in ("", "unknown status")
    assert m.k3moe_status_string(99) == "unknown status"


def test_product_path_has_no_oracle_reference():
    """The CUDA library and its binding never reach the oracle or a CPU fallback."""
    pkg = os.path.join(ROOT, "mxfp4_routed_expert_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


@pytest.mark.parametrize("flag", ["K3MOE_STRICT", "K3MOE_RENORM_TOPK", "K3MOE_BIAS_SELECT_ONLY", "K3MOE_ONE_LAUNCH"])
def test_option_flags_are_accepted(m, flag):
    """The option flags pass validation (the call then fails only on the tiny
    workspace size, before anything is launched)."""
    d = m.make_dims(256, 128, 32, 4, 128, getattr(m, flag) | m.K3MOE_OUT_FP32)
    st = m.lib.k3moe_layer(A16, 4, A16, None, A16, A16, A16, A16, ctypes.byref(d), A16, None, None,
                           A16 * 16, 16, None)
    assert st == m.K3MOE_ERR_WORKSPACE_TOO_SMALL


def test_fault_hook_validates_and_resets(m):
    assert m.k3moe_debug_set_fault(2, 0) == m.K3MOE_ERR_INVALID_ARGUMENT
    assert m.k3moe_debug_set_fault(-1, 0) == m.K3MOE_ERR_INVALID_ARGUMENT
    assert m.k3moe_debug_set_fault(1, 1000000) == m.K3MOE_OK
    assert m.k3moe_debug_set_fault(0, 0) == m.K3MOE_OK
