"""The expert cache's policy (host-side bookkeeping, no GPU): least recently
used over the slots, no requested expert evicted by another of the same
request, free slots first, lowest slot on ties; refused requests change
nothing.  Checked against a plain Python model of the same policy on random
request streams, and on hand cases."""
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def m():
    spec = importlib.util.spec_from_file_location(
        "k3moe_build", os.path.join(ROOT, "mxfp4_routed_expert_softmax_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import mxfp4_routed_expert_softmax_b200 as m
    return m


class FakeSlots:
    """A stand-in for the slot memory: an aligned address that is never used
    (plan() makes no copy)."""

    def __init__(self, nbytes):
        self.addr = 1 << 40
        self.nbytes = nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def make(m, E, S, d=256, ff=128):
    dims = m.make_dims(d, ff, E, min(4, E), 128)
    sb = m.k3moe_cache_slot_bytes(dims)
    assert sb % 256 == 0 and sb >= 3 * d * ff * 17 // 32
    return m.ExpertCache(dims, S, FakeSlots(S * sb), [0x1000 + 64 * e for e in range(E)])


class LruModel:
    def __init__(self, S):
        self.S = S
        self.slot_expert = [-1] * S
        self.last = [0] * S
        self.clock = 0

    def plan(self, req):
        distinct = list(dict.fromkeys(req))
        if len(distinct) > self.S:
            return None
        self.clock += 1
        now = self.clock
        for e in distinct:
            if e in self.slot_expert:
                self.last[self.slot_expert.index(e)] = now
        fills = []
        for e in distinct:
            if e in self.slot_expert:
                continue
            cand = [s for s in range(self.S) if self.last[s] != now]
            s = min(cand, key=lambda q: (self.last[q], q))
            self.slot_expert[s] = e
            self.last[s] = now
            fills.append(e)
        return fills


def test_cache_matches_lru_model(m):
    rng = np.random.default_rng(5)
    E, S = 40, 12
    c = make(m, E, S)
    model = LruModel(S)
    req_total = hit_total = 0
    for step in range(400):
        n = int(rng.integers(1, 14))
        # skewed popularity, as routed tokens are
        req = (rng.zipf(1.3, n) - 1) % E
        want = model.plan(req.tolist())
        st, got = c.plan(req)
        if want is None:
            assert st == m.K3MOE_ERR_INVALID_ARGUMENT
            continue
        assert st == m.K3MOE_OK
        assert got == want, (step, req.tolist())
        d = len(set(req.tolist()))
        req_total += d
        hit_total += d - len(want)
    s = c.stats()
    assert s["requests"] == req_total and s["hits"] == hit_total
    assert s["fills"] == req_total - hit_total
    assert s["evictions"] == s["fills"] - S  # every slot was filled once before evictions began


def test_cache_hand_cases(m):
    c = make(m, 10, 3)
    assert c.plan([1, 2, 1]) == (m.K3MOE_OK, [1, 2])        # free slots, repeats once
    assert c.plan([3]) == (m.K3MOE_OK, [3])                 # the last free slot
    assert c.plan([1, 4]) == (m.K3MOE_OK, [4])              # 1 is used now: evict 2 (older than 3)
    assert c.plan([2, 3, 4]) == (m.K3MOE_OK, [2])           # 3, 4 requested: 1 goes
    st, _ = c.plan([5, 6, 7, 8])                             # more than the slots: refused
    assert st == m.K3MOE_ERR_INVALID_ARGUMENT
    assert c.plan([2, 3, 4]) == (m.K3MOE_OK, [])            # unchanged by the refusal
    st, _ = c.plan([10])                                     # out of range
    assert st == m.K3MOE_ERR_INVALID_ARGUMENT
    assert c.stats()["evictions"] == 2


def test_cache_rejects_bad_arguments(m):
    import ctypes
    dims = m.make_dims(256, 128, 8, 2, 128)
    sb = m.k3moe_cache_slot_bytes(dims)
    h = ctypes.c_void_p()
    ptrs = (ctypes.c_void_p * 8)(*[0x1000] * 8)
    assert m.lib.k3moe_cache_create(ctypes.byref(dims), 2, 1 << 40, 2 * sb - 1, ptrs, ctypes.byref(h)) == 1
    assert m.lib.k3moe_cache_create(ctypes.byref(dims), 0, 1 << 40, 2 * sb, ptrs, ctypes.byref(h)) == 1
    assert m.lib.k3moe_cache_create(ctypes.byref(dims), 2, (1 << 40) + 16, 2 * sb, ptrs, ctypes.byref(h)) == 1
    ptrs[3] = None
    assert m.lib.k3moe_cache_create(ctypes.byref(dims), 2, 1 << 40, 2 * sb, ptrs, ctypes.byref(h)) == 1
