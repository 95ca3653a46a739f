"""Host-side LRU slot manager (ft_slot_*), exercised in its host-only mode:
bookkeeping against a small reference LRU, the capacity guard, missing banks
and injected copy failures.  No GPU is needed."""
import collections
import ctypes

import numpy as np
import pytest

from moe_expert_layer_renorm_b200 import _lib
from moe_expert_layer_renorm_b200.build import build
from moe_expert_layer_renorm_b200.layer import SlotManager


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


class RefLRU:
    """Reference policy: an OrderedDict from key to slot, most recent last."""

    def __init__(self, cap):
        self.cap = cap
        self.d = collections.OrderedDict()
        self.free = list(range(cap - 1, -1, -1))
        self.hits = self.misses = self.evictions = 0

    def acquire(self, layer, ids):
        want = list(dict.fromkeys(ids))
        assert len(want) <= self.cap
        keys = [(layer, e) for e in want]
        for k in keys:
            if k in self.d:
                self.d.move_to_end(k)
                self.hits += 1
        table = {}
        for k in keys:
            if k in self.d:
                table[k[1]] = self.d[k]
                continue
            if self.free:
                slot = self.free.pop()
            else:
                victim = next(v for v in self.d if v not in keys)
                slot = self.d.pop(victim)
                self.evictions += 1
            self.d[k] = slot
            table[k[1]] = slot
            self.misses += 1
        return table


def _mgr(cap, E=16, layers=3):
    lay = _lib.slot_layout(256, 512, cap)
    m = SlotManager(cap, lay, host_only=True)
    bank = (ctypes.c_uint8 * 16)()
    for layer in range(layers):
        for e in range(E):
            m.register_host(layer, e, ctypes.addressof(bank))
    return m, bank


def _acquire(m, layer, ids, E=16):
    table = (ctypes.c_int32 * E)()
    m.acquire(layer, ids, ctypes.addressof(table), E)
    return list(table)


def test_lru_policy_matches_reference():
    cap, E = 6, 16
    m, _bank = _mgr(cap, E)
    ref = RefLRU(cap)
    g = np.random.default_rng(0)
    for step in range(400):
        layer = int(g.integers(0, 3))
        n = int(g.integers(1, cap + 1))
        ids = [int(v) for v in g.integers(0, E, size=n)]
        want = ref.acquire(layer, ids)
        got = _acquire(m, layer, ids, E)
        for e in range(E):
            assert got[e] == want.get(e, -1), (step, e)
        slots = [got[e] for e in set(ids)]
        assert len(set(slots)) == len(slots)          # distinct experts, distinct slots
        assert all(0 <= s < cap for s in slots)
    st = m.stats()
    assert (st["hits"], st["misses"], st["evictions"]) == (ref.hits, ref.misses, ref.evictions)
    assert st["bytes_h2d"] == ref.misses * int(_lib.slot_layout(256, 512, cap).slot_bytes)
    m.close()


def test_repeated_request_is_all_hits():
    m, _bank = _mgr(4)
    _acquire(m, 0, [1, 2, 3])
    before = m.stats()
    t1 = _acquire(m, 0, [3, 2, 1, 1])
    after = m.stats()
    assert after["misses"] == before["misses"] and after["hits"] == before["hits"] + 3
    assert sorted(t1[e] for e in (1, 2, 3)) == [0, 1, 2]


def test_capacity_guard():
    m, _bank = _mgr(3)
    with pytest.raises(_lib.FtError) as ei:
        _acquire(m, 0, [0, 1, 2, 3])
    assert ei.value.code == _lib.FT_ERR_CAPACITY
    assert m.stats()["misses"] == 0          # nothing changed
    _acquire(m, 0, [0, 1, 2])                 # exactly full works


def test_missing_host_bank_is_reported():
    lay = _lib.slot_layout(256, 512, 4)
    m = SlotManager(4, lay, host_only=True)
    with pytest.raises(_lib.FtError) as ei:
        _acquire(m, 0, [5])
    assert ei.value.code == _lib.FT_ERR_NOT_RESIDENT


def test_injected_copy_failure_leaves_state_consistent():
    m, _bank = _mgr(4)
    _acquire(m, 0, [0, 1])
    m.inject_copy_failures(1)
    with pytest.raises(_lib.FtError) as ei:
        _acquire(m, 0, [2])
    assert ei.value.code == _lib.FT_ERR_CUDA
    # the failed fill is not resident; a retry misses again and succeeds
    misses = m.stats()["misses"]
    t = _acquire(m, 0, [2, 0, 1])
    assert m.stats()["misses"] == misses + 1
    assert len({t[0], t[1], t[2]}) == 3


def test_bad_expert_id():
    m, _bank = _mgr(4)
    with pytest.raises(_lib.FtError) as ei:
        _acquire(m, 0, [16])
    assert ei.value.code == _lib.FT_ERR_INVALID_ARG


def test_layers_are_separate_keys():
    m, _bank = _mgr(4)
    a = _acquire(m, 0, [7])
    b = _acquire(m, 1, [7])
    assert a[7] != b[7]
    assert m.stats()["misses"] == 2


def test_fills_coalesce_into_runs_of_consecutive_slots_and_banks():
    # banks of one layer in one block: the misses of a call become one copy per run of
    # consecutive slots whose banks are consecutive too, whatever the request order
    cap, E = 8, 16
    lay = _lib.slot_layout(256, 512, cap)
    m = SlotManager(cap, lay, host_only=True)
    nbytes = int(lay.slot_bytes)
    block = (ctypes.c_uint8 * (nbytes * E))()
    base = ctypes.addressof(block)
    for e in range(E):
        m.register_host(0, e, base + e * nbytes)
    t = _acquire(m, 0, [3, 0, 2, 1])            # four free slots, banks 0..3: one run
    st = m.stats()
    assert st["misses"] == 4 and st["copies"] == 1
    assert [t[e] for e in range(4)] == [0, 1, 2, 3]   # slots follow the banks' order
    t = _acquire(m, 0, [9, 5])                   # banks 5 and 9 are not adjacent: two copies
    st2 = m.stats()
    assert st2["misses"] == 6 and st2["copies"] == 3
    assert sorted([t[5], t[9]]) == [4, 5]
