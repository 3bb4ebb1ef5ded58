"""The bounded expert cache's bookkeeping, without a GPU (pool in host memory).

"Red Lite dev72 - bounded verify, profiling", section 1: one prepare of the
union of the rows' experts, which must not evict any expert of that union;
per-row plans of each row's experts in its own selection order.  These tests
check the slot assignment (empty slots first, then least recently used
outside the union), the union's protection, the capacity limit, the plans and
the copied bytes.
"""
import ctypes

import numpy as np
import pytest

from bit_routed_expert_top_b200 import api, synth

FMT, H, I, E = synth.FMT_Q2, 256, 128, 8
NB = synth.expert_bytes(FMT, H, I)


def make_cache(slots):
    rng = np.random.default_rng(3)
    blobs = rng.integers(0, 256, (E, NB), dtype=np.uint8)
    return api.ExpertCache(FMT, H, I, E, slots, blobs, host_pool=True), blobs


def test_empty_slots_then_least_recently_used():
    c, _ = make_cache(3)
    c.prepare([0, 1, 2])
    assert [c.slot_of(e) for e in range(E)] == [0, 1, 2, -1, -1, -1, -1, -1]
    c.prepare([3])                                  # every slot used at the same time: the first is evicted
    assert c.slot_of(0) == -1 and c.slot_of(3) == 0
    c.prepare([1, 4])                               # 1 is a hit; 2 (slot 2) is now the oldest
    assert c.slot_of(2) == -1 and c.slot_of(4) == 2 and c.slot_of(1) == 1
    st = c.stats()
    assert st == dict(hits=1, misses=5, bytes_copied=5 * NB, evictions=2)


def test_union_members_are_never_evicted():
    c, _ = make_cache(2)
    c.prepare([5])
    c.prepare([6])                                  # 5 is now the least recently used
    c.prepare([5, 7, 5])                            # union {5, 7}: 7 must take 6's slot, not 5's
    assert c.slot_of(5) >= 0 and c.slot_of(7) >= 0 and c.slot_of(6) == -1


def test_union_larger_than_the_cache_is_refused():
    c, _ = make_cache(2)
    with pytest.raises(api.RlMoeError, match="union"):
        c.prepare([1, 2, 3])
    with pytest.raises(api.RlMoeError):
        c.prepare([E])                              # expert id out of range


def test_plans_follow_each_rows_selection_order_and_hold_the_blobs():
    c, blobs = make_cache(4)
    idx = np.array([[3, 1], [1, 6]], dtype=np.int32)
    c.prepare(idx.ravel())
    plans = c.plan(idx)
    for t in range(2):
        for j in range(2):
            e = idx[t, j]
            assert ctypes.string_at(plans[t][j], NB) == blobs[e].tobytes()
    assert plans[0][1] == plans[1][0]               # expert 1, one slot for both rows
    with pytest.raises(api.RlMoeError, match="not resident"):
        c.plan(np.array([[0, 3]], dtype=np.int32))


def test_host_pool_has_no_device_table():
    c, _ = make_cache(2)
    with pytest.raises(api.RlMoeError, match="host-pool"):
        c.table()


def test_bad_arguments():
    blobs = np.zeros((E, NB), np.uint8)
    with pytest.raises(api.RlMoeError):
        api.ExpertCache(FMT, H, I, E, 0, blobs, host_pool=True)        # no slot
    with pytest.raises(api.RlMoeError):
        api.ExpertCache(FMT, H, I, E, E + 1, blobs, host_pool=True)    # more slots than experts
    with pytest.raises(api.RlMoeError):
        api.ExpertCache(7, H, I, E, 2, blobs, host_pool=True)          # unknown format
