"""Residency manager bookkeeping on a host-only pool (no device: page tables and
LRU order only).  A batch's adapters become resident, missing ones are loaded,
and when pages run out the least recently used adapters outside the batch are
evicted (ties: lowest id); a batch that cannot fit, or names an unknown
adapter, changes nothing."""
import ctypes

import pytest

import segmented_rank_gemm_sgmv_b200 as sg

R = 16
PROJ = [(512, 512)]
PER_ADAPTER = sg.AdapterPool.pages_needed(PROJ, R)  # 32 pages


def _resident(pool, ids):
    out = []
    for a in ids:
        r = ctypes.c_int32()
        if sg.load_library().sgmv_pool_adapter_rank(pool.handle, a, ctypes.byref(r)) == 0:
            out.append(a)
    return out


@pytest.fixture()
def setup():
    pool = sg.AdapterPool(PROJ, num_pages=2 * PER_ADAPTER, page_elems=512, max_rank=R, device=-1)
    res = sg.Residency(pool)
    for a in range(5):
        res.register(a, R)
    return pool, res


def test_lru_eviction_order(setup):
    pool, res = setup
    assert res.prepare([0, 1, 1, -1]) == 2
    assert _resident(pool, range(5)) == [0, 1]
    assert res.prepare([0]) == 0                      # hit: 0 becomes the most recent
    assert res.prepare([2]) == 1                      # evicts 1 (least recently used)
    assert _resident(pool, range(5)) == [0, 2]
    assert res.prepare([1, 2]) == 1                   # evicts 0, never 2 (in the batch)
    assert _resident(pool, range(5)) == [1, 2]
    s = res.stats()
    assert (s.hits, s.misses, s.evictions, s.bytes_loaded) == (2, 4, 2, 0)


def test_ties_take_the_lowest_id_first(setup):
    pool, res = setup
    assert res.prepare([3, 4]) == 2                   # both last used in the same batch
    assert res.prepare([0]) == 1
    assert _resident(pool, range(5)) == [0, 4]       # 3 went first


def test_batch_that_cannot_fit_changes_nothing(setup):
    pool, res = setup
    res.prepare([0, 1])
    with pytest.raises(sg.SgmvError) as e:
        res.prepare([2, 3, 4])                       # three adapters, room for two
    assert e.value.status == 4                       # SGMV_ERR_OUT_OF_PAGES
    assert _resident(pool, range(5)) == [0, 1]
    assert res.stats().evictions == 0


def test_unknown_adapter_is_refused(setup):
    pool, res = setup
    with pytest.raises(sg.SgmvError) as e:
        res.prepare([0, 9])
    assert e.value.status == 3                       # SGMV_ERR_NOT_RESIDENT
    assert _resident(pool, range(5)) == []
    res.unregister(4)
    with pytest.raises(sg.SgmvError):
        res.prepare([4])


def test_adapters_loaded_directly_are_the_oldest():
    pool = sg.AdapterPool(PROJ, num_pages=2 * PER_ADAPTER, page_elems=512, max_rank=R, device=-1)
    pool.load(7, R)                                  # resident before the manager exists
    res = sg.Residency(pool)
    for a in range(3):
        res.register(a, R)
    res.prepare([0])
    res.prepare([1])                                 # evicts 7, not 0
    assert _resident(pool, [0, 1, 2, 7]) == [0, 1]


# ---------------------------------------------------------------- property-based
from hypothesis import given, settings, HealthCheck
from hypothesis import strategies as st


@settings(max_examples=120, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(batches=st.lists(st.lists(st.sampled_from([-1, 0, 1, 2, 3, 4, 5]), min_size=1, max_size=6),
                        min_size=1, max_size=25),
       room=st.integers(1, 4))
def test_lru_against_a_simulation(batches, room):
    """Random batches over six equal-rank adapters with room for `room` of them: the
    residency manager's result (what is resident, what each batch loaded, hits, misses,
    evictions) equals an independent LRU simulation -- batch adapters touched, misses
    loaded, least recently used outside the batch evicted first (ties: lowest id), a
    batch that cannot fit refused with nothing changed."""
    pool = sg.AdapterPool(PROJ, num_pages=room * PER_ADAPTER, page_elems=512, max_rank=R, device=-1)
    res = sg.Residency(pool)
    for a in range(6):
        res.register(a, R)
    resident, last, tick = set(), {}, 0
    hits = misses = evictions = 0
    for batch in batches:
        want = sorted({a for a in batch if a >= 0})
        tick += 1
        if len(want) > room:
            with pytest.raises(sg.SgmvError) as e:
                res.prepare(batch)
            assert e.value.status == 4
        else:
            miss = [a for a in want if a not in resident]
            hits += len(want) - len(miss)
            misses += len(miss)
            for a in want:
                if a in resident:
                    last[a] = tick
            while len(resident) + len(miss) > room:
                victim = min((a for a in resident if a not in want), key=lambda a: (last[a], a))
                resident.discard(victim)
                evictions += 1
            for a in miss:
                resident.add(a)
                last[a] = tick
            assert res.prepare(batch) == len(miss)
        assert _resident(pool, range(6)) == sorted(resident)
        s = res.stats()
        assert (s.hits, s.misses, s.evictions) == (hits, misses, evictions)
