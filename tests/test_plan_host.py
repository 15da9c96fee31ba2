"""Segment builder and dispatch (host, no GPU), bit-exact against the oracle's
brute-force grouping ("SGMV: the kernel that holds it all up": tokens grouped by
adapter; large segments to tensor cores, small ones to the gather path)."""
import json
import os

import numpy as np
import pytest

import oracle
import segmented_rank_gemm_sgmv_b200 as sg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _pool(ranks, projs=((512, 1024), (1024, 512))):
    pool = sg.AdapterPool(list(projs), num_pages=200000, page_elems=512, max_rank=128, device=-1)
    pool.shuffle_free_pages(11)
    for a, r in ranks.items():
        pool.load(a, r)
    return pool


def _check_plan(plan, pool, ids, ranks, thr):
    tix, off, seg_ad = oracle.group_by_adapter(ids)
    assert plan.token_idx.tolist() == tix
    assert plan.seg_offsets.tolist() == (off if seg_ad else [0])
    assert plan.seg_adapter.tolist() == seg_ad
    assert plan.seg_rank.tolist() == [ranks[a] for a in seg_ad]
    assert plan.num_rows == len(tix)
    assert plan.max_rank == max([ranks[a] for a in seg_ad], default=0)
    # every work record repeats its segment's rank and page-table bases, per projection
    a_pt, b_pt = plan.seg_pt(0), plan.seg_pt(1)
    for recs in (plan.simt_records, plan.tc_records):
        for rec in recs:
            for p in range(len(pool.projections)):
                seg = int(rec[p, 0])
                assert rec[p, 3] == ranks[seg_ad[seg]]
                assert rec[p, 4] == a_pt[seg, p] and rec[p, 5] == b_pt[seg, p]
                assert tuple(rec[p, :3]) == tuple(rec[0, :3])
    # dispatch covers every row of every non-empty, non-zero-rank segment exactly once
    covered = []
    for items, lim, is_tc in ((plan.simt_items, 4, False), (plan.tc_tiles, 128, True)):
        for s, b, e in items.tolist():
            n = off[s + 1] - off[s]
            assert off[s] <= b < e <= off[s + 1] and e - b <= lim
            assert (n >= thr) == is_tc
            assert ranks[seg_ad[s]] > 0
            covered.extend(range(b, e))
    want = [i for s, a in enumerate(seg_ad) if ranks[a] > 0 for i in range(off[s], off[s + 1])]
    assert sorted(covered) == want


@pytest.mark.parametrize("seed", range(6))
def test_plan_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    ranks = {a: int(rng.choice([0, 8, 16, 24, 64, 128])) for a in range(0, 60, 3)}
    pool = _pool(ranks)
    T = int(rng.choice([1, 7, 64, 300, 1000]))
    resident = list(ranks)
    ids = rng.choice(resident + [-1], size=T).astype(np.int32)
    if seed % 2 == 0:   # a long segment
        ids[: T // 2] = resident[1]
    for thr in (0, 1, 16, 10 ** 9):
        plan = pool.plan(ids, long_threshold=thr)
        _check_plan(plan, pool, ids.tolist(), ranks, plan.plan.long_threshold)


def test_segment_figure_plan():
    with open(os.path.join(GOLDEN, "segment_figure.json")) as f:
        g = json.load(f)
    ranks = {int(k): v for k, v in g["adapter_rank"].items()}
    pool = _pool(ranks)
    ids = [r["adapter"] for r in g["requests"]]
    plan = pool.plan(ids)
    assert plan.seg_adapter.tolist() == [s["adapter"] for s in g["expected_segments"]]
    assert plan.seg_rank.tolist() == [s["rank"] for s in g["expected_segments"]]
    assert np.diff(plan.seg_offsets).tolist() == [len(s["requests"]) for s in g["expected_segments"]]


def test_seg_pt_points_at_the_adapters_pages():
    ranks = {5: 16, 9: 8}
    pool = _pool(ranks)
    plan = pool.plan([9, 5, 9])
    a_pt, b_pt = plan.seg_pt(0), plan.seg_pt(1)
    # entries of one (adapter, projection, matrix) are contiguous from the base
    assert a_pt[0, 0] < b_pt[0, 0] < a_pt[0, 1] < b_pt[0, 1]
    assert b_pt[0, 0] - a_pt[0, 0] == 16 * 512 // 512
    assert a_pt[0, 1] - b_pt[0, 0] == 16 * 1024 // 512


def test_empty_and_all_minus_one():
    pool = _pool({1: 8})
    for ids in ([], [-1, -1, -1]):
        plan = pool.plan(ids)
        assert plan.num_rows == 0 and plan.plan.num_segments == 0
        assert plan.plan.num_simt_items == 0 and plan.plan.num_tc_tiles == 0


def test_errors():
    pool = _pool({1: 8})
    with pytest.raises(sg.SgmvError) as e:
        pool.plan([1, 2])
    assert e.value.status == 3
    with pytest.raises(sg.SgmvError) as e:
        pool.plan([1, -2])
    assert e.value.status == 1


def test_simt_items_largest_rank_first():
    """SIMT work items come largest rank first (stable within a rank), so that
    their CTAs are scheduled before the smaller ones."""
    ranks = {0: 8, 1: 64, 2: 16, 3: 64, 4: 32}
    pool = _pool(ranks)
    ids = np.asarray([0, 1, 2, 3, 4] * 3 + [1, 3], dtype=np.int32)
    plan = pool.plan(ids, long_threshold=10 ** 9)
    rec_ranks = [int(r[0, 3]) for r in plan.simt_records]
    assert rec_ranks == sorted(rec_ranks, reverse=True)
    segs = [int(r[0, 0]) for r in plan.simt_records]
    for a, b in zip(range(len(segs) - 1), range(1, len(segs))):
        if rec_ranks[a] == rec_ranks[b]:
            assert segs[a] <= segs[b]


def test_default_dispatch_needs_one_full_tile_of_long_rows():
    """With the default threshold (16 rows), segments go to the tensor-core kernels only
    when the long segments hold at least 128 rows in total; otherwise every segment is
    cut into SIMT items and the plan reports the threshold as never reached.  An
    explicit threshold is applied as given."""
    ranks = {0: 8, 1: 16, 2: 16, 3: 8}
    few = [0] * 16 + [1] * 16 + [2] * 16 + [3] * 16                    # 64 long rows
    pool = _pool(ranks)
    plan = pool.plan(few)
    assert plan.plan.num_tc_tiles == 0 and plan.plan.num_simt_items == 16
    assert plan.plan.long_threshold == 2 ** 31 - 1
    _check_plan(plan, pool, few, ranks, plan.plan.long_threshold)
    plan = pool.plan(few, long_threshold=16)                             # explicit: applied as given
    assert plan.plan.num_tc_tiles == 4 and plan.plan.long_threshold == 16
    many = [0] * 100 + [1] * 28 + [2] * 3                                # 128 long rows
    plan = pool.plan(many)
    assert plan.plan.long_threshold == 16 and plan.plan.num_tc_tiles == 2 and plan.plan.num_simt_items == 1
    _check_plan(plan, pool, many, ranks, 16)


# ---------------------------------------------------------------- property-based
from hypothesis import given, settings, HealthCheck
from hypothesis import strategies as st

_RANKS = {a: r for a, r in zip(range(0, 24, 2), [0, 8, 16, 5, 24, 64, 128, 1, 32, 16, 8, 40])}
_POOL = None


def _shared_pool():
    global _POOL
    if _POOL is None:
        _POOL = _pool(_RANKS)
    return _POOL


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(ids=st.lists(st.sampled_from(list(_RANKS) + [-1]), min_size=0, max_size=400),
       runs=st.lists(st.tuples(st.sampled_from(list(_RANKS)), st.integers(1, 200)), max_size=3),
       thr=st.sampled_from([0, 1, 2, 5, 16, 17, 129, 10 ** 9]))
def test_plan_properties(ids, runs, thr):
    """Any batch (with long same-adapter runs mixed in), any threshold: the plan equals the
    brute-force grouping and every row of a segment with rank > 0 is covered exactly once
    by items of <= 4 rows or tiles of <= 128 rows, on the side the threshold says."""
    batch = list(ids)
    for a, n in runs:
        batch += [a] * n
    plan = _shared_pool().plan(np.asarray(batch, dtype=np.int32), long_threshold=thr)
    _check_plan(plan, _shared_pool(), batch, _RANKS, plan.plan.long_threshold)
    if thr > 0:
        assert plan.plan.long_threshold == thr


def test_plan_carries_each_adapter_scale():
    """sgmv_pool_set_adapter_scale: the factor belongs to the adapter id (resident or
    not, kept across evictions and reloads) and the builder copies it per segment."""
    pool = sg.AdapterPool([(1024, 512)], num_pages=4000, page_elems=512, max_rank=64, device=-1)
    for a, r in ((3, 16), (7, 8), (9, 32)):
        pool.load(a, r)
    pool.set_scale(7, 0.25)
    pool.set_scale(9, -2.0)
    pool.set_scale(11, 5.0)                      # an id that is not resident yet
    plan = pool.plan([9, 3, -1, 7, 9, 7])
    assert plan.seg_adapter.tolist() == [3, 7, 9]
    assert plan.seg_scale.tolist() == [1.0, 0.25, -2.0]
    pool.evict(7)
    pool.load(7, 8)
    pool.load(11, 16)
    plan = pool.plan([11, 7])
    assert plan.seg_scale.tolist() == [0.25, 5.0]
    pool.set_scale(7, 1.0)
    assert pool.scale_of(7) == 1.0 and pool.scale_of(11) == 5.0 and pool.scale_of(12345) == 1.0
    for bad in (float("inf"), float("nan")):
        with pytest.raises(sg.SgmvError) as e:
            pool.set_scale(3, bad)
        assert e.value.status == 1


@pytest.mark.parametrize("projs,n_items,want_table", [
    ([(512, 512)], 64, 0), ([(512, 512)], 256, 0), ([(512, 512)], 257, 1),
    ([(512, 512), (512, 1024)], 64, 0), ([(512, 512), (512, 1024)], 65, 1),
])
def test_launch_argument_threshold(projs, n_items, want_table):
    """Up to 256 SIMT items travel as launch arguments for a single-projection pool; a pool
    of several projections keeps its device table above 64 (its grouped calls need it)."""
    pool = sg.AdapterPool(projs, num_pages=20000, page_elems=512, max_rank=8, device=-1)
    for a in range(n_items):
        pool.load(a, 8)
    plan = pool.plan(np.arange(n_items, dtype=np.int32))
    assert plan.plan.num_simt_items == n_items and plan.plan.num_tc_tiles == 0
    assert plan.plan.needs_device_table == want_table
    pool.close()
