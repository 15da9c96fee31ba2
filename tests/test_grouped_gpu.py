"""sgmv_lora_delta_grouped: several projections of one layer over the same
batch plan in one call.  Each entry's result is checked against the fp64
oracle of its projection (the gates of tests/sgmv_cases.py); the grouped path
takes one SIMT shrink and one SIMT expand launch for all entries, the
tensor-core tiles one pair per entry."""
import ctypes

import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import GATE_REL, build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu

PROJS = [("a", 1024, 1536), ("b", 2048, 512), ("c", 1536, 3072)]


class _Bank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def _case(seg_lens, ranks, seed, minus_one=3):
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(seg_lens)] + [np.full(minus_one, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("grouped", seed, int(ids.size), PROJS, np.arange(len(seg_lens), dtype=np.int32),
                            np.asarray(ranks, np.int32), ids)
    bank = _Bank()
    g = torch.Generator(device="cuda").manual_seed(seed)
    for a, r in enumerate(ranks):
        for p, (_, di, do) in enumerate(PROJS):
            A = (torch.randn(r, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
            B = (torch.randn(do, r, generator=g, device="cuda") / max(r, 1) ** 0.5).to(torch.bfloat16)
            bank.m[(a, p)] = (A, B)
    acts = []
    for p, (_, di, do) in enumerate(PROJS):
        x = (torch.randn(wl.T, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
        y = torch.randn(wl.T, do, generator=g, device="cuda").to(torch.bfloat16)
        acts.append((x, y))
    return wl, bank, acts


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
@pytest.mark.parametrize("thr", [0, 10 ** 9, 1], ids=["dispatch", "simt", "tc"])
def test_grouped_matches_oracle_per_projection(thr, y_dtype):
    # segments from 1 to 150 rows (SIMT items and tensor tiles), ranks 8 .. 128
    wl, bank, acts = _case([1, 3, 5, 17, 150, 40, 2, 9], [8, 16, 24, 64, 128, 32, 16, 8], seed=31)
    pool = build_pool(wl, bank)
    plan = pool.plan(wl.adapter_ids, long_threshold=thr)
    plan.upload()
    ys = [y.to(y_dtype).clone() for _, y in acts]
    entries = [(acts[p][0], ys[p], p) for p in range(len(PROJS))]
    vs = sg.lora_delta_grouped(entries, plan, pool, 1.0)
    assert sg.check_errors() == 0
    for p in range(len(PROJS)):
        ref = run_oracle(wl, bank, p, acts[p][0], acts[p][1])
        compare(plan, vs[p], ys[p], acts[p][1], ref)


def test_grouped_small_plan_without_device_table():
    """A decode-sized plan (work items as launch arguments, no device table): the
    entries run one by one."""
    wl, bank, acts = _case([1, 2, 3, 4], [16, 8, 32, 16], seed=5, minus_one=0)
    pool = build_pool(wl, bank)
    plan = pool.plan(wl.adapter_ids)
    assert not plan.plan.needs_device_table
    ys = [y.clone() for _, y in acts]
    vs = sg.lora_delta_grouped([(acts[p][0], ys[p], p) for p in range(3)], plan, pool)
    assert sg.check_errors() == 0
    for p in range(3):
        compare(plan, vs[p], ys[p], acts[p][1], run_oracle(wl, bank, p, acts[p][0], acts[p][1]))


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_grouped_llama70b_layer(y_dtype):
    """The 70B layer's 7 projections in one grouped call -- the launch configuration the
    benchmark times (the full pool of 2000 rank-16 adapters, 256 tokens on distinct
    adapters) -- against the oracle on every token of every projection: Gate A on bf16
    y, Gate B (relative to the delta) on fp32 y."""
    wl = workloads.make("llama70b_layer")
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    acts = [workloads.activations(wl, p, device="cuda") for p in range(len(wl.projections))]
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    ys = [y.to(y_dtype).clone() for _, y in acts]
    vs = sg.lora_delta_grouped([(acts[p][0], ys[p], p) for p in range(len(acts))], plan, pool)
    assert sg.check_errors() == 0
    for p in range(len(acts)):
        ref = run_oracle(wl, bank, p, acts[p][0], acts[p][1])
        compare(plan, vs[p], ys[p], acts[p][1], ref)


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_grouped_llama70b_layer_shared_x(y_dtype):
    """The layer with a real layer's inputs: q, k, v name one x and gate, up another, so
    the grouped call stacks them in one shrink pass over each shared x.  Every token of
    every projection against the oracle."""
    wl = workloads.make("llama70b_layer_shared_x")
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    acts = [workloads.activations(wl, p, device="cuda") for p in range(len(wl.projections))]
    xs = [acts[wl.x_of(p)][0] for p in range(len(acts))]          # one tensor per shared input
    assert xs[1] is xs[0] and xs[2] is xs[0] and xs[5] is xs[4]
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    ys = [y.to(y_dtype).clone() for _, y in acts]
    vs = sg.lora_delta_grouped([(xs[p], ys[p], p) for p in range(len(acts))], plan, pool)
    assert sg.check_errors() == 0
    for p in range(len(acts)):
        compare(plan, vs[p], ys[p], acts[p][1], run_oracle(wl, bank, p, xs[p], acts[p][1]))


SHARED = [("a", 1024, 1536), ("b", 1024, 512), ("c", 1024, 3072), ("d", 2048, 1024), ("e", 2048, 1536)]


@pytest.mark.parametrize("fmt", ["bf16", "fp8_e4m3", "int4"])
@pytest.mark.parametrize("thr", [0, 10 ** 9], ids=["dispatch", "simt"])
def test_grouped_shared_x_matches_oracle(thr, fmt):
    """Projections a, b, c read one x and d, e another (the shrink stacks 3 and 2
    projections), with ragged segments, ranks 8 .. 128, long segments on the tensor
    cores under the dispatch, and quantised pools."""
    seg_lens, ranks = [1, 3, 5, 17, 150, 40, 2, 9], [8, 16, 24, 64, 128, 32, 16, 8]
    rng = np.random.default_rng(61)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(seg_lens)] + [np.full(3, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("shared", 61, int(ids.size), SHARED, np.arange(len(seg_lens), dtype=np.int32),
                            np.asarray(ranks, np.int32), ids, x_source=[0, 0, 0, 3, 3])
    bank = _Bank()
    g = torch.Generator(device="cuda").manual_seed(61)
    for a, r in enumerate(ranks):
        for p, (_, di, do) in enumerate(SHARED):
            bank.m[(a, p)] = ((torch.randn(r, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16),
                              (torch.randn(do, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16))
    x0 = (torch.randn(wl.T, 1024, generator=g, device="cuda") / 32).to(torch.bfloat16)
    x1 = (torch.randn(wl.T, 2048, generator=g, device="cuda") / 45).to(torch.bfloat16)
    xs = [x0, x0, x0, x1, x1]
    y_in = [torch.randn(wl.T, do, generator=g, device="cuda").to(torch.bfloat16) for _, _, do in SHARED]
    pool = build_pool(wl, bank, weight_format=fmt)
    plan = pool.plan(wl.adapter_ids, long_threshold=thr)
    plan.upload()
    ys = [y.to(torch.float32).clone() for y in y_in]
    vs = sg.lora_delta_grouped([(xs[p], ys[p], p) for p in range(5)], plan, pool, 1.0)
    assert sg.check_errors() == 0
    for p in range(5):
        compare(plan, vs[p], ys[p], y_in[p], run_oracle(wl, bank, p, xs[p], y_in[p], weight_format=fmt))


def test_grouped_argument_errors():
    wl, bank, acts = _case([20, 3], [16, 8], seed=2)
    pool = build_pool(wl, bank)
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    v = plan.new_v()
    with pytest.raises(sg.SgmvError) as e:  # one workspace for two entries
        sg.lora_delta_grouped([(acts[0][0], acts[0][1].clone(), 0, v), (acts[1][0], acts[1][1].clone(), 1, v)],
                              plan, pool)
    assert e.value.status == 1
    lib = sg.load_library()
    arr = (sg.DeltaEntry * 9)()
    assert lib.sgmv_lora_delta_grouped(arr, 9, plan.T, ctypes.byref(plan.plan), plan.table_ptr(), pool.handle,
                                       1.0, 0, None) == 1
    assert lib.sgmv_lora_delta_grouped(arr, 0, plan.T, ctypes.byref(plan.plan), plan.table_ptr(), pool.handle,
                                       1.0, 0, None) == 1
