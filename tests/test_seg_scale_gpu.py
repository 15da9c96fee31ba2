"""Per-adapter scale (each adapter's LoRA alpha / r, set with sgmv_pool_set_adapter_scale):
a token on adapter a gets y_t + (scale * s_a) B_a A_a x_t.  Checked through the C ABI
against the fp64 oracle with the same factors per segment, under the gates of
tests/sgmv_cases.py, on both kernel paths and the size-based dispatch, with bf16, FP8 and
INT4 pools, bf16 and fp32 y, one call or two, the decode-sized plan whose work items
travel as launch arguments, and the grouped call."""
import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

SIMT, TC = 1 << 30, 1
# negative, fractional, zero, above one; the factor of the last adapter is left unset (1)
SCALES = {0: 0.5, 1: 2.0, 2: -1.25, 3: 0.0, 4: 3.0, 5: 0.125}


class _Bank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def _case(seg_lens, ranks, projs, seed, minus_one=2):
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(seg_lens)] +
                         [np.full(minus_one, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("seg_scale", seed, int(ids.size), projs, np.arange(len(seg_lens), dtype=np.int32),
                            np.asarray(ranks, np.int32), ids, scale=0.75)
    bank = _Bank()
    g = torch.Generator(device="cuda").manual_seed(seed)
    for a, r in enumerate(ranks):
        for p, (_, di, do) in enumerate(projs):
            A = (torch.randn(r, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
            B = (torch.randn(do, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16)
            bank.m[(a, p)] = (A, B)
    acts = []
    for _, di, do in projs:
        x = (torch.randn(wl.T, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
        y = torch.randn(wl.T, do, generator=g, device="cuda").to(torch.bfloat16)
        acts.append((x, y))
    return wl, bank, acts


def _pool(wl, bank, fmt):
    pool = build_pool(wl, bank, weight_format=fmt)
    for a, s in SCALES.items():
        pool.set_scale(a, s)
    return pool


@pytest.mark.parametrize("mode", ["separate", "lora_delta"])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
@pytest.mark.parametrize("path", [0, SIMT, TC], ids=["dispatch", "simt", "tc"])
@pytest.mark.parametrize("fmt", ["bf16", "fp8_e4m3", "int4"])
def test_adapter_scales_match_oracle(fmt, path, y_dtype, mode):
    # segments of 1 .. 150 rows: SIMT items and tensor-core tiles under the dispatch
    wl, bank, acts = _case([1, 3, 150, 17, 40, 2, 9], [8, 16, 64, 24, 32, 16, 128],
                           [("p", 1024, 1536)], seed=41)
    pool = _pool(wl, bank, fmt)
    x, y = acts[0]
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, path, y_dtype, mode=mode)
    assert np.allclose(plan.seg_scale, [np.float32(SCALES.get(int(a), 1.0)) for a in plan.seg_adapter])
    ref = run_oracle(wl, bank, 0, x, y, weight_format=fmt, adapter_scale=SCALES)
    compare(plan, v, y_out, y, ref)
    if path == 0:
        assert plan.plan.num_tc_tiles > 0 and plan.plan.num_simt_items > 0


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_adapter_scales_on_a_decode_plan_without_device_table(y_dtype):
    """Decode-sized batch: the work items and their factors travel as launch arguments."""
    wl, bank, acts = _case([1, 2, 1, 3, 1, 4, 2], [16] * 7, [("q", 2048, 2048)], seed=42, minus_one=1)
    pool = _pool(wl, bank, "bf16")
    x, y = acts[0]
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, 0, y_dtype, mode="lora_delta")
    assert not plan.plan.needs_device_table
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y, adapter_scale=SCALES))


@pytest.mark.parametrize("thr", [0, TC], ids=["dispatch", "tc"])
def test_adapter_scales_grouped(thr):
    projs = [("a", 1024, 1536), ("b", 2048, 512)]
    wl, bank, acts = _case([1, 3, 130, 5, 2, 7, 1], [8, 16, 32, 64, 16, 8, 24], projs, seed=43)
    pool = _pool(wl, bank, "bf16")
    plan = pool.plan(wl.adapter_ids, long_threshold=thr)
    plan.upload()
    ys = [y.to(torch.float32).clone() for _, y in acts]
    vs = sg.lora_delta_grouped([(acts[p][0], ys[p], p) for p in range(2)], plan, pool, wl.scale)
    assert sg.check_errors() == 0
    for p in range(2):
        compare(plan, vs[p], ys[p], acts[p][1],
                run_oracle(wl, bank, p, acts[p][0], acts[p][1], adapter_scale=SCALES))


def test_scale_change_needs_a_new_plan_and_survives_reload():
    """A factor set after a plan was built does not change that plan; a plan built
    afterwards carries it, and an evicted and reloaded adapter keeps it."""
    wl, bank, acts = _case([2, 3], [16, 8], [("p", 1024, 1024)], seed=44, minus_one=0)
    pool = build_pool(wl, bank)
    old = pool.plan(wl.adapter_ids)
    pool.set_scale(1, 4.0)
    pool.evict(1)
    A, B = bank.get(1, 0)
    pool.load(1, 8, [A], [B])
    assert pool.scale_of(1) == 4.0 and pool.scale_of(0) == 1.0
    assert old.seg_scale.tolist() == [1.0, 1.0]
    x, y = acts[0]
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, 0, torch.float32, mode="lora_delta")
    assert plan.seg_scale.tolist() == [1.0, 4.0]
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y, adapter_scale={1: 4.0}))
