"""Large decode-shaped batches: about 600 SIMT items of 1 to 4 tokens with ranks from 5 to
128 (enough CTAs that the shrink takes one CTA per item over the whole of d_in, C = 1),
checked against the fp64 oracle under the gates of tests/sgmv_cases.py: one projection
and grouped projections with a shared x, bf16, FP8 and INT4 pools, bf16 and fp32 y."""
import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu

RANKS = (5, 8, 16, 24, 40, 64, 128)


class _Bank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def _case(projs, seed, x_source=None, n_seg=600):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 5, size=n_seg)
    ranks = rng.choice(RANKS, size=n_seg)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(lens)] + [np.full(5, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("large", seed, int(ids.size), projs, np.arange(n_seg, dtype=np.int32),
                            ranks.astype(np.int32), ids, x_source=x_source)
    bank = _Bank()
    g = torch.Generator(device="cuda").manual_seed(seed)
    for p, (_, di, do) in enumerate(projs):
        for r in RANKS:
            members = [a for a in range(n_seg) if ranks[a] == r]
            A = (torch.randn(len(members), r, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
            B = (torch.randn(len(members), do, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16)
            for i, a in enumerate(members):
                bank.m[(a, p)] = (A[i], B[i])
    xs, ys = {}, []
    for p, (_, di, do) in enumerate(projs):
        src = wl.x_of(p)
        if src not in xs:
            xs[src] = (torch.randn(wl.T, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16)
        ys.append(torch.randn(wl.T, do, generator=g, device="cuda").to(torch.bfloat16))
    return wl, bank, [xs[wl.x_of(p)] for p in range(len(projs))], ys


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
@pytest.mark.parametrize("fmt", ["bf16", "fp8_e4m3", "int4"])
def test_large_batch_one_projection(fmt, y_dtype):
    wl, bank, xs, ys = _case([("p", 4096, 1024)], seed=71)
    pool = build_pool(wl, bank, weight_format=fmt)
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    assert plan.plan.num_tc_tiles == 0 and plan.plan.num_simt_items > 500
    y_out = ys[0].to(y_dtype).clone()
    v = plan.new_v()
    v.fill_(float("nan"))
    sg.lora_delta(xs[0], plan, pool, y_out, 0, 1.0, v=v)
    assert sg.check_errors() == 0
    compare(plan, v, y_out, ys[0], run_oracle(wl, bank, 0, xs[0], ys[0], weight_format=fmt))


@pytest.mark.parametrize("fmt", ["bf16", "int4"])
def test_large_batch_grouped_shared_x(fmt):
    """Three projections over one x (stacked) and one over its own x of another width
    (3072 columns: three passes, the last of them full)."""
    projs = [("a", 4096, 1024), ("b", 4096, 512), ("c", 4096, 2048), ("d", 3072, 1536)]
    wl, bank, xs, ys = _case(projs, seed=72, x_source=[0, 0, 0, 3])
    pool = build_pool(wl, bank, weight_format=fmt)
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    outs = [y.to(torch.float32).clone() for y in ys]
    vs = sg.lora_delta_grouped([(xs[p], outs[p], p) for p in range(4)], plan, pool, 1.0)
    assert sg.check_errors() == 0
    for p in range(4):
        compare(plan, vs[p], outs[p], ys[p], run_oracle(wl, bank, p, xs[p], ys[p], weight_format=fmt))
