"""sgmv_lora_delta_host: the whole step from host buffers (segment builder, copies in,
grouped delta, copy out) in one library call.  Checked through the C ABI against
sgmv_lora_delta_grouped on device copies of the same inputs (bit for bit: the same
kernels), and against the fp64 oracle, with shared inputs, bf16 and fp32 y, a
decode-sized plan (no device table) and a batch large enough for the tensor-core tiles."""
import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu

PROJS = [("a", 1024, 1536), ("b", 1024, 512), ("c", 2048, 1024)]


class _Bank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def _case(seg_lens, ranks, seed):
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(seg_lens)] + [np.full(2, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("host", seed, int(ids.size), PROJS, np.arange(len(seg_lens), dtype=np.int32),
                            np.asarray(ranks, np.int32), ids, x_source=[0, 0, 2])
    bank = _Bank()
    g = torch.Generator(device="cuda").manual_seed(seed)
    for a, r in enumerate(ranks):
        for p, (_, di, do) in enumerate(PROJS):
            bank.m[(a, p)] = ((torch.randn(r, di, generator=g, device="cuda") / di ** 0.5).to(torch.bfloat16),
                              (torch.randn(do, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16))
    x0 = (torch.randn(wl.T, 1024, generator=g, device="cuda") / 32).to(torch.bfloat16)
    x2 = (torch.randn(wl.T, 2048, generator=g, device="cuda") / 45).to(torch.bfloat16)
    xs = [x0, x0, x2]
    ys = [torch.randn(wl.T, do, generator=g, device="cuda").to(torch.bfloat16) for _, _, do in PROJS]
    return wl, bank, xs, ys


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
@pytest.mark.parametrize("shape", ["decode", "mixed"])
def test_host_step_matches_grouped_call_and_oracle(shape, y_dtype):
    if shape == "decode":   # few items: the work items travel as launch arguments
        wl, bank, xs, ys = _case([1, 2, 1, 3], [16, 8, 32, 16], seed=81)
    else:                   # ragged segments, one long enough for tensor-core tiles
        wl, bank, xs, ys = _case([1, 3, 150, 17, 40, 2, 9], [8, 16, 64, 24, 32, 16, 128], seed=82)
    pool = build_pool(wl, bank)
    # reference: the grouped call on device copies
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    y_dev = [y.to(y_dtype).clone() for y in ys]
    sg.lora_delta_grouped([(xs[p], y_dev[p], p) for p in range(3)], plan, pool, 0.5)
    # the host step, twice (the second call reuses the table and workspace)
    x_host = {id(xs[0]): xs[0].cpu().pin_memory(), id(xs[2]): xs[2].cpu().pin_memory()}
    step = sg.HostStep(pool, capacity_tokens=wl.T)
    for _ in range(2):
        y_host = [y.to(y_dtype).cpu().pin_memory() for y in ys]
        h2d, d2h = step.run(wl.adapter_ids, [(x_host[id(xs[p])], y_host[p], p) for p in range(3)], 0.5)
        torch.cuda.synchronize()
        assert sg.check_errors() == 0
        for p in range(3):
            assert torch.equal(y_host[p].view(torch.int16 if y_dtype == torch.bfloat16 else torch.int32),
                               y_dev[p].cpu().view(torch.int16 if y_dtype == torch.bfloat16 else torch.int32))
    esz = 2 if y_dtype == torch.bfloat16 else 4
    T = wl.T
    table = int(step.plan.table_bytes) if step.plan.needs_device_table else 0
    assert h2d == table + T * (1024 + 2048) * 2 + T * (1536 + 512 + 1024) * esz   # x0 crosses once
    assert d2h == T * (1536 + 512 + 1024) * esz
    if y_dtype == torch.float32:
        for p in range(3):
            ref = run_oracle(wl, bank, p, xs[p], ys[p], scale=0.5)
            compare(plan, _v_of(pool, wl, xs, p), y_host[p], ys[p], ref)


def _v_of(pool, wl, xs, p):
    """v of projection p from a plain shrink, for Gate V of the comparison."""
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    v = plan.new_v()
    sg.shrink(xs[p], plan, pool, v, p)
    return v


def test_host_step_rejects_a_small_workspace():
    wl, bank, xs, ys = _case([1, 2], [16, 8], seed=83)
    pool = build_pool(wl, bank)
    step = sg.HostStep(pool, capacity_tokens=wl.T)
    step.workspace = torch.empty(256, dtype=torch.uint8, device="cuda")
    import ctypes
    lib = sg.load_library()
    arr = (sg.HostEntry * 1)(sg.HostEntry(0, 1024, 1536, 0, xs[0].cpu().pin_memory().data_ptr(),
                                          ys[0].cpu().pin_memory().data_ptr()))
    ids = np.ascontiguousarray(wl.adapter_ids)
    st = lib.sgmv_lora_delta_host(ids.ctypes.data, int(ids.size), pool.handle, arr, 1, 1.0, 0,
                                  step.host_table.data_ptr(), step.table_bytes, step.workspace.data_ptr(), 256,
                                  None, None, None, None)
    assert st == 8                                            # SGMV_ERR_CAPACITY, nothing enqueued
