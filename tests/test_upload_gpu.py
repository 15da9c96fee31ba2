"""sgmv_upload_table: the device copy of a plan's table equals the host table byte for byte,
from pinned host memory (read by the upload kernel) and from pageable memory (a copy-engine
transfer), and a delta call reading the uploaded table passes the oracle's gates."""
import ctypes

import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu


def test_upload_pinned_and_pageable():
    wl = workloads.make("prefill_long", seed=5, requests=3, seq=200, d=1024)
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    plan = sg.BatchPlan(pool, capacity_tokens=wl.T)
    plan.build(wl.adapter_ids)
    assert plan.plan.needs_device_table
    n = int(plan.plan.table_bytes)
    assert plan.host.is_pinned()
    dev = plan.upload()
    torch.cuda.synchronize()
    assert torch.equal(dev[:n].cpu(), plan.host[:n])
    # the same table from pageable memory
    page = torch.empty(n + 64, dtype=torch.uint8)
    off = (-page.data_ptr()) % 16
    page[off:off + n].copy_(plan.host[:n])
    p2 = sg.Plan.from_buffer_copy(plan.plan)
    p2.host_table = page[off:].data_ptr()
    dst = torch.zeros(n, dtype=torch.uint8, device="cuda")
    lib = sg.load_library()
    assert lib.sgmv_upload_table(ctypes.byref(p2), dst.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), plan.host[:n])
    # and the delta reads it
    x, y = workloads.activations(wl, 0, device="cuda")
    v = plan.new_v()
    y_out = y.clone()
    sg.lora_delta(x, plan, pool, y_out, 0, wl.scale, v=v)
    sg.check_errors()
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y))
    pool.close()
