"""sgmv_lora_delta_noalloc: the variant for callers that cannot give the library
device memory (a fixed arena owned by another runtime, or a rule against
growing the process's device footprint).  Its workspace is a fixed array inside
the library instead of a caller buffer.

Checked through the C ABI against sgmv_lora_delta (the same computation with a
caller-provided workspace) on two calls in a row -- different batches, so a
stale workspace from the first call would show in the second -- within the
parity tolerance, and the size limit is refused with SGMV_ERR_CAPACITY.
This file is collected last on purpose; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
from sgmv_cases import GATE_REL

pytestmark = pytest.mark.gpu


def _case(seed, lens, ranks, d_in, d_out):
    g = torch.Generator(device="cuda").manual_seed(seed)
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(lens)] + [np.full(3, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    pool = sg.AdapterPool([(d_in, d_out)], num_pages=sum(r * (d_in + d_out) // 512 for r in ranks) + 16,
                          page_elems=512, max_rank=128, device=0)
    pool.shuffle_free_pages(seed)
    for a, r in enumerate(ranks):
        A = (torch.randn(r, d_in, generator=g, device="cuda") / d_in ** 0.5).to(torch.bfloat16)
        B = (torch.randn(d_out, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16)
        pool.load(a, r, [A], [B])
    x = (torch.randn(ids.size, d_in, generator=g, device="cuda") / d_in ** 0.5).to(torch.bfloat16)
    y = torch.randn(ids.size, d_out, generator=g, device="cuda").to(torch.bfloat16)
    plan = pool.plan(ids)
    plan.upload()
    return pool, plan, x, y


def _call_noalloc(x, plan, pool, y):
    lib = sg.load_library()
    return lib.sgmv_lora_delta_noalloc(x.data_ptr(), x.stride(0), plan.T, x.shape[1], y.shape[1], 0,
                                       ctypes.byref(plan.plan), plan.table_ptr(), pool.handle, 1.0,
                                       y.data_ptr(), y.stride(0), 0, torch.cuda.current_stream().cuda_stream)


def _rows_close(a, b):
    a, b = a.double(), b.double()
    rel = (a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30)
    return float(rel.max())


def test_noalloc_matches_lora_delta_on_two_calls():
    # first call: mixed ranks up to 128 and a 140-row segment (tensor-core tiles use the workspace too)
    # second call: a smaller batch with other ranks, after the first one left its contents behind
    for seed, lens, ranks, d_in, d_out in ((1, [1, 3, 7, 140, 2], [16, 128, 8, 64, 32], 2048, 3072),
                                           (2, [5, 1, 2], [24, 16, 8], 1024, 1536)):
        pool, plan, x, y = _case(seed, lens, ranks, d_in, d_out)
        y_ref = y.clone()
        sg.lora_delta(x, plan, pool, y_ref, 0, 1.0)       # caller-provided workspace
        y_na = y.clone()
        st = _call_noalloc(x, plan, pool, y_na)
        assert st == 0, sg.load_library().sgmv_last_error()
        assert sg.check_errors() == 0
        assert _rows_close(y_na, y_ref) <= GATE_REL
        untouched = torch.from_numpy(np.where(np.asarray([t not in set(plan.token_idx.tolist())
                                                          for t in range(plan.T)]))[0]).cuda()
        assert torch.equal(y_na[untouched], y[untouched])


def test_noalloc_refuses_batches_above_its_workspace():
    pool = sg.AdapterPool([(512, 512)], num_pages=300, page_elems=512, max_rank=128, device=0)
    g = torch.Generator(device="cuda").manual_seed(3)
    pool.load(0, 128, [torch.randn(128, 512, generator=g, device="cuda").to(torch.bfloat16)],
              [torch.randn(512, 128, generator=g, device="cuda").to(torch.bfloat16)])
    T = 5000                                              # 5000 rows x 128 > 2^19 floats
    plan = pool.plan(np.zeros(T, np.int32))
    plan.upload()
    x = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(T, 512, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(x, plan, pool, y) == 8          # SGMV_ERR_CAPACITY, nothing launched
    assert b"workspace" in sg.load_library().sgmv_last_error()
