"""sgmv_lora_delta_noalloc: the variant for callers that cannot give the library
device memory (a fixed arena owned by another runtime, or a rule against
growing the process's device footprint).  Its workspace is a fixed array inside
the library instead of a caller buffer.

Checked through the C ABI on two calls in a row -- different batches, shapes and
ranks, so a stale workspace left by the first call would show in the second:
  * bit for bit against sgmv_lora_delta (the same kernels with a caller-provided
    workspace: both are deterministic, so any difference is a workspace fault);
  * against the fp64 oracle with fp32 y (Gate B, relative to the delta itself, at
    the parity tolerance of tests/sgmv_cases.py), for both entry points;
and the size limit is refused with SGMV_ERR_CAPACITY.
This file is collected last on purpose; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu


class _Bank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def _case(seed, lens, ranks, d_in, d_out):
    g = torch.Generator(device="cuda").manual_seed(seed)
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, np.int32) for a, n in enumerate(lens)] + [np.full(3, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("noalloc", seed, int(ids.size), [("p", d_in, d_out)],
                            np.arange(len(lens), dtype=np.int32), np.asarray(ranks, np.int32), ids)
    bank = _Bank()
    for a, r in enumerate(ranks):
        A = (torch.randn(r, d_in, generator=g, device="cuda") / d_in ** 0.5).to(torch.bfloat16)
        B = (torch.randn(d_out, r, generator=g, device="cuda") / r ** 0.5).to(torch.bfloat16)
        bank.m[(a, 0)] = (A, B)
    pool = build_pool(wl, bank, shuffle_seed=seed)
    x = (torch.randn(wl.T, d_in, generator=g, device="cuda") / d_in ** 0.5).to(torch.bfloat16)
    y = torch.randn(wl.T, d_out, generator=g, device="cuda").to(torch.bfloat16)
    plan = pool.plan(ids)
    plan.upload()
    return wl, bank, pool, plan, x, y


def _call_noalloc(x, plan, pool, y):
    lib = sg.load_library()
    return lib.sgmv_lora_delta_noalloc(x.data_ptr(), x.stride(0), plan.T, x.shape[1], y.shape[1], 0,
                                       ctypes.byref(plan.plan), plan.table_ptr(), pool.handle, 1.0,
                                       y.data_ptr(), y.stride(0), 0 if y.dtype == torch.bfloat16 else 1,
                                       torch.cuda.current_stream().cuda_stream)


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


# first call: mixed ranks up to 128 and a 140-row segment (tensor-core tiles use the workspace
# too); second call: a smaller batch with other ranks, after the first left its contents behind
CALLS = ((1, [1, 3, 7, 140, 2], [16, 128, 8, 64, 32], 2048, 3072),
         (2, [5, 1, 2], [24, 16, 8], 1024, 1536))


@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_noalloc_matches_lora_delta_and_oracle_on_two_calls(y_dtype):
    for seed, lens, ranks, d_in, d_out in CALLS:
        wl, bank, pool, plan, x, y = _case(seed, lens, ranks, d_in, d_out)
        y_in = y.to(y_dtype)
        y_ref = y_in.clone()
        v_ref = sg.lora_delta(x, plan, pool, y_ref, 0, 1.0)        # caller-provided workspace
        y_na = y_in.clone()
        st = _call_noalloc(x, plan, pool, y_na)
        assert st == 0, sg.load_library().sgmv_last_error()
        assert sg.check_errors() == 0
        assert torch.equal(_bits(y_na), _bits(y_ref)), "the two entry points differ"
        if y_dtype == torch.float32:                                 # Gate B against the oracle
            ref = run_oracle(wl, bank, 0, x, y)
            compare(plan, v_ref, y_na, y, ref)
        untouched = [t for t in range(plan.T) if t not in set(plan.token_idx.tolist())]
        assert torch.equal(_bits(y_na[untouched]), _bits(y_in[untouched]))


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
