"""Residency manager on the GPU: a pool with room for three adapters serves
batches over six, loading missing adapters from pinned host copies on a copy
stream (evicting the least recently used) while the deltas run on the compute
stream; every batch's delta matches the fp64 oracle, so the pages written
after evictions hold the right adapters."""
import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import compare, run_oracle

pytestmark = pytest.mark.gpu

D_IN, D_OUT = 1024, 1536
RANKS = [16, 32, 8, 16, 64, 16]


class _Bank:
    def __init__(self, m):
        self.m = m

    def get(self, a, p):
        return self.m[(a, p)]


def test_batches_over_more_adapters_than_fit():
    g = torch.Generator().manual_seed(11)
    host, dev = {}, {}
    for a, r in enumerate(RANKS):
        A = (torch.randn(r, D_IN, generator=g) / D_IN ** 0.5).to(torch.bfloat16).pin_memory()
        B = (torch.randn(D_OUT, r, generator=g) / r ** 0.5).to(torch.bfloat16).pin_memory()
        host[a] = (A, B)
        dev[(a, 0)] = (A.cuda(), B.cuda())            # the oracle's copy
    per = [sg.AdapterPool.pages_needed([(D_IN, D_OUT)], r) for r in RANKS]
    pool = sg.AdapterPool([(D_IN, D_OUT)], num_pages=sum(sorted(per)[-3:]), page_elems=512, max_rank=64, device=0)
    pool.shuffle_free_pages(3)
    res = sg.Residency(pool)
    for a, r in enumerate(RANKS):
        res.register(a, r, [host[a][0]], [host[a][1]])
    copy_stream = torch.cuda.Stream()
    compute = torch.cuda.current_stream()
    rng = np.random.default_rng(4)
    batches = [[0, 1, 2], [3, 4], [0, 5], [1, 2, 3], [4, 5, 0], [2, 4]]
    for i, adapters in enumerate(batches):
        ids = rng.choice(adapters, size=24).astype(np.int32)
        ids[:2] = -1
        res.prepare(ids, copy_stream, compute)
        wl = workloads.Workload("res", i, ids.size, [("p", D_IN, D_OUT)], np.arange(len(RANKS), dtype=np.int32),
                                np.asarray(RANKS, np.int32), ids)
        x = (torch.randn(ids.size, D_IN, device="cuda") / D_IN ** 0.5).to(torch.bfloat16)
        y = torch.randn(ids.size, D_OUT, device="cuda").to(torch.bfloat16)
        plan = pool.plan(ids)
        y_out = y.clone()
        v = sg.lora_delta(x, plan, pool, y_out, 0, 1.0)
        assert sg.check_errors() == 0
        compare(plan, v, y_out, y, run_oracle(wl, _Bank(dev), 0, x, y))
    # the policy, simulated independently: hits, misses, evictions and bytes loaded
    total = sum(sorted(per)[-3:])
    resident, tick, hits, misses, evict, nbytes = {}, 0, 0, 0, 0, 0
    rng = np.random.default_rng(4)
    for adapters in batches:
        ids = rng.choice(adapters, size=24).astype(np.int32)
        ids[:2] = -1
        batch = sorted(set(int(a) for a in ids if a >= 0))
        tick += 1
        miss = [a for a in batch if a not in resident]
        hits += len(batch) - len(miss)
        for a in batch:
            if a in resident:
                resident[a] = tick
        free = total - sum(per[a] for a in resident)
        need = sum(per[a] for a in miss)
        while need > free:
            victim = min((t, a) for a, t in resident.items() if a not in batch)[1]
            free += per[victim]
            del resident[victim]
            evict += 1
        for a in miss:
            resident[a] = tick
            misses += 1
            nbytes += 2 * RANKS[a] * (D_IN + D_OUT)
    s = res.stats()
    assert (s.hits, s.misses, s.evictions, s.bytes_loaded) == (hits, misses, evict, nbytes)
    assert evict >= 3
    res.close()
