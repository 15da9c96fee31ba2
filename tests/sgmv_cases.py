"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare them.

Tolerances (written here, used by every parity test):
  GATE_REL = 1e-3  relative L2 error per output row, the bar the work is held to.
  Gate V:  v rows        ||v_gpu - v_ref|| / ||v_ref||
  Gate A:  bf16 y rows   ||y_gpu - bf16(y_ref)|| / ||bf16(y_ref)||
  Gate B:  fp32 y rows   ||y_gpu - y_ref|| / ||y_ref - y_in||   (relative to the delta itself)
Rows of tokens that use no adapter (or a rank-0 adapter) must be bit-identical to y_in.

Quantised pools (weight_format "fp8_e4m3" / "int4"): the oracle computes the delta with
the dequantised weights of oracle/quant.py (codes x row scale, fp64), under the same gates.
"""
from __future__ import annotations

import os
from typing import Dict, List, Optional

import numpy as np
import torch

import oracle
from oracle import quant as oquant
import segmented_rank_gemm_sgmv_b200 as sg
import workloads

GATE_REL = 1e-3


def build_pool(wl: workloads.Workload, bank: workloads.AdapterBank, page_elems: int = 512,
               shuffle_seed: Optional[int] = 1, extra_pages: int = 64, weight_format: str = "bf16") -> sg.AdapterPool:
    projs = [(d_in, d_out) for _, d_in, d_out in wl.projections]
    need = sum(sg.AdapterPool.pages_needed(projs, int(r), page_elems) for r in wl.pool_ranks)
    pool = sg.AdapterPool(projs, num_pages=need + extra_pages, page_elems=page_elems,
                          max_rank=max(16, int(wl.pool_ranks.max(initial=0))), device=0,
                          weight_format=weight_format)
    if shuffle_seed is not None:
        pool.shuffle_free_pages(shuffle_seed)
    for a, r in zip(wl.pool_ids.tolist(), wl.pool_ranks.tolist()):
        if r == 0:
            pool.load(a, 0)
            continue
        A, B = zip(*[bank.get(a, p) for p in range(len(wl.projections))])
        pool.load(a, int(r), list(A), list(B))
    return pool


def run_gpu(pool, wl, proj, x, y, long_threshold=0, y_dtype=torch.bfloat16, scale=None,
            adapter_ids=None, mode="separate"):
    """mode "separate": sgmv_shrink then sgmv_expand; "lora_delta": both in one call."""
    ids = wl.adapter_ids if adapter_ids is None else adapter_ids
    plan = pool.plan(ids, long_threshold=long_threshold)
    plan.upload()
    v = plan.new_v()
    v.fill_(float("nan"))
    y_out = y.to(y_dtype).clone()
    sc = wl.scale if scale is None else scale
    if mode == "separate":
        sg.shrink(x, plan, pool, v, proj)
        sg.expand(v, plan, pool, y_out, proj, sc)
    else:
        sg.lora_delta(x, plan, pool, y_out, proj, sc, v=v)
    sg.check_errors()
    return plan, v, y_out


def oracle_weights(bank, a, proj, weight_format: str = "bf16"):
    """(A, B) of adapter a for the oracle, float64: the bf16 values, or their quantised and
    dequantised form (oracle/quant.py) for a quantised pool."""
    A16, B16 = bank.get(a, proj)
    A, B = workloads.bf16_to_f64(A16), workloads.bf16_to_f64(B16)
    if weight_format == "bf16":
        return A, B
    *_, Ad, Bd = oquant.quantize_adapter(A.astype(np.float32), B.astype(np.float32), weight_format)
    return Ad, Bd


def run_oracle(wl, bank, proj, x, y, rows_of_tokens: Optional[List[int]] = None, scale=None,
               adapter_ids=None, threads: int = 0, weight_format: str = "bf16",
               adapter_scale: Optional[Dict[int, float]] = None):
    """fp64 oracle on the whole batch, or on the listed tokens only (each token's
    result depends only on its own row and adapter).  adapter_scale: the multiplier of
    each adapter's delta (absent ids: 1), as set on the pool with set_scale."""
    ids = (wl.adapter_ids if adapter_ids is None else adapter_ids).tolist()
    tix, off, seg_ad = oracle.group_by_adapter(ids)
    if rows_of_tokens is not None:
        keep = set(rows_of_tokens)
        sub_ids = [a if t in keep else -1 for t, a in enumerate(ids)]
        tix, off, seg_ad = oracle.group_by_adapter(sub_ids)
    ranks = [wl.rank_of(a) for a in seg_ad]
    AB = [oracle_weights(bank, a, proj, weight_format) for a in seg_ad]
    A = [ab[0] for ab in AB]
    B = [ab[1] for ab in AB]
    seg_scale = None
    if adapter_scale:
        seg_scale = [float(np.float32(adapter_scale.get(int(a), 1.0))) for a in seg_ad]
    v_ref, y_ref = oracle.lora_delta(workloads.bf16_to_f64(x), workloads.bf16_to_f64(y), off, ranks, A, B,
                                     token_idx=tix, scale=wl.scale if scale is None else scale,
                                     threads=threads or (os.cpu_count() or 1), seg_scale=seg_scale)
    return dict(tix=tix, off=off, seg_ad=seg_ad, ranks=ranks, v=v_ref, y=y_ref)


def row_rel(a: np.ndarray, b: np.ndarray, denom: np.ndarray) -> np.ndarray:
    num = np.sqrt(((a - b) ** 2).sum(axis=1))
    den = np.sqrt((denom ** 2).sum(axis=1))
    return num / np.maximum(den, 1e-300)


def compare(plan, v_gpu, y_gpu, y_in, ref, check_rows: Optional[List[int]] = None) -> Dict[str, float]:
    """Bookkeeping bit-exact, then Gates V and A/B. Returns the worst errors."""
    out = {}
    tix, off, ranks = ref["tix"], ref["off"], ref["ranks"]
    if check_rows is None:
        assert plan.token_idx.tolist() == tix
        assert plan.seg_offsets.tolist() == (off if ref["seg_ad"] else [0])
        assert plan.seg_rank.tolist() == ranks
    v_gpu = v_gpu.double().cpu().numpy()
    y_gpu_np = y_gpu.double().cpu().numpy()
    y_in_np = workloads.bf16_to_f64(y_in)
    # map token -> (gpu row, ref row)
    plan_row = {t: i for i, t in enumerate(plan.token_idx.tolist())}
    worst_v, worst_y = 0.0, 0.0
    touched = set()
    for s, r in enumerate(ranks):
        for i in range(off[s], off[s + 1]):
            t = tix[i]
            if r == 0:
                continue
            touched.add(t)
            gi = plan_row[t]
            ev = row_rel(v_gpu[gi:gi + 1, :r], ref["v"][i:i + 1, :r], ref["v"][i:i + 1, :r])[0]
            worst_v = max(worst_v, ev)
            if y_gpu.dtype == torch.bfloat16:
                yr = torch.from_numpy(ref["y"][t:t + 1]).to(torch.bfloat16).double().numpy()
                ey = row_rel(y_gpu_np[t:t + 1], yr, yr)[0]
            else:
                ey = row_rel(y_gpu_np[t:t + 1], ref["y"][t:t + 1], ref["y"][t:t + 1] - y_in_np[t:t + 1])[0]
            worst_y = max(worst_y, ey)
    out["v"], out["y"] = worst_v, worst_y
    assert worst_v <= GATE_REL, f"Gate V: worst per-row relative L2 {worst_v:.3e}"
    assert worst_y <= GATE_REL, f"Gate {'A' if y_gpu.dtype == torch.bfloat16 else 'B'}: worst {worst_y:.3e}"
    if check_rows is None:
        untouched = [t for t in range(y_in.shape[0]) if t not in touched]
        if untouched:
            a = y_gpu.cpu()[untouched]
            b = y_in.to(y_gpu.dtype).cpu()[untouched]
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), \
                "rows without an adapter changed"
    return out
