"""Benchmark of the multi-LoRA delta (SGMV shrink + expand) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--weights bf16|fp8_e4m3|int4] [--per-projection] [--split-phases]

One step is one pass of the whole hot path over one batch: the host segment
builder (run every step, overlapped with the previous device work), one
host-to-device copy of the segment table, then SGMV-shrink and SGMV-expand for
every adapted projection of the workload (one grouped call for a multi-projection
workload unless --per-projection).  The default workload is the Llama-3-70B-shaped
layer (7 adapted projections, 256 decode tokens each on its own rank-16 adapter of a
pool of 2000): tokens/s per adapted layer.  At N = 1 the same run also measures every
other workload (tiny, decode_q_proj, decode_q_proj_12, mixed_rank_mlp_up,
prefill_long) and reports each under `per_workload` with its own step time, roofline
and clocks (--no-per-workload skips them).  The device time of a step (CUDA events on the
launching stream, from the table copy to the last expand) is what `value`
measures; L2 is flushed (a 512 MiB write, then read back so that L2 holds clean
lines) between steps, outside the timed windows.  --weights runs the same batch on a pool of FP8 E4M3 or INT4 codes.  `e2e` repeats
the step through the library's host-buffer entry (sgmv_lora_delta_host): the host
builder, the copies of every distinct x and every y from pinned memory, the delta and
the copy of y back, all enqueued by the library in one call inside the timed window.

With N > 1 (torchrun) every rank runs its own batch of the same shape (weak
scaling, no collective on the data path: the tokens of a batch are
independent); the reported time is the max over ranks.

The CPU baseline is the oracle on the machine's host cores, on the whole batch or, for the
layer, on a bounded sample of its tokens (named in `cpu_baseline.sample`).

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "LoRA-delta tokens/s per adapted layer; SGMV achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


class L2Flush:
    """Between timed steps: write a 512 MiB buffer (more than four times the 126 MB L2), then
    read it back.  The write evicts every line a step could reuse; the read leaves L2 holding
    clean lines, so the next step does not pay for writing back the flush's own dirty data
    (measured on the 70B layer: 263 us per step after a write-only flush, 251 us after write
    + read; the empty-launch floor 7.0 / 6.3 us)."""

    def __init__(self, device):
        self.buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.sink = torch.empty((), dtype=torch.int64, device=device)

    def zero_(self):
        self.buf.zero_()
        torch.sum(self.buf.view(torch.int64), dim=0, out=self.sink)


# ---------------------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# bytes of one stored weight value, by pool weight format
WEIGHT_BYTES = {"bf16": 2.0, "fp8_e4m3": 1.0, "int4": 0.5}


def algorithmic_bytes(wl: workloads.Workload, proj: int, weights: str = "bf16"):
    """Minimum bytes of one shrink and one expand: each distinct adapter's A and B
    once (codes plus one fp32 scale per rank row in a quantised pool), x read once
    (a projection that reads another's x (wl.x_source) adds none), v written and read
    in fp32, y read and written."""
    wb = WEIGHT_BYTES[weights]
    sb = 0 if weights == "bf16" else 4
    _, d_in, d_out = wl.projections[proj]
    ids = wl.adapter_ids[wl.adapter_ids >= 0]
    distinct = np.unique(ids)
    r_of = {int(a): wl.rank_of(int(a)) for a in distinct}
    sum_r_adapters = sum(r_of.values())
    rows = [t for t in range(wl.T) if wl.adapter_ids[t] >= 0 and r_of[int(wl.adapter_ids[t])] > 0]
    sum_r_tokens = sum(r_of[int(wl.adapter_ids[t])] for t in rows)
    x_bytes = 2 * len(rows) * d_in if wl.x_of(proj) == proj else 0
    shrink = int(wb * sum_r_adapters * d_in) + sb * sum_r_adapters + x_bytes + 4 * sum_r_tokens
    expand = int(wb * sum_r_adapters * d_out) + sb * sum_r_adapters + 4 * sum_r_tokens + 4 * len(rows) * d_out
    flops = 2 * sum_r_tokens * (d_in + d_out)
    return shrink, expand, flops, 4 * sum_r_tokens


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report what is known
            self.err = str(e)
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def source_digest() -> str:
    """sha256 (first 16 hex digits) of the library's code: csrc/* by name, with `//`
    comments, trailing blanks and empty lines removed, so that a comment edit keeps
    the counters while any code change drops them."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "segmented_rank_gemm_sgmv_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8", errors="replace") as f:
            for line in f:
                code = re.sub(r"//.*", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def read_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and parts[0] == workload and parts[1] == kernel and parts[3] == digest:
                return float(parts[2])
    return None


# ---------------------------------------------------------------------------- ranks
def reduce_max(x: float, device) -> float:
    """Max of a per-rank number over all ranks (identity without a process group).
    Every rank must call it at the same point."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    if torch.distributed.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch of the same shape each
    step (weak scaling); the job's time is the slowest rank's."""
    return world * tokens_per_rank * steps / (total_ms * 1e-3)


# ---------------------------------------------------------------------------- our arm
def setup(wl_name: str, rank: int, device: int, pool_override: int = 0, weights: str = "bf16"):
    import segmented_rank_gemm_sgmv_b200 as sg
    wl = workloads.make(wl_name, seed=rank, **({"pool": pool_override} if pool_override else {}))
    bank = workloads.AdapterBank(wl, device=f"cuda:{device}")
    projs = [(d_in, d_out) for _, d_in, d_out in wl.projections]
    need = sum(sg.AdapterPool.pages_needed(projs, int(r)) for r in wl.pool_ranks)
    pool = sg.AdapterPool(projs, num_pages=need + 64, page_elems=512,
                          max_rank=max(16, int(wl.pool_ranks.max())), device=device, weight_format=weights)
    pool.shuffle_free_pages(1234 + rank)
    for a, r in zip(wl.pool_ids.tolist(), wl.pool_ranks.tolist()):
        A, B = zip(*[bank.get(a, p) for p in range(len(projs))])
        pool.load(a, int(r), list(A), list(B))
    acts = [workloads.activations(wl, p, device=f"cuda:{device}") for p in range(len(projs))]
    # projections that read another's input get that very tensor (the grouped call then
    # stacks them in one shrink pass over it)
    acts = [(acts[wl.x_of(p)][0], acts[p][1]) for p in range(len(projs))]
    del bank
    torch.cuda.empty_cache()
    return sg, wl, pool, acts


def run_ours(args, rank, world, device, with_e2e=True):
    sg, wl, pool, acts = setup(args.workload, rank, device, args.pool, args.weights)
    n_proj = len(wl.projections)
    stream = torch.cuda.current_stream(device)
    plans = [sg.BatchPlan(pool, capacity_tokens=wl.T) for _ in range(2)]
    for pl in plans:
        pl.build(wl.adapter_ids)
        pl.upload(stream)
    v = plans[0].new_v()
    grouped = getattr(args, "grouped", False) and n_proj > 1
    vs = [plans[0].new_v() for _ in range(n_proj)] if grouped else None
    flush = L2Flush(f"cuda:{device}")
    # Hold the stream for ~200 us after the flush so that the host has enqueued the
    # whole step before the device reaches it: event times are then device times.
    gate_cycles = int(2e-4 * 2.0e9)
    split = args.split_phases

    # Events per step: `start` before the table upload, `end` after the kernels.  Every
    # event recorded between kernels adds device time (2-4 us measured between the table
    # upload and the kernels), so the timed steps record no others; the kernels' own time
    # (the roofline) of a plan that needs a table copy comes from a second loop of the same
    # steps whose upload is enqueued before `start` (kernels_only).  --split-phases adds
    # events around each projection's phases.
    def step(i, ev=None, kernels_only=False):
        pl = plans[i % 2]
        pl.build(wl.adapter_ids)                     # host segment builder + dispatch
        if kernels_only:
            pl.upload(stream)
        if ev:
            ev["start"].record(stream)
        if not kernels_only:
            pl.upload(stream)                        # the table to the device (plans that need one)
        if grouped:                                  # every projection in one call
            sg.lora_delta_grouped([(acts[p][0], acts[p][1], p, vs[p]) for p in range(n_proj)], pl, pool,
                                  wl.scale, stream)
        else:
            for p in range(n_proj):
                x, y = acts[p]
                if split:                            # events around and between the phases (no overlap)
                    ev and ev["ph"][p][0].record(stream)
                    sg.shrink(x, pl, pool, v, p, stream)
                    ev and ev["ph"][p][1].record(stream)
                    sg.expand(v, pl, pool, y, p, wl.scale, stream)
                    ev and ev["ph"][p][2].record(stream)
                else:                                # shrink, then expand overlapping it (PDL)
                    sg.lora_delta(x, pl, pool, y, p, wl.scale, v=v, stream=stream)
        if ev:
            ev["end"].record(stream)

    def new_events():
        mk = lambda: torch.cuda.Event(enable_timing=True)
        ev = {"start": mk(), "end": mk()}
        if split:
            ev["ph"] = [[mk(), mk(), mk()] for _ in range(n_proj)]
        return ev

    for i in range(args.warmup):
        flush.zero_()
        step(i)
    sg.check_errors(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    records = []
    with ClockSampler(device) as clk:
        for i in range(args.steps):
            flush.zero_()                            # L2 flush, outside the timed window
            torch.cuda._sleep(gate_cycles)
            ev = new_events()
            step(i, ev)
            records.append(ev)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sg.check_errors(stream)
    step_ms = [e["start"].elapsed_time(e["end"]) for e in records]
    total_ms = reduce_max(float(sum(step_ms)), f"cuda:{device}")
    # the kernels' own time (roofline): the timed steps themselves when there is no table
    # copy, else the same steps again with the copy enqueued before the start event
    if plans[0].plan.needs_device_table and not split:
        krec = []
        for i in range(args.steps):
            flush.zero_()
            torch.cuda._sleep(gate_cycles)
            ev = new_events()
            step(i, ev, kernels_only=True)
            krec.append(ev)
        torch.cuda.synchronize(device)
        sg.check_errors(stream)
        proj_ms = [e["start"].elapsed_time(e["end"]) for e in krec]
    else:
        proj_ms = step_ms

    shrink_b = expand_b = flops = 0
    for p in range(n_proj):
        s_b, e_b, f, _ = algorithmic_bytes(wl, p, args.weights)
        shrink_b += s_b
        expand_b += e_b
        flops += f
    peak, peak_kind = measured_peaks()
    # the kernels the calls launch, as the library reports them (sgmv_lora_delta_kernels)
    y_dt = acts[0][1].dtype
    if split:                                        # separate shrink and expand calls
        plan0 = plans[0].plan
        mask = (sg.KERNELS_SIMT if plan0.num_simt_items > 0 else 0) | (sg.KERNELS_TC if plan0.num_tc_tiles > 0 else 0)
        launches = 2 * n_proj * bin(mask).count("1")
    elif grouped:
        mask, launches = sg.lora_delta_kernels(plans[0], pool, list(range(n_proj)), y_dt, stream)
    else:
        mask = launches = 0
        for p in range(n_proj):
            k, n_l = sg.lora_delta_kernels(plans[0], pool, [p], y_dt, stream)
            mask |= k
            launches += n_l
    simt_pair = ("shrink_slab_kernel" if mask & sg.KERNELS_SLAB else "shrink_simt_kernel") + " + expand_simt_kernel"
    if plans[0].plan.needs_device_table:
        launches += 1                                # the table upload (sgmv_upload_table) of every step
    names = " + ".join(n for bit, n in ((sg.KERNELS_FUSED, "fused_simt_kernel"), (sg.KERNELS_SIMT, simt_pair),
                                        (sg.KERNELS_TC, "shrink_tc_kernel + expand_tc_kernel")) if mask & bit)
    api = "sgmv_lora_delta_grouped" if grouped else "sgmv_lora_delta"
    res = dict(total_ms=total_ms, proj_ms=float(np.mean(proj_ms)), kernel_name=f"{api} ({names})",
               step_bytes=shrink_b + expand_b, flops=flops, peak=peak, peak_kind=peak_kind,
               launches=launches,
               clocks=clk.summary(), dom_launches=1 if grouped else n_proj,
               traffic=read_traffic(args.workload, ("lora_delta_grouped" if grouped else "lora_delta") +
                                    ("" if args.weights == "bf16" else "@" + args.weights)), split=split)
    if split:
        ph = lambda e, p, k: e["ph"][p][k].elapsed_time(e["ph"][p][k + 1])
        res["phase_us_per_proj"] = {
            name: [round(1e3 * float(np.mean([ph(e, p, 0) for e in records])), 2),
                   round(1e3 * float(np.mean([ph(e, p, 1) for e in records])), 2)]
            for p, (name, _, _) in enumerate(wl.projections)}
        res["phase_ms"] = {"shrink": float(np.mean([sum(ph(e, p, 0) for p in range(n_proj)) for e in records])),
                           "expand": float(np.mean([sum(ph(e, p, 1) for p in range(n_proj)) for e in records]))}
    res["achieved"] = res["step_bytes"] / (res["proj_ms"] * 1e-3) / 1e9
    if with_e2e:
        res["e2e"] = e2e_ours(sg, wl, pool, acts, args, device, stream, world)
    pool.close()
    return wl, res


def e2e_ours(sg, wl, pool, acts, args, device, stream, world):
    """The step through the library's host-buffer entry (sgmv_lora_delta_host): the segment
    builder, the copies of every distinct x and every y from pinned host memory, the delta
    and the copy of y back, enqueued by the library in one call (one call per projection
    with --per-projection).  Timed from an event before the call to an event after the
    last copy, with the stream idle before the call."""
    n_proj = len(wl.projections)
    host_x = {s: acts[s][0].cpu().pin_memory() for s in sorted(set(wl.x_of(p) for p in range(n_proj)))}
    host_y = [y.cpu().pin_memory() for _, y in acts]   # updated in place every step
    step = sg.HostStep(pool, capacity_tokens=wl.T)
    grouped = getattr(args, "grouped", False) and n_proj > 1
    entries = [(host_x[wl.x_of(p)], host_y[p], p) for p in range(n_proj)]
    h2d = d2h = 0
    flush = L2Flush(f"cuda:{device}")

    def one():
        nonlocal h2d, d2h
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        b_in = b_out = 0
        for group in ([entries] if grouped else [[e] for e in entries]):
            i, o = step.run(wl.adapter_ids, group, wl.scale, stream)
            b_in += i
            b_out += o
        e1.record(stream)
        e1.synchronize()
        h2d, d2h = b_in, b_out
        return e0.elapsed_time(e1)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        torch.cuda.synchronize(device)
        one()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda.synchronize(device)
        times.append(one())
    total = reduce_max(float(sum(times)), f"cuda:{device}")
    return dict(total_ms=total, h2d=h2d, d2h=d2h, breakdown=e2e_breakdown(sg, wl, pool, host_x, host_y, stream, flush))


def e2e_breakdown(sg, wl, pool, host_x, host_y, stream, flush, reps: int = 10):
    """Where an end-to-end step's time goes: the same work as sgmv_lora_delta_host, issued
    phase by phase through the binding with events between the phases (the stream idle
    before each step): the host segment builder (host clock), the host-to-device copies
    (table, distinct x, y), the kernels, and the copy of y back.  Median microseconds."""
    n_proj = len(wl.projections)
    dev_x = {s: torch.empty_like(h, device=f"cuda:{pool.device}") for s, h in host_x.items()}
    dev_y = [torch.empty_like(h, device=f"cuda:{pool.device}") for h in host_y]
    plan = sg.BatchPlan(pool, capacity_tokens=wl.T)
    plan.build(wl.adapter_ids)
    vs = [plan.new_v() for _ in range(n_proj)]
    rows = {"build": [], "h2d": [], "kernels": [], "d2h": []}
    for i in range(reps + 2):
        flush.zero_()
        torch.cuda.synchronize(pool.device)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        t0 = time.perf_counter()
        plan.build(wl.adapter_ids)
        t1 = time.perf_counter()
        ev[0].record(stream)
        plan.upload(stream)
        for s_, h in host_x.items():
            dev_x[s_].copy_(h, non_blocking=True)
        for p in range(n_proj):
            dev_y[p].copy_(host_y[p], non_blocking=True)
        ev[1].record(stream)
        if n_proj > 1:
            sg.lora_delta_grouped([(dev_x[wl.x_of(p)], dev_y[p], p, vs[p]) for p in range(n_proj)], plan, pool,
                                  wl.scale, stream)
        else:
            sg.lora_delta(dev_x[wl.x_of(0)], plan, pool, dev_y[0], 0, wl.scale, v=vs[0], stream=stream)
        ev[2].record(stream)
        for p in range(n_proj):
            host_y[p].copy_(dev_y[p], non_blocking=True)
        ev[3].record(stream)
        ev[3].synchronize()
        if i >= 2:
            rows["build"].append((t1 - t0) * 1e6)
            rows["h2d"].append(ev[0].elapsed_time(ev[1]) * 1e3)
            rows["kernels"].append(ev[1].elapsed_time(ev[2]) * 1e3)
            rows["d2h"].append(ev[2].elapsed_time(ev[3]) * 1e3)
    return {k + "_us": round(float(statistics.median(v)), 1) for k, v in rows.items()}


# ---------------------------------------------------------------------------- oracle arm
def oracle_inputs(wl, device, weights: str = "bf16", max_tokens: int = 0):
    """fp64 host copies of the batch's inputs (x, y, A, B of the adapters in use; in a
    quantised pool's format, the dequantised weights, quantised here outside any timing).
    max_tokens > 0 keeps only the batch's first max_tokens adapted tokens (a bounded
    sample: every token's delta depends on its own row and adapter only)."""
    bank = workloads.AdapterBank(wl, device=device)
    import oracle
    from oracle import quant as oquant
    ids = wl.adapter_ids.tolist()
    if max_tokens > 0:
        keep = [t for t, a in enumerate(ids) if a >= 0][:max_tokens]
        ids = [a if t in set(keep) else -1 for t, a in enumerate(ids)]
    tix, off, seg_ad = oracle.group_by_adapter(ids)
    per_proj = []

    def weights_of(a, p):
        A, B = (workloads.bf16_to_f64(m) for m in bank.get(a, p))
        if weights == "bf16":
            return A, B
        return oquant.quantize_adapter(A.astype(np.float32), B.astype(np.float32), weights)[4:]

    for p in range(len(wl.projections)):
        x, y = workloads.activations(wl, p, device=device)
        AB = [weights_of(a, p) for a in seg_ad]
        A = [ab[0] for ab in AB]
        B = [ab[1] for ab in AB]
        per_proj.append((workloads.bf16_to_f64(x), workloads.bf16_to_f64(y), A, B))
    ranks = [wl.rank_of(a) for a in seg_ad]
    del bank
    return tix, off, ranks, per_proj


def time_oracle(prepared, wl, budget_s: float, threads: int):
    """Run the oracle over the whole batch (all projections) until about budget_s
    seconds have passed; returns (tokens/s, reps, elapsed, threads used)."""
    import oracle
    tix, off, ranks, per_proj = prepared
    used = oracle.threads_used(threads)
    reps, t0 = 0, time.perf_counter()
    while True:
        for x, y, A, B in per_proj:
            oracle.lora_delta(x, y, off, ranks, A, B, token_idx=tix, scale=wl.scale, threads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return len(tix) * reps / el, reps, el, used


def run_reference(args, rank, world, device):
    if rank != 0:
        return
    wl = workloads.make(args.workload, seed=0)
    threads = os.cpu_count() or 1
    dev = f"cuda:{device}" if torch.cuda.is_available() else "cpu"
    prepared = oracle_inputs(wl, dev, args.weights, ORACLE_SAMPLE_TOKENS.get(wl.name, 0))
    for _ in range(args.warmup):
        time_oracle(prepared, wl, 0.0, threads)
    per_step_budget = max(0.05, getattr(args, "ref_budget", 60.0) / max(args.steps, 1))
    t_all, reps_all, used = 0.0, 0, 1
    for _ in range(args.steps):
        _, reps, el, used = time_oracle(prepared, wl, per_step_budget, threads)
        t_all += el
        reps_all += reps
    n_tok = len(prepared[0])
    value = reps_all * n_tok / t_all
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_all / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, args.weights),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": f"{sample_text(wl, n_tok)} repeated {reps_all} times over "
                                       f"{args.steps} steps"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# adapted tokens of the oracle's bounded sample, by workload (0: the whole batch)
ORACLE_SAMPLE_TOKENS = {"llama70b_layer": 64, "llama70b_layer_shared_x": 64}
# workloads measured besides the headline one, each in the same process
PER_WORKLOAD = ("tiny", "decode_q_proj", "decode_q_proj_12", "mixed_rank_mlp_up", "prefill_long",
                "llama70b_layer_shared_x", "llama70b_layer")


def sample_text(wl, n_tok: int) -> str:
    whole = int((wl.adapter_ids >= 0).sum())
    what = "whole batch" if n_tok == whole else f"first {n_tok} of the batch's {whole} tokens"
    return f"{what} ({n_tok} tokens x {len(wl.projections)} projections)"


def roofline_of(res) -> dict:
    return {"bound": "hbm", "kernel": res["kernel_name"], "achieved": res["achieved"],
            "peak": res["peak"], "unit": "GB/s", "frac": res["achieved"] / res["peak"],
            "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs)" if res["peak_kind"] == "measured"
            else "fallback 6650 GB/s",
            "algorithmic_bytes_per_step": res["step_bytes"],
            "calls_per_step": res["dom_launches"],
            "launches_per_step": res["launches"],
            "traffic": res["traffic"]}


def per_workload_entry(wl, res, args, world) -> dict:
    n_tok = int((wl.adapter_ids >= 0).sum())
    return {"tokens": n_tok, "distinct_adapters": wl.distinct_adapters,
            "value": job_value(world, n_tok, args.steps, res["total_ms"]), "unit": "tokens/s",
            "ms_per_step": res["total_ms"] / args.steps, "roofline": roofline_of(res), "clocks": res["clocks"]}


def config_of(wl, weights: str = "bf16"):
    ranks = sorted(set(int(wl.rank_of(a)) for a in np.unique(wl.adapter_ids[wl.adapter_ids >= 0])))
    return {"workload": wl.name, "tokens": wl.T,
            "projections": [f"{n}:{a}->{b}" for n, a, b in wl.projections],
            "ranks": ranks, "pool_adapters": int(wl.pool_ids.size),
            "distinct_adapters": wl.distinct_adapters, "page_elems": 512, "adapter_weights": weights,
            "l2": "flushed between steps (512 MiB write, then read back, outside the timed window)",
            "parallelism": "replicas"}


# ---------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama70b_layer", choices=workloads.WORKLOAD_NAMES)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pool", type=int, default=0,
                    help="resident adapters of the pool (llama70b_layer only; for small profiler captures, "
                         "the kernels see the same batch shape)")
    ap.add_argument("--per-projection", action="store_true",
                    help="one sgmv_lora_delta call per projection instead of one sgmv_lora_delta_grouped call "
                         "for all projections of a multi-projection workload (the default)")
    ap.add_argument("--split-phases", action="store_true",
                    help="record an event between shrink and expand (times each phase; removes their overlap)")
    ap.add_argument("--weights", default="bf16", choices=sorted(WEIGHT_BYTES),
                    help="adapter storage of the pool: bf16, or FP8 E4M3 / INT4 codes with a scale per rank row")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the other workloads' lines (per_workload; measured at N = 1 only)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-budget", type=float, default=60.0,
                    help="seconds of oracle time over all steps of --impl reference")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.grouped = not args.per_projection and not args.split_phases

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        if torch.cuda.is_available():
            torch.cuda.set_device(0)

    try:
        if args.impl == "reference":
            run_reference(args, rank, world, local)
            return
        wl, res = run_ours(args, rank, world, local)
        if rank != 0:
            return
        n_tok = int((wl.adapter_ids >= 0).sum())
        value = job_value(world, n_tok, args.steps, res["total_ms"])
        e2e = res["e2e"]
        e2e_value = job_value(world, n_tok, args.steps, e2e["total_ms"])
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["total_ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_of(wl, args.weights),
            "hbm_gbs_step": res["step_bytes"] / (res["total_ms"] / args.steps * 1e-3) / 1e9,
            "roofline": roofline_of(res),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d"],
                    "d2h_bytes_per_step": e2e["d2h"], "breakdown": e2e["breakdown"]},
            "gpu_launches": res["launches"] * args.steps,
            "clocks": res["clocks"],
        }
        if "phase_ms" in res:
            line["phase_ms"] = res["phase_ms"]
            line["phase_us_per_proj"] = res["phase_us_per_proj"]
        if not args.no_cpu_baseline and world == 1:
            prepared = oracle_inputs(wl, f"cuda:{local}", args.weights, ORACLE_SAMPLE_TOKENS.get(wl.name, 0))
            rate, reps, el, used = time_oracle(prepared, wl, args.cpu_budget, os.cpu_count() or 1)
            line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": used, "kind": "oracle",
                                    "sample": f"{sample_text(wl, len(prepared[0]))} repeated {reps} times"
                                              f" in {el:.1f} s"}
        if not args.no_per_workload and world == 1:
            import copy
            line["per_workload"] = {}
            for name in PER_WORKLOAD:
                if name == wl.name:
                    continue
                a2 = copy.copy(args)
                a2.workload, a2.pool = name, 0
                a2.grouped = not args.per_projection and not args.split_phases
                wl2, res2 = run_ours(a2, rank, world, local, with_e2e=False)
                line["per_workload"][name] = per_workload_entry(wl2, res2, a2, world)
                del res2
                torch.cuda.empty_cache()
        print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
