"""sgmv_lora_delta_kernels: the kernels the library reports for a call are the kernels the
call launches.  Checked with the CUDA profiler's kernel list for a decode-sized call (one
fused launch), mixed-rank and larger decode batches (the SIMT pair, with the slab shrink
where it applies), a prefill batch (tensor-core pair) and a grouped call over a layer's
projections (one SIMT pair for all of them)."""
import pytest
import torch
from torch.profiler import ProfilerActivity, profile

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool

pytestmark = pytest.mark.gpu


def _kernels_launched(fn):
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    ours = ("shrink_simt_kernel", "expand_simt_kernel", "fused_simt_kernel", "shrink_slab_kernel",
            "shrink_tc_kernel", "expand_tc_kernel")
    return [n for n in names if any(k in n for k in ours)]


@pytest.mark.parametrize("name,kw,want", [
    ("decode_q_proj", {}, sg.KERNELS_FUSED),
    ("mixed_rank_mlp_up", {}, sg.KERNELS_SIMT),
    ("mixed_rank_mlp_up", dict(T=64), sg.KERNELS_SIMT),
    ("decode_q_proj", dict(T=200), sg.KERNELS_SIMT),
    ("prefill_long", dict(requests=2, seq=256, d=2048), sg.KERNELS_TC),
])
def test_single_projection_calls(name, kw, want):
    wl = workloads.make(name, seed=3, **kw)
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    x, y = workloads.activations(wl, 0, device="cuda")
    plan = sg.BatchPlan(pool, capacity_tokens=wl.T)
    plan.build(wl.adapter_ids)
    plan.upload()
    kinds_all, launches = sg.lora_delta_kernels(plan, pool, [0], y.dtype)
    kinds = kinds_all & ~sg.KERNELS_SLAB
    assert kinds == want
    assert not (kinds_all & sg.KERNELS_SLAB) or kinds == sg.KERNELS_SIMT
    v = plan.new_v()
    seen = _kernels_launched(lambda: sg.lora_delta(x, plan, pool, y, 0, 1.0, v=v))
    assert len(seen) == launches, seen
    if want == sg.KERNELS_FUSED:
        assert all("fused_simt_kernel" in n for n in seen)
    elif want == sg.KERNELS_SIMT:
        shrink = "shrink_slab_kernel" if kinds_all & sg.KERNELS_SLAB else "shrink_simt_kernel"
        assert sorted(n.split("<")[0].split("::")[-1] for n in seen) == ["expand_simt_kernel", shrink]
    else:
        assert sorted(n.split("<")[0].split("::")[-1] for n in seen) == ["expand_tc_kernel", "shrink_tc_kernel"]
    sg.check_errors()
    pool.close()


def test_grouped_layer_call():
    wl = workloads.make("llama70b_layer", seed=4, T=40, pool=64)
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    acts = [workloads.activations(wl, p, device="cuda") for p in range(len(wl.projections))]
    plan = sg.BatchPlan(pool, capacity_tokens=wl.T)
    plan.build(wl.adapter_ids)
    plan.upload()
    projs = list(range(len(wl.projections)))
    kinds, launches = sg.lora_delta_kernels(plan, pool, projs, torch.bfloat16)
    vs = [plan.new_v() for _ in projs]
    seen = _kernels_launched(lambda: sg.lora_delta_grouped([(acts[p][0], acts[p][1], p, vs[p]) for p in projs],
                                                           plan, pool, 1.0))
    assert len(seen) == launches, seen
    if plan.plan.needs_device_table:
        assert kinds == sg.KERNELS_SIMT and launches == 2
    else:  # entries run one at a time, each its own (possibly fused) call
        assert launches >= len(projs)
    sg.check_errors()
    pool.close()
