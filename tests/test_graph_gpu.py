"""CUDA-graph capture of a delta step: the library's launches (the fused decode kernel with its
work items as launch arguments, the SIMT pair, the tensor-core pair reading a device table)
are captured into a graph and replayed; every replay must equal the eager call bit for bit
(the kernels are deterministic), and the result must pass the oracle's gates.  A graph bakes
in its launch configuration and launch arguments, so a serving loop replays one per batch
shape; the device table of a plan that needs one may be rewritten between replays."""
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw,kind", [
    ("decode_q_proj", {}, sg.KERNELS_FUSED),
    ("mixed_rank_mlp_up", dict(T=128), sg.KERNELS_SIMT),
    ("prefill_long", dict(requests=2, seq=256, d=2048), sg.KERNELS_TC),
])
def test_captured_step_replays_like_the_eager_call(name, kw, kind):
    wl = workloads.make(name, seed=21, **kw)
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    x, y0 = workloads.activations(wl, 0, device="cuda")
    plan = sg.BatchPlan(pool, capacity_tokens=wl.T)
    plan.build(wl.adapter_ids)
    plan.upload()
    kinds, _ = sg.lora_delta_kernels(plan, pool, [0], y0.dtype)
    assert kinds & kind
    v = plan.new_v()

    y_eager = y0.clone()
    sg.lora_delta(x, plan, pool, y_eager, 0, wl.scale, v=v)  # also sets every kernel attribute once
    torch.cuda.synchronize()
    sg.check_errors()

    y_static = y0.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            sg.lora_delta(x, plan, pool, y_static, 0, wl.scale, v=v)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        y_static.copy_(y0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_static.view(torch.int16), y_eager.view(torch.int16))
    sg.check_errors()
    ref = run_oracle(wl, bank, 0, x, y0)
    compare(plan, v, y_static, y0, ref)
    del g
    pool.close()
