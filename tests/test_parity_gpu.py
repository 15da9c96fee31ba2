"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element.  Gates and tolerances: tests/sgmv_cases.py.

The five workloads are the pages' shapes (see workloads/): tiny, decode q_proj,
mixed ranks (MLP up), long prefill segments, and a full Llama-3-70B layer; the
rest are edge cases of the method: ragged segment lengths around the 4-row
SIMT items, the 16-row dispatch threshold and the 128-row tensor-core tiles,
ranks that are not multiples of 8 or 16, the largest rank, tokens without an
adapter, empty batches, page sizes other than 512 elements, and the pins that
fix the arithmetic exactly (integer inputs, zero B, zero scale).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import GATE_REL, build_pool, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

TC = 1                 # long_threshold that sends every segment to the tensor-core path
SIMT = 1 << 30  # long_threshold that keeps every segment on the SIMT path


class DictBank:
    def __init__(self):
        self.m = {}

    def get(self, a, p):
        return self.m[(a, p)]


def custom_case(seg_lens, ranks, d_in, d_out, seed=0, minus_one=0, shuffle=True, device="cuda", ints=False,
                scale=1.0):
    """Workload with given segment lengths and ranks (one adapter per segment)."""
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.full(n, a, dtype=np.int32) for a, n in enumerate(seg_lens)] +
                         [np.full(minus_one, -1, dtype=np.int32)])
    if shuffle:
        ids = ids[rng.permutation(ids.size)]
    wl = workloads.Workload("custom", seed, int(ids.size), [("p", d_in, d_out)],
                            np.arange(len(seg_lens), dtype=np.int32), np.asarray(ranks, dtype=np.int32), ids,
                            scale=scale)
    bank = DictBank()
    g = torch.Generator(device=device).manual_seed(seed)
    for a, r in enumerate(ranks):
        if ints:
            A = torch.randint(-1, 2, (r, d_in), generator=g, device=device).to(torch.bfloat16)
            B = torch.randint(-1, 2, (d_out, r), generator=g, device=device).to(torch.bfloat16)
        else:
            A = (torch.randn(r, d_in, generator=g, device=device) / d_in ** 0.5).to(torch.bfloat16)
            B = (torch.randn(d_out, r, generator=g, device=device) / max(r, 1) ** 0.5).to(torch.bfloat16)
        bank.m[(a, 0)] = (A, B)
    T = wl.T
    if ints:
        x = torch.zeros(T, d_in, device=device)
        for t in range(T):
            nz = torch.randperm(d_in, generator=g, device=device)[:8]
            x[t, nz] = torch.randint(0, 2, (8,), generator=g, device=device).float() * 2 - 1
        x = x.to(torch.bfloat16)
        y = torch.randint(-8, 9, (T, d_out), generator=g, device=device).to(torch.bfloat16)
    else:
        x = (torch.randn(T, d_in, generator=g, device=device) / d_in ** 0.5).to(torch.bfloat16)
        y = torch.randn(T, d_out, generator=g, device=device).to(torch.bfloat16)
    return wl, bank, x, y


def check(wl, bank, x, y, long_threshold, y_dtype=torch.bfloat16, proj=0, mode="separate", **kw):
    pool = build_pool(wl, bank)
    plan, v, y_out = run_gpu(pool, wl, proj, x, y, long_threshold, y_dtype, mode=mode, **kw)
    ref = run_oracle(wl, bank, proj, x, y, **kw)
    errs = compare(plan, v, y_out, y, ref)
    return plan, v, y_out, ref, errs


# ------------------------------------------------------------------ workloads
MODES = pytest.mark.parametrize("mode", ["separate", "lora_delta"])


@MODES
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_tiny(path, y_dtype, mode):
    wl = workloads.make("tiny")
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    plan, *_ = check(wl, bank, x, y, path, y_dtype, mode=mode)
    assert (plan.plan.num_tc_tiles > 0) == (path == TC)


@MODES
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_decode_q_proj(y_dtype, mode):
    """Gate A on bf16 y, and Gate B on fp32 y: relative to the delta itself, which is
    only ~1 % of y at d = 8192."""
    wl = workloads.make("decode_q_proj")
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    plan, *_ = check(wl, bank, x, y, 0, y_dtype, mode=mode)
    assert plan.plan.num_tc_tiles == 0 and plan.plan.num_segments == wl.distinct_adapters


def test_decode_q_proj_12():
    """The decode batch with about 12 distinct adapters among 32 requests (Zipf s = 1.5)."""
    wl = workloads.make("decode_q_proj_12")
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    plan, *_ = check(wl, bank, x, y, 0, mode="lora_delta")
    assert plan.plan.num_tc_tiles == 0 and plan.plan.num_segments == wl.distinct_adapters < 20


@MODES
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_mixed_rank_mlp_up(y_dtype, mode):
    wl = workloads.make("mixed_rank_mlp_up")
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    plan, *_ = check(wl, bank, x, y, 0, y_dtype, mode=mode)
    assert len(set(plan.seg_rank.tolist())) == 4


@pytest.mark.parametrize("path,mode,y_dtype",
                         [(0, "separate", torch.bfloat16), (0, "lora_delta", torch.bfloat16),
                          (0, "lora_delta", torch.float32), (SIMT, "separate", torch.bfloat16)],
                         ids=["dispatch", "dispatch-lora_delta", "dispatch-lora_delta-yfp32", "simt"])
def test_prefill_long(path, mode, y_dtype):
    wl = workloads.make("prefill_long")
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    plan, *_ = check(wl, bank, x, y, path, y_dtype, mode=mode)
    if path == 0:
        assert plan.plan.num_tc_tiles == 32 and plan.plan.num_simt_items == 0


@MODES
def test_llama70b_layer_sampled(mode):
    """Full-size layer (pool of 2000 rank-16 adapters, 7 projections, 256 tokens on
    distinct adapters), one call per projection (the benchmark's grouped call over all
    seven is checked on every token in tests/test_grouped_gpu.py); the oracle recomputes
    a sample of 32 tokens one by one for every projection."""
    wl = workloads.make("llama70b_layer")
    bank = workloads.AdapterBank(wl, device="cuda")
    pool = build_pool(wl, bank)
    rng = np.random.default_rng(123)
    sample = sorted(rng.choice(wl.T, size=32, replace=False).tolist())
    for p in range(len(wl.projections)):
        x, y = workloads.activations(wl, p, device="cuda")
        plan, v, y_out = run_gpu(pool, wl, p, x, y, mode=mode)
        ref = run_oracle(wl, bank, p, x, y, rows_of_tokens=sample)
        compare(plan, v, y_out, y, ref, check_rows=sample)
        # every token is its own segment; untouched rows do not exist in this workload
        assert plan.plan.num_segments == 256 and plan.plan.num_simt_items == 256


# ------------------------------------------------------------------ slab shrink
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
@pytest.mark.parametrize("case", ["decode200", "mixed64", "ragged"])
def test_slab_shrink(case, y_dtype):
    """Single-projection batches that take the one-shot slab shrink (each CTA's whole slice of
    A staged at once, contracted with warp-level mma): 200 decode tokens, 64 mixed-rank tokens,
    and ragged segments with ranks that are not multiples of 16 (padding rows of the mma
    tiles) and a d_in of 3 pages (cluster of 3)."""
    if case == "decode200":
        wl = workloads.make("decode_q_proj", T=200)
    elif case == "mixed64":
        wl = workloads.make("mixed_rank_mlp_up", T=64)
    if case == "ragged":
        wl, bank, x, y = custom_case([1, 2, 3, 4, 5, 7, 9, 2, 1], [3, 24, 40, 57, 64, 9, 16, 1, 33], 1536, 1024,
                                     seed=11, minus_one=3)
    else:
        bank = workloads.AdapterBank(wl, device="cuda")
        x, y = workloads.activations(wl, 0, device="cuda")
    pool = build_pool(wl, bank)
    plan = pool.plan(wl.adapter_ids, long_threshold=SIMT)
    kinds, _ = sg.lora_delta_kernels(plan, pool, [0], y_dtype)
    assert kinds == sg.KERNELS_SIMT | sg.KERNELS_SLAB, kinds
    pool.close()
    for mode in ("separate", "lora_delta"):
        check(wl, bank, x, y, SIMT, y_dtype, mode=mode)


# ------------------------------------------------------------------ exact pins
@MODES
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("d", [512, 1024, 1536])
def test_exact_integer_inputs_bit_exact(path, d, mode):
    """Integer inputs whose every partial sum is exact in bf16/fp32/fp64: the GPU must
    equal the oracle bit for bit, in v and in y, on both paths."""
    wl, bank, x, y = custom_case([3, 70, 1, 130, 5, 8], [4, 3, 1, 2, 16, 9], d, 2 * d, seed=5, minus_one=5,
                                 ints=True)
    pool = build_pool(wl, bank)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, path, mode=mode)
    ref = run_oracle(wl, bank, 0, x, y)
    vg = v.double().cpu().numpy()
    row = {t: i for i, t in enumerate(plan.token_idx.tolist())}
    for s, r in enumerate(ref["ranks"]):
        for i in range(ref["off"][s], ref["off"][s + 1]):
            assert np.array_equal(vg[row[ref["tix"][i]], :r], ref["v"][i, :r])
    assert np.array_equal(y_out.double().cpu().numpy(), ref["y"])


@MODES
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_zero_B_and_zero_scale_leave_y_unchanged(path, mode):
    wl, bank, x, y = custom_case([5, 90], [8, 16], 512, 1024, seed=6)
    for a in range(2):
        A, B = bank.m[(a, 0)]
        bank.m[(a, 0)] = (A, torch.zeros_like(B))
    pool = build_pool(wl, bank)
    _, _, y_out = run_gpu(pool, wl, 0, x, y, path, mode=mode)
    assert torch.equal(y_out.view(torch.int16), y.view(torch.int16))
    wl2, bank2, x2, y2 = custom_case([5, 90], [8, 16], 512, 1024, seed=7)
    pool2 = build_pool(wl2, bank2)
    _, _, y_out2 = run_gpu(pool2, wl2, 0, x2, y2, path, scale=0.0, mode=mode)
    assert torch.equal(y_out2.view(torch.int16), y2.view(torch.int16))


# ------------------------------------------------------------------ edge cases
@MODES
@pytest.mark.parametrize("path", [0, SIMT, TC], ids=["dispatch", "simt", "tc"])
def test_ragged_lengths_and_odd_ranks(path, mode):
    lens = [1, 63, 64, 65, 127, 128, 129, 200, 2, 3, 5, 7, 8, 9, 15, 16, 17]
    ranks = [5, 24, 100, 128, 16, 8, 40, 64, 128, 8, 16, 32, 64, 12, 72, 8, 16]
    wl, bank, x, y = custom_case(lens, ranks, 1536, 2560, seed=8, minus_one=11)
    check(wl, bank, x, y, path, torch.float32, mode=mode)


@MODES
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_single_token_and_rank_zero(path, mode):
    wl, bank, x, y = custom_case([1], [16], 512, 512, seed=9)
    check(wl, bank, x, y, path, mode=mode)
    wl, bank, x, y = custom_case([3, 4], [0, 8], 512, 512, seed=10, minus_one=2)
    check(wl, bank, x, y, path, mode=mode)


def test_empty_batches():
    wl, bank, x, y = custom_case([], [], 512, 512, seed=11, minus_one=7)
    pool = build_pool(wl, bank) if len(wl.pool_ids) else sg.AdapterPool([(512, 512)], 16, 512, 16, 0)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y)
    assert torch.equal(y_out, y)
    wl0 = workloads.Workload("e", 0, 0, [("p", 512, 512)], np.zeros(0, np.int32), np.zeros(0, np.int32),
                             np.zeros(0, np.int32))
    x0 = torch.zeros(0, 512, dtype=torch.bfloat16, device="cuda")
    run_gpu(pool, wl0, 0, x0, x0.clone())


@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_padded_rank_within_gate(path):
    """An adapter zero-padded to a larger rank gives the same delta (no-padding claim)."""
    wl, bank, x, y = custom_case([7, 80], [8, 16], 1024, 512, seed=12)
    _, v1, y1, _, _ = check(wl, bank, x, y, path, torch.float32)
    for a, r in ((0, 8), (1, 16)):
        A, B = bank.m[(a, 0)]
        bank.m[(a, 0)] = (torch.cat([A, torch.zeros(r, A.shape[1], dtype=A.dtype, device=A.device)]),
                          torch.cat([B, torch.zeros(B.shape[0], r, dtype=B.dtype, device=B.device)], dim=1))
    wl.pool_ranks = wl.pool_ranks * 2
    _, v2, y2, _, _ = check(wl, bank, x, y, path, torch.float32)
    d = (y1.double() - y.double()).norm(dim=1)
    assert ((y2.double() - y1.double()).norm(dim=1) <= GATE_REL * d + 1e-30).all()


def test_permuted_batch():
    wl, bank, x, y = custom_case([9, 3, 70], [16, 32, 8], 512, 1024, seed=13, minus_one=4)
    _, _, y1, _, _ = check(wl, bank, x, y, 0)
    perm = torch.randperm(wl.T, generator=torch.Generator().manual_seed(1))
    wl.adapter_ids = wl.adapter_ids[perm.numpy()]
    xp, yp = x[perm.cuda()].contiguous(), y[perm.cuda()].contiguous()
    _, _, y2, _, _ = check(wl, bank, xp, yp, 0)
    y1p = y1[perm.cuda()].float()
    assert ((y2.float() - y1p).abs() <= y1p.abs() * 2 ** -7 + 1e-30).all()   # at most one bf16 ulp


def test_pool_pages_hold_A_rows_and_Bt_rows():
    wl, bank, x, y = custom_case([2, 2], [8, 24], 1024, 1536, seed=14)
    pool = build_pool(wl, bank)
    pages = pool.pages_tensor()
    P = pool.page_elems
    for a, r in ((0, 8), (1, 24)):
        A, B = bank.m[(a, 0)]
        ids_a = torch.from_numpy(pool.page_ids(a, 0, 0)).long().cuda()
        ids_b = torch.from_numpy(pool.page_ids(a, 0, 1)).long().cuda()
        assert torch.equal(pages[ids_a].reshape(r, 1024).view(torch.int16), A.view(torch.int16))
        assert torch.equal(pages[ids_b].reshape(r, 1536).view(torch.int16), B.t().contiguous().view(torch.int16))
    assert P == 512


@MODES
def test_device_bounds_checks_report_without_faulting(mode):
    """A corrupted device table (token row past the batch) is caught by the kernels'
    own bounds checks: the access is skipped and sgmv_check_errors reports it."""
    for path in (SIMT, TC):
        wl, bank, x, y = custom_case([3, 130], [8, 16], 512, 512, seed=15)
        pool = build_pool(wl, bank)
        plan = pool.plan(wl.adapter_ids, long_threshold=path)
        if plan.plan.needs_device_table:     # the kernels read the device copy: corrupt that
            table = plan.upload()
            torch.cuda.synchronize()
            tix = table[plan.plan.off_token_idx:plan.plan.off_token_idx + 4 * plan.num_rows].view(torch.int32)
        else:                                # the work items travel as launch arguments, built from the host table
            tix = plan.host[plan.plan.off_token_idx:plan.plan.off_token_idx + 4 * plan.num_rows].view(torch.int32)
        tix[0] = wl.T + 5
        v = plan.new_v()
        y2 = y.clone()
        if mode == "separate":
            sg.shrink(x, plan, pool, v, 0)
            sg.expand(v, plan, pool, y2, 0)
        else:
            sg.lora_delta(x, plan, pool, y2, 0, v=v)
        with pytest.raises(sg.SgmvError) as e:
            sg.check_errors()
        assert e.value.status == 6
        assert sg.check_errors() == 0   # cleared


def test_lora_delta_requires_workspace():
    wl, bank, x, y = custom_case([1, 2, 3], [16, 8, 32], 1024, 1024, seed=21, minus_one=3)
    pool = build_pool(wl, bank)
    plan = pool.plan(wl.adapter_ids)
    plan.upload()
    lib = sg.load_library()
    import ctypes
    st = lib.sgmv_lora_delta(x.data_ptr(), x.stride(0), plan.T, 1024, 1024, 0, ctypes.byref(plan.plan),
                             plan.table_ptr(), pool.handle, 1.0, y.data_ptr(), y.stride(0), 0, None, 0,
                             None)
    assert st == 1


@pytest.mark.parametrize("page_elems,d_in,d_out", [(64, 1536, 2560), (256, 1536, 2560), (1024, 2048, 3072)],
                         ids=["P64", "P256", "P1024"])
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_page_sizes(page_elems, d_in, d_out, path, y_dtype):
    """Other page sizes: a B^T block or an A chunk spans several small pages, or a
    CTA's column range starts inside a large one."""
    wl, bank, x, y = custom_case([1, 3, 5, 17, 130, 40], [8, 16, 24, 64, 128, 32], d_in, d_out, seed=21,
                                 minus_one=4)
    pool = build_pool(wl, bank, page_elems=page_elems)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, path, y_dtype, mode="lora_delta")
    ref = run_oracle(wl, bank, 0, x, y)
    errs = compare(plan, v, y_out, y, ref)
    assert errs["v"] <= GATE_REL and errs["y"] <= GATE_REL, errs
    assert sg.check_errors() == 0
