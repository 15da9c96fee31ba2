"""Quantised adapter pools (FP8 E4M3 / INT4 codes, one fp32 scale per rank row) on the GPU.

1. The codes and scales the pool stores (quantised on the device as it loads bf16
   weights) are bit-identical to the oracle's quantiser (oracle/quant.py): the integer
   decisions are taken in fp32 on both sides.
2. The delta through every path (SIMT, tensor cores, one call or two, grouped
   projections, the residency manager) matches the fp64 oracle computed with the
   dequantised weights, under the gates of tests/sgmv_cases.py.
"""
import numpy as np
import pytest
import torch

from oracle import quant as oquant
import segmented_rank_gemm_sgmv_b200 as sg
import workloads
from sgmv_cases import build_pool, compare, run_gpu, run_oracle
from test_parity_gpu import SIMT, TC, custom_case
from test_grouped_gpu import PROJS, _case

pytestmark = pytest.mark.gpu

FMTS = pytest.mark.parametrize("fmt", ["fp8_e4m3", "int4"])


def _f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


@FMTS
@pytest.mark.parametrize("page_elems", [64, 512])
@pytest.mark.parametrize("src", ["device", "host"])
def test_codes_and_scales_bit_exact(fmt, page_elems, src):
    d_in, d_out = 1024, 1536
    pool = sg.AdapterPool([(d_in, d_out)], num_pages=4096, page_elems=page_elems, max_rank=32, device=0,
                          weight_format=fmt)
    pool.shuffle_free_pages(7)
    g = torch.Generator(device="cuda").manual_seed(3)
    for a, r in enumerate([5, 16, 32]):
        A = (torch.randn(r, d_in, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
        B = (torch.randn(d_out, r, generator=g, device="cuda") * 0.2).to(torch.bfloat16)
        if r == 5:
            A[2].zero_()                 # a zero row: scale 0, codes 0
            B[:, 1].zero_()              # a zero rank column of B = a zero row of B^T
            A[3, 7] = 1000.0             # one huge value: the rest of the row rounds to small codes
            A[4, ::3] = -A[4, ::3]       # ties and signs
        if src == "host":
            pool.load(a, r, [A.cpu()], [B.cpu()])
        else:
            pool.load(a, r, [A], [B])
        for m, W in ((0, _f32(A)), (1, _f32(B).T.copy())):
            codes, scales = pool.read(a, 0, m)
            want_codes, want_scales = oquant.quantize_rows(W, fmt)
            assert np.array_equal(scales.view(np.uint32), want_scales.view(np.uint32)), (a, m)
            assert np.array_equal(codes, want_codes), (a, m, np.argwhere(codes != want_codes)[:5])
    s = pool.stats()
    assert s.weight_format == sg.WEIGHT_FORMATS[fmt]
    assert s.page_bytes == (page_elems if fmt == "fp8_e4m3" else page_elems // 2)


@FMTS
@pytest.mark.parametrize("mode", ["separate", "lora_delta"])
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32], ids=["ybf16", "yfp32"])
def test_ragged_segments(fmt, path, y_dtype, mode):
    # segment lengths around the 4-row SIMT items and the 128-row tiles, ranks not multiples of 8/16
    wl, bank, x, y = custom_case([1, 3, 4, 5, 17, 130, 2], [8, 12, 16, 5, 64, 128, 33], 1024, 1536, seed=9,
                                 minus_one=3)
    pool = build_pool(wl, bank, weight_format=fmt)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, path, y_dtype, mode=mode)
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y, weight_format=fmt))


@FMTS
@pytest.mark.parametrize("page_elems", [64, 256, 1024])
@pytest.mark.parametrize("path", [SIMT, TC], ids=["simt", "tc"])
def test_page_sizes(fmt, page_elems, path):
    wl, bank, x, y = custom_case([2, 6, 40], [16, 8, 32], 2048, 1024, seed=4)
    pool = build_pool(wl, bank, page_elems=page_elems, weight_format=fmt)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, path, mode="lora_delta")
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y, weight_format=fmt))


@FMTS
@pytest.mark.parametrize("name", ["decode_q_proj", "mixed_rank_mlp_up", "prefill_long"])
def test_workloads(fmt, name):
    wl = workloads.make(name)
    bank = workloads.AdapterBank(wl, device="cuda")
    x, y = workloads.activations(wl, 0, device="cuda")
    pool = build_pool(wl, bank, weight_format=fmt)
    plan, v, y_out = run_gpu(pool, wl, 0, x, y, 0, mode="lora_delta")
    compare(plan, v, y_out, y, run_oracle(wl, bank, 0, x, y, weight_format=fmt))


@FMTS
@pytest.mark.parametrize("thr", [0, 10 ** 9, 1], ids=["dispatch", "simt", "tc"])
def test_grouped(fmt, thr):
    wl, bank, acts = _case([1, 3, 5, 17, 150, 40, 2, 9], [8, 16, 24, 64, 128, 32, 16, 8], seed=31)
    pool = build_pool(wl, bank, weight_format=fmt)
    plan = pool.plan(wl.adapter_ids, long_threshold=thr)
    plan.upload()
    ys = [y.clone() for _, y in acts]
    vs = sg.lora_delta_grouped([(acts[p][0], ys[p], p) for p in range(len(PROJS))], plan, pool, 1.0)
    assert sg.check_errors() == 0
    for p in range(len(PROJS)):
        compare(plan, vs[p], ys[p], acts[p][1], run_oracle(wl, bank, p, acts[p][0], acts[p][1], weight_format=fmt))


@FMTS
def test_residency_loads_quantise_like_direct_loads(fmt):
    d_in, d_out, r = 1024, 512, 16
    pool = sg.AdapterPool([(d_in, d_out)], num_pages=2 * r * (d_in + d_out) // 512 + 8, page_elems=512,
                          max_rank=r, device=0, weight_format=fmt)
    res = sg.Residency(pool)
    g = torch.Generator().manual_seed(1)
    host = {}
    for a in range(3):
        A = (torch.randn(r, d_in, generator=g) * 0.1).to(torch.bfloat16).pin_memory()
        B = (torch.randn(d_out, r, generator=g) * 0.1).to(torch.bfloat16).pin_memory()
        host[a] = (A, B)
        res.register(a, r, [A], [B])
    copy = torch.cuda.Stream()
    for a in (0, 1, 2, 0):   # room for two: the third evicts, the fourth reloads
        res.prepare(np.array([a], np.int32), copy_stream=copy)
        torch.cuda.synchronize()
        A, B = host[a]
        codes, scales = pool.read(a, 0, 0)
        want_codes, want_scales = oquant.quantize_rows(_f32(A), fmt)
        assert np.array_equal(codes, want_codes) and np.array_equal(scales, want_scales)
        codes, scales = pool.read(a, 0, 1)
        want_codes, want_scales = oquant.quantize_rows(_f32(B).T.copy(), fmt)
        assert np.array_equal(codes, want_codes) and np.array_equal(scales, want_scales)
    assert res.stats().evictions >= 2
    res.close()


def test_quantised_pool_memory():
    projs = [(8192, 8192)]
    for fmt, per_page in (("bf16", 1024), ("fp8_e4m3", 512), ("int4", 256)):
        pool = sg.AdapterPool(projs, num_pages=64, page_elems=512, max_rank=16, device=0, weight_format=fmt)
        assert pool.stats().page_bytes == per_page
        pool.close()


def test_bf16_pool_read_returns_the_stored_weights():
    d_in, d_out, r = 1024, 512, 12
    pool = sg.AdapterPool([(d_in, d_out)], num_pages=256, page_elems=512, max_rank=16, device=0)
    pool.shuffle_free_pages(5)
    g = torch.Generator(device="cuda").manual_seed(2)
    A = torch.randn(r, d_in, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(d_out, r, generator=g, device="cuda").to(torch.bfloat16)
    pool.load(3, r, [A], [B])
    codes, scales = pool.read(3, 0, 0)
    assert np.array_equal(codes, A.view(torch.int16).cpu().numpy().view(np.uint16)) and np.all(scales == 1.0)
    codes, _ = pool.read(3, 0, 1)
    assert np.array_equal(codes, B.t().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
