"""The roofline numerator of bench.py: algorithmic bytes per step, pinned to closed forms
(CPU only).  Each distinct adapter's A and B once, x read once, v written and read in fp32,
y read and written; the adapter bytes of a rank-16 Llama-3-70B layer are those of the
memory table in "Multi-LoRA serving: the single translator with a thousand glossaries
..." (section "The maths that matters")."""
import json
import os

import bench
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _total(wl, weights="bf16"):
    return sum(sum(bench.algorithmic_bytes(wl, p, weights)[:2]) for p in range(len(wl.projections)))


def test_tiny_bytes_closed_form():
    wl = workloads.make("tiny")            # 64 tokens, 512 -> 512, 4 adapters of rank 8
    shrink, expand, flops, _ = bench.algorithmic_bytes(wl, 0)
    assert shrink == 2 * 4 * 8 * 512 + 2 * 64 * 512 + 4 * 64 * 8 == 100352
    assert expand == 2 * 4 * 8 * 512 + 4 * 64 * 8 + 4 * 64 * 512 == 165888
    assert flops == 2 * 64 * 8 * (512 + 512)


def test_prefill_bytes_by_term():
    wl = workloads.make("prefill_long")    # 8 x 512 tokens, 8192 -> 8192, 8 adapters of rank 64
    T, d, r = 4096, 8192, 64
    x, y, w, v = 2 * T * d, 4 * T * d, 2 * 8 * r * (d + d), 8 * T * r
    assert _total(wl) == x + y + w + v == 220200960


def test_llama70b_layer_weight_bytes_match_the_memory_table():
    with open(os.path.join(GOLDEN, "memory_table_llama3_70b_r16.json")) as f:
        per_adapter = json.load(f)["sum_per_layer_bytes"]
    wl = workloads.make("llama70b_layer")  # 256 tokens, each on its own rank-16 adapter
    T, r = 256, 16
    act = sum(2 * T * d_in + 4 * T * d_out + 8 * T * r for _, d_in, d_out in wl.projections)
    assert _total(wl) - act == 256 * per_adapter == 1325400064


def test_quantised_weight_bytes():
    wl = workloads.make("prefill_long")
    w16 = 2 * 8 * 64 * (8192 + 8192)
    rest = _total(wl) - w16
    scales = 2 * 4 * 8 * 64                # one fp32 scale per rank row of A and of B^T
    assert _total(wl, "fp8_e4m3") == rest + w16 // 2 + scales
    assert _total(wl, "int4") == rest + w16 // 4 + scales


def test_shared_x_layer_counts_each_input_once():
    """The layer with a real layer's inputs (q, k, v read one x; gate, up one x): the
    same bytes as the layer with seven inputs, less the x reads of k, v and up."""
    shared, own = workloads.make("llama70b_layer_shared_x"), workloads.make("llama70b_layer")
    assert shared.adapter_ids.tolist() == own.adapter_ids.tolist()
    T = 256
    assert [shared.x_of(p) for p in range(7)] == [0, 0, 0, 3, 4, 4, 6]
    assert _total(own) - _total(shared) == 3 * 2 * T * 8192
