"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a result the pages print, a closed form, a textbook routine, exact
integer arithmetic or an invariant of the definition -- so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them.

Pages, by title:
  [SGMV post] "Multi-LoRA serving: the single translator with a thousand glossaries --
              shared base, thousands of concurrent adapters and the SGMV kernel"
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, T, d_in, d_out, ranks, token_perm=True):
    """Random fp64 case with one segment per rank entry and random token order."""
    S = len(ranks)
    sizes = rng.multinomial(T, np.ones(S) / S) if S else np.zeros(0, dtype=int)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    A = [rng.standard_normal((r, d_in)) for r in ranks]
    B = [rng.standard_normal((d_out, r)) for r in ranks]
    x = rng.standard_normal((T, d_in))
    W = rng.standard_normal((d_out, d_in))
    y_in = x @ W.T
    tix = rng.permutation(T) if token_perm else np.arange(T)
    return dict(x=x, W=W, y_in=y_in, off=off, ranks=list(ranks), A=A, B=B, tix=tix)


# -- p1: merged weights ----------------------------------------------------------------
def test_merged_weights_identity():
    """[SGMV post] "The bare mechanism": W' = W + BA and y = Wx + B(Ax) are the same map.
    Oracle result (unmerged, shrink then expand) vs the explicitly merged (W + s*B A) x."""
    rng = np.random.default_rng(1)
    T, d_in, d_out = 23, 40, 56
    c = _rand_case(rng, T, d_in, d_out, [3, 7, 1, 5])
    scale = 0.75
    v, y = oracle.lora_delta(c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"],
                             token_idx=c["tix"], scale=scale)
    for s in range(len(c["ranks"])):
        Wm = c["W"] + scale * (c["B"][s] @ c["A"][s])
        for i in range(c["off"][s], c["off"][s + 1]):
            t = c["tix"][i]
            ref = Wm @ c["x"][t]
            np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


# -- p2: zero B ------------------------------------------------------------------------
def test_zero_B_gives_zero_delta():
    """B = 0 makes the delta B(Ax) vanish: y must equal y_in bit for bit."""
    rng = np.random.default_rng(2)
    c = _rand_case(rng, 17, 32, 24, [4, 2])
    B0 = [np.zeros_like(b) for b in c["B"]]
    _, y = oracle.lora_delta(c["x"], c["y_in"], c["off"], c["ranks"], c["A"], B0,
                             token_idx=c["tix"])
    assert np.array_equal(y, c["y_in"])


# -- p3: one adapter for the whole batch is one dense GEMM ----------------------------
def test_single_adapter_batch_is_dense_gemm():
    """[SGMV post] "SGMV: the kernel that holds it all up": when every request uses the
    same adapter the work is the single-large-segment case.  Compare with numpy's
    matmul of the whole batch: Y + s * (X A^T) B^T."""
    rng = np.random.default_rng(3)
    T, d_in, d_out, r = 37, 48, 20, 6
    x = rng.standard_normal((T, d_in))
    y_in = rng.standard_normal((T, d_out))
    A = rng.standard_normal((r, d_in))
    B = rng.standard_normal((d_out, r))
    v, y = oracle.lora_delta(x, y_in, [0, T], [r], [A], [B], scale=1.5)
    ref_v = x @ A.T
    ref_y = y_in + 1.5 * (ref_v @ B.T)
    np.testing.assert_allclose(v[:, :r], ref_v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, ref_y, rtol=1e-12, atol=1e-12)


# -- p4: zero-padded rank --------------------------------------------------------------
def test_zero_padded_rank_changes_nothing():
    """[SGMV post] TL;DR: a batch may mix ranks "without padding".  Padding an adapter to
    a larger rank with zero rows of A and zero columns of B leaves y bit-identical."""
    rng = np.random.default_rng(4)
    c = _rand_case(rng, 19, 24, 16, [3, 5])
    _, y1 = oracle.lora_delta(c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"],
                              token_idx=c["tix"])
    A2 = [np.vstack([a, np.zeros((4, a.shape[1]))]) for a in c["A"]]
    B2 = [np.hstack([b, np.zeros((b.shape[0], 4))]) for b in c["B"]]
    v2, y2 = oracle.lora_delta(c["x"], c["y_in"], c["off"], [r + 4 for r in c["ranks"]],
                               A2, B2, token_idx=c["tix"])
    assert np.array_equal(y1, y2)
    assert np.all(v2[:, -4:] == 0.0)


# -- p5: exact small integers ----------------------------------------------------------
def _int_case(rng, T, d_in, d_out, ranks):
    S = len(ranks)
    sizes = rng.multinomial(T, np.ones(S) / S)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    x = np.zeros((T, d_in), dtype=np.int64)
    for t in range(T):
        nz = rng.choice(d_in, size=min(8, d_in), replace=False)
        x[t, nz] = rng.choice([-1, 1], size=nz.size)
    A = [rng.integers(-1, 2, size=(r, d_in)) for r in ranks]
    B = [rng.integers(-1, 2, size=(d_out, r)) for r in ranks]
    y_in = rng.integers(-8, 9, size=(T, d_out))
    tix = rng.permutation(T)
    return off, x, A, B, y_in, tix


def test_exact_integer_inputs_match_brute_force():
    """Integer inputs small enough that every product and partial sum is exact in fp64:
    the oracle must equal Python integer arithmetic done element by element."""
    rng = np.random.default_rng(5)
    T, d_in, d_out, ranks = 11, 64, 24, [4, 1, 3]
    off, x, A, B, y_in, tix = _int_case(rng, T, d_in, d_out, ranks)
    v, y = oracle.lora_delta(x.astype(float), y_in.astype(float), off, ranks,
                             [a.astype(float) for a in A], [b.astype(float) for b in B],
                             token_idx=tix, scale=1.0)
    for s, r in enumerate(ranks):
        for i in range(off[s], off[s + 1]):
            t = int(tix[i])
            vv = [sum(int(A[s][k][c]) * int(x[t][c]) for c in range(d_in)) for k in range(r)]
            assert [int(q) for q in v[i, :r]] == vv
            for j in range(d_out):
                want = int(y_in[t][j]) + sum(int(B[s][j][k]) * vv[k] for k in range(r))
                assert y[t, j] == want


# -- p6: permutation invariance --------------------------------------------------------
def test_token_order_does_not_matter():
    """The per-token equation of [SGMV post] ("SGMV: the kernel that holds it all up")
    makes each token's result depend on its own row only: shuffling the batch permutes
    the rows of the result and changes no value."""
    rng = np.random.default_rng(6)
    c = _rand_case(rng, 29, 16, 12, [2, 3, 4])
    _, y = oracle.lora_delta(c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"],
                             token_idx=c["tix"])
    perm = rng.permutation(29)          # new position p holds old token perm[p]
    inv = np.argsort(perm)
    _, yp = oracle.lora_delta(c["x"][perm], c["y_in"][perm], c["off"], c["ranks"], c["A"],
                              c["B"], token_idx=inv[c["tix"]])
    assert np.array_equal(yp, y[perm])


# -- p7: scale -------------------------------------------------------------------------
def test_scale_zero_and_two():
    """scale = 0 leaves y unchanged; scale = 2 doubles the delta (exact on integers)."""
    rng = np.random.default_rng(7)
    off, x, A, B, y_in, tix = _int_case(rng, 9, 64, 16, [2, 3])
    args = (x.astype(float), y_in.astype(float), off, [2, 3],
            [a.astype(float) for a in A], [b.astype(float) for b in B])
    _, y0 = oracle.lora_delta(*args, token_idx=tix, scale=0.0)
    _, y1 = oracle.lora_delta(*args, token_idx=tix, scale=1.0)
    _, y2 = oracle.lora_delta(*args, token_idx=tix, scale=2.0)
    assert np.array_equal(y0, y_in.astype(float))
    assert np.array_equal(y2 - y_in, 2.0 * (y1 - y_in))


# -- degenerate cases ------------------------------------------------------------------
def test_tokens_outside_segments_and_rank_zero_untouched():
    rng = np.random.default_rng(8)
    T, d_in, d_out = 10, 16, 8
    x = rng.standard_normal((T, d_in))
    y_in = rng.standard_normal((T, d_out))
    A = [rng.standard_normal((0, d_in)), rng.standard_normal((2, d_in))]
    B = [rng.standard_normal((d_out, 0)), rng.standard_normal((d_out, 2))]
    # segment 0 (rank 0) holds tokens 1, 4; segment 1 holds token 7; others use no adapter
    v, y = oracle.lora_delta(x, y_in, [0, 2, 3], [0, 2], A, B, token_idx=[1, 4, 7])
    untouched = [t for t in range(T) if t != 7]
    assert np.array_equal(y[untouched], y_in[untouched])
    np.testing.assert_allclose(y[7], y_in[7] + B[1] @ (A[1] @ x[7]), rtol=1e-13)


def test_empty_batch():
    v, y = oracle.lora_delta(np.zeros((0, 8)), np.zeros((0, 4)), [0], [], [], [])
    assert v.shape[0] == 0 and y.shape == (0, 4)


# -- p8: segment builder ---------------------------------------------------------------
def test_segment_figure_golden():
    """[SGMV post], figure of "SGMV: the kernel that holds it all up": four requests over
    adapters A12, A12, A47, A89 form three segments A12 (2 requests), A47, A89."""
    with open(os.path.join(GOLDEN, "segment_figure.json")) as f:
        g = json.load(f)
    ids = [r["adapter"] for r in g["requests"]]
    names = [r["request"] for r in g["requests"]]
    tix, off, seg_ad = oracle.group_by_adapter(ids)
    got = []
    for s, a in enumerate(seg_ad):
        got.append({"adapter": a, "requests": [names[t] for t in tix[off[s]:off[s + 1]]],
                    "rank": g["adapter_rank"][str(a)]})
    assert got == g["expected_segments"]


def test_group_by_adapter_invariants():
    rng = np.random.default_rng(9)
    for T in (0, 1, 5, 64, 300):
        ids = rng.integers(-1, 12, size=T)
        tix, off, seg_ad = oracle.group_by_adapter(ids.tolist())
        covered = sorted(tix)
        assert covered == [t for t in range(T) if ids[t] >= 0]          # each token once
        assert off[0] == 0 and all(a < b for a, b in zip(off, off[1:]))  # no empty segment
        assert seg_ad == sorted(set(int(a) for a in ids if a >= 0))     # ascending ids
        for s, a in enumerate(seg_ad):
            seg = tix[off[s]:off[s + 1]]
            assert all(ids[t] == a for t in seg)
            assert seg == sorted(seg)                                   # stable


# -- p9: memory table ------------------------------------------------------------------
def test_memory_table_golden():
    """[SGMV post], "The maths that matters": bytes per matrix (d_in r + r d_out) b and the
    Llama-3-70B rank-16 table that sums to 5,177,344 B per layer (~395 MB over 80 layers)."""
    with open(os.path.join(GOLDEN, "memory_table_llama3_70b_r16.json")) as f:
        g = json.load(f)
    total = 0
    for m in g["matrices"]:
        got = oracle.adapter_bytes(m["d_in"], m["d_out"], g["rank"], g["bytes_per_param"])
        assert got == m["bytes"], m
        total += got
    assert total == g["sum_per_layer_bytes"]
    assert round(total * g["layers"] / 2 ** 20) == g["adapter_total_approx_MB"]


@pytest.mark.parametrize("threads", [1, 4])
def test_threads_give_identical_bits(threads):
    rng = np.random.default_rng(10)
    c = _rand_case(rng, 40, 32, 16, [3, 8, 2])
    args = (c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"])
    v1, y1 = oracle.lora_delta(*args, token_idx=c["tix"], threads=1)
    vn, yn = oracle.lora_delta(*args, token_idx=c["tix"], threads=threads)
    assert np.array_equal(y1, yn) and np.array_equal(v1, vn)


# -- per-segment scale (LoRA's alpha / r of each adapter) -------------------------------
# The pages give no LoRA scaling.  Reading: each adapter carries one multiplier applied to
# its own delta, on top of the call's scale: y_t = y_t + (scale * s_{a(t)}) B A x_t.
def test_segment_scale_merged_weights_identity():
    """[SGMV post] "The bare mechanism": W' = W + BA, with each adapter's delta scaled by
    its own factor c_s: the oracle equals the explicitly merged (W + scale c_s B_s A_s) x
    for the tokens of each segment."""
    rng = np.random.default_rng(11)
    c = _rand_case(rng, 31, 40, 56, [3, 7, 1, 5])
    scale, seg_scale = 0.75, [2.0, 0.125, -1.5, 3.25]
    _, y = oracle.lora_delta(c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"],
                             token_idx=c["tix"], scale=scale, seg_scale=seg_scale)
    for s in range(len(c["ranks"])):
        Wm = c["W"] + scale * seg_scale[s] * (c["B"][s] @ c["A"][s])
        for i in range(c["off"][s], c["off"][s + 1]):
            t = c["tix"][i]
            ref = Wm @ c["x"][t]
            np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_equal_segment_scales_are_one_call_scale():
    """Every segment with the same factor c is the per-call form with scale * c, bit for
    bit; all ones is the form without per-segment factors."""
    rng = np.random.default_rng(12)
    c = _rand_case(rng, 27, 24, 16, [2, 5, 3])
    args = (c["x"], c["y_in"], c["off"], c["ranks"], c["A"], c["B"])
    _, y_seg = oracle.lora_delta(*args, token_idx=c["tix"], scale=0.75, seg_scale=[1.5] * 3)
    _, y_call = oracle.lora_delta(*args, token_idx=c["tix"], scale=0.75 * 1.5)
    assert np.array_equal(y_seg, y_call)
    _, y_one = oracle.lora_delta(*args, token_idx=c["tix"], scale=0.5, seg_scale=[1.0] * 3)
    _, y_none = oracle.lora_delta(*args, token_idx=c["tix"], scale=0.5)
    assert np.array_equal(y_one, y_none)


def test_segment_scale_exact_integers_match_brute_force():
    """Integer inputs and integer factors: every value is exact in fp64, so the oracle must
    equal Python integers y_in + scale * c_s * B (A x) element by element."""
    rng = np.random.default_rng(13)
    T, d_in, d_out, ranks = 13, 64, 20, [4, 1, 3, 2]
    off, x, A, B, y_in, tix = _int_case(rng, T, d_in, d_out, ranks)
    seg_scale, scale = [3, -2, 0, 1], 2
    v, y = oracle.lora_delta(x.astype(float), y_in.astype(float), off, ranks,
                             [a.astype(float) for a in A], [b.astype(float) for b in B],
                             token_idx=tix, scale=float(scale), seg_scale=[float(q) for q in seg_scale])
    for s, r in enumerate(ranks):
        for i in range(off[s], off[s + 1]):
            t = int(tix[i])
            vv = [sum(int(A[s][k][cc]) * int(x[t][cc]) for cc in range(d_in)) for k in range(r)]
            for j in range(d_out):
                want = int(y_in[t][j]) + scale * seg_scale[s] * sum(int(B[s][j][k]) * vv[k] for k in range(r))
                assert y[t, j] == want


def test_segment_scale_acts_on_its_own_segment_only():
    """With y_in = 0 the result is the scaled delta itself: doubling one segment's factor
    doubles exactly that segment's rows (exact in fp64), a zero factor leaves its rows
    at y_in, and every other row keeps its bits."""
    rng = np.random.default_rng(14)
    c = _rand_case(rng, 25, 16, 12, [2, 3, 4])
    y0 = np.zeros_like(c["y_in"])
    args = (c["x"], y0, c["off"], c["ranks"], c["A"], c["B"])
    _, y_a = oracle.lora_delta(*args, token_idx=c["tix"], seg_scale=[1.0, 0.5, 1.25])
    _, y_b = oracle.lora_delta(*args, token_idx=c["tix"], seg_scale=[1.0, 1.0, 1.25])
    _, y_z = oracle.lora_delta(*args, token_idx=c["tix"], seg_scale=[1.0, 0.0, 1.25])
    rows1 = c["tix"][c["off"][1]:c["off"][2]]
    others = [t for t in range(25) if t not in set(rows1.tolist())]
    assert np.array_equal(y_b[rows1], 2.0 * y_a[rows1])
    assert np.array_equal(y_b[others], y_a[others])
    assert np.array_equal(y_z[rows1], y0[rows1]) and np.array_equal(y_z[others], y_a[others])
