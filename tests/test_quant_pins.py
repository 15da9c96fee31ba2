"""Pins of the oracle's adapter quantisation (oracle/quant.py) against what the FP8 E4M3
format definition, hand-worked rows, a library conversion (torch.float8_e4m3fn) and the
mathematics fix.  CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle import quant as q
import oracle


def test_e4m3_closed_form_values():
    # sign | 4 exponent bits (bias 7) | 3 mantissa bits; subnormals at exponent 0
    assert q.e4m3_value(0x00) == 0.0
    assert q.e4m3_value(0x01) == 2.0 ** -9          # smallest subnormal 0.001b * 2^-6
    assert q.e4m3_value(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert q.e4m3_value(0x08) == 2.0 ** -6          # smallest normal
    assert q.e4m3_value(0x38) == 1.0                # exponent 7 = bias
    assert q.e4m3_value(0x3C) == 1.5
    assert q.e4m3_value(0x7E) == 448.0              # 1.110b * 2^8, the largest finite value
    assert math.isnan(q.e4m3_value(0x7F)) and math.isnan(q.e4m3_value(0xFF))
    assert q.e4m3_value(0xC0) == -2.0
    assert q.e4m3_value(0x80) == 0.0 and math.copysign(1.0, q.e4m3_value(0x80)) == -1.0


def test_e4m3_table_matches_library_decode():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = q.e4m3_decode(np.arange(256, dtype=np.uint8))
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2
    assert np.array_equal(lib[~nan], ours[~nan])


def test_e4m3_encode_matches_library_in_range():
    rng = np.random.default_rng(1)
    pos = q._E4M3_POS
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)           # every tie
    v = np.concatenate([
        (rng.standard_normal(50000) * 60).astype(np.float32),
        (rng.standard_normal(20000) * 2.0 ** -8).astype(np.float32),  # subnormal range
        mids, -mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
        pos.astype(np.float32)])
    v = v[np.abs(v) <= 448]
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q.e4m3_encode(v), lib)


def test_e4m3_encode_ties_saturation_and_sign():
    v = np.array([1.0625, 1.1875, 3 * 2.0 ** -11, 2.0 ** -10, 448.0, 460.0, 500.0, 1e30, -1e30,
                  0.0, -0.0, -2.0 ** -12], dtype=np.float32)
    # 1.0625 lies half way between 1.0 (0x38, even) and 1.125 (0x39): even wins; 1.1875
    # between 1.125 (0x39) and 1.25 (0x3A): 0x3A; 1.5 * 2^-10 between 2^-10... (sub-
    # normals step 2^-9): 3 * 2^-11 = 1.5 * 2^-10 rounds to 2^-9 (0x01); 2^-10 is the
    # tie between 0 and 2^-9: 0 (even).  Beyond 448: saturated (satfinite).
    want = [0x38, 0x3A, 0x01, 0x00, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80, 0x80]
    assert q.e4m3_encode(v).tolist() == want


def test_int4_packing_golden():
    codes = np.array([[1, -1, 7, -7, 0, -8, 3, 2]])
    packed = q.int4_pack(codes)
    assert packed.tolist() == [[0xF1, 0x97, 0x80, 0x23]]   # value 2i in the low nibble
    assert np.array_equal(q.int4_unpack(packed), codes)


def test_int4_hand_worked_row():
    w = np.array([[1.75, -0.875, 0.25, 0.125, -1.75, 0.625, 0.0, 1.125]], dtype=np.float32)
    codes, s = q.quantize_rows(w, q.INT4)
    assert s.tolist() == [0.25]                              # 1.75 / 7
    # ratios 7, -3.5, 1, 0.5, -7, 2.5, 0, 4.5: halves go to the even integer
    assert q.int4_unpack(codes).tolist() == [[7, -4, 1, 0, -7, 2, 0, 4]]
    assert q.dequantize_rows(codes, s, q.INT4).tolist() == [[1.75, -1.0, 0.25, 0.0, -1.75, 0.5, 0.0, 1.0]]


def test_fp8_hand_worked_row():
    w = np.array([[7.0, -1.0, 1.0625 / 64, 4.5 / 64, -7.0, 0.0, 2.0 ** -15, 300.0 / 64]], dtype=np.float32)
    codes, s = q.quantize_rows(w, q.FP8_E4M3)
    assert s.tolist() == [7.0 / 448]                         # 2^-6
    # ratios 448, -64, 1.0625 (tie -> 1.0), 4.5, -448, 0, 2^-9, 300 (-> 288: step 32 in [256, 448])
    assert q.e4m3_decode(codes).tolist() == [[448.0, -64.0, 1.0, 4.5, -448.0, 0.0, 2.0 ** -9, 288.0]]


def test_zero_row_and_scale_per_row():
    w = np.zeros((3, 16), dtype=np.float32)
    w[1, 3] = -5.0
    w[2] = np.linspace(-1, 1, 16, dtype=np.float32)
    for fmt in (q.INT4, q.FP8_E4M3):
        codes, s = q.quantize_rows(w, fmt)
        assert s[0] == 0 and not codes[0].any()
        assert np.float32(s[1]) == np.float32(np.float32(5.0) / np.float32(q.QMAX[fmt]))
        deq = q.dequantize_rows(codes, s, fmt)
        assert deq[1, 3] == pytest.approx(-5.0, rel=1e-6) and np.count_nonzero(deq[1]) == 1


@pytest.mark.parametrize("fmt", [q.INT4, q.FP8_E4M3])
def test_error_bounds_and_brute_force(fmt):
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((12, 256)) * rng.uniform(1e-3, 10, (12, 1))).astype(np.float32)
    w[3, :] *= 1e-6                                             # tiny row: subnormal codes for E4M3
    codes, s = q.quantize_rows(w, fmt)
    deq = q.dequantize_rows(codes, s, fmt)
    ratio = (w / s[:, None]).astype(np.float32).astype(np.float64)
    amax = np.abs(w).max(axis=1)
    # the largest element of each row maps to +-Q and comes back (up to the scale's rounding)
    np.testing.assert_allclose(np.abs(deq).max(axis=1), amax, rtol=2e-7)
    if fmt == q.INT4:
        qv = q.int4_unpack(codes)
        assert qv.min() >= -7 and qv.max() <= 7
        # brute force: the code is the nearest of the 15 integers (ties: even)
        grid = np.arange(-7, 8)
        d = np.abs(ratio[..., None] - grid)
        best = d.min(axis=-1)
        assert np.array_equal(np.abs(ratio - qv), best)
        assert np.all(np.abs(w - deq) <= s[:, None] / 2 * (1 + 1e-6))
    else:
        val = q.e4m3_decode(codes)
        # half a unit in the last place: 2^-4 relative for normals, 2^-10 absolute below 2^-6
        half_ulp = np.maximum(np.abs(ratio) * 2.0 ** -4, 2.0 ** -10)
        assert np.all(np.abs(val - ratio) <= half_ulp)
        assert np.all(np.abs(val) <= 448.0)


def test_transpose_orientation_of_B():
    rng = np.random.default_rng(3)
    A = rng.standard_normal((4, 32)).astype(np.float32)
    B = rng.standard_normal((64, 4)).astype(np.float32)
    B2 = B.copy()
    B2[:, 2] *= 1000.0                                          # one rank column of B
    _, _, _, sB, _, _ = q.quantize_adapter(A, B, q.INT4)
    _, _, _, sB2, _, _ = q.quantize_adapter(A, B2, q.INT4)
    # B^T rows are B's columns: only scale 2 changes
    assert np.array_equal(np.delete(sB, 2), np.delete(sB2, 2))
    assert sB2[2] == pytest.approx(sB[2] * 1000.0, rel=1e-6)


@pytest.mark.parametrize("fmt", [q.INT4, q.FP8_E4M3])
def test_row_scales_factor_out_of_the_delta(fmt):
    """The delta on the dequantised weights equals the codes-then-scales order the
    kernels use: v_k = s^A_k sum_c q_kc x_c and y += sum_k (v_k s^B_k) q^B_kj."""
    rng = np.random.default_rng(11)
    T, d_in, d_out, r = 5, 64, 96, 6
    x = rng.standard_normal((T, d_in)).astype(np.float32).astype(np.float64)
    y0 = rng.standard_normal((T, d_out))
    A = rng.standard_normal((r, d_in)).astype(np.float32)
    B = rng.standard_normal((d_out, r)).astype(np.float32)
    cA, sA, cB, sB, Ad, Bd = q.quantize_adapter(A, B, fmt)
    v, y = oracle.lora_delta(x, y0, [0, T], [r], [Ad], [Bd], scale=0.5)
    if fmt == q.INT4:
        qa, qb = q.int4_unpack(cA), q.int4_unpack(cB)
    else:
        qa, qb = q.e4m3_decode(cA), q.e4m3_decode(cB)
    v2 = np.zeros((T, r))
    y2 = y0.copy()
    for t in range(T):                      # plain loops, the kernels' order of the scales
        for k in range(r):
            v2[t, k] = float(sA[k]) * sum(float(qa[k, c]) * x[t, c] for c in range(d_in))
        for j in range(d_out):
            y2[t, j] += 0.5 * sum(v2[t, k] * float(sB[k]) * float(qb[k, j]) for k in range(r))
    np.testing.assert_allclose(v[:, :r], v2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-12)
