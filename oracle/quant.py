"""Adapter weight quantisation of the oracle -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py`
may import this module; the CUDA library never calls it.

Pages cited by title:
  [ClusterBid]  "Multi-LoRA Inference Serving: Serving Thousands of Fine-Tuned Models on
                One GPU" (clusterbid.com): the paragraph on the GPU memory budget (adapters
                stored in FP8 take half the memory) and the paragraph on adapter weight
                quantization (INT4 adapters, dequantised at inference).

The pages name the two formats and nothing else about them.  Readings (the plainest
ones the rest supports):
  * FP8 is E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
    no infinities, largest finite value 448): the FP8 format used for weights.
  * Symmetric quantisation with one real scale per rank row of A and of B^T:
      s_k  = max_c |w_kc| / Q                 Q = 448 (E4M3) or 7 (INT4)
      q_kc = RN(w_kc / s_k)                   E4M3: nearest, ties to even, saturating
                                              INT4: nearest, ties to even, in [-7, 7]
      w'_kc = value(q_kc) * s_k
    A row of zeros has s_k = 0 and all codes 0.
  * The decisions (the scale and each code) are taken in fp32 on both sides, as the
    stored weights are bf16 (exact in fp32).
  * INT4 codes are two's complement nibbles, value 2i in the low nibble of byte i.

Every function is pinned by `tests/test_quant_pins.py`: the E4M3 table against the
format's closed form and torch's float8_e4m3fn conversion (a library routine),
hand-worked rows, error bounds, and brute force over the code grid.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

FP8_E4M3 = "fp8_e4m3"
INT4 = "int4"
QMAX = {FP8_E4M3: 448.0, INT4: 7.0}


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code from the format's definition (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6          # subnormal: 0.mmm * 2^(1 - bias)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)   # normal: 1.mmm * 2^(e - bias)


# the 127 finite non-negative values, by code 0x00 .. 0x7E (ascending)
_E4M3_POS = np.array([e4m3_value(c) for c in range(0x7F)], dtype=np.float64)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each float32 value, ties to the even code (mantissa bit 0
    clear), magnitudes above 448 saturated to 448, sign kept (also for zero).
    Brute force: the distance to every finite code is computed and the smallest taken."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64)).reshape(-1)
    out = np.empty(a.shape, dtype=np.uint8)
    even = (np.arange(_E4M3_POS.size) & 1) == 0
    for i0 in range(0, a.size, 1 << 15):
        x = a[i0:i0 + (1 << 15)]
        d = np.abs(x[:, None] - _E4M3_POS[None, :])
        cand = d == d.min(axis=1, keepdims=True)
        c = np.where(cand.sum(axis=1) > 1, np.argmax(cand & even[None, :], axis=1), np.argmax(cand, axis=1))
        out[i0:i0 + x.size] = np.where(x >= 448.0, 0x7E, c)
    sign = np.signbit(v.reshape(-1))
    out[sign] |= 0x80
    return out.reshape(v.shape)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def int4_pack(q: np.ndarray) -> np.ndarray:
    """[rows][d] int codes in [-8, 7] -> [rows][d/2] bytes, value 2i in the low nibble."""
    q = np.asarray(q, dtype=np.int64)
    assert q.shape[-1] % 2 == 0
    nib = (q & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def int4_unpack(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    lo, hi = b & 0xF, b >> 4
    q = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    q[..., 0::2], q[..., 1::2] = lo, hi
    return np.where(q >= 8, q - 16, q)


def quantize_rows(w: np.ndarray, fmt: str) -> Tuple[np.ndarray, np.ndarray]:
    """Quantise each row of w (float32-exact values, e.g. widened bf16) with its own
    scale.  Returns (codes, scales): E4M3 codes uint8 [rows][d], or packed INT4 bytes
    uint8 [rows][d/2]; scales float32 [rows]."""
    w = np.asarray(w, dtype=np.float32)
    rows, d = w.shape
    qmax = np.float32(QMAX[fmt])
    scales = np.zeros(rows, dtype=np.float32)
    q = np.zeros((rows, d), dtype=np.int64)
    codes8 = np.zeros((rows, d), dtype=np.uint8)
    for k in range(rows):
        amax = np.float32(np.max(np.abs(w[k]))) if d else np.float32(0)
        if amax == 0:
            continue                                          # s = 0, codes 0
        s = np.float32(amax / qmax)                           # fp32 division
        scales[k] = s
        ratio = (w[k] / s).astype(np.float32)                 # fp32 division per value
        if fmt == FP8_E4M3:
            codes8[k] = e4m3_encode(ratio)
        else:
            q[k] = np.clip(np.rint(ratio), -7, 7).astype(np.int64)  # rint: half to even
    if fmt == FP8_E4M3:
        return codes8, scales
    return int4_pack(q), scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, fmt: str) -> np.ndarray:
    """float64 [rows][d] values code * scale."""
    if fmt == FP8_E4M3:
        vals = e4m3_decode(codes)
    else:
        vals = int4_unpack(codes).astype(np.float64)
    return vals * np.asarray(scales, dtype=np.float64)[:, None]


def quantize_adapter(A: np.ndarray, B: np.ndarray, fmt: str):
    """One adapted matrix pair in the pool's orientation: A [r][d_in] row by row, and
    B [d_out][r] through its transpose B^T [r][d_out] row by row.  Returns
    (codes_A, scales_A, codes_BT, scales_BT, A', B') with A' [r][d_in] and
    B' [d_out][r] the dequantised float64 weights the delta is computed with."""
    cA, sA = quantize_rows(A, fmt)
    cB, sB = quantize_rows(np.asarray(B).T, fmt)
    return cA, sA, cB, sB, dequantize_rows(cA, sA, fmt), dequantize_rows(cB, sB, fmt).T
