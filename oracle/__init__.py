"""CPU oracle for the multi-LoRA delta -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The CUDA library never calls it and it
imports nothing from the CUDA library.

Contents
  lora_delta(...)        fp64 loops of y_t = W x_t + s * s_{a(t)} B_{a(t)} A_{a(t)} x_t (C, sgmv_oracle.c)
  group_by_adapter(ids)  one segment per adapter, by brute-force sorting
  adapter_bytes(...)     the bytes-per-matrix formula of section "The maths that matters"

Citations name the pages by title:
  [SGMV post]  "Multi-LoRA serving: the single translator with a thousand glossaries --
                shared base, thousands of concurrent adapters and the SGMV kernel" (blog.lo0.es)
  [Glossary]   "Multi-LoRA Serving" (skillsintelligence.tools glossary entry)

Pins: every function here is pinned by `tests/test_oracle_pins.py` against
results the pages or the mathematics fix (merged weights, a textbook dense
GEMM, exact integer arithmetic, zero-padding, permutations, the memory table
and the segment figure of the [SGMV post]).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sgmv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (plain gcc, fp64, no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-o", _LIB, _SRC]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, dp = ctypes.c_int64, ctypes.POINTER(ctypes.c_double)
        lib.oracle_lora_delta.restype = ctypes.c_int
        lib.oracle_lora_delta.argtypes = [
            i64, i64, i64, dp, i64, dp, i64, i64,
            ctypes.POINTER(i64), ctypes.POINTER(i64),
            ctypes.POINTER(dp), ctypes.POINTER(dp), ctypes.POINTER(i64),
            ctypes.c_double, dp, dp, i64, dp, ctypes.c_int]
        lib.oracle_threads.restype = ctypes.c_int
        lib.oracle_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def threads_used(threads: int) -> int:
    return int(_load().oracle_threads(int(threads)))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def lora_delta(x: np.ndarray, y_in: np.ndarray, seg_offsets: Sequence[int],
               seg_rank: Sequence[int], A: List[np.ndarray], B: List[np.ndarray],
               token_idx: Optional[Sequence[int]] = None, scale: float = 1.0,
               ldv: Optional[int] = None, threads: int = 1,
               seg_scale: Optional[Sequence[float]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 reference of the per-token delta ([SGMV post], "SGMV: the kernel that holds
    it all up": per-token equation, shrink then expand).

    x      float64 [T][d_in]   (exact widening of the bf16 inputs)
    y_in   float64 [T][d_out]  (holds W x)
    A[s]   float64 [r_s][d_in],  B[s] float64 [d_out][r_s]   (logical orientation of
           "The bare mechanism": A in R^{r x d_in}, B in R^{d_out x r})
    seg_offsets [S+1], seg_rank [S], token_idx [rows] (row -> token) or None (identity)
    scale      one multiplier for the whole call
    seg_scale  [S] multiplier of each segment's adapter (LoRA's alpha/r), or None (all 1):
               a token of segment s gets y_t + (scale * seg_scale[s]) * B_s A_s x_t.  The
               pages give no scaling; one number per adapter, applied to its delta, is the
               plainest reading of "W' = W + BA" with LoRA's usual alpha/r factor.
    Returns (v [rows][ldv] float64, y [T][d_out] float64).
    """
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    y_in = np.ascontiguousarray(y_in, dtype=np.float64)
    T, d_in = x.shape
    d_out = y_in.shape[1]
    assert y_in.shape[0] == T
    S = len(seg_rank)
    off = np.ascontiguousarray(np.asarray(seg_offsets, dtype=np.int64))
    rk = np.ascontiguousarray(np.asarray(seg_rank, dtype=np.int64))
    assert off.size == S + 1 or (S == 0 and off.size <= 1)
    if off.size == 0:
        off = np.zeros(1, dtype=np.int64)
    rows = int(off[S]) if S > 0 else 0
    R = int(rk.max()) if S > 0 else 0
    ldv = max(R, 1) if ldv is None else int(ldv)
    As = [np.ascontiguousarray(a, dtype=np.float64) for a in A]
    Bs = [np.ascontiguousarray(b, dtype=np.float64) for b in B]
    for s in range(S):
        assert As[s].shape == (rk[s], d_in), (As[s].shape, rk[s], d_in)
        assert Bs[s].shape == (d_out, rk[s]), (Bs[s].shape, d_out, rk[s])
    dp_t = ctypes.POINTER(ctypes.c_double)
    A_ptrs = (dp_t * max(S, 1))(*[_dp(a) for a in As])
    B_ptrs = (dp_t * max(S, 1))(*[_dp(b) for b in Bs])
    if token_idx is None:
        tix = None
        tix_p = None
    else:
        tix = np.ascontiguousarray(np.asarray(token_idx, dtype=np.int64))
        assert tix.size == rows
        tix_p = tix.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    if seg_scale is None:
        ss, ss_p = None, None
    else:
        ss = np.ascontiguousarray(np.asarray(seg_scale, dtype=np.float64))
        assert ss.size == S
        ss_p = _dp(ss)
    v = np.zeros((max(rows, 0), ldv), dtype=np.float64)
    y = np.empty_like(y_in)
    rc = lib.oracle_lora_delta(
        T, d_in, d_out, _dp(x), d_in, _dp(y_in), d_out, S,
        off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        rk.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        A_ptrs, B_ptrs, tix_p, float(scale), ss_p, _dp(v), ldv, _dp(y), int(threads))
    if rc != 0:
        raise ValueError(f"oracle_lora_delta rejected its arguments (code {rc})")
    return v, y


def group_by_adapter(adapter_ids: Sequence[int]) -> Tuple[List[int], List[int], List[int]]:
    """One segment per distinct adapter ([SGMV post], "SGMV: the kernel that holds it all
    up": SGMV "groups the batch's tokens by adapter"; the figure of that section shows
    segment A12 with its two requests, then A47, then A89).

    Readings where the pages are silent: segments are ordered by ascending adapter id,
    tokens inside a segment keep their batch order, tokens with id -1 use no adapter
    and belong to no segment.

    Returns (token_idx, seg_offsets, seg_adapter) computed by brute force: every
    (adapter, position) pair sorted with Python's sort.
    """
    pairs = sorted((int(a), i) for i, a in enumerate(adapter_ids) if int(a) >= 0)
    token_idx = [i for _, i in pairs]
    seg_adapter: List[int] = []
    seg_offsets: List[int] = [0]
    for n, (a, _) in enumerate(pairs):
        if not seg_adapter or seg_adapter[-1] != a:
            if seg_adapter:
                seg_offsets.append(n)
            seg_adapter.append(a)
    if seg_adapter:
        seg_offsets.append(len(pairs))
    return token_idx, seg_offsets, seg_adapter


def adapter_bytes(d_in: int, d_out: int, r: int, b: int = 2) -> int:
    """Bytes of one adapted matrix: (d_in * r + r * d_out) * b
    ([SGMV post], "The maths that matters", memory-per-adapter formula)."""
    return (d_in * r + r * d_out) * b
