"""Python binding of libsgmv_b200.so -- the multi-LoRA delta on one B200.

Argument marshalling only: every step of the computation runs in the CUDA
library behind the C ABI declared in include/sgmv.h.  PyTorch supplies device
memory and streams.  If the compiled library is missing this module raises on
import of any entry point; there is no fallback.

    pool = AdapterPool([(d_in, d_out), ...], num_pages=..., device=0)
    pool.load(adapter_id, rank, [A_p ...], [B_p ...])    # A_p: [r, d_in], B_p: [d_out, r] bf16
    plan = pool.plan(adapter_ids)                         # segment builder + dispatch (host)
    plan.upload()                                         # one host->device copy of the table
    v = plan.new_v()
    shrink(x, plan, pool, v, proj)                        # v = A_{a(t)} x_t
    expand(v, plan, pool, y, proj, scale)                 # y_t += scale * B_{a(t)} v_t
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsgmv_b200.so")

_STATUS = {0: "SGMV_OK", 1: "SGMV_ERR_INVALID", 2: "SGMV_ERR_UNSUPPORTED", 3: "SGMV_ERR_NOT_RESIDENT",
           4: "SGMV_ERR_OUT_OF_PAGES", 5: "SGMV_ERR_CUDA", 6: "SGMV_ERR_BOUNDS", 7: "SGMV_ERR_TIMEOUT",
           8: "SGMV_ERR_CAPACITY"}

EXPORTED = ("sgmv_status_string", "sgmv_last_error", "sgmv_pool_create", "sgmv_pool_create_ex",
            "sgmv_pool_destroy", "sgmv_pool_load", "sgmv_pool_read",
            "sgmv_pool_evict", "sgmv_pool_get_stats", "sgmv_pool_adapter_rank", "sgmv_pool_adapter_pages",
            "sgmv_pool_set_adapter_scale", "sgmv_pool_get_adapter_scale",
            "sgmv_pool_shuffle_free_pages", "sgmv_pool_pages_device", "sgmv_plan_table_capacity",
            "sgmv_build_plan", "sgmv_shrink", "sgmv_expand", "sgmv_lora_delta", "sgmv_lora_delta_grouped",
            "sgmv_lora_delta_noalloc", "sgmv_lora_delta_kernels", "sgmv_upload_table", "sgmv_host_workspace_bytes",
            "sgmv_lora_delta_host",
            "sgmv_check_errors", "sgmv_residency_create", "sgmv_residency_destroy",
            "sgmv_residency_register", "sgmv_residency_unregister", "sgmv_residency_prepare",
            "sgmv_residency_get_stats")


class SgmvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "num_segments", "num_rows", "max_rank", "n_proj", "num_simt_items", "num_tc_tiles",
        "long_threshold", "max_item_rows", "needs_device_table")] + [(n, ctypes.c_int64) for n in (
            "table_bytes", "off_token_idx", "off_seg_offsets", "off_seg_adapter", "off_seg_rank",
            "off_seg_a_pt", "off_seg_b_pt", "off_simt_items", "off_tc_tiles")] + [("host_table", ctypes.c_void_p),
                                                                                   ("off_seg_scale", ctypes.c_int64)]


class DeltaEntry(ctypes.Structure):
    _fields_ = [("proj", ctypes.c_int32), ("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("x", ctypes.c_void_p), ("ldx", ctypes.c_int64),
                ("y", ctypes.c_void_p), ("ldy", ctypes.c_int64), ("v", ctypes.c_void_p), ("ldv", ctypes.c_int64)]


class HostEntry(ctypes.Structure):
    _fields_ = [("proj", ctypes.c_int32), ("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("x_host", ctypes.c_void_p), ("y_host", ctypes.c_void_p)]


class ResidencyStats(ctypes.Structure):
    _fields_ = [("hits", ctypes.c_int64), ("misses", ctypes.c_int64), ("evictions", ctypes.c_int64),
                ("bytes_loaded", ctypes.c_int64)]


class PoolStats(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int64), ("free_pages", ctypes.c_int64), ("page_bytes", ctypes.c_int64),
                ("payload_bytes", ctypes.c_int64), ("resident_adapters", ctypes.c_int32),
                ("page_elems", ctypes.c_int32), ("weight_format", ctypes.c_int32), ("reserved", ctypes.c_int32)]


# weight formats of a pool (sgmv_weight_format)
WEIGHT_FORMATS = {"bf16": 0, "fp8_e4m3": 1, "int4": 2}


_lib = None


def load_library() -> ctypes.CDLL:
    """Load the compiled library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with segmented_rank_gemm_sgmv_b200/build.py "
                          "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    i32, i64, vp, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float
    st = ctypes.c_int
    sig = {
        "sgmv_status_string": (ctypes.c_char_p, [st]),
        "sgmv_last_error": (ctypes.c_char_p, []),
        "sgmv_pool_create": (st, [ctypes.c_int, i64, i32, i32, vp, vp, i32, ctypes.POINTER(vp)]),
        "sgmv_pool_create_ex": (st, [ctypes.c_int, i64, i32, i32, vp, vp, i32, i32, ctypes.POINTER(vp)]),
        "sgmv_pool_read": (st, [vp, i32, i32, i32, vp, i64, vp, i64, vp]),
        "sgmv_pool_destroy": (st, [vp]),
        "sgmv_pool_load": (st, [vp, i32, i32, vp, vp, ctypes.c_int, vp]),
        "sgmv_pool_evict": (st, [vp, i32]),
        "sgmv_pool_get_stats": (st, [vp, ctypes.POINTER(PoolStats)]),
        "sgmv_pool_adapter_rank": (st, [vp, i32, ctypes.POINTER(i32)]),
        "sgmv_pool_set_adapter_scale": (st, [vp, i32, f32]),
        "sgmv_pool_get_adapter_scale": (st, [vp, i32, ctypes.POINTER(f32)]),
        "sgmv_pool_adapter_pages": (st, [vp, i32, i32, i32, vp, i64, ctypes.POINTER(i64)]),
        "sgmv_pool_shuffle_free_pages": (st, [vp, ctypes.c_uint64]),
        "sgmv_pool_pages_device": (vp, [vp]),
        "sgmv_plan_table_capacity": (i64, [i32, i32]),
        "sgmv_build_plan": (st, [vp, i32, vp, i32, vp, i64, ctypes.POINTER(Plan)]),
        "sgmv_shrink": (st, [vp, i64, i32, i32, i32, ctypes.POINTER(Plan), vp, vp, vp, i64, vp]),
        "sgmv_expand": (st, [vp, i64, i32, i32, i32, ctypes.POINTER(Plan), vp, vp, f32, vp, i64, i32, vp]),
        "sgmv_lora_delta": (st, [vp, i64, i32, i32, i32, i32, ctypes.POINTER(Plan), vp, vp, f32, vp, i64, i32,
                                 vp, i64, vp]),
        "sgmv_lora_delta_grouped": (st, [ctypes.POINTER(DeltaEntry), i32, i32, ctypes.POINTER(Plan), vp, vp, f32,
                                         i32, vp]),
        "sgmv_lora_delta_noalloc": (st, [vp, i64, i32, i32, i32, i32, ctypes.POINTER(Plan), vp, vp, f32, vp, i64,
                                         i32, vp]),
        "sgmv_lora_delta_kernels": (st, [ctypes.POINTER(Plan), vp, vp, i32, vp, i32, ctypes.POINTER(i32),
                                         ctypes.POINTER(i32)]),
        "sgmv_upload_table": (st, [ctypes.POINTER(Plan), vp, vp]),
        "sgmv_host_workspace_bytes": (i64, [i32, vp, ctypes.POINTER(HostEntry), i32, i32]),
        "sgmv_lora_delta_host": (st, [vp, i32, vp, ctypes.POINTER(HostEntry), i32, f32, i32, vp, i64, vp, i64,
                                      ctypes.POINTER(Plan), ctypes.POINTER(i64), ctypes.POINTER(i64), vp]),
        "sgmv_check_errors": (st, [vp, ctypes.POINTER(ctypes.c_uint32)]),
        "sgmv_residency_create": (st, [vp, ctypes.POINTER(vp)]),
        "sgmv_residency_destroy": (st, [vp]),
        "sgmv_residency_register": (st, [vp, i32, i32, vp, vp]),
        "sgmv_residency_unregister": (st, [vp, i32]),
        "sgmv_residency_prepare": (st, [vp, vp, i32, vp, vp, ctypes.POINTER(i32)]),
        "sgmv_residency_get_stats": (st, [vp, ctypes.POINTER(ResidencyStats)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        msg = load_library().sgmv_last_error().decode(errors="replace")
        raise SgmvError(status, msg)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


class AdapterPool:
    """Paged adapter pool (see include/sgmv.h, "Paged adapter pool")."""

    def __init__(self, projections: Sequence[Tuple[int, int]], num_pages: int, page_elems: int = 512,
                 max_rank: int = 128, device: int = 0, weight_format: str = "bf16"):
        """weight_format: "bf16" (default), "fp8_e4m3" or "int4" -- a quantised pool stores
        codes with one fp32 scale per rank row and quantises bf16 weights as it loads them."""
        lib = load_library()
        self.projections = [(int(a), int(b)) for a, b in projections]
        self.device = device
        self.page_elems = page_elems
        if weight_format not in WEIGHT_FORMATS:
            raise ValueError(f"weight_format must be one of {sorted(WEIGHT_FORMATS)}")
        self.weight_format = weight_format
        n = len(self.projections)
        d_in = (ctypes.c_int32 * n)(*[p[0] for p in self.projections])
        d_out = (ctypes.c_int32 * n)(*[p[1] for p in self.projections])
        h = ctypes.c_void_p()
        _check(lib.sgmv_pool_create_ex(device, int(num_pages), int(page_elems), n,
                                       ctypes.cast(d_in, ctypes.c_void_p), ctypes.cast(d_out, ctypes.c_void_p),
                                       int(max_rank), WEIGHT_FORMATS[weight_format], ctypes.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            load_library().sgmv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def pages_needed(projections, rank: int, page_elems: int = 512) -> int:
        return sum(rank * (a // page_elems + b // page_elems) for a, b in projections)

    def load(self, adapter_id: int, rank: int, A: Optional[Sequence[torch.Tensor]] = None,
             B: Optional[Sequence[torch.Tensor]] = None, stream=None) -> None:
        """A[p]: bf16 [rank, d_in_p]; B[p]: bf16 [d_out_p, rank]; all on the pool's device or all on the
        host.  A host-only pool (device=-1) takes A = B = None and records the bookkeeping only."""
        n = len(self.projections)
        if rank > 0 and self.device < 0 and A is None and B is None:
            _check(load_library().sgmv_pool_load(self.handle, int(adapter_id), int(rank), None, None, 0, None))
        elif rank > 0:
            assert len(A) == n and len(B) == n
            on_dev = A[0].is_cuda
            keep = []
            for p, (d_in, d_out) in enumerate(self.projections):
                a = A[p].contiguous()
                b = B[p].contiguous()
                assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16
                assert tuple(a.shape) == (rank, d_in) and tuple(b.shape) == (d_out, rank), (a.shape, b.shape)
                assert a.is_cuda == on_dev and b.is_cuda == on_dev
                keep += [a, b]
            a_ptrs = (ctypes.c_void_p * n)(*[keep[2 * p].data_ptr() for p in range(n)])
            b_ptrs = (ctypes.c_void_p * n)(*[keep[2 * p + 1].data_ptr() for p in range(n)])
            _check(load_library().sgmv_pool_load(self.handle, int(adapter_id), int(rank),
                                                  ctypes.cast(a_ptrs, ctypes.c_void_p),
                                                  ctypes.cast(b_ptrs, ctypes.c_void_p), 1 if on_dev else 0,
                                                  _stream(stream) if self.device >= 0 else None))
            del keep
        else:
            _check(load_library().sgmv_pool_load(self.handle, int(adapter_id), 0, None, None, 0,
                                                  _stream(stream) if self.device >= 0 else None))

    def evict(self, adapter_id: int) -> None:
        _check(load_library().sgmv_pool_evict(self.handle, int(adapter_id)))

    def shuffle_free_pages(self, seed: int) -> None:
        _check(load_library().sgmv_pool_shuffle_free_pages(self.handle, int(seed)))

    def stats(self) -> PoolStats:
        s = PoolStats()
        _check(load_library().sgmv_pool_get_stats(self.handle, ctypes.byref(s)))
        return s

    def read(self, adapter_id: int, proj: int, matrix: int, stream=None) -> Tuple[np.ndarray, np.ndarray]:
        """Stored form of (adapter, projection, matrix 0 = A / 1 = B^T): (codes, scales).
        codes: uint16 bf16 words [r][d] (bf16 pool), uint8 E4M3 codes [r][d] or packed INT4
        bytes [r][d/2]; scales: float32 [r] (ones for a bf16 pool)."""
        r = self.rank_of(adapter_id)
        d = self.projections[proj][matrix]
        nbytes = {"bf16": 2 * d, "fp8_e4m3": d, "int4": d // 2}[self.weight_format]
        codes = np.zeros((max(r, 1), nbytes), dtype=np.uint8)
        scales = np.zeros(max(r, 1), dtype=np.float32)
        _check(load_library().sgmv_pool_read(self.handle, int(adapter_id), int(proj), int(matrix),
                                             codes.ctypes.data, codes.size, scales.ctypes.data, scales.size,
                                             _stream(stream) if self.device >= 0 else None))
        codes, scales = codes[:r], scales[:r]
        if self.weight_format == "bf16":
            codes = codes.view(np.uint16)
        return codes, scales

    def set_scale(self, adapter_id: int, scale: float) -> None:
        """Multiplier of the adapter's delta (its LoRA alpha / r), kept by id across
        evictions and reloads; plans built afterwards carry it (sgmv_pool_set_adapter_scale)."""
        _check(load_library().sgmv_pool_set_adapter_scale(self.handle, int(adapter_id), float(scale)))

    def scale_of(self, adapter_id: int) -> float:
        s = ctypes.c_float()
        _check(load_library().sgmv_pool_get_adapter_scale(self.handle, int(adapter_id), ctypes.byref(s)))
        return float(s.value)

    def rank_of(self, adapter_id: int) -> int:
        r = ctypes.c_int32()
        _check(load_library().sgmv_pool_adapter_rank(self.handle, int(adapter_id), ctypes.byref(r)))
        return r.value

    def page_ids(self, adapter_id: int, proj: int, matrix: int) -> np.ndarray:
        n = ctypes.c_int64()
        lib = load_library()
        st = lib.sgmv_pool_adapter_pages(self.handle, adapter_id, proj, matrix, None, 0, ctypes.byref(n))
        if st not in (0, 8):
            _check(st)
        out = np.zeros(max(n.value, 1), dtype=np.int32)
        _check(lib.sgmv_pool_adapter_pages(self.handle, adapter_id, proj, matrix, out.ctypes.data, n.value,
                                           ctypes.byref(n)))
        return out[:n.value]

    def pages_tensor(self) -> torch.Tensor:
        """The page buffer as a tensor view (device pools only): bf16 [num_pages, page_elems]
        for a bf16 pool, uint8 [num_pages, page_bytes] for a quantised one."""
        addr = load_library().sgmv_pool_pages_device(self.handle)
        s = self.stats()
        storage = torch.cuda.memory  # noqa: F841  (keeps torch.cuda initialised)
        arr = _DevicePtr(addr, s.num_pages * s.page_bytes, self.device)
        t = torch.as_tensor(arr, device=f"cuda:{self.device}")
        if self.weight_format != "bf16":
            return t.view(s.num_pages, s.page_bytes)
        return t.view(torch.bfloat16).view(s.num_pages, s.page_elems)

    def plan(self, adapter_ids, long_threshold: int = 0) -> "BatchPlan":
        return BatchPlan(self, adapter_ids, long_threshold)


class _DevicePtr:
    """__cuda_array_interface__ wrapper around a raw device address (read-only inspection)."""

    def __init__(self, addr: int, nbytes: int, device: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (addr, False),
                                         "version": 3}


class BatchPlan:
    """Segment table + dispatch for one batch (see include/sgmv.h, "Segment builder").

    The host table lives in pinned memory and the device copy in a device buffer,
    both reused by later build() calls; build() first waits for the previous
    upload from the host buffer to finish, so a plan can be rebuilt every step.
    """

    def __init__(self, pool: AdapterPool, adapter_ids=None, long_threshold: int = 0,
                 capacity_tokens: Optional[int] = None):
        self.pool = pool
        self.long_threshold = int(long_threshold)
        ids = None if adapter_ids is None else np.asarray(adapter_ids, dtype=np.int32).reshape(-1)
        cap_t = capacity_tokens if capacity_tokens is not None else (0 if ids is None else ids.size)
        self.capacity = int(load_library().sgmv_plan_table_capacity(int(cap_t), len(pool.projections)))
        pinned = torch.cuda.is_available() and pool.device >= 0
        self.host = torch.empty(self.capacity, dtype=torch.uint8, pin_memory=pinned)
        self.plan = Plan()
        self.device_table: Optional[torch.Tensor] = None
        self._uploaded: Optional[torch.cuda.Event] = None
        self.T = 0
        if ids is not None:
            self.build(ids)

    def build(self, adapter_ids, long_threshold: Optional[int] = None) -> "BatchPlan":
        ids = np.ascontiguousarray(np.asarray(adapter_ids, dtype=np.int32).reshape(-1))
        if self._uploaded is not None:
            self._uploaded.synchronize()      # the previous upload has read the host buffer
        lt = self.long_threshold if long_threshold is None else int(long_threshold)
        _check(load_library().sgmv_build_plan(ids.ctypes.data if ids.size else None, int(ids.size),
                                              self.pool.handle, lt, self.host.data_ptr(), self.capacity,
                                              ctypes.byref(self.plan)))
        self.T = int(ids.size)
        return self

    # -- host views of the table
    def _arr(self, off: int, count: int, dtype) -> np.ndarray:
        nbytes = count * np.dtype(dtype).itemsize
        return self.host.numpy()[off:off + nbytes].view(dtype).copy()

    @property
    def token_idx(self) -> np.ndarray:
        return self._arr(self.plan.off_token_idx, self.plan.num_rows, np.int32)

    @property
    def seg_offsets(self) -> np.ndarray:
        return self._arr(self.plan.off_seg_offsets, self.plan.num_segments + 1, np.int32)

    @property
    def seg_adapter(self) -> np.ndarray:
        return self._arr(self.plan.off_seg_adapter, self.plan.num_segments, np.int32)

    @property
    def seg_rank(self) -> np.ndarray:
        return self._arr(self.plan.off_seg_rank, self.plan.num_segments, np.int32)

    @property
    def seg_scale(self) -> np.ndarray:
        return self._arr(self.plan.off_seg_scale, self.plan.num_segments, np.float32)

    def seg_pt(self, matrix: int) -> np.ndarray:
        off = self.plan.off_seg_a_pt if matrix == 0 else self.plan.off_seg_b_pt
        return self._arr(off, self.plan.num_segments * self.plan.n_proj, np.int64).reshape(
            self.plan.num_segments, self.plan.n_proj)

    def _records(self, off: int, n: int) -> np.ndarray:
        """[n][n_proj] records as an int64 array [..., 6]: seg, row_begin, row_end, rank, a_pt, b_pt."""
        npj = self.plan.n_proj
        raw = self._arr(off, 8 * n * npj, np.int32).reshape(n, npj, 8)
        out = np.zeros((n, npj, 6), dtype=np.int64)
        out[..., :4] = raw[..., :4]
        out[..., 4] = raw[..., 4:6].copy().view(np.int64)[..., 0]
        out[..., 5] = raw[..., 6:8].copy().view(np.int64)[..., 0]
        return out

    @property
    def simt_records(self) -> np.ndarray:
        return self._records(self.plan.off_simt_items, self.plan.num_simt_items)

    @property
    def tc_records(self) -> np.ndarray:
        return self._records(self.plan.off_tc_tiles, self.plan.num_tc_tiles)

    @property
    def simt_items(self) -> np.ndarray:
        """[n][3]: segment, row_begin, row_end of each SIMT item."""
        return self.simt_records[:, 0, :3].astype(np.int32).reshape(-1, 3)

    @property
    def tc_tiles(self) -> np.ndarray:
        """[n][3]: segment, row_begin, row_end of each tensor-core tile."""
        return self.tc_records[:, 0, :3].astype(np.int32).reshape(-1, 3)

    @property
    def num_rows(self) -> int:
        return self.plan.num_rows

    @property
    def max_rank(self) -> int:
        return self.plan.max_rank

    def launches(self, projections: int = 1) -> int:
        """Kernel launches one shrink + expand pass makes per projection, times `projections`."""
        per = 2 * (int(self.plan.num_simt_items > 0) + int(self.plan.num_tc_tiles > 0))
        return per * projections

    # -- device side
    def table_ptr(self, stream=None) -> Optional[int]:
        """Device address of the table for the kernel calls, or None when the plan's work
        items travel as launch arguments (no copy needed)."""
        if not self.plan.needs_device_table:
            return None
        if self.device_table is None:
            self.upload(stream)
        return self.device_table.data_ptr()

    def upload(self, stream=None) -> Optional[torch.Tensor]:
        """Copy the table to the device on `stream` (sgmv_upload_table: a small kernel reading
        the pinned host table); nothing to do when the plan's work items travel as launch
        arguments."""
        if not self.plan.needs_device_table:
            return None
        n = max(int(self.plan.table_bytes), 16)
        dev = torch.device("cuda", self.pool.device)
        if self.device_table is None or self.device_table.numel() < max(n, self.capacity):
            self.device_table = torch.empty(max(n, self.capacity), dtype=torch.uint8, device=dev)
        s = torch.cuda.current_stream(dev) if stream is None else stream
        _check(load_library().sgmv_upload_table(ctypes.byref(self.plan), self.device_table.data_ptr(), _stream(s)))
        with torch.cuda.stream(s):
            if self._uploaded is None:
                self._uploaded = torch.cuda.Event()
            self._uploaded.record(s)
        return self.device_table

    def new_v(self, ldv: Optional[int] = None) -> torch.Tensor:
        ldv = ldv or max(4, (self.plan.max_rank + 3) // 4 * 4)
        return torch.empty(max(self.plan.num_rows, 1), ldv, dtype=torch.float32,
                           device=torch.device("cuda", self.pool.device))


class Residency:
    """Adapters kept in host memory, made resident in `pool` batch by batch with
    least-recently-used eviction (see include/sgmv.h, "Residency manager")."""

    def __init__(self, pool: AdapterPool):
        self.pool = pool
        h = ctypes.c_void_p()
        _check(load_library().sgmv_residency_create(pool.handle, ctypes.byref(h)))
        self.handle = h
        self._host = {}  # adapter -> host tensors kept alive while registered

    def close(self):
        if getattr(self, "handle", None):
            load_library().sgmv_residency_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def register(self, adapter_id: int, rank: int, A: Optional[Sequence[torch.Tensor]] = None,
                 B: Optional[Sequence[torch.Tensor]] = None) -> None:
        """A[p]: bf16 [rank, d_in_p], B[p]: bf16 [d_out_p, rank] on the host (pinned if possible);
        None for a host-only pool."""
        if A is None:
            _check(load_library().sgmv_residency_register(self.handle, int(adapter_id), int(rank), None, None))
            return
        n = len(self.pool.projections)
        keep = []
        for p, (d_in, d_out) in enumerate(self.pool.projections):
            a, b = A[p].contiguous(), B[p].contiguous()
            assert not a.is_cuda and not b.is_cuda and a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16
            assert tuple(a.shape) == (rank, d_in) and tuple(b.shape) == (d_out, rank)
            keep += [a, b]
        a_ptrs = (ctypes.c_void_p * n)(*[keep[2 * p].data_ptr() for p in range(n)])
        b_ptrs = (ctypes.c_void_p * n)(*[keep[2 * p + 1].data_ptr() for p in range(n)])
        _check(load_library().sgmv_residency_register(self.handle, int(adapter_id), int(rank),
                                                      ctypes.cast(a_ptrs, ctypes.c_void_p),
                                                      ctypes.cast(b_ptrs, ctypes.c_void_p)))
        self._host[int(adapter_id)] = keep

    def unregister(self, adapter_id: int) -> None:
        _check(load_library().sgmv_residency_unregister(self.handle, int(adapter_id)))
        self._host.pop(int(adapter_id), None)

    def prepare(self, adapter_ids, copy_stream=None, compute_stream=None) -> int:
        """Make the batch's adapters resident (see sgmv_residency_prepare); returns how many were loaded."""
        ids = np.ascontiguousarray(np.asarray(adapter_ids, dtype=np.int32))
        loaded = ctypes.c_int32(0)
        dev = self.pool.device >= 0
        _check(load_library().sgmv_residency_prepare(
            self.handle, ids.ctypes.data if ids.size else None, int(ids.size),
            _stream(copy_stream) if dev else None, _stream(compute_stream) if dev else None, ctypes.byref(loaded)))
        return int(loaded.value)

    def stats(self) -> ResidencyStats:
        s = ResidencyStats()
        _check(load_library().sgmv_residency_get_stats(self.handle, ctypes.byref(s)))
        return s


def shrink(x: torch.Tensor, plan: BatchPlan, pool: AdapterPool, v: torch.Tensor, proj: int = 0,
           stream=None) -> None:
    """v[i, k] = sum_c A_s[k, c] x[token_idx[i], c]  (SGMV-shrink)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert v.dtype == torch.float32 and v.dim() == 2 and v.stride(1) == 1
    _check(load_library().sgmv_shrink(_ptr(x), x.stride(0), plan.T, x.shape[1], int(proj), ctypes.byref(plan.plan),
                                      plan.table_ptr(stream), pool.handle, _ptr(v), v.stride(0), _stream(stream)))


def expand(v: torch.Tensor, plan: BatchPlan, pool: AdapterPool, y: torch.Tensor, proj: int = 0,
           scale: float = 1.0, stream=None) -> None:
    """y[t, j] += scale * sum_k B_s[j, k] v[i, k]  (SGMV-expand, in place, one rounding)."""
    assert v.dtype == torch.float32 and v.dim() == 2 and v.stride(1) == 1
    assert y.dim() == 2 and y.stride(1) == 1 and y.dtype in (torch.bfloat16, torch.float32)
    _check(load_library().sgmv_expand(_ptr(v), v.stride(0), plan.T, y.shape[1], int(proj), ctypes.byref(plan.plan),
                                      plan.table_ptr(stream), pool.handle, float(scale), _ptr(y), y.stride(0),
                                      0 if y.dtype == torch.bfloat16 else 1, _stream(stream)))


def lora_delta_grouped(entries, plan: BatchPlan, pool: AdapterPool, scale: float = 1.0, stream=None):
    """lora_delta for several projections over the same plan in one call (one SIMT
    shrink and one SIMT expand launch for all of them).  `entries`: (x, y, proj) or
    (x, y, proj, v) tuples, all y of one dtype.  Returns the workspaces v."""
    assert 1 <= len(entries) <= 8
    arr = (DeltaEntry * len(entries))()
    vs, ydt = [], None
    for i, e in enumerate(entries):
        x, y, proj = e[0], e[1], int(e[2])
        v = e[3] if len(e) > 3 and e[3] is not None else plan.new_v()
        assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
        assert y.dim() == 2 and y.stride(1) == 1 and y.dtype in (torch.bfloat16, torch.float32)
        assert v.dtype == torch.float32 and v.dim() == 2 and v.stride(1) == 1
        assert ydt is None or ydt == y.dtype
        ydt = y.dtype
        arr[i] = DeltaEntry(proj, x.shape[1], y.shape[1], 0, _ptr(x), x.stride(0), _ptr(y), y.stride(0), _ptr(v),
                            v.stride(0))
        vs.append(v)
    _check(load_library().sgmv_lora_delta_grouped(arr, len(entries), plan.T, ctypes.byref(plan.plan),
                                                  plan.table_ptr(stream), pool.handle, float(scale),
                                                  0 if ydt == torch.bfloat16 else 1, _stream(stream)))
    return vs


# kernel kinds reported by lora_delta_kernels (SGMV_KERNELS_* in include/sgmv.h)
KERNELS_FUSED, KERNELS_SIMT, KERNELS_TC, KERNELS_SLAB = 1, 2, 4, 8


def lora_delta_kernels(plan: BatchPlan, pool: AdapterPool, projs: Sequence[int], y_dtype=torch.bfloat16,
                       stream=None) -> Tuple[int, int]:
    """(kinds, launches): which kernels lora_delta (one projection) or lora_delta_grouped (the
    projections `projs`) launch for this plan and pool -- a mask of KERNELS_FUSED,
    KERNELS_SIMT (with KERNELS_SLAB when its shrink is the slab kernel) and KERNELS_TC --
    and how many launches; nothing is launched."""
    n = len(projs)
    arr = (ctypes.c_int32 * n)(*[int(p) for p in projs])
    kinds, launches = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().sgmv_lora_delta_kernels(ctypes.byref(plan.plan), pool.handle,
                                                  ctypes.cast(arr, ctypes.c_void_p), n, plan.table_ptr(stream),
                                                  0 if y_dtype == torch.bfloat16 else 1, ctypes.byref(kinds),
                                                  ctypes.byref(launches)))
    return int(kinds.value), int(launches.value)


def lora_delta_noalloc(x: torch.Tensor, plan: BatchPlan, pool: AdapterPool, y: torch.Tensor, proj: int = 0,
                       scale: float = 1.0, stream=None) -> None:
    """lora_delta with the intermediate in the library's fixed device array (no workspace
    argument, nothing allocated); see sgmv_lora_delta_noalloc in include/sgmv.h."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert y.dim() == 2 and y.stride(1) == 1 and y.dtype in (torch.bfloat16, torch.float32)
    _check(load_library().sgmv_lora_delta_noalloc(
        _ptr(x), x.stride(0), plan.T, x.shape[1], y.shape[1], int(proj), ctypes.byref(plan.plan),
        plan.table_ptr(stream), pool.handle, float(scale), _ptr(y), y.stride(0),
        0 if y.dtype == torch.bfloat16 else 1, _stream(stream)))


class HostStep:
    """The whole step from host buffers in one library call (sgmv_lora_delta_host): the
    segment builder, the copies of x and y to the device, the grouped delta and the copy
    of y back, all enqueued on the stream by the library.  Holds the pinned host table
    and the device workspace, grown as needed and reused across steps."""

    def __init__(self, pool: AdapterPool, capacity_tokens: int):
        self.pool = pool
        lib = load_library()
        self.table_bytes = int(lib.sgmv_plan_table_capacity(int(capacity_tokens), len(pool.projections)))
        self.host_table = torch.empty(self.table_bytes, dtype=torch.uint8, pin_memory=torch.cuda.is_available())
        self.workspace: Optional[torch.Tensor] = None
        self.plan = Plan()
        self.capacity = int(capacity_tokens)
        self._done: Optional[torch.cuda.Event] = None

    def run(self, adapter_ids, entries, scale: float = 1.0, stream=None) -> Tuple[int, int]:
        """entries: (x_host, y_host, proj) with contiguous host tensors (pinned for asynchronous
        copies), all y of one dtype; entries naming the same x_host tensor share its copy and
        one stacked shrink pass.  y_host holds the result once the stream has completed.
        Returns the (host-to-device, device-to-host) bytes the step's copies move."""
        ids = np.ascontiguousarray(np.asarray(adapter_ids, dtype=np.int32).reshape(-1))
        assert ids.size <= self.capacity and 1 <= len(entries) <= 8
        if self._done is not None:
            self._done.synchronize()          # the previous step's copies have read the host table
        arr = (HostEntry * len(entries))()
        ydt = None
        for i, (x, y, proj) in enumerate(entries):
            assert not x.is_cuda and not y.is_cuda and x.is_contiguous() and y.is_contiguous()
            assert x.dtype == torch.bfloat16 and y.dtype in (torch.bfloat16, torch.float32)
            assert ydt is None or ydt == y.dtype
            ydt = y.dtype
            arr[i] = HostEntry(int(proj), x.shape[1], y.shape[1], 0, x.data_ptr(), y.data_ptr())
        y_dtype = 0 if ydt == torch.bfloat16 else 1
        lib = load_library()
        need = int(lib.sgmv_host_workspace_bytes(self.capacity, self.pool.handle, arr, len(entries), y_dtype))
        if need < 0:
            _check(1)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", self.pool.device))
        h2d, d2h = ctypes.c_int64(), ctypes.c_int64()
        _check(lib.sgmv_lora_delta_host(ids.ctypes.data if ids.size else None, int(ids.size), self.pool.handle, arr,
                                        len(entries), float(scale), y_dtype, self.host_table.data_ptr(),
                                        self.table_bytes, self.workspace.data_ptr(), self.workspace.numel(),
                                        ctypes.byref(self.plan), ctypes.byref(h2d), ctypes.byref(d2h),
                                        _stream(stream)))
        if self._done is None:
            self._done = torch.cuda.Event()
        s = torch.cuda.current_stream(self.pool.device) if stream is None else stream
        if isinstance(s, torch.cuda.Stream):
            self._done.record(s)
        else:
            self._done.record(torch.cuda.ExternalStream(int(s)))
        return int(h2d.value), int(d2h.value)


def check_errors(stream=None) -> int:
    """Wait for the stream; raise SgmvError if a device-side check failed, else return 0."""
    bits = ctypes.c_uint32()
    _check(load_library().sgmv_check_errors(_stream(stream), ctypes.byref(bits)))
    return bits.value


def lora_delta(x: torch.Tensor, plan: BatchPlan, pool: AdapterPool, y: torch.Tensor, proj: int = 0,
               scale: float = 1.0, v: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y_t += scale * B_{a(t)} A_{a(t)} x_t for every token in one call (SGMV-shrink into the
    workspace v, then SGMV-expand).  Returns v."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert y.dim() == 2 and y.stride(1) == 1 and y.dtype in (torch.bfloat16, torch.float32)
    if v is None:
        v = plan.new_v()
    assert v.dtype == torch.float32 and v.dim() == 2 and v.stride(1) == 1
    _check(load_library().sgmv_lora_delta(
        _ptr(x), x.stride(0), plan.T, x.shape[1], y.shape[1], int(proj), ctypes.byref(plan.plan),
        plan.table_ptr(stream), pool.handle, float(scale), _ptr(y), y.stride(0),
        0 if y.dtype == torch.bfloat16 else 1, _ptr(v), v.stride(0), _stream(stream)))
    return v
