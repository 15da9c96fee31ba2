"""Host-side checks of the C ABI: the library loads without a GPU, exports every
entry point include/sgmv.h declares, and rejects malformed arguments with a
status code instead of launching anything."""
import ctypes
import os
import re

import pytest

import segmented_rank_gemm_sgmv_b200 as sg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "sgmv.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"SGMV_API\s+[\w\s\*]*?\b(sgmv_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_entry_points()
    assert len(names) >= 16
    lib = ctypes.CDLL(sg.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sg.EXPORTED)


def test_status_strings():
    lib = sg.load_library()
    assert lib.sgmv_status_string(0) == b"SGMV_OK"
    assert lib.sgmv_status_string(3) == b"SGMV_ERR_NOT_RESIDENT"


@pytest.mark.parametrize("kw,err", [
    (dict(page_elems=500), "power of two"),
    (dict(page_elems=32), "power of two"),
    (dict(projections=[(512, 700)]), "multiple of page_elems"),
    (dict(max_rank=129), "max_rank"),
    (dict(num_pages=0), "num_pages"),
])
def test_pool_create_rejects(kw, err):
    args = dict(projections=[(512, 512)], num_pages=16, page_elems=64, max_rank=16, device=-1)
    args.update(kw)
    with pytest.raises(sg.SgmvError) as e:
        sg.AdapterPool(**args)
    assert e.value.status == 1 and err in str(e.value)


def test_kernel_entry_points_reject_host_only_pool():
    pool = sg.AdapterPool([(512, 512)], num_pages=64, page_elems=512, max_rank=16, device=-1)
    pool.load(0, 8)
    plan = pool.plan([0, 0, -1])
    lib = sg.load_library()
    st = lib.sgmv_shrink(None, 512, 3, 512, 0, ctypes.byref(plan.plan), None, pool.handle, None, 8, None)
    assert st == 1 and b"no device memory" in lib.sgmv_last_error()
    st = lib.sgmv_expand(None, 8, 3, 512, 0, ctypes.byref(plan.plan), None, pool.handle, 1.0, None, 512, 0, None)
    assert st == 1


def test_plan_table_capacity_bounds():
    lib = sg.load_library()
    assert lib.sgmv_plan_table_capacity(-1, 1) == -1
    assert lib.sgmv_plan_table_capacity(0, 1) >= 16
    assert lib.sgmv_plan_table_capacity(1000, 7) >= 1000 * 4 * 3 + 1000 * 7 * 16 + 1000 * 32


def test_host_step_workspace_and_argument_checks():
    """sgmv_host_workspace_bytes: the table, each distinct x, each y and each v, every
    region rounded up to 256 bytes; sgmv_lora_delta_host refuses bad arguments before
    enqueueing anything."""
    pool = sg.AdapterPool([(1024, 512), (1024, 1536), (2048, 512)], num_pages=4096, page_elems=512, max_rank=16,
                          device=-1)
    pool.load(0, 16)
    lib = sg.load_library()
    T = 37
    r256 = lambda n: (n + 255) // 256 * 256
    x0, x2 = ctypes.c_void_p(4096), ctypes.c_void_p(8192)          # host addresses are not touched here
    ents = (sg.HostEntry * 3)(sg.HostEntry(0, 1024, 512, 0, x0, ctypes.c_void_p(1 << 20)),
                              sg.HostEntry(1, 1024, 1536, 0, x0, ctypes.c_void_p(2 << 20)),
                              sg.HostEntry(2, 2048, 512, 0, x2, ctypes.c_void_p(3 << 20)))
    table = lib.sgmv_plan_table_capacity(T, 3)
    for y_dtype, esz in ((0, 2), (1, 4)):
        want = (r256(table) + r256(T * 1024 * 2) + r256(T * 2048 * 2) +
                sum(r256(T * d * esz) for d in (512, 1536, 512)) + 3 * r256(T * 16 * 4))
        assert lib.sgmv_host_workspace_bytes(T, pool.handle, ents, 3, y_dtype) == want
    assert lib.sgmv_host_workspace_bytes(T, pool.handle, ents, 0, 0) == -1
    bad = (sg.HostEntry * 1)(sg.HostEntry(0, 1024, 1536, 0, x0, ctypes.c_void_p(1 << 20)))   # d_out of proj 1
    assert lib.sgmv_host_workspace_bytes(T, pool.handle, bad, 1, 0) == -1
    ids = (ctypes.c_int32 * 2)(0, -1)
    host = ctypes.create_string_buffer(4096)
    st = lib.sgmv_lora_delta_host(ids, 2, pool.handle, ents, 3, 1.0, 0, host, 4096, None, 0, None, None, None, None)
    assert st == 1 and b"workspace" in lib.sgmv_last_error()


def test_kernels_query_argument_checks():
    """sgmv_lora_delta_kernels refuses malformed arguments before any CUDA call."""
    lib = sg.load_library()
    pool = sg.AdapterPool([(512, 512)], num_pages=64, page_elems=512, max_rank=16, device=-1)
    pool.load(0, 8)
    plan = pool.plan([0, 0, -1])
    projs = (ctypes.c_int32 * 1)(0)
    kinds, launches = ctypes.c_int32(7), ctypes.c_int32(7)
    pp = ctypes.cast(projs, ctypes.c_void_p)
    st = lib.sgmv_lora_delta_kernels(None, pool.handle, pp, 1, None, 0, ctypes.byref(kinds), ctypes.byref(launches))
    assert st == 1 and b"required" in lib.sgmv_last_error()
    st = lib.sgmv_lora_delta_kernels(ctypes.byref(plan.plan), pool.handle, pp, 1, None, 0, None, ctypes.byref(launches))
    assert st == 1
    st = lib.sgmv_lora_delta_kernels(ctypes.byref(plan.plan), pool.handle, pp, 1, None, 0, ctypes.byref(kinds),
                                     ctypes.byref(launches))
    assert st == 1 and b"no device memory" in lib.sgmv_last_error()
    pool.close()


def test_upload_table_argument_checks():
    """sgmv_upload_table refuses null or misaligned tables before any CUDA call."""
    lib = sg.load_library()
    pool = sg.AdapterPool([(512, 512)], num_pages=64, page_elems=512, max_rank=16, device=-1)
    pool.load(0, 8)
    plan = pool.plan([0, 0, -1])
    assert lib.sgmv_upload_table(None, 16, None) == 1
    assert lib.sgmv_upload_table(ctypes.byref(plan.plan), None, None) == 1
    assert lib.sgmv_upload_table(ctypes.byref(plan.plan), 17, None) == 1
    assert b"aligned" in lib.sgmv_last_error()
    pool.close()
