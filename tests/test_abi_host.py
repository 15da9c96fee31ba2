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
