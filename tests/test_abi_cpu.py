"""CPU-side checks of the boundary: the library loads and exports every entry
point that include/pa.h declares, and plan validation rejects unsupported
geometry before touching the device."""
import ctypes
import os
import re

import pytest

from paged_kv_gqa_fmha_b200 import _build, binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    return sorted(set(re.findall(r"PA_API\s+[\w\s\*]*?\b(pa_\w+)\s*\(", src)))


def test_library_builds_and_exports_every_declared_symbol():
    _build.build()
    lib = ctypes.CDLL(binding.LIB_PATH)
    names = declared_entry_points()
    assert set(names) == set(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_binding_declares_signatures():
    lib = binding.load_library()
    assert lib.pa_run.restype is ctypes.c_int
    assert lib.pa_last_error() is not None


@pytest.mark.parametrize("args,msg", [
    ((0, 32, 8, 128, 16, 128), "must be > 0"),
    ((4, 32, 8, 96, 16, 128), "unsupported head_dim"),
    ((4, 32, 8, 128, 8, 128), "unsupported page_size"),
    ((4, 32, 6, 128, 16, 128), "not a multiple"),
    ((4, 128, 2, 128, 16, 128), "GQA ratio 64"),
    ((4, 32, 8, 128, 16, -3), "must be > 0"),
])
def test_plan_rejects_unsupported_geometry_on_host(args, msg):
    lib = binding.load_library()
    h = lib.pa_create_plan(*args)
    assert not h
    assert msg in lib.pa_last_error().decode()


def test_setters_reject_null_plan():
    lib = binding.load_library()
    assert lib.pa_set_scale(None, 1.0) == binding.PA_ERR_INVALID
    assert lib.pa_set_num_pages(None, 3) == binding.PA_ERR_INVALID
    assert lib.pa_set_num_splits(None, 2) == binding.PA_ERR_INVALID
    assert lib.pa_run(None, None, None, None, None, None, None, None, None, None) == \
        binding.PA_ERR_INVALID
    assert lib.pa_workspace_bytes(None) == 0
    lib.pa_destroy(None)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        binding.load_library(str(tmp_path / "nope.so"))


def test_every_plan_entry_point_rejects_null_plan():
    """Each call that takes a plan checks it before anything else (no device
    work is attempted)."""
    lib = binding.load_library()
    E = binding.PA_ERR_INVALID
    assert lib.pa_set_two_stage_prefill(None, 1) == E
    assert lib.pa_set_decode_kernel(None, 1) == E
    assert lib.pa_set_causal(None, 0) == E
    assert lib.pa_set_fused_merge(None, 1) == E
    assert lib.pa_set_page_table_stride(None, 256) == E
    assert lib.pa_set_kv_fp8(None, 1, 1.0, 1.0) == E
    assert lib.pa_append_kv(None, None, None, None, None, None, None, None, None) == E
    assert lib.pa_profile_start(None, 4) == E
    f, n, k = ctypes.c_float(), ctypes.c_int(), ctypes.c_int()
    assert lib.pa_profile_read(None, ctypes.byref(f), ctypes.byref(n), ctypes.byref(k)) == E
    s = ctypes.c_uint32()
    assert lib.pa_get_status(None, None, ctypes.byref(s), 0) == E
    assert lib.pa_max_splits(None) == 0
    assert "NULL" in lib.pa_last_error().decode()


def test_selftest_wait_timeout_validates_arguments_on_host():
    lib = binding.load_library()
    s, t = ctypes.c_uint32(), ctypes.c_uint32()
    assert lib.pa_selftest_wait_timeout(100, None, ctypes.byref(t)) == binding.PA_ERR_INVALID
    assert lib.pa_selftest_wait_timeout(0, ctypes.byref(s), ctypes.byref(t)) == \
        binding.PA_ERR_INVALID
    assert "limit_us" in lib.pa_last_error().decode()
    assert lib.pa_selftest_wait_timeout(1000001, ctypes.byref(s), ctypes.byref(t)) == \
        binding.PA_ERR_INVALID


# Fake device addresses: every case below is rejected by the host-side checks
# before any pointer is used, so none of them is ever dereferenced.
_A = 0x10000          # 16-byte aligned
_M = 0x10008          # not 16-byte aligned


@pytest.mark.parametrize("geom,ptrs,code,msg", [
    ((0, 32, 8, 128, 16, 8, 0, 0.0), (_A,) * 6, binding.PA_ERR_INVALID, "must be > 0"),
    ((2, 32, 8, 96, 16, 8, 0, 0.0), (_A,) * 6, binding.PA_ERR_UNSUPPORTED, "unsupported geometry"),
    ((2, 128, 2, 128, 16, 8, 0, 0.0), (_A,) * 6, binding.PA_ERR_UNSUPPORTED, "unsupported geometry"),
    ((2, 32, 8, 128, 16, 8, 0, float("nan")), (_A,) * 6, binding.PA_ERR_INVALID, "scale"),
    ((4096, 32, 8, 128, 16, 4096, 0, 0.0), (_A,) * 6, binding.PA_ERR_UNSUPPORTED, "scratch"),
    ((2, 32, 8, 128, 16, 8, 0, 0.0), (_A, _A, None, _A, _A, _A), binding.PA_ERR_INVALID, "NULL"),
    ((2, 32, 8, 128, 16, 8, 0, 0.0), (_A, _A, _A, _M, _A, _A), binding.PA_ERR_INVALID, "aligned"),
])
def test_run_noalloc_rejects_bad_arguments_on_host(geom, ptrs, code, msg):
    """pa_run_noalloc validates geometry, scale, its scratch bound, NULL and
    misaligned pointers before it looks for a device."""
    lib = binding.load_library()
    B, Hq, Hkv, D, ps, C, P, scale = geom
    q, k, v, table, lens, out = ptrs
    rc = lib.pa_run_noalloc(B, Hq, Hkv, D, ps, C, P, scale, q, k, v, table, lens, None, out,
                            None, None)
    assert rc == code
    assert msg in lib.pa_last_error().decode()
