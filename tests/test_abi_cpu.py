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
