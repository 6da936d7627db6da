"""The C-ABI library builds for sm_100a, loads, and exports every entry point
that include/cqa.h declares (no compute call: runs without a GPU)."""

import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_entry_points():
    src = open(os.path.join(ROOT, "include", "cqa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(cqa_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def libpath():
    from certified_quantized_kv_int8_b200.build import build
    return build()


def test_header_declares_the_boundary():
    names = _declared_entry_points()
    for n in ("cqa_cache_create", "cqa_cache_destroy", "cqa_quantize_append", "cqa_decode",
              "cqa_dense_reference", "cqa_debug_export", "cqa_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(cqa_[a-z_0-9]+)$", out, flags=re.M))
    missing = [n for n in _declared_entry_points() if n not in exported]
    assert not missing, missing


def test_library_loads_and_binding_matches(libpath):
    import certified_quantized_kv_int8_b200 as cqa
    lib = cqa.load_library()
    for n in _declared_entry_points():
        assert hasattr(lib, n)
    assert set(cqa.EXPORTED_SYMBOLS) == set(_declared_entry_points())
    assert cqa.cqa_error_string(0) == "ok"
    assert "capacity" in cqa.cqa_error_string(-4)
    assert cqa.cqa_error_string(12345) == "unknown error"


def test_binding_reports_a_missing_library(tmp_path, monkeypatch):
    import certified_quantized_kv_int8_b200 as cqa
    monkeypatch.setattr(cqa, "_lib", None)
    monkeypatch.setattr(cqa, "LIB", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        cqa.load_library()


def test_sources_use_no_closed_calls():
    """The library issues one plain copy per transfer; no batched-copy runtime call appears."""
    bad = re.compile("cu(da)?" + "Memcpy" + "(3D)?" + "Batch" + "Async")
    for dirpath, _, files in os.walk(os.path.join(ROOT, "certified_quantized_kv_int8_b200")):
        for f in files:
            if f.endswith((".cu", ".cuh", ".h", ".py", ".cpp")):
                assert not bad.search(open(os.path.join(dirpath, f)).read()), f
