"""The C-ABI library loads on a machine without a GPU and exports every entry
point that include/fa_b200.h declares (no compute calls here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_b200.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_fa_build", os.path.join(ROOT, "io_aware_exact_27_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.build()
    return ctypes.CDLL(path)


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ("fa_fwd", "fa_fwd_varlen", "fa_fwd_fp8", "fa_bwd", "fa_bwd_varlen", "fa_bwd_workspace_size",
                 "fa_get_status", "fa_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in fa_b200.h but not exported"


def test_status_strings(lib):
    lib.fa_status_string.restype = ctypes.c_char_p
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(4) == b"FA_ERR_TIMEOUT"
    assert lib.fa_status_string(99) == b"FA_ERR_UNKNOWN"


def test_workspace_size_host_logic(lib):
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    ws = lib.fa_bwd_workspace_size(4 * 2048, 4, 16, 128)
    # two fp32 vectors per (query head, token) (LSE in base 2 and dot(dO, O));
    # per head: tokens rounded up to 4, 4 floats of alignment room per
    # sequence and 128 trailing entries; each vector 256-byte aligned
    per_head = (4 * 2048 + 3) // 4 * 4 + 4 * 4 + 128
    assert ws == 2 * ((16 * per_head * 4 + 255) // 256 * 256)
    assert ws % 256 == 0
    assert lib.fa_bwd_workspace_size(0, 1, 16, 128) == 0


def test_binding_imports_and_names_match():
    import io_aware_exact_27_b200 as fa
    for name in declared_functions():
        assert hasattr(fa, name), f"binding lacks {name}"
