"""The C-ABI library loads on a machine without a GPU and exports every entry
point that include/fa_b200.h declares; its pure host logic (workspace sizes,
status strings, argument checks that return before any device work) answers
there too. No compute calls here."""

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


def test_kvcache_workspace_size_host_logic(lib):
    """Split-KV decode scratch: per split, one fp32 partial O row (d floats)
    and its LSE for every (batch, query, head); nothing for a single split."""
    f = lib.fa_fwd_kvcache_workspace_size
    f.restype = ctypes.c_size_t
    assert f(16, 1, 32, 128, 1) == 0 and f(16, 1, 32, 128, 0) == 0
    for B, Nq, Hq, d, s in ((16, 1, 32, 128, 4), (2, 3, 8, 64, 7)):
        assert f(B, Nq, Hq, d, s) == s * B * Nq * Hq * (d + 1) * 4
    assert f(0, 1, 32, 128, 4) == 0 and f(16, 1, 32, 128, 8) == 2 * f(16, 1, 32, 128, 4)


def test_argument_checks_before_any_device_work(lib):
    """Calls rejected (or empty) by their host-side checks return before
    touching a device, so they answer on a machine without one."""
    P = ctypes.c_void_p
    lib.fa_fwd_blocksparse.argtypes = [P] * 6 + [ctypes.c_int] * 6 + [ctypes.c_float, P]
    fake = P(16)
    # negative sizes: invalid; an empty batch: nothing to do
    assert lib.fa_fwd_blocksparse(fake, fake, fake, fake, fake, fake, -1, 1, 1, 128, 64, 0, 0.125, None) == 1
    assert lib.fa_fwd_blocksparse(fake, fake, fake, fake, fake, fake, 0, 1, 1, 128, 64, 0, 0.125, None) == 0
    # no mask: invalid; more than 1024 key blocks: unsupported
    assert lib.fa_fwd_blocksparse(fake, fake, fake, None, fake, fake, 1, 1, 1, 128, 64, 0, 0.125, None) == 1
    assert lib.fa_fwd_blocksparse(fake, fake, fake, fake, fake, fake, 1, 1, 1, 131073, 64, 0, 0.125, None) == 2
    lib.fa_fwd.argtypes = [P] * 5 + [ctypes.c_int] * 6 + [ctypes.c_float, P]
    assert lib.fa_fwd(fake, fake, fake, fake, fake, -2, 1, 1, 128, 64, 0, 0.125, None) == 1
    assert lib.fa_fwd(fake, fake, fake, fake, fake, 3, 1, 1, 0, 64, 0, 0.125, None) == 0
    # fp8 backward: code pointers required; d = 128 only
    lib.fa_bwd_fp8.argtypes = [P] * 14 + [ctypes.c_size_t] + [ctypes.c_int] * 6 + [ctypes.c_float, P]
    args = [fake] * 14 + [1 << 20]
    assert lib.fa_bwd_fp8(*([None] + args[1:]), 1, 2, 2, 256, 128, 1, 0.125, None) == 1
    assert lib.fa_bwd_fp8(*args, 1, 2, 2, 256, 64, 1, 0.125, None) == 2
    assert lib.fa_bwd_fp8(*args, 0, 2, 2, 256, 128, 1, 0.125, None) == 0


def test_torch_wrappers_reject_what_the_library_cannot_read():
    """The C entry points see only data pointers: the torch-level calls refuse
    non-contiguous views, other element types and host tensors before any
    library call (so this runs without a GPU)."""
    import torch
    import io_aware_exact_27_b200 as fa
    x = torch.zeros((2, 256, 4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="contiguous"):
        fa.attention_fwd(x[:, ::2], x[:, ::2], x[:, ::2])
    with pytest.raises(ValueError, match="bfloat16"):
        fa.attention_fwd(x.float(), x, x)
    with pytest.raises(ValueError, match="CUDA"):
        fa.attention_fwd(x, x, x)
    lse = torch.zeros((2, 4, 256), dtype=torch.float32)
    with pytest.raises(ValueError, match="float32"):
        fa.attention_bwd(x, x, x, x, lse.double(), x)
    with pytest.raises(ValueError, match="int32"):
        fa.attention_fwd_varlen(x[0], x[0], x[0], torch.zeros(3, dtype=torch.int64), 128)
    with pytest.raises(ValueError, match="uint8"):
        fa.attention_fwd_blocksparse(x, x, x, torch.ones((4, 2, 2), dtype=torch.int32))
    with pytest.raises(ValueError, match="1-byte"):
        fa.attention_fwd_fp8(x, x, x, lse, lse, lse)


def test_noalloc_size_limit_on_the_host(lib):
    """fa_bwd_noalloc's size check runs before any device call: a problem
    whose workspace (fa_bwd_workspace_size) exceeds the 8 MiB array is refused with
    FA_ERR_WORKSPACE; one that just fits passes the check and then stops
    at a later host-side check (null tensors), launching nothing."""
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.fa_bwd_noalloc.argtypes = [P] * 9 + [I] * 6 + [ctypes.c_float, P]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    fake = P(256)
    limit = 8 << 20
    H, d = 16, 128
    # largest N (B = 1) whose workspace fits, found from the size function itself
    fits = max(n for n in range(60000, 70000, 4) if lib.fa_bwd_workspace_size(n, 1, H, d) <= limit)
    assert lib.fa_bwd_workspace_size(fits + 4, 1, H, d) > limit
    assert lib.fa_bwd_noalloc(*([fake] * 9), 1, H, H, fits + 4, d, 1, 0.1, None) == 5
    # null tensors: past the size check the call stops at the device lookup
    # (no GPU) or at the pointer checks (GPU): nothing is launched either way
    st = lib.fa_bwd_noalloc(*([None] * 9), 1, H, H, fits, d, 1, 0.1, None)
    assert st in (1, 3)
    # about Hq * (B*N + 4*B + 131) fp32 pairs: 8 MiB / 8 bytes / 16 heads
    assert abs(fits - (limit // 8 // H - 4 - 131)) <= 8

