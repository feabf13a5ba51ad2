"""The C-ABI library builds, loads, and exports every entry point include/attn.h declares.

No call here reaches the GPU: only pure host functions and argument checks that fail before any
CUDA call are exercised.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "attn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def raw():
    from exact_io_aware_41_b200 import build

    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("attn_fwd", "attn_decode_splitkv", "attn_decode_combine", "attn_decode_workspace_bytes",
                 "attn_get_last_error", "attn_status_string", "attn_kernel_name"):
        assert must in names


def test_library_exports_every_declared_symbol(raw):
    for name in _declared_functions():
        assert hasattr(raw, name), name


def test_binding_covers_every_declared_symbol(raw):
    import exact_io_aware_41_b200 as pkg

    assert set(_declared_functions()) == set(pkg.SIGNATURES)
    for name in _declared_functions():
        assert callable(getattr(pkg, name, None)) or name in ("attn_status_string", "attn_kernel_name")


def test_status_strings_and_kernel_names():
    import exact_io_aware_41_b200 as pkg

    assert pkg.status_string(0) == "ok"
    assert "timed out" in pkg.status_string(pkg.ATTN_ERR_TIMEOUT)
    assert pkg.status_string(99) == "unknown status"
    assert pkg.kernel_name(0).startswith("attn::attn_fwd_kernel")
    assert pkg.kernel_name(1).startswith("attn::decode_split_tc_kernel")
    assert pkg.kernel_name(7) is None


def test_decode_workspace_sizing():
    import exact_io_aware_41_b200 as pkg

    # n_splits = ceil(1000 / 64) = 16; part_o = 2*8*16*128*4 = 131072 bytes (already 256-aligned);
    # part_lse = 2*8*16*4 = 1024 bytes
    assert pkg.attn_decode_workspace_bytes(2, 8, 2, 128, 1000, 64) == 131072 + 1024
    assert pkg.attn_decode_workspace_bytes(0, 8, 2, 128, 1000, 64) == 0
    assert pkg.attn_decode_workspace_bytes(2, 8, 3, 128, 1000, 64) == 0
    c = pkg.attn_decode_default_chunk(8, 8, 131072)
    assert c % 64 == 0 and 64 <= c <= 2048
    assert pkg.attn_decode_workspace_bytes(8, 32, 8, 128, 131072, 0) == \
        pkg.attn_decode_workspace_bytes(8, 32, 8, 128, 131072, c)


def test_argument_errors_are_reported_before_any_launch(raw):
    import exact_io_aware_41_b200 as pkg

    lib = pkg.lib_handle()
    p = 1 << 20  # aligned, never dereferenced: every call below fails validation first
    # null pointer
    assert lib.attn_fwd(0, p, p, p, p, 1, 2, 2, 16, 16, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    # misaligned pointer
    assert lib.attn_fwd(p + 2, p, p, p, p, 1, 2, 2, 16, 16, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    # Hq not a multiple of Hkv, zero sizes, bad scale, bad causal flag
    assert lib.attn_fwd(p, p, p, p, p, 1, 3, 2, 16, 16, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd(p, p, p, p, p, 1, 2, 2, 0, 16, 64, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd(p, p, p, p, p, 1, 2, 2, 16, 16, 64, -1.0, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd(p, p, p, p, p, 1, 2, 2, 16, 16, 64, float("nan"), 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd(p, p, p, p, p, 1, 2, 2, 16, 16, 64, 0.125, 2, None) == pkg.ATTN_ERR_INVALID_ARG
    # unsupported head dim
    assert lib.attn_fwd(p, p, p, p, p, 1, 2, 2, 16, 16, 48, 0.125, 0, None) == pkg.ATTN_ERR_UNSUPPORTED
    # decode: chunk not a multiple of 64, unsupported group, too little workspace
    args = [p, p, p, p, 1024, p, p, 2, 8, 2, 128, 0.1]
    assert lib.attn_decode_splitkv(*args, 100, p, 1 << 30, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_decode_splitkv(p, p, p, p, 1024, p, p, 2, 6, 2, 128, 0.1, 64, p, 1 << 30, None) == \
        pkg.ATTN_ERR_UNSUPPORTED
    assert lib.attn_decode_splitkv(p, p, p, p, 1024, p, p, 2, 8, 2, 48, 0.1, 64, p, 1 << 30, None) == \
        pkg.ATTN_ERR_UNSUPPORTED
    assert lib.attn_decode_splitkv(*args, 64, p, 16, None) == pkg.ATTN_ERR_WORKSPACE
    assert lib.attn_decode_splitkv(*args, 64, 0, 1 << 30, None) == pkg.ATTN_ERR_WORKSPACE
    assert lib.attn_decode_combine(p, p, 0, 4, 128, p, p, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_decode_combine(p, p, 4, 4, 96, p, p, None) == pkg.ATTN_ERR_UNSUPPORTED
    assert lib.attn_decode_combine(p, p, 4, 25601, 128, p, p, None) == pkg.ATTN_ERR_UNSUPPORTED
    assert lib.attn_selftest_bounded_wait(0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_pair_wait(0, 1, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_pair_wait(1000, 2, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_exp2_poly(None, p, 4, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_exp2_poly(p, p, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_selftest_exp2_poly(p + 2, p, 4, None) == pkg.ATTN_ERR_INVALID_ARG


def test_decode_sizes_the_combine_cannot_take_are_refused_before_any_launch(raw):
    """More than 25600 splits per row (the combine kernel's shared-memory limit) is refused by both
    decode entry points before the split kernel is enqueued: no CUDA call is reached here, on a
    host without a GPU."""
    import exact_io_aware_41_b200 as pkg

    lib = pkg.lib_handle()
    p = 1 << 20
    cap = 64 * 25601  # chunk 64: 25601 splits
    assert lib.attn_decode_splitkv(p, p, p, p, cap, p, p, 1, 1, 1, 32, 0.1, 64, p, 1 << 40, None) == \
        pkg.ATTN_ERR_UNSUPPORTED
    assert lib.attn_decode_splitkv_static(p, p, p, p, cap, p, p, 1, 1, 1, 32, 0.1, 64, None) == \
        pkg.ATTN_ERR_UNSUPPORTED
    # one split fewer passes the check and reaches the workspace check (too small here)
    assert lib.attn_decode_splitkv(p, p, p, p, cap - 64, p, p, 1, 1, 1, 32, 0.1, 64, p, 16, None) == \
        pkg.ATTN_ERR_WORKSPACE


def test_backward_and_8bit_argument_errors_are_reported_before_any_launch(raw):
    """The backward and 8-bit entry points refuse bad arguments on the host, before any CUDA call."""
    import exact_io_aware_41_b200 as pkg

    lib = pkg.lib_handle()
    p = 1 << 20  # aligned, never dereferenced
    big = 1 << 40

    def bwd(*, q=p, lse=p, B=1, Hq=2, Hkv=2, Nq=16, Nkv=16, d=128, scale=0.125, causal=0, ws=p, ws_bytes=big):
        return lib.attn_bwd(q, p, p, p, lse, p, p, p, p, B, Hq, Hkv, Nq, Nkv, d, scale, causal, ws, ws_bytes, None)

    assert bwd(q=0) == pkg.ATTN_ERR_INVALID_ARG
    assert bwd(q=p + 8) == pkg.ATTN_ERR_INVALID_ARG           # operands 16-byte aligned
    assert bwd(lse=p + 2) == pkg.ATTN_ERR_INVALID_ARG         # lse 4-byte aligned
    assert bwd(Hq=3) == pkg.ATTN_ERR_INVALID_ARG              # Hq a multiple of Hkv
    assert bwd(Nkv=0) == pkg.ATTN_ERR_INVALID_ARG
    assert bwd(scale=0.0) == pkg.ATTN_ERR_INVALID_ARG
    assert bwd(causal=3) == pkg.ATTN_ERR_INVALID_ARG
    assert bwd(d=64) == pkg.ATTN_ERR_UNSUPPORTED
    assert bwd(ws=0) == pkg.ATTN_ERR_WORKSPACE
    assert bwd(ws=p + 16) == pkg.ATTN_ERR_WORKSPACE           # workspace 256-byte aligned
    assert bwd(ws_bytes=pkg.attn_bwd_workspace_bytes(1, 2, 16, 128) - 1) == pkg.ATTN_ERR_WORKSPACE
    # 8-bit quantization and attention
    assert lib.attn_fp8_quantize(0, None, p, p, 1, 16, 2, 128, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fp8_quantize(p, None, p, p + 2, 1, 16, 2, 128, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fp8_quantize(p, None, p, p, 1, 20, 2, 128, 1, None) == pkg.ATTN_ERR_INVALID_ARG  # N % 16
    assert lib.attn_fp8_quantize(p, None, p, p, 1, 16, 2, 128, 2, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fp8_quantize(p, None, p, p, 1, 16, 2, 64, 0, None) == pkg.ATTN_ERR_UNSUPPORTED
    f8 = [p, p, p, p, p, p, p, p]
    assert lib.attn_fwd_fp8(*f8, 1, 2, 2, 16, 24, 128, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG  # Nkv % 16
    assert lib.attn_fwd_fp8(*f8, 1, 3, 2, 16, 16, 128, 0.125, 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_fp8(*f8, 1, 2, 2, 16, 16, 128, float("inf"), 0, None) == pkg.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_fp8(*f8, 1, 2, 2, 16, 16, 64, 0.125, 0, None) == pkg.ATTN_ERR_UNSUPPORTED


def test_backward_workspace_sizing():
    import exact_io_aware_41_b200 as pkg

    # fp32 dQ accumulator [B, Nq, Hq, d] rounded up to 256 bytes, then LSE' and D rows of whole
    # 128-row tiles: B=2, Hq=3, Nq=130, d=128 -> 399360 + 2 * 2*3*256*4 = 411648
    assert pkg.attn_bwd_workspace_bytes(2, 3, 130, 128) == 2 * 130 * 3 * 128 * 4 + 2 * (2 * 3 * 256 * 4)
    assert pkg.attn_bwd_workspace_bytes(1, 1, 1, 128) == 512 + 2 * 128 * 4
    assert pkg.attn_bwd_workspace_bytes(0, 1, 1, 128) == 0
