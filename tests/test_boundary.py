"""The C ABI without a GPU: the library loads, exports every entry point that
include/*.h declares, sizes workspaces, and rejects bad arguments before any
CUDA call."""
import ctypes
import glob
import os
import re

import pytest

from expert_ffn_layer_moe_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names.update(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward"} <= names
    L = moe.lib()
    missing = [n for n in sorted(names) if not hasattr(L, n)]
    assert not missing, missing


def test_workspace_bytes():
    f = moe.moe_workspace_bytes
    assert f(156, 6144, 16384, 8, 2) > 156 * 2 * (6144 * 2 * 2 + 16384 * 2)
    assert f(156, 6144, 16384, 8, 2, 3072) > f(156, 6144, 16384, 8, 2, 0)
    assert f(2000, 256, 512, 8, 2) > f(1000, 256, 512, 8, 2)
    # invalid sizes -> 0
    assert f(10, 100, 512, 8, 2) == 0        # H not a multiple of 64
    assert f(10, 256, 512, 0, 1) == 0        # no experts
    assert f(10, 256, 512, 4, 5) == 0        # k > E
    assert f(10, 256, 512, 300, 2) == 0      # E > 256
    assert f(10, 256, 512, 16, 9) == 0       # k > 8
    assert f(-1, 256, 512, 8, 2) == 0
    assert f(10, 256, 512, 8, 2, 100) == 0   # shared width not a multiple of 64
    # fp8 activations: the same layout plus the quantized rows (N*k*(H+I) bytes) and their scales
    g = moe.moe_workspace_bytes_w8a8
    assert g(156, 6144, 16384, 8, 2) - f(156, 6144, 16384, 8, 2) >= 312 * (6144 + 16384)
    assert g(10, 100, 512, 8, 2) == 0 and g(10, 256, 512, 4, 5) == 0
    w = moe.moe_expert_ffn_w8a8_ws_bytes
    assert w(312, 6144, 16384) >= 312 * 16384 * 2 + 312 * (6144 + 16384) + 2 * 312 * 4
    assert w(312, 100, 512) == 0 and w(-1, 256, 512) == 0


def test_invalid_arguments_are_rejected_before_any_launch():
    L = moe.lib()
    nullp = None
    s = ctypes.c_void_p(0)
    # bad sizes: every call returns MOE_ERR_INVALID_ARG (1) without touching CUDA
    assert L.moe_route(nullp, nullp, nullp, 4, 256, 0, 1, nullp, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_route(nullp, nullp, nullp, 4, 256, 8, 9, nullp, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_route(nullp, nullp, nullp, 4, 100, 8, 2, nullp, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_route(nullp, nullp, nullp, 4, 256, 8, 2, nullp, nullp, nullp, nullp, 0, s) == 1  # null ptrs
    assert L.moe_permute(nullp, nullp, 4, 256, 8, 2, nullp, nullp, nullp, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_expert_ffn(nullp, nullp, nullp, nullp, nullp, -1, 256, 512, 8, nullp, nullp, 0, s) == 1
    assert L.moe_expert_ffn(nullp, nullp, nullp, nullp, nullp, 8, 256, 500, 8, nullp, nullp, 0, s) == 1
    assert L.moe_combine(nullp, nullp, nullp, nullp, 4, 256, 0, nullp, s) == 1
    # fp8 weights: bad K, negative rows, null pointers, missing scales
    assert L.moe_quantize_fp8(nullp, 4, 100, nullp, nullp, s) == 1
    assert L.moe_quantize_fp8(nullp, -1, 256, nullp, nullp, s) == 1
    assert L.moe_quantize_fp8(nullp, 4, 256, nullp, nullp, s) == 1
    assert L.moe_quantize_fp8(nullp, 0, 256, nullp, nullp, s) == 0          # nothing to do
    assert L.moe_expert_ffn_fp8(*([nullp] * 8), 8, 256, 500, 8, nullp, nullp, 0, s) == 1
    assert L.moe_expert_ffn_fp8(*([nullp] * 8), 8, 256, 512, 8, nullp, nullp, 0, s) == 1
    assert L.moe_layer_forward_fp8_ex(*([nullp] * 12), 4, 256, 512, 8, 2, 0, nullp, nullp, nullp, 0, s,
                                      nullp) == 1
    assert L.moe_expert_ffn_w8a8(*([nullp] * 8), 8, 256, 500, 8, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_expert_ffn_w8a8(*([nullp] * 8), 8, 256, 512, 8, nullp, nullp, nullp, 0, s) == 1
    assert L.moe_expert_ffn_w8a8(*([nullp] * 8), 0, 256, 512, 8, nullp, nullp, nullp, 0, s) == 0
    assert L.moe_layer_forward_w8a8_ex(*([nullp] * 12), 4, 256, 512, 8, 2, 0, nullp, nullp, nullp, 0, s,
                                       nullp) == 1
    assert L.moe_layer_forward_w8a8_ex(*([nullp] * 12), 4, 256, 512, 8, 9, 0, nullp, nullp, nullp, 0, s,
                                       nullp) == 1
    assert L.moe_layer_forward(nullp, nullp, nullp, nullp, nullp, 4, 256, 512, 8, 2, nullp) == 1
    # row scatter: width a positive multiple of 8, rows >= 0, pointers present
    assert L.moe_scatter_rows(nullp, nullp, 4, 12, nullp, 4, s) == 1
    assert L.moe_scatter_rows(nullp, nullp, -1, 64, nullp, 4, s) == 1
    assert L.moe_scatter_rows(nullp, nullp, 4, 64, nullp, -1, s) == 1
    assert L.moe_scatter_rows(nullp, nullp, 4, 64, nullp, 4, s) == 1
    assert L.moe_scatter_rows(nullp, nullp, 0, 64, nullp, 4, s) == 0
    assert L.moe_layer_forward_ex(*([nullp] * 9), 4, 256, 512, 8, 2, 64, nullp, nullp, nullp, 0, s,
                                  nullp) == 1
    # N == 0 is a no-op where no output needs defining
    assert L.moe_route(nullp, nullp, nullp, 0, 256, 8, 2, nullp, nullp, nullp, nullp, 0, s) == 0
    assert L.moe_combine(nullp, nullp, nullp, nullp, 0, 256, 2, nullp, s) == 0
    assert L.moe_expert_ffn(nullp, nullp, nullp, nullp, nullp, 0, 256, 512, 8, nullp, nullp, 0, s) == 0


def test_misaligned_pointers_are_unsupported():
    L = moe.lib()
    fake = ctypes.c_void_p(0x1000 + 8)   # never dereferenced: the check comes first
    ok = ctypes.c_void_p(0x2000)
    s = ctypes.c_void_p(0)
    assert L.moe_route(fake, ok, None, 4, 256, 8, 2, None, ok, ok, None, 0, s) == 2
    assert L.moe_combine(fake, ok, ok, None, 4, 256, 2, ok, s) == 2
    assert L.moe_quantize_fp8(fake, 4, 256, ok, ok, s) == 2
    assert L.moe_quantize_fp8(ok, 4, 256, fake, ok, s) == 2
    # fp8 activations: a misaligned h output is refused before the workspace is looked at
    assert L.moe_expert_ffn_w8a8(*([ok] * 8), 8, 256, 512, 8, ok, fake, None, 0, s) == 2
    assert L.moe_scatter_rows(fake, ok, 4, 64, ok, 4, s) == 2
    # and a missing or short workspace is refused
    assert L.moe_expert_ffn_w8a8(*([ok] * 8), 8, 256, 512, 8, ok, None, None, 0, s) == 3


def test_status_strings():
    L = moe.lib()
    assert L.moe_status_string(0) == b"ok"
    assert L.moe_status_string(3).startswith(b"workspace")


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "_LIB_PATH", "/nonexistent/libmoe_b200.so")
    with pytest.raises(RuntimeError, match="not built"):
        moe.lib()


def test_process_wide_options_round_trip_and_reject_bad_values():
    """Every option setter returns the previous setting, takes effect for later calls,
    and refuses values outside its range (-1 from C, ValueError from the binding),
    all without a GPU."""
    L = moe.lib()
    cases = [  # (setter, valid values, default, a rejected value)
        (L.moe_set_gather_mode, [moe.MOE_GATHER_OFF, moe.MOE_GATHER_ON, moe.MOE_GATHER_AUTO], moe.MOE_GATHER_AUTO, 7),
        (L.moe_set_microbatches, [2, 1], 1, 3),
        (L.moe_set_shared_stream, [0, 1], 1, 2),
        (L.moe_set_decode_gemv, [moe.MOE_DECODE_OFF, moe.MOE_DECODE_ON, moe.MOE_DECODE_AUTO], moe.MOE_DECODE_AUTO, -1),
    ]
    for setter, values, default, bad in cases:
        prev = setter(default)
        try:
            assert prev == default          # nothing else in this process changed it
            last = default
            for v in values:
                assert setter(v) == last
                last = v
            assert setter(bad) == -1        # refused, and the setting is unchanged
            assert setter(default) == last
        finally:
            setter(default)
    with pytest.raises(ValueError):
        moe.moe_set_decode_gemv(5)
    with pytest.raises(ValueError):
        moe.moe_set_gather_mode(9)
    with pytest.raises(ValueError):
        moe.moe_set_microbatches(0)
