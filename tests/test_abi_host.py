"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/moe_route.h declares, and rejects invalid arguments
on the host before touching the device."""
import ctypes
import os
import re

import pytest

import permute_fp4_dispatch_b200 as moe
from permute_fp4_dispatch_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "moe_route.h")) as f:
        text = f.read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    build()
    return moe.library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 13
    raw = ctypes.CDLL(moe.library_path)
    for n in names:
        assert hasattr(raw, n), n
        assert n in moe._SIGS, n            # and the binding marshals it


def test_binding_names_match_the_header():
    names = set(declared_entry_points())
    exported = {n for n in moe.__all__ if n.startswith("moe_")}
    assert names == exported


def test_status_strings(lib):
    assert moe.moe_status_string(0) == "ok"
    assert "architecture" in moe.moe_status_string(2)
    assert moe.moe_version() >= 100


def test_host_validation_runs_before_any_device_work(lib):
    # invalid shapes are refused on the host (no CUDA call is needed for the verdict)
    P = 16  # any non-null, aligned dummy address
    assert lib.moe_mask_padding(P, -1, 2, P, 0, None) == 1
    assert lib.moe_create_indices(P, 8, 0, P, P, P, P, P, None, P, 256, None) == 1
    assert lib.moe_create_indices(P, 8, 4, P, P, P, P, P, None, None, 0, None) == 3
    assert lib.moe_create_indices_static(P, 8, 2000, P, P, P, P, P, None, None) == 1
    assert lib.moe_dispatch_mxfp4(P, 4, 48, 2, 4, P, P, P, P, P, 8, P, None) == 1   # K % 32
    assert lib.moe_quantize_activations_nvfp4(P, 4, 24, 1.0, P, P, None) == 1      # K % 16
    assert lib.moe_quantize_activations_nvfp4(P, 4, 32, 0.0, P, P, None) == 1      # g > 0
    gemv = lambda *a: lib.moe_grouped_gemv_nvfp4(*a)  # noqa: E731
    G = (P, P, P, P)                                   # a full step-2 grouping
    assert gemv(0, P, None, 1.0, P, 4, 2, P, P, None, 4, 12, 64, *G, P, None, 0, None) == 1  # N % 8
    assert gemv(0, P, None, 1.0, P, 4, 2, P, P, None, 4, 16, 80, *G, P, None, 0, None) == 1  # K % 32
    assert gemv(0, 8 + 1, None, 1.0, P, 4, 2, P, P, None, 4, 16, 64, *G, P, None, 0,
                None) == 1                                                            # alignment
    assert gemv(0, P, None, 1.0, P, 4, 2, P, P, None, 4, 16, 64, P, None, P, P, P, None, 0,
                None) == 1                                                            # partial grouping
    assert gemv(0, P, None, 1.0, None, 4, 2, P, P, None, 4, 16, 64, None, None, None, None, P,
                None, 0, None) == 1                                                   # no map at all
    # the grouping's part of the workspace (the rest holds converted activations)
    ws = moe.moe_grouped_gemv_workspace_bytes(4, 2, 4, 64) - 256 - 512
    assert gemv(0, P, None, 1.0, P, 4, 2, P, P, None, 4, 16, 64, None, None, None, None, P,
                P * 16, ws - 1, None) == 3                                            # workspace size
    assert gemv(0, P, None, 1.0, P, 4, 2, P, P, None, 4, 16, 64, None, None, None, None, P,
                P * 16 + 16, ws, None) == 3                                           # workspace align
    assert lib.moe_combine(P, P, P, 4, 2, 12, 4, 0, 1.0, P, None) == 1              # H % 8
    assert lib.moe_combine(P, P, P, 4, 2, 16, 4, 7, 1.0, P, None) == 1              # epilogue


def test_workspace_sizing(lib):
    assert moe.moe_create_indices_workspace_bytes(1024, 128) == 256
    big = moe.moe_create_indices_workspace_bytes(98304, 64)
    assert big == 256 + 12 * 64 * 4
    assert moe.moe_mxfp4_row_stride(2048) == 1088
    assert moe.moe_mxfp4_row_stride(2880) == 1536
    # grouped GEMV workspace: order, restore [S] u32, starts [E+1], ids [E], stats [2],
    # the grouping call's own workspace, then W4A16 activations converted once
    # (per-token offsets [M] int32, fp16 rows [M, K]), each section 256-byte aligned
    r = lambda n: -(-n // 256) * 256  # noqa: E731
    S, E, M, K = 1024, 128, 128, 2048
    assert moe.moe_grouped_gemv_workspace_bytes(M, 8, E, K) == (
        2 * r(4 * S) + r(4 * (E + 1)) + r(4 * E) + r(8) + 256 + r(4 * M) + r(2 * M * K))
    S, E, M, K = 98304, 64, 16384, 4096
    assert moe.moe_grouped_gemv_workspace_bytes(M, 6, E, K) == (
        2 * r(4 * S) + r(4 * (E + 1)) + r(4 * E) + r(8) + r(256 + 12 * 64 * 4) + r(4 * M) +
        r(2 * M * K))
