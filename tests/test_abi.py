"""The C-ABI library loads and exports every entry point that include/pbsa.h declares;
host-side argument checks answer without a GPU."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pbsa.h")


def declared():
    src = open(HEADER).read()
    return re.findall(r"^PBSA_API\s+[\w\s\*]+?\b(pbsa_\w+)\s*\(", src, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(_lib.LIB_PATH)


def test_header_declares_the_entry_points():
    names = set(declared())
    assert {"pbsa_blockify", "pbsa_score_select", "pbsa_attend", "pbsa_memory_update",
            "pbsa_get_device_error", "pbsa_status_string", "pbsa_workspace_bytes"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    for name in declared():
        assert hasattr(_lib, name) and hasattr(P, name), name   # bound, and exported by the package


def test_host_side_checks_without_gpu(lib):
    P.load()
    assert P.pbsa_status_string(0) == "ok" and P.pbsa_status_string(5).startswith("index")
    g = P.make_geom(12, 128, 32, 48, 8, 8, 128 ** -0.5, "bf16")
    # error word + per-head column partial sums of four-row groups (18 for 72 query blocks)
    assert P.pbsa_workspace_bytes(g, 72, 360) >= 256 + 12 * 18 * 360 * 4
    assert P.pbsa_workspace_bytes(g, 72, 360) >= P.pbsa_workspace_bytes(g, 8, 40) > 256
    bad = P.make_geom(12, 128, 32, 48, 8, 7, 0.1, "bf16")        # tile is not 64 tokens
    assert _lib.load().pbsa_blockify(ctypes.byref(bad), None, 1, None, 1, None, None, 0, None, None) == 1
    assert _lib.load().pbsa_workspace_bytes(ctypes.byref(bad), 1, 1) == 0
    # null pointers are rejected before any CUDA call
    assert _lib.load().pbsa_attend(ctypes.byref(g), None, 1, None, None, 10, None, None, 8, None, None,
                                   None, None) == 1
    odd = P.make_geom(12, 96, 32, 48, 8, 8, 0.1, "bf16")          # head_dim 96 is not built
    assert _lib.load().pbsa_blockify(ctypes.byref(odd), None, 1, None, 1, None, None, 0, None, None) == 2
    # the fused blockify + select entry point checks its pointers the same way
    assert _lib.load().pbsa_blockify_score_select(ctypes.byref(g), None, 1, None, None, 10, None, None, 0,
                                                  0, None, None, 0, None, None, 0, None, None, None) == 1
