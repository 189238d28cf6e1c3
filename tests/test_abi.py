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


def test_new_entry_points_reject_bad_arguments_on_the_host(lib):
    """pbsa_blockify_kv, pbsa_memory_update_plan and pbsa_memory_update_apply validate their
    scalars and flags on the host and return before any launch (the well-aligned fake pointers
    below are never dereferenced)."""
    L = _lib.load()
    g = P.make_geom(12, 128, 32, 48, 8, 8, 128 ** -0.5, "bf16")
    fake = ctypes.c_void_p(0x10000)
    gp = ctypes.byref(g)
    # blockify_kv: unknown flag bit, a null K pool, a misaligned V, no frames
    assert L.pbsa_blockify_kv(gp, fake, fake, 3, fake, None, 100, None, fake, fake, 100, 2, fake, None) == 1
    assert L.pbsa_blockify_kv(gp, fake, fake, 3, fake, None, 100, None, None, fake, 100, 0, fake, None) == 1
    assert L.pbsa_blockify_kv(gp, fake, ctypes.c_void_p(0x10004), 3, fake, None, 100, None, fake, fake, 100, 0,
                              fake, None) == 1
    assert L.pbsa_blockify_kv(gp, fake, fake, 0, fake, None, 100, None, fake, fake, 100, 0, fake, None) == 1
    # too few slots for the frames when no destination list is given (3 frames = 72 blocks)
    assert L.pbsa_blockify_kv(gp, fake, fake, 3, fake, None, 71, None, fake, fake, 71, 0, fake, None) == 1
    # plan: unknown flag bit, gamma outside [0, 1], capacity above the pool, no workspace
    args = lambda flags=0, gamma=0.9, cap=96, ws=fake: (  # noqa: E731
        gp, fake, 72, fake, 312, fake, fake, cap, 24, fake, fake, 72, ctypes.c_float(gamma), None, None,
        flags, ws, None)
    assert L.pbsa_memory_update_plan(*args(flags=4)) == 1
    assert L.pbsa_memory_update_plan(*args(gamma=1.5)) == 1
    assert L.pbsa_memory_update_plan(*args(cap=400)) == 1
    assert L.pbsa_memory_update_plan(*args(ws=None)) == 1
    assert L.pbsa_memory_update_plan(gp, fake, 72, fake, 312, fake, fake, 2000, 24, fake, fake, 100,
                                     ctypes.c_float(0.9), None, None, 0, fake, None) == 1   # capacity > pool
    big = P.make_geom(12, 128, 32, 48, 8, 8, 128 ** -0.5, "bf16")
    assert L.pbsa_memory_update_plan(ctypes.byref(big), fake, 72, fake, 4000, fake, fake, 96, 24, fake, fake,
                                     2000, ctypes.c_float(0.9), None, None, 0, fake, None) == 2   # pool > 2048
    # apply: null pools, capacity above the pool, a misaligned K pool
    assert L.pbsa_memory_update_apply(gp, fake, None, fake, 312, 96, 72, fake, None) == 1
    assert L.pbsa_memory_update_apply(gp, fake, fake, fake, 50, 96, 72, fake, None) == 1
    assert L.pbsa_memory_update_apply(gp, fake, ctypes.c_void_p(0x10008), fake, 312, 96, 72, fake, None) == 1

