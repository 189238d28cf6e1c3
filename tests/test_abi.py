"""The C-ABI library loads and exports every entry point that include/pbsa.h declares;
host-side argument checks answer without a GPU."""
import ctypes
import os
import re

import pytest
import torch

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


# The next two tests hand the library fake (never dereferenced) device pointers; every case must
# fail in a host-side check.  They never run where a GPU is visible, so that a case which slipped
# past the checks could not launch a kernel on a real device.
host_only = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device pointers: CPU-only check")


@host_only
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



@host_only
def test_every_entry_point_checks_its_arguments_on_the_host(lib):
    """Each entry point's host-side rules, case by case, with the status they must return
    (1 = PBSA_ERR_INVALID_ARG, 2 = PBSA_ERR_UNSUPPORTED).  Every case fails before any CUDA
    call; the aligned fake pointers are never dereferenced."""
    L = _lib.load()
    f, m = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10004)   # aligned / misaligned
    F = ctypes.c_float
    g = P.make_geom(12, 128, 32, 48, 8, 8, 128 ** -0.5, "bf16")
    g32 = P.make_geom(12, 128, 32, 48, 8, 8, 128 ** -0.5, "f32")
    gp, gp32 = ctypes.byref(g), ctypes.byref(g32)

    # geometry (through pbsa_blockify): invalid shapes are 1, unbuilt ones 2
    def blk(geom):
        return L.pbsa_blockify(ctypes.byref(geom), f, 1, f, 24, None, None, 0, f, None)
    bad = {
        "scale 0": (P.make_geom(12, 128, 32, 48, 8, 8, 0.0, "bf16"), 1),
        "frame not a multiple of the tile": (P.make_geom(12, 128, 30, 48, 8, 8, 0.1, "bf16"), 1),
        "unknown dtype": (P.make_geom(12, 128, 32, 48, 8, 8, 0.1, 7), 1),
        "no heads": (P.make_geom(0, 128, 32, 48, 8, 8, 0.1, "bf16"), 1),
        "bf16 with d = 32": (P.make_geom(12, 32, 32, 48, 8, 8, 0.1, "bf16"), 2),
        "more than 4096 heads": (P.make_geom(4097, 128, 32, 48, 8, 8, 0.1, "bf16"), 2),
        "frame above 2^24 tokens": (P.make_geom(1, 128, 8192, 4096, 8, 8, 0.1, "bf16"), 2),
    }
    for what, (geom, want) in bad.items():
        assert blk(geom) == want, what
        assert L.pbsa_workspace_bytes(ctypes.byref(geom), 8, 8) == 0, what
        assert L.pbsa_bwd_workspace_bytes(ctypes.byref(geom), 1, 8, 8) == 0, what
    assert L.pbsa_bwd_workspace_bytes(gp, 0, 8, 8) == 0
    # the backward keeps one 8 KB bf16 dS tile per (head, query block, list entry): 12 heads,
    # 24 blocks per frame, 8 more entries per row
    ws8, ws16 = L.pbsa_bwd_workspace_bytes(gp, 1, 8, 8), L.pbsa_bwd_workspace_bytes(gp, 1, 8, 16)
    assert ws16 - ws8 >= 12 * 24 * 8 * 8192

    # score + top-k: gp, q_reps, nq, k_reps, pool, cand_slot, cand_gid, ncand, k, prefix_slot,
    # prefix_cnt, prefix_ld, out_slot, out_cnt, out_ld, out_score, ws, stream
    def ss(nq=72, ncand=144, cs=f, cg=f, k=32, ps=f, pc=f, pld=96, out_ld=128, q=f):
        return L.pbsa_score_select(gp, q, nq, f, 400, cs, cg, ncand, k, ps, pc, pld, f, f, out_ld, None, f, None)
    assert ss(nq=0) == 1
    assert ss(cs=None) == 1
    assert ss(ps=None) == 1                   # a count without its list
    assert ss(out_ld=127) == 1                # no room for prefix + k
    assert ss(ncand=1025) == 2
    assert ss(q=m) == 1

    # general selection: ..., k, top_frames, n_recent, prefix_slot, prefix_cnt, prefix_ld,
    # suffix_slot, suffix_n, out_slot, out_cnt, out_ld, out_score, ws, stream
    def sx(ncand=144, top=-1, recent=1, suffix=None, sn=0, out_ld=128):
        return L.pbsa_blockify_select_ex(gp, f, 3, f, f, 400, f, f, ncand, 32, top, recent, f, f, 96, suffix, sn,
                                         f, f, out_ld, None, f, None)
    assert sx(sn=4) == 1                      # suffix count without its list
    assert sx(top=2, ncand=100) == 1          # frame-level selection needs whole frames
    assert sx(top=2, recent=-1) == 1
    assert sx(suffix=f, sn=4, out_ld=131) == 1
    assert sx(ncand=24 * 50) == 2
    assert L.pbsa_blockify_hsa_select(gp, f, 3, f, f, 400, f, f, 144, -1, 1, 32, f, f, 96, f, f, 128, None, f,
                                      None) == 1

    # trainable-path lists: gp, q, q_frames, q_reps, k_reps, pool, seq_frames, chunk_frames, sink_frames,
    # k, out_slot, out_cnt, out_ld, out_score, ws, stream (18 frames = 2 sequences of 9, 432 blocks)
    def ts(qf=18, pool=432, seq=9, chunk=3, sink=1, k=16, out_ld=112, q=f):
        return L.pbsa_blockify_train_select(gp, q, qf, f, f, pool, seq, chunk, sink, k, f, f, out_ld, None, f, None)
    assert ts(qf=17) == 1                     # not a whole number of sequences
    assert ts(pool=431) == 1                  # slot = block id needs every block in the pool
    assert ts(sink=4) == 1                    # sinks beyond the first chunk
    assert ts(sink=-1) == 1
    assert ts(out_ld=111) == 1                # 24 sinks + 16 + 72 own
    assert ts(k=-1) == 1
    assert ts(q=m) == 1
    assert ts(qf=48, seq=48, pool=1152) == 2  # last chunk: 44 earlier non-sink frames = 1056 candidates

    # attention: gp, q, q_frames, k_pool, v_pool, pool, kv_slot, kv_cnt, kv_ld, o, lse, ws, stream
    def at(geom=gp, qf=3, pool=400, ld=128, o=f):
        return L.pbsa_attend(geom, f, qf, f, f, pool, f, f, ld, o, None, f, None)
    assert at(qf=0) == 1
    assert at(o=m) == 1
    assert at(pool=(1 << 31) // (12 * 64) + 1) == 1   # pool rows overflow 31 bits
    assert at(ld=513) == 2                              # the bf16 kernel merges two lists of <= 512
    assert at(geom=gp32, ld=4097) == 2

    # backward: ..., kv_ld, o, d_o, lse, dq, dk_pool, dv_pool, ws, stream
    def bw(geom=gp, qf=3, ld=128, ws=f, dq=f):
        return L.pbsa_attend_bwd(geom, f, qf, f, f, 400, f, f, ld, f, f, f, dq, f, f, ws, None)
    assert bw(ws=None) == 1
    assert bw(dq=m) == 1
    assert bw(ld=513) == 2
    assert bw(qf=22) == 2                     # 528 query blocks
    assert bw(geom=gp32) == 2

    # memory update: gp, q_reps, nq, k_reps, k_pool, v_pool, pool, slot_gid, slot_ema, capacity,
    # n_sink_gid, cand_slot, cand_gid, ncand, gamma, p_list, p_cnt, ws, stream
    def mu(gamma=0.9, cap=96, ncand=72, cs=f, pool=400):
        return L.pbsa_memory_update(gp, f, 72, f, f, f, pool, f, f, cap, 24, cs, f, ncand, F(gamma), None, None,
                                    f, None)
    assert mu(gamma=-0.1) == 1
    assert mu(gamma=float("nan")) == 1
    assert mu(cap=401) == 1                   # capacity above the pool
    assert mu(cs=None) == 1
    assert mu(ncand=1953, pool=4000) == 2     # 96 + 1953 entries > 2048

    # the scratch-free update: same scalars, and pools whose workspace exceeds its 4 MiB scratch
    def na(nq=72, ncand=72):
        return L.pbsa_memory_update_noalloc(gp, f, nq, f, f, f, 4000, f, f, 96, 24, f, f, ncand, F(0.9), None, None,
                                            None)
    assert na(nq=0) == 1
    assert na(nq=4000, ncand=1900) == 2

    # bounded-wait self test and the error word
    assert L.pbsa_selftest_wait_timeout(None, 1000, None) == 1
    assert L.pbsa_selftest_wait_timeout(f, 0, None) == 1
    assert L.pbsa_selftest_wait_timeout(f, 2_000_000, None) == 1
    assert L.pbsa_get_device_error(None, None) == 1
