"""Thin ctypes binding of libpbsa.so: argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but
check tensor placement/dtype, take device pointers and the current CUDA stream, and
raise ``PBSAError`` on a non-OK status.  All computation happens in the library's CUDA
kernels; there is no fallback of any kind -- if the library is missing or was not built,
``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpbsa.so")

PBSA_F32, PBSA_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "device wait timed out", 5: "index out of range on the device"}


class PBSAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)} (status {code})")
        self.code = code


class Geom(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("frame_h", ctypes.c_int),
                ("frame_w", ctypes.c_int), ("tile_h", ctypes.c_int), ("tile_w", ctypes.c_int),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int)]

    @property
    def bpf(self) -> int:
        return (self.frame_h // self.tile_h) * (self.frame_w // self.tile_w)

    @property
    def tpf(self) -> int:
        return self.frame_h * self.frame_w


def make_geom(heads, head_dim, frame_h, frame_w, tile_h, tile_w, scale, dtype) -> Geom:
    dt = dtype if isinstance(dtype, int) else (PBSA_BF16 if dtype in ("bf16", torch.bfloat16) else PBSA_F32)
    return Geom(heads, head_dim, frame_h, frame_w, tile_h, tile_w, float(scale), dt)


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "pbsa_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Geom), _I, _I]),
    "pbsa_blockify": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _I, _P, _P, _I, _P, _P]),
    "pbsa_blockify_kv": (_I, [ctypes.POINTER(Geom), _P, _P, _I, _P, _P, _I, _P, _P, _P, _I, _I, _P, _P]),
    "pbsa_score_select": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _I, _P, _P, _I, _I, _P, _P, _I,
                               _P, _P, _I, _P, _P, _P]),
    "pbsa_blockify_score_select": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _P, _P, _I, _I, _P,
                                        _P, _I, _P, _P, _I, _P, _P, _P]),
    "pbsa_blockify_hsa_select": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I,
                                      _P, _P, _I, _P, _P, _I, _P, _P, _P]),
    "pbsa_blockify_select_ex": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I,
                                     _P, _P, _I, _P, _I, _P, _P, _I, _P, _P, _P]),
    "pbsa_blockify_train_select": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I,
                                        _P, _P, _P]),
    "pbsa_attend": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P]),
    "pbsa_memory_update": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _P, _I, _P, _P, _I, _I, _P,
                                _P, _I, ctypes.c_float, _P, _P, _P, _P]),
    "pbsa_memory_update_plan": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _I, _P, _P, _I, _I, _P, _P, _I,
                                     ctypes.c_float, _P, _P, _I, _P, _P]),
    "pbsa_memory_update_apply": (_I, [ctypes.POINTER(Geom), _P, _P, _P, _I, _I, _I, _P, _P]),
    "pbsa_memory_update_noalloc": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _P, _I, _P, _P, _I, _I,
                                        _P, _P, _I, ctypes.c_float, _P, _P, _P]),
    "pbsa_memory_update_noalloc_error": (_I, [_P]),
    "pbsa_get_device_error": (_I, [_P, _P]),
    "pbsa_selftest_wait_timeout": (_I, [_P, ctypes.c_uint, _P]),
    "pbsa_status_string": (ctypes.c_char_p, [_I]),
    "pbsa_bwd_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Geom), _I, _I, _I]),
    "pbsa_attend_bwd": (_I, [ctypes.POINTER(Geom), _P, _I, _P, _P, _I, _P, _P, _I, _P, _P, _P,
                             _P, _P, _P, _P, _P]),
}
OPTIONAL = {}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpbsa.so (raises if it is absent: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libpbsa.so not found at {path}; build it with "
                           "`python -m block_sparse_attention_pbsa_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in {**_SIGS, **OPTIONAL}.items():
        if not hasattr(lib, name):
            if name in _SIGS:
                raise RuntimeError(f"{path} does not export {name}")
            continue
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise PBSAError(fn, code)


def _tok_dtype(g: Geom):
    return torch.bfloat16 if g.dtype == PBSA_BF16 else torch.float32


def pbsa_workspace_bytes(g: Geom, max_q_blocks: int, max_pool_entries: int) -> int:
    return int(load().pbsa_workspace_bytes(ctypes.byref(g), max_q_blocks, max_pool_entries))


def pbsa_blockify(g: Geom, x, n_frames, reps, rep_slots, dst_slot=None, pool=None, pool_slots=0,
                  ws=None, stream=None):
    _check("pbsa_blockify", load().pbsa_blockify(
        ctypes.byref(g), _ptr(x, _tok_dtype(g), "x"), n_frames, _ptr(reps, torch.float32, "reps"),
        rep_slots, _ptr(dst_slot, torch.int32, "dst_slot"), _ptr(pool, _tok_dtype(g), "pool"),
        pool_slots, _ptr(ws, None, "ws"), _stream(stream)))


PBSA_OVERLAP_PREVIOUS = 1


def pbsa_blockify_kv(g: Geom, k, v, n_frames, k_reps, v_reps, rep_slots, dst_slot, k_pool, v_pool,
                     pool_slots, flags=0, ws=None, stream=None):
    _check("pbsa_blockify_kv", load().pbsa_blockify_kv(
        ctypes.byref(g), _ptr(k, _tok_dtype(g), "k"), _ptr(v, _tok_dtype(g), "v"), n_frames,
        _ptr(k_reps, torch.float32, "k_reps"), _ptr(v_reps, torch.float32, "v_reps"), rep_slots,
        _ptr(dst_slot, torch.int32, "dst_slot"), _ptr(k_pool, _tok_dtype(g), "k_pool"),
        _ptr(v_pool, _tok_dtype(g), "v_pool"), pool_slots, flags, _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_score_select(g: Geom, q_reps, nq, k_reps, pool_slots, cand_slot, cand_gid, ncand, k,
                      prefix_slot, prefix_cnt, prefix_ld, out_slot, out_cnt, out_ld,
                      out_score=None, ws=None, stream=None):
    _check("pbsa_score_select", load().pbsa_score_select(
        ctypes.byref(g), _ptr(q_reps, torch.float32, "q_reps"), nq,
        _ptr(k_reps, torch.float32, "k_reps"), pool_slots, _ptr(cand_slot, torch.int32, "cand_slot"),
        _ptr(cand_gid, torch.int32, "cand_gid"), ncand, k, _ptr(prefix_slot, torch.int32, "prefix_slot"),
        _ptr(prefix_cnt, torch.int32, "prefix_cnt"), prefix_ld, _ptr(out_slot, torch.int32, "out_slot"),
        _ptr(out_cnt, torch.int32, "out_cnt"), out_ld, _ptr(out_score, torch.float32, "out_score"),
        _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_blockify_score_select(g: Geom, q, q_frames, q_reps, k_reps, pool_slots, cand_slot, cand_gid,
                               ncand, k, prefix_slot, prefix_cnt, prefix_ld, out_slot, out_cnt, out_ld,
                               out_score=None, ws=None, stream=None):
    _check("pbsa_blockify_score_select", load().pbsa_blockify_score_select(
        ctypes.byref(g), _ptr(q, _tok_dtype(g), "q"), q_frames, _ptr(q_reps, torch.float32, "q_reps"),
        _ptr(k_reps, torch.float32, "k_reps"), pool_slots, _ptr(cand_slot, torch.int32, "cand_slot"),
        _ptr(cand_gid, torch.int32, "cand_gid"), ncand, k, _ptr(prefix_slot, torch.int32, "prefix_slot"),
        _ptr(prefix_cnt, torch.int32, "prefix_cnt"), prefix_ld, _ptr(out_slot, torch.int32, "out_slot"),
        _ptr(out_cnt, torch.int32, "out_cnt"), out_ld, _ptr(out_score, torch.float32, "out_score"),
        _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_blockify_hsa_select(g: Geom, q, q_frames, q_reps, k_reps, pool_slots, cand_slot, cand_gid,
                             ncand, top_frames, n_recent_frames, k, prefix_slot, prefix_cnt, prefix_ld,
                             out_slot, out_cnt, out_ld, out_score=None, ws=None, stream=None):
    _check("pbsa_blockify_hsa_select", load().pbsa_blockify_hsa_select(
        ctypes.byref(g), _ptr(q, _tok_dtype(g), "q"), q_frames, _ptr(q_reps, torch.float32, "q_reps"),
        _ptr(k_reps, torch.float32, "k_reps"), pool_slots, _ptr(cand_slot, torch.int32, "cand_slot"),
        _ptr(cand_gid, torch.int32, "cand_gid"), ncand, top_frames, n_recent_frames, k,
        _ptr(prefix_slot, torch.int32, "prefix_slot"), _ptr(prefix_cnt, torch.int32, "prefix_cnt"),
        prefix_ld, _ptr(out_slot, torch.int32, "out_slot"), _ptr(out_cnt, torch.int32, "out_cnt"), out_ld,
        _ptr(out_score, torch.float32, "out_score"), _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_blockify_select_ex(g: Geom, q, q_frames, q_reps, k_reps, pool_slots, cand_slot, cand_gid, ncand,
                            k, top_frames, n_recent_frames, prefix_slot, prefix_cnt, prefix_ld,
                            suffix_slot, suffix_n, out_slot, out_cnt, out_ld, out_score=None, ws=None,
                            stream=None):
    _check("pbsa_blockify_select_ex", load().pbsa_blockify_select_ex(
        ctypes.byref(g), _ptr(q, _tok_dtype(g), "q"), q_frames, _ptr(q_reps, torch.float32, "q_reps"),
        _ptr(k_reps, torch.float32, "k_reps"), pool_slots, _ptr(cand_slot, torch.int32, "cand_slot"),
        _ptr(cand_gid, torch.int32, "cand_gid"), ncand, k, top_frames, n_recent_frames,
        _ptr(prefix_slot, torch.int32, "prefix_slot"), _ptr(prefix_cnt, torch.int32, "prefix_cnt"),
        prefix_ld, _ptr(suffix_slot, torch.int32, "suffix_slot"), suffix_n,
        _ptr(out_slot, torch.int32, "out_slot"), _ptr(out_cnt, torch.int32, "out_cnt"), out_ld,
        _ptr(out_score, torch.float32, "out_score"), _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_blockify_train_select(g: Geom, q, q_frames, q_reps, k_reps, pool_slots, seq_frames, chunk_frames,
                               sink_frames, k, out_slot, out_cnt, out_ld, out_score=None, ws=None, stream=None):
    _check("pbsa_blockify_train_select", load().pbsa_blockify_train_select(
        ctypes.byref(g), _ptr(q, _tok_dtype(g), "q"), q_frames, _ptr(q_reps, torch.float32, "q_reps"),
        _ptr(k_reps, torch.float32, "k_reps"), pool_slots, seq_frames, chunk_frames, sink_frames, k,
        _ptr(out_slot, torch.int32, "out_slot"), _ptr(out_cnt, torch.int32, "out_cnt"), out_ld,
        _ptr(out_score, torch.float32, "out_score"), _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_attend(g: Geom, q, q_frames, k_pool, v_pool, pool_slots, kv_slot, kv_cnt, kv_ld, o,
                lse=None, ws=None, stream=None):
    dt = _tok_dtype(g)
    _check("pbsa_attend", load().pbsa_attend(
        ctypes.byref(g), _ptr(q, dt, "q"), q_frames, _ptr(k_pool, dt, "k_pool"),
        _ptr(v_pool, dt, "v_pool"), pool_slots, _ptr(kv_slot, torch.int32, "kv_slot"),
        _ptr(kv_cnt, torch.int32, "kv_cnt"), kv_ld, _ptr(o, dt, "o"), _ptr(lse, torch.float32, "lse"),
        _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_memory_update(g: Geom, q_reps, nq, k_reps, k_pool, v_pool, pool_slots, slot_gid, slot_ema,
                       capacity, n_sink_gid, cand_slot, cand_gid, ncand, gamma, p_list=None,
                       p_cnt=None, ws=None, stream=None):
    dt = _tok_dtype(g)
    _check("pbsa_memory_update", load().pbsa_memory_update(
        ctypes.byref(g), _ptr(q_reps, torch.float32, "q_reps"), nq, _ptr(k_reps, torch.float32, "k_reps"),
        _ptr(k_pool, dt, "k_pool"), _ptr(v_pool, dt, "v_pool"), pool_slots,
        _ptr(slot_gid, torch.int32, "slot_gid"), _ptr(slot_ema, torch.float32, "slot_ema"), capacity,
        n_sink_gid, _ptr(cand_slot, torch.int32, "cand_slot"), _ptr(cand_gid, torch.int32, "cand_gid"),
        ncand, float(gamma), _ptr(p_list, torch.int32, "p_list"), _ptr(p_cnt, torch.int32, "p_cnt"),
        _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_memory_update_plan(g: Geom, q_reps, nq, k_reps, pool_slots, slot_gid, slot_ema, capacity, n_sink_gid,
                            cand_slot, cand_gid, ncand, gamma, p_list=None, p_cnt=None, flags=0, ws=None,
                            stream=None):
    _check("pbsa_memory_update_plan", load().pbsa_memory_update_plan(
        ctypes.byref(g), _ptr(q_reps, torch.float32, "q_reps"), nq, _ptr(k_reps, torch.float32, "k_reps"),
        pool_slots, _ptr(slot_gid, torch.int32, "slot_gid"), _ptr(slot_ema, torch.float32, "slot_ema"),
        capacity, n_sink_gid, _ptr(cand_slot, torch.int32, "cand_slot"), _ptr(cand_gid, torch.int32, "cand_gid"),
        ncand, float(gamma), _ptr(p_list, torch.int32, "p_list"), _ptr(p_cnt, torch.int32, "p_cnt"), flags,
        _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_memory_update_apply(g: Geom, k_reps, k_pool, v_pool, pool_slots, capacity, ncand, ws=None, stream=None):
    _check("pbsa_memory_update_apply", load().pbsa_memory_update_apply(
        ctypes.byref(g), _ptr(k_reps, torch.float32, "k_reps"), _ptr(k_pool, _tok_dtype(g), "k_pool"),
        _ptr(v_pool, _tok_dtype(g), "v_pool"), pool_slots, capacity, ncand, _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_memory_update_noalloc(g: Geom, q_reps, nq, k_reps, k_pool, v_pool, pool_slots, slot_gid,
                               slot_ema, capacity, n_sink_gid, cand_slot, cand_gid, ncand, gamma,
                               p_list=None, p_cnt=None, stream=None):
    """pbsa_memory_update with the library's built-in scratch instead of a workspace."""
    dt = _tok_dtype(g)
    _check("pbsa_memory_update_noalloc", load().pbsa_memory_update_noalloc(
        ctypes.byref(g), _ptr(q_reps, torch.float32, "q_reps"), nq, _ptr(k_reps, torch.float32, "k_reps"),
        _ptr(k_pool, dt, "k_pool"), _ptr(v_pool, dt, "v_pool"), pool_slots,
        _ptr(slot_gid, torch.int32, "slot_gid"), _ptr(slot_ema, torch.float32, "slot_ema"), capacity,
        n_sink_gid, _ptr(cand_slot, torch.int32, "cand_slot"), _ptr(cand_gid, torch.int32, "cand_gid"),
        ncand, float(gamma), _ptr(p_list, torch.int32, "p_list"), _ptr(p_cnt, torch.int32, "p_cnt"),
        _stream(stream)))


def pbsa_memory_update_noalloc_error(stream=None) -> int:
    """Read and clear the error word of pbsa_memory_update_noalloc's built-in scratch."""
    return int(load().pbsa_memory_update_noalloc_error(_stream(stream)))


def pbsa_bwd_workspace_bytes(g: Geom, q_frames: int, pool_slots: int, kv_ld: int) -> int:
    return int(load().pbsa_bwd_workspace_bytes(ctypes.byref(g), q_frames, pool_slots, kv_ld))


def pbsa_attend_bwd(g: Geom, q, q_frames, k_pool, v_pool, pool_slots, kv_slot, kv_cnt, kv_ld, o,
                    d_o, lse, dq, dk_pool, dv_pool, ws, stream=None):
    dt = _tok_dtype(g)
    _check("pbsa_attend_bwd", load().pbsa_attend_bwd(
        ctypes.byref(g), _ptr(q, dt, "q"), q_frames, _ptr(k_pool, dt, "k_pool"), _ptr(v_pool, dt, "v_pool"),
        pool_slots, _ptr(kv_slot, torch.int32, "kv_slot"), _ptr(kv_cnt, torch.int32, "kv_cnt"), kv_ld,
        _ptr(o, dt, "o"), _ptr(d_o, dt, "d_o"), _ptr(lse, torch.float32, "lse"), _ptr(dq, dt, "dq"),
        _ptr(dk_pool, dt, "dk_pool"), _ptr(dv_pool, dt, "dv_pool"), _ptr(ws, None, "ws"), _stream(stream)))


def pbsa_selftest_wait_timeout(ws, limit_us: int, stream=None):
    _check("pbsa_selftest_wait_timeout", load().pbsa_selftest_wait_timeout(_ptr(ws, None, "ws"), int(limit_us),
                                                                           _stream(stream)))


def pbsa_get_device_error(ws, stream=None) -> int:
    return int(load().pbsa_get_device_error(_ptr(ws, None, "ws"), _stream(stream)))


def pbsa_status_string(code: int) -> str:
    return load().pbsa_status_string(code).decode()
