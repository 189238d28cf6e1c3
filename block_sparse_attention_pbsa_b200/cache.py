"""Per-layer PBSA KV cache in HBM and its host-side bookkeeping.

Sparse Forcing (gist.science English page, 2.B "Structured Memory Decomposition"): the KV
cache of a layer is the persistent memory P_t (capacity C: the sink blocks of frame 0
plus the best-scored older blocks, shared by all diffusion steps of a chunk) and the
local window L_t (the last W frames, frame 0 excluded).  This module owns the device
buffers of one layer and sequences the C-ABI calls; every number is computed by the
library's kernels.

Pool layout (slots of 64 tokens, per head): ``[0, C)`` persistent slots, then a ring of
``W + chunk_frames`` frames (frame f -> ring position f mod (W + chunk_frames)), then an
optional staging area used only by ``prefill``.  The ring holds the window plus the
chunk being committed, so the blocks leaving the window are still intact while the
memory update scores and copies them.
"""
from __future__ import annotations

import collections
import dataclasses

import torch

from . import _lib as L


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    heads: int
    head_dim: int
    frame_h: int
    frame_w: int
    tile_h: int
    tile_w: int
    capacity: int
    window_frames: int
    chunk_frames: int
    topk: int
    gamma: float
    dtype: str = "bf16"           # "bf16" or "f32"
    staging_blocks: int = 0       # extra slots for prefill (history beyond the ring)
    scale: float | None = None
    # local selection policy: -1 = flat top-k over the window; >= 0 = two-level (hierarchical)
    # selection: the hsa_recent latest window frames + the hsa_top_frames best other frames,
    # then the top-k blocks of those frames
    hsa_top_frames: int = -1
    hsa_recent: int = 1
    # own-chunk variant: every query block also attends the chunk's own blocks, written into
    # their ring positions at the current step before the selection (the chunk-wise
    # self-attention of the trainable path, applied at inference)
    own_chunk: bool = False
    # largest local top-k a per-chunk schedule may set (set_topk); -1: topk
    max_topk: int = -1

    @property
    def bpf(self) -> int:
        return (self.frame_h // self.tile_h) * (self.frame_w // self.tile_w)

    @property
    def tpf(self) -> int:
        return self.frame_h * self.frame_w


class PBSALayerCache:
    def __init__(self, cfg: LayerConfig, device="cuda"):
        self.cfg = cfg
        self.device = torch.device(device)
        self.geom = L.make_geom(cfg.heads, cfg.head_dim, cfg.frame_h, cfg.frame_w, cfg.tile_h,
                                cfg.tile_w, cfg.scale or cfg.head_dim ** -0.5, cfg.dtype)
        self.tdtype = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        H, d, bpf, C = cfg.heads, cfg.head_dim, cfg.bpf, cfg.capacity
        self.ring_frames = cfg.window_frames + cfg.chunk_frames
        self.ring_base = C
        self.stage_base = C + self.ring_frames * bpf
        self.pool_slots = self.stage_base + cfg.staging_blocks
        dev = self.device
        self.k_pool = torch.zeros((H, self.pool_slots, 64, d), dtype=self.tdtype, device=dev)
        self.v_pool = torch.zeros_like(self.k_pool)
        self.k_reps = torch.zeros((H, self.pool_slots, d), dtype=torch.float32, device=dev)
        self.slot_gid = torch.full((H, C), -1, dtype=torch.int32, device=dev)
        self.slot_ema = torch.zeros((H, C), dtype=torch.float32, device=dev)
        self.p_list = torch.zeros((H, C), dtype=torch.int32, device=dev)
        self.p_cnt = torch.zeros((H,), dtype=torch.int32, device=dev)
        nq = cfg.chunk_frames * bpf
        self.max_pool_entries = C + max(self.ring_frames * bpf, cfg.staging_blocks)
        self.ws = torch.zeros(L.pbsa_workspace_bytes(self.geom, nq, self.max_pool_entries),
                              dtype=torch.uint8, device=dev)
        self.topk = cfg.topk
        self.max_topk = max(cfg.topk, cfg.max_topk)
        self.kv_ld = C + max(self.max_topk, 0) + (nq if cfg.own_chunk else 0)
        self.kv_ld_own = max(self.kv_ld, nq)
        # flat buffers, viewed per call as [H, nq, ...] for chunks of up to chunk_frames frames
        self._q_reps_buf = torch.zeros(H * nq * d, dtype=torch.float32, device=dev)
        self._kv_slot_buf = torch.zeros(H * nq * self.kv_ld_own, dtype=torch.int32, device=dev)
        self._kv_cnt_buf = torch.zeros(H * nq, dtype=torch.int32, device=dev)
        self.q_reps = self._q_reps_buf.view(H, nq, d)
        self.kv_slot = self._kv_slot_buf.view(H, nq, self.kv_ld_own)
        self.kv_cnt = self._kv_cnt_buf.view(H, nq)
        self.hist = 0
        self._cand = None      # (cand_slot, cand_gid, n) of the current local window
        self._dst_cache = {}

    # ------------------------------------------------------------------ layout helpers
    def ring_slot(self, frame: int, tile: int) -> int:
        return self.ring_base + (frame % self.ring_frames) * self.cfg.bpf + tile

    def window_frames(self, hist: int | None = None) -> list[int]:
        h = self.hist if hist is None else hist
        return list(range(max(1, h - self.cfg.window_frames), h))

    def _ints(self, rows) -> torch.Tensor:
        t = torch.tensor(rows, dtype=torch.int32).pin_memory()
        return t.to(self.device, non_blocking=True)

    # Candidate lists depend only on the ring geometry and the frame schedule, which every
    # layer of a model shares: they are built once per (device, heads, ring, list) and reused by
    # the layers.  Their gids change with every chunk, so only the most recent lists are kept
    # (the device memory they hold stays bounded over a rollout of any length).
    _LIST_MEMO: "collections.OrderedDict" = collections.OrderedDict()
    _LIST_MEMO_MAX = 8

    def _list_pair(self, pairs) -> tuple[torch.Tensor, torch.Tensor]:
        """Device tensors [H, n] of the slots and gids of ``pairs`` (a list of (slot, gid))."""
        H = self.cfg.heads
        memo = PBSALayerCache._LIST_MEMO
        key = (str(self.device), H, self.ring_frames, self.cfg.bpf, self.ring_base, tuple(pairs))
        hit = memo.get(key)
        if hit is None:
            n = len(pairs)
            hit = (self._ints([[s for s, _ in pairs]] * H).view(H, n),
                   self._ints([[g for _, g in pairs]] * H).view(H, n))
            memo[key] = hit
            while len(memo) > PBSALayerCache._LIST_MEMO_MAX:
                memo.popitem(last=False)
        else:
            memo.move_to_end(key)
        return hit

    def _frames_dst(self, first: int, n: int) -> torch.Tensor:
        key = (first % self.ring_frames, n)
        if key not in self._dst_cache:
            bpf = self.cfg.bpf
            self._dst_cache[key] = self._ints(
                [self.ring_slot(first + f, t) for f in range(n) for t in range(bpf)])
        return self._dst_cache[key]

    def _refresh_window(self):
        bpf, H = self.cfg.bpf, self.cfg.heads
        frames = self.window_frames()
        pairs = [(self.ring_slot(f, t), f * bpf + t) for f in frames for t in range(bpf)]
        if not pairs:
            self._cand = (None, None, 0)
            return
        cs, cg = self._list_pair(pairs)
        self._cand = (cs, cg, len(pairs))

    @property
    def kv_bytes(self) -> int:
        """Bytes of K and V held for the persistent memory and the ring (prefill staging excluded)."""
        c = self.cfg
        slots = c.capacity + self.ring_frames * c.bpf
        return 2 * c.heads * slots * 64 * c.head_dim * self.k_pool.element_size()

    # ------------------------------------------------------------------ the hot path
    def frames_of(self, x: torch.Tensor) -> int:
        n, rem = divmod(x.shape[0], self.cfg.tpf)
        if rem or not 0 < n <= self.cfg.chunk_frames:
            raise ValueError(f"a chunk holds 1..{self.cfg.chunk_frames} whole frames, got {x.shape[0]} tokens")
        return n

    def query_reps(self, q: torch.Tensor, stream=None) -> torch.Tensor:
        """a1: representatives of the chunk's query blocks -> self.q_reps [H, nq, d]."""
        c = self.cfg
        nq = self.frames_of(q) * c.bpf
        self.q_reps = self._q_reps_buf[:c.heads * nq * c.head_dim].view(c.heads, nq, c.head_dim)
        L.pbsa_blockify(self.geom, q, nq // c.bpf, self.q_reps, nq, ws=self.ws, stream=stream)
        return self.q_reps

    def select(self, q_reps: torch.Tensor, stream=None):
        """a2: per query block, persistent slots + top-k local slots -> (kv_slot, kv_cnt, kv_ld)."""
        c = self.cfg
        nq = q_reps.shape[1]
        self.kv_slot = self._kv_slot_buf[:c.heads * nq * self.kv_ld_own].view(c.heads, nq, self.kv_ld_own)
        self.kv_cnt = self._kv_cnt_buf[:c.heads * nq].view(c.heads, nq)
        cs, cg, n = self._cand
        if n == 0:
            # no local window yet: persistent slots only (score_select with no candidates)
            L.pbsa_score_select(self.geom, q_reps, nq, self.k_reps, self.pool_slots, None, None, 0, 0,
                                self.p_list, self.p_cnt, c.capacity, self.kv_slot, self.kv_cnt,
                                self.kv_ld_own, ws=self.ws, stream=stream)
        else:
            L.pbsa_score_select(self.geom, q_reps, nq, self.k_reps, self.pool_slots, cs, cg, n, self.topk,
                                self.p_list, self.p_cnt, c.capacity, self.kv_slot, self.kv_cnt,
                                self.kv_ld_own, ws=self.ws, stream=stream)
        return self.kv_slot, self.kv_cnt, self.kv_ld_own

    def set_topk(self, k: int):
        """Local top-k of the following selections (a per-chunk schedule; at most max_topk)."""
        if not 0 <= k <= self.max_topk:
            raise ValueError(f"top-k must lie in [0, {self.max_topk}], got {k}")
        self.topk = int(k)

    def query_select(self, q: torch.Tensor, stream=None):
        """a1 + a2 in one launch: q_reps of the chunk and, per query block, persistent slots +
        top-k local slots -> (q_reps, kv_slot, kv_cnt, kv_ld)."""
        c = self.cfg
        nf = self.frames_of(q)
        nq = nf * c.bpf
        self.q_reps = self._q_reps_buf[:c.heads * nq * c.head_dim].view(c.heads, nq, c.head_dim)
        self.kv_slot = self._kv_slot_buf[:c.heads * nq * self.kv_ld_own].view(c.heads, nq, self.kv_ld_own)
        self.kv_cnt = self._kv_cnt_buf[:c.heads * nq].view(c.heads, nq)
        self._select_fused(q, nf, self.q_reps, self.kv_slot, self.kv_cnt, self.kv_ld_own, stream)
        return self.q_reps, self.kv_slot, self.kv_cnt, self.kv_ld_own

    def _select_fused(self, q, nf, q_reps, kv_slot, kv_cnt, kv_ld, stream=None):
        """The one-launch blockify + selection of the configured policy (and, for the own-chunk
        variant, the chunk's ring slots appended to every row)."""
        c = self.cfg
        cs, cg, n = self._cand
        top = c.hsa_top_frames if (c.hsa_top_frames >= 0 and n) else -1
        own = self._frames_dst(self.hist, nf) if c.own_chunk else None
        L.pbsa_blockify_select_ex(self.geom, q, nf, q_reps, self.k_reps, self.pool_slots, cs, cg, n,
                                  self.topk if n else 0, top, c.hsa_recent, self.p_list, self.p_cnt, c.capacity,
                                  own, own.numel() if own is not None else 0, kv_slot, kv_cnt, kv_ld,
                                  ws=self.ws, stream=stream)

    def attend(self, q, kv_slot, kv_cnt, kv_ld, o=None, lse=None, stream=None):
        """a3: fine attention over the listed slots."""
        if o is None:
            o = torch.empty_like(q)
        L.pbsa_attend(self.geom, q, self.frames_of(q), self.k_pool, self.v_pool, self.pool_slots,
                      kv_slot, kv_cnt, kv_ld, o, lse, ws=self.ws, stream=stream)
        return o

    def decode_step(self, q, k=None, v=None, o=None, lse=None, stream=None):
        """One denoising step of the current chunk: returns O (raster, like q).

        With an empty history the chunk attends its own blocks (``k``, ``v`` of this step,
        written to the chunk's ring positions); otherwise P_t + top-k of L_t.
        """
        if self._cand is None:
            self._refresh_window()
        if self.hist > 0:
            if self.cfg.own_chunk:
                if k is None or v is None:
                    raise ValueError("the own-chunk variant attends the chunk's blocks: pass its k and v")
                self._write_chunk(k, v, stream)
            _, kv_slot, kv_cnt, kv_ld = self.query_select(q, stream)
            return self.attend(q, kv_slot, kv_cnt, kv_ld, o, lse, stream)
        # empty history: the chunk attends its own blocks
        if k is None or v is None:
            raise ValueError("the first chunk attends its own blocks: pass its k and v")
        q_reps = self.query_reps(q, stream)
        self._write_chunk(k, v, stream)
        nq = q_reps.shape[1]
        own = self._ints([[self.ring_slot(b // self.cfg.bpf, b % self.cfg.bpf) for b in range(nq)]] * nq)
        kv_slot = torch.zeros((self.cfg.heads, nq, nq), dtype=torch.int32, device=self.device)
        kv_slot[:] = own.view(nq, nq)
        kv_cnt = torch.full((self.cfg.heads, nq), nq, dtype=torch.int32, device=self.device)
        return self.attend(q, kv_slot, kv_cnt, nq, o, lse, stream)

    def _write_chunk(self, k, v, stream=None, flags=0):
        n = self.frames_of(k)
        dst = self._frames_dst(self.hist, n)
        # K and V blocks in one launch; value representatives are not used by the method
        L.pbsa_blockify_kv(self.geom, k, v, n, self.k_reps, None, self.pool_slots, dst, self.k_pool,
                           self.v_pool, self.pool_slots, flags=flags, ws=self.ws, stream=stream)

    def commit(self, k, v, q_reps_last=None, stream=None, overlap=False, split=False):
        """a4: commit the finished chunk (its last-step K, V) and update the persistent memory.

        The chunk's blocks enter the ring; the frames that leave the window, and frame 0's
        sink blocks when frame 0 is in the chunk, are the candidates of the memory update,
        scored by the chunk's last-step query representatives.

        ``overlap``: the call directly follows this cache's last ``decode_step`` on the stream,
        with nothing launched in between.  The memory update's plan and the write of the chunk
        then run as programmatic dependents of that attend, on the SMs its last wave leaves idle,
        and the copies of promoted blocks follow it.  (A chunk whose own blocks were attended --
        the first chunk, the own-chunk variant -- takes the serial order: the write would
        overlap their reads.)  ``split``: the memory update as plan + apply without the overlap.
        """
        c = self.cfg
        bpf, H = c.bpf, c.heads
        q_reps_last = self.q_reps if q_reps_last is None else q_reps_last
        first, n = self.hist, self.frames_of(k)
        old_win = set(self.window_frames(first))
        new_hist = first + n
        new_win = set(self.window_frames(new_hist))
        entering = {f for f in range(first, new_hist) if f != 0}
        evicted = sorted((old_win | entering) - new_win)
        cand = [(self.ring_slot(f, t), f * bpf + t) for f in evicted for t in range(bpf)]
        if first == 0:
            cand = [(self.ring_slot(0, t), t) for t in range(bpf)] + cand
        if overlap and not (first == 0 or c.own_chunk):
            # the candidates are the frames leaving the window, never the chunk's own slots
            self._update(q_reps_last, cand, stream, split=True, plan_flags=L.PBSA_OVERLAP_PREVIOUS, apply=False)
            self._write_chunk(k, v, stream, flags=L.PBSA_OVERLAP_PREVIOUS)
            L.pbsa_memory_update_apply(self.geom, self.k_reps, self.k_pool, self.v_pool, self.pool_slots,
                                       c.capacity, len(cand), ws=self.ws, stream=stream)
        else:
            self._write_chunk(k, v, stream)
            self._update(q_reps_last, cand, stream, split=split or overlap)
        self.hist = new_hist
        self._refresh_window()

    def _update(self, q_reps, cand, stream=None, split=False, plan_flags=0, apply=True):
        c, H = self.cfg, self.cfg.heads
        ncand = len(cand)
        cs, cg = self._list_pair(cand) if ncand else (None, None)
        if not split:
            L.pbsa_memory_update(self.geom, q_reps, q_reps.shape[1], self.k_reps, self.k_pool, self.v_pool,
                                 self.pool_slots, self.slot_gid, self.slot_ema, c.capacity, c.bpf, cs, cg,
                                 ncand, c.gamma, self.p_list, self.p_cnt, ws=self.ws, stream=stream)
            return
        L.pbsa_memory_update_plan(self.geom, q_reps, q_reps.shape[1], self.k_reps, self.pool_slots, self.slot_gid,
                                  self.slot_ema, c.capacity, c.bpf, cs, cg, ncand, c.gamma, self.p_list, self.p_cnt,
                                  flags=plan_flags, ws=self.ws, stream=stream)
        if apply:
            L.pbsa_memory_update_apply(self.geom, self.k_reps, self.k_pool, self.v_pool, self.pool_slots,
                                       c.capacity, ncand, ws=self.ws, stream=stream)

    def prefill(self, k_hist, v_hist, hist_frames: int, q_reps, stream=None):
        """Load a history of ``hist_frames`` frames at once (single-step decode workloads).

        The sinks and every middle frame (older than the window) go to the staging area and
        one memory update with no prior EMA selects the persistent set among them, scored by
        ``q_reps``; the window frames go to their ring positions.
        """
        c = self.cfg
        bpf = c.bpf
        win = self.window_frames(hist_frames)
        middle = list(range(1, win[0] if win else hist_frames))
        staged = [0] + middle
        if len(staged) * bpf > c.staging_blocks:
            raise ValueError(f"prefill needs {len(staged) * bpf} staging blocks, have {c.staging_blocks}")
        dst = []
        for f in range(hist_frames):
            for t in range(bpf):
                dst.append(self.stage_base + staged.index(f) * bpf + t if f in staged else self.ring_slot(f, t))
        dst_t = self._ints(dst)
        L.pbsa_blockify_kv(self.geom, k_hist, v_hist, hist_frames, self.k_reps, None, self.pool_slots, dst_t,
                           self.k_pool, self.v_pool, self.pool_slots, ws=self.ws, stream=stream)
        cand = [(self.stage_base + i * bpf + t, f * bpf + t) for i, f in enumerate(staged) for t in range(bpf)]
        self._update(q_reps, cand, stream)
        self.hist = hist_frames
        self._refresh_window()

    # ------------------------------------------------------------------ checkpoint / resume
    _STATE = ("k_pool", "v_pool", "k_reps", "slot_gid", "slot_ema", "p_list", "p_cnt")

    def state_dict(self, device="cpu") -> dict:
        """Everything a rollout needs to continue from here: the pools, key representatives and
        slot tables (copied to ``device``), the number of committed frames and the local top-k.
        The ring holds the window, so a copy taken after a commit resumes the rollout exactly."""
        st = {name: getattr(self, name).to(device, copy=True) for name in self._STATE}
        st["hist"] = self.hist
        st["topk"] = self.topk
        st["config"] = dataclasses.asdict(self.cfg)
        return st

    def load_state_dict(self, st: dict):
        """Restore a ``state_dict`` taken from a cache of the same configuration."""
        if st.get("config") != dataclasses.asdict(self.cfg):
            raise ValueError("the state was taken from a cache of another configuration")
        for name in self._STATE:
            dst = getattr(self, name)
            if tuple(st[name].shape) != tuple(dst.shape) or st[name].dtype != dst.dtype:
                raise ValueError(f"{name}: shape or dtype does not match the cache")
            dst.copy_(st[name])
        self.hist = int(st["hist"])
        self.topk = int(st["topk"])
        self._refresh_window()

    # ------------------------------------------------------------------ inspection
    def persistent_gids(self) -> list[set[int]]:
        g = self.slot_gid.cpu()
        return [set(int(x) for x in row if x >= 0) for row in g]

    def slot_to_gid(self) -> dict[int, int]:
        """Map of ring/stage slots to global block ids for the current window (host bookkeeping)."""
        bpf = self.cfg.bpf
        return {self.ring_slot(f, t): f * bpf + t for f in self.window_frames() for t in range(bpf)}


class ChunkDecodeStep:
    """One chunk decode plus its commit, with every device-side index array prepared up front.

    ``run(q, k, v)`` issues only C-ABI launches on one stream -- blockify(Q), score+top-k,
    attend, blockify(K), blockify(V) into the chunk's ring positions, memory update (2
    kernels) -- with no host synchronisation or allocation, so it can be timed per kernel
    or captured in a CUDA graph.  It does not advance the cache's host bookkeeping: the same
    step can be replayed on a restored state (see ``snapshot``/``restore``).
    """

    def __init__(self, cache: PBSALayerCache, q_frames: int | None = None, fused_select: bool = True):
        c = cache.cfg
        if cache.hist == 0:
            # the first chunk attends its own blocks, and frame 0's blocks are candidates of its
            # update, which must then follow their commit: decode_step + commit cover that case
            raise ValueError("a chunk decode step needs a history: use decode_step for the first chunk")
        self.cache = cache
        self.fused_select = fused_select
        # kernels per run(): [blockify(Q) + select] (1 fused or 2) + attend + commit of K and V (1)
        # + memory update (plan + apply)
        self.LAUNCHES = (1 if fused_select else 2) + 1 + 1 + 2
        self.q_frames = q_frames or c.chunk_frames
        if cache._cand is None:
            cache._refresh_window()
        bpf, H = c.bpf, c.heads
        nq = self.q_frames * bpf
        self.nq = nq
        dev = cache.device
        self.q_reps = torch.zeros((H, nq, c.head_dim), dtype=torch.float32, device=dev)
        self.kv_slot = torch.zeros((H, nq, cache.kv_ld), dtype=torch.int32, device=dev)
        self.kv_cnt = torch.zeros((H, nq), dtype=torch.int32, device=dev)
        first = cache.hist
        self.dst = cache._frames_dst(first, self.q_frames)
        old_win = set(cache.window_frames(first))
        new_win = set(cache.window_frames(first + self.q_frames))
        entering = {f for f in range(first, first + self.q_frames) if f != 0}
        evicted = sorted((old_win | entering) - new_win)
        cand = [(cache.ring_slot(f, t), f * bpf + t) for f in evicted for t in range(bpf)]
        if first == 0:
            cand = [(cache.ring_slot(0, t), t) for t in range(bpf)] + cand
        self.ncand = len(cand)
        self.cs = cache._ints([[s for s, _ in cand]] * H).view(H, -1) if cand else None
        self.cg = cache._ints([[g for _, g in cand]] * H).view(H, -1) if cand else None

    def flops(self) -> float:
        """Selected-block attention FLOPs of one run (QK^T and PV, 2 flops per MAC)."""
        c = self.cache.cfg
        cnt = int(self.kv_cnt.sum().item())
        return 4.0 * 64 * 64 * c.head_dim * cnt

    def run(self, q, k, v, o, lse=None, stream=None, marks=None):
        """``marks``: optional list of 7 torch.cuda.Event recorded around the kernel groups:
        0 | blockify Q (+ select) | 1 | select | 2 | attend | 3 | commit blockify K+V | 4 | memory
        update plan | 5 | memory update apply (copies) | 6.  For the own-chunk variant the chunk's
        blockify K+V runs first (between marks 0 and 1), the fused selection between 1 and 2, and
        nothing between 3 and 4.  Without marks the plan and the commit overlap attend."""
        ca, c = self.cache, self.cache.cfg
        g, ws, ps = ca.geom, ca.ws, ca.pool_slots
        if marks is not None:
            ev_stream = stream or torch.cuda.current_stream(self.cache.device)
            mk = lambda i: marks[i].record(ev_stream)  # noqa: E731
        else:
            mk = lambda i: None  # noqa: E731
        own = c.own_chunk
        mk(0)
        if own:   # the chunk's K, V go to their ring positions first: every row attends them
            L.pbsa_blockify_kv(g, k, v, self.q_frames, ca.k_reps, None, ps, self.dst, ca.k_pool, ca.v_pool, ps,
                               ws=ws, stream=stream)
            mk(1)
        cs, cg, n = ca._cand
        if self.fused_select:
            ca._select_fused(q, self.q_frames, self.q_reps, self.kv_slot, self.kv_cnt, ca.kv_ld, stream)
            if not own:
                mk(1)
        else:
            L.pbsa_blockify(g, q, self.q_frames, self.q_reps, self.nq, ws=ws, stream=stream)
            if not own:
                mk(1)
            L.pbsa_score_select(g, self.q_reps, self.nq, ca.k_reps, ps, cs, cg, n, ca.topk if n else 0,
                                ca.p_list, ca.p_cnt, c.capacity, self.kv_slot, self.kv_cnt, ca.kv_ld,
                                ws=ws, stream=stream)
        mk(2)
        L.pbsa_attend(g, q, self.q_frames, ca.k_pool, ca.v_pool, ps, self.kv_slot, self.kv_cnt, ca.kv_ld,
                      o, lse, ws=ws, stream=stream)
        mk(3)
        if marks is None:
            # Programmatic dependents of attend: the memory update's plan (scores, ranking, slot
            # table; no pool access) and the commit of K, V (free ring slots, which the attend
            # lists never name) run on the SMs that attend's last wave leaves idle; the copies
            # of promoted blocks into persistent slots wait until attend has finished.
            L.pbsa_memory_update_plan(g, self.q_reps, self.nq, ca.k_reps, ps, ca.slot_gid, ca.slot_ema, c.capacity,
                                      c.bpf, self.cs, self.cg, self.ncand, c.gamma, ca.p_list, ca.p_cnt,
                                      flags=L.PBSA_OVERLAP_PREVIOUS, ws=ws, stream=stream)
            if not own:
                L.pbsa_blockify_kv(g, k, v, self.q_frames, ca.k_reps, None, ps, self.dst, ca.k_pool, ca.v_pool, ps,
                                   flags=L.PBSA_OVERLAP_PREVIOUS, ws=ws, stream=stream)
            L.pbsa_memory_update_apply(g, ca.k_reps, ca.k_pool, ca.v_pool, ps, c.capacity, self.ncand, ws=ws,
                                       stream=stream)
        else:
            # the same kernels, serialised between the timing events
            if not own:
                L.pbsa_blockify_kv(g, k, v, self.q_frames, ca.k_reps, None, ps, self.dst, ca.k_pool, ca.v_pool, ps,
                                   ws=ws, stream=stream)
            mk(4)
            L.pbsa_memory_update_plan(g, self.q_reps, self.nq, ca.k_reps, ps, ca.slot_gid, ca.slot_ema, c.capacity,
                                      c.bpf, self.cs, self.cg, self.ncand, c.gamma, ca.p_list, ca.p_cnt, ws=ws,
                                      stream=stream)
            mk(5)
            L.pbsa_memory_update_apply(g, ca.k_reps, ca.k_pool, ca.v_pool, ps, c.capacity, self.ncand, ws=ws,
                                       stream=stream)
        mk(6)
        return o

    def capture(self, q, k, v, o, lse=None, marks=None, ends=None) -> torch.cuda.CUDAGraph:
        """Capture ``run`` in a CUDA graph (one launch replays all kernels of the step).

        Call ``run`` once before capturing (kernel attributes are set on first use).  With
        ``marks`` (7 events between the kernel groups) or ``ends`` (2 events around the whole
        step, which leave the commit free to overlap attend), pass events created with
        ``external=True`` so they time inside the graph.
        """
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=self.cache.device)
        side.wait_stream(torch.cuda.current_stream(self.cache.device))
        with torch.cuda.graph(graph, stream=side):
            if ends is not None:
                ends[0].record(side)
            self.run(q, k, v, o, lse, stream=None, marks=marks)
            if ends is not None:
                ends[1].record(side)
        torch.cuda.current_stream(self.cache.device).wait_stream(side)
        return graph

    def capture_pipeline(self, q, k, v, o, qh, kh, vh, oh, parts=None):
        """Capture one end-to-end step, transfers included, as one CUDA graph for
        ``run_pipelined``: pinned host Q, K, V (``qh``, ``kh``, ``vh``) -> the device buffers
        ``q``, ``k``, ``v`` -> the step -> O (``o``) -> pinned host ``oh``.

        Q goes up first, then K and V, on one copy stream; [blockify(Q) + selection + attend]
        starts as soon as Q has landed, and O goes down on a second copy stream as soon as it is
        computed.  The memory update reads neither K nor V of the chunk (its candidates are
        blocks leaving the window, never the chunk's ring positions), so it runs while they
        upload, and only the commit waits for them.  With ``parts`` > 1, Q goes up in that many
        slices of whole frames, each followed by the selection and attention of its frames, and
        the memory update recomputes the chunk's representatives from the resident Q (the same
        kernel and order as the fused selection's, so the same bits).  Every query block's
        selection and attention are independent of the others', so the results equal ``run``'s
        bit for bit.  The graph holds the host buffers' addresses: ``run_pipelined`` takes the
        same four buffers.  (The own-chunk variant, which needs K, V before the selection, is
        not split.)"""
        if self.cache.cfg.own_chunk:
            raise ValueError("the own-chunk variant writes K, V before the selection: use capture()")
        for t in (qh, kh, vh, oh):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("the host buffers must be pinned CPU tensors")
        ca, c = self.cache, self.cache.cfg
        parts = parts or 1
        if self.q_frames % parts:
            raise ValueError(f"{self.q_frames} frames do not split into {parts} equal parts")
        fpp = self.q_frames // parts                 # frames per part
        rows, nqp = fpp * c.tpf, fpp * c.bpf
        dev = ca.device
        g, ws, ps = ca.geom, ca.ws, ca.pool_slots
        H = c.heads
        if parts == 1:   # the step's own buffers: the same kernels as run()
            part_bufs = [(self.q_reps, self.kv_slot, self.kv_cnt)]
        else:
            part_bufs = [(torch.zeros((H, nqp, c.head_dim), dtype=torch.float32, device=dev),
                          torch.zeros((H, nqp, ca.kv_ld), dtype=torch.int32, device=dev),
                          torch.zeros((H, nqp), dtype=torch.int32, device=dev)) for _ in range(parts)]
        main, h2d, d2h = (torch.cuda.Stream(device=dev) for _ in range(3))
        main.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=main):
            h2d.wait_stream(main)
            d2h.wait_stream(main)
            landed = []
            with torch.cuda.stream(h2d):
                for i in range(parts):
                    q[i * rows:(i + 1) * rows].copy_(qh[i * rows:(i + 1) * rows], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d)
                    landed.append(ev)
                k.copy_(kh, non_blocking=True)
                v.copy_(vh, non_blocking=True)
            for i, (qr, kv, cnt) in enumerate(part_bufs):
                main.wait_event(landed[i])
                qp, op = q[i * rows:(i + 1) * rows], o[i * rows:(i + 1) * rows]
                ca._select_fused(qp, fpp, qr, kv, cnt, ca.kv_ld)
                L.pbsa_attend(g, qp, fpp, ca.k_pool, ca.v_pool, ps, kv, cnt, ca.kv_ld, op, None, ws=ws)
                done = torch.cuda.Event()
                done.record(main)
                d2h.wait_event(done)
                with torch.cuda.stream(d2h):
                    oh[i * rows:(i + 1) * rows].copy_(op, non_blocking=True)
            # the memory update: the same kernels as run(), the same results bit for bit
            if parts > 1:
                L.pbsa_blockify(g, q, self.q_frames, self.q_reps, self.nq, ws=ws)
            L.pbsa_memory_update_plan(g, self.q_reps, self.nq, ca.k_reps, ps, ca.slot_gid, ca.slot_ema, c.capacity,
                                      c.bpf, self.cs, self.cg, self.ncand, c.gamma, ca.p_list, ca.p_cnt, ws=ws)
            L.pbsa_memory_update_apply(g, ca.k_reps, ca.k_pool, ca.v_pool, ps, c.capacity, self.ncand, ws=ws)
            main.wait_stream(h2d)                   # K, V uploaded
            L.pbsa_blockify_kv(g, k, v, self.q_frames, ca.k_reps, None, ps, self.dst, ca.k_pool, ca.v_pool, ps,
                               ws=ws)
            main.wait_stream(d2h)                   # O downloaded
        torch.cuda.current_stream(dev).wait_stream(main)
        self._pipe = {"graph": graph, "host": (qh, kh, vh, oh), "bufs": part_bufs}
        # launches per pipelined step: per part the fused selection and attend; [blockify(Q)], plan,
        # apply; the commit
        self.PIPELINED_LAUNCHES = 2 * parts + (3 if parts > 1 else 2) + 1

    def run_pipelined(self, qh, kh, vh, oh):
        """One step from the pinned host buffers given to ``capture_pipeline`` to the pinned
        host result, with the transfers overlapped with the kernels: one graph launch on the
        current stream (asynchronous; ``oh`` holds O once the stream reaches this point)."""
        p = self._pipe
        if any(a.data_ptr() != b.data_ptr() for a, b in zip((qh, kh, vh, oh), p["host"])):
            raise ValueError("run_pipelined takes the host buffers the step was captured with")
        p["graph"].replay()
        return oh

    def snapshot(self):
        """Copies of everything ``run`` mutates outside the chunk's own ring positions."""
        ca, C = self.cache, self.cache.cfg.capacity
        return [t.clone() for t in (ca.slot_gid, ca.slot_ema, ca.p_list, ca.p_cnt, ca.k_reps[:, :C],
                                    ca.k_pool[:, :C], ca.v_pool[:, :C])]

    def restore(self, snap):
        ca, C = self.cache, self.cache.cfg.capacity
        for dst, src in zip((ca.slot_gid, ca.slot_ema, ca.p_list, ca.p_cnt, ca.k_reps[:, :C],
                             ca.k_pool[:, :C], ca.v_pool[:, :C]), snap):
            dst.copy_(src, non_blocking=True)
