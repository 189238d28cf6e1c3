"""Seeded synthetic workloads for PBSA (Persistent Block-Sparse Attention).

This module only *draws numbers* and describes shapes. It holds none of the
method's arithmetic (no pooling, scoring, selection, softmax or update), so the
CPU oracle under ``oracle/`` and the CUDA path can both be fed from it without
sharing any computation.

Workload shapes follow the five synthetic configurations used to exercise the
method of *Sparse Forcing: Native Trainable Sparse Attention for Real-time
Autoregressive Diffusion Video Generation* (gist.science English explainer,
section 2.B "Structured Memory Decomposition" and 2.C "Persistent Block-Sparse
Attention"): a latent video of frames of ``frame_h x frame_w`` tokens, each
frame cut into 64-token tiles ("spatiotemporal blocks"), a persistent memory of
capacity ``C`` that always holds frame 0's blocks (the sinks), and a sliding
local window of ``W`` frames.

Random values come from ``torch.Generator`` (Philox on CUDA, MT19937 on CPU),
seeded per tensor from a fixed integer recipe, so that every tensor is
reproducible on its own.  bf16 workloads are drawn in fp32 and rounded once
(round-to-nearest-even); both sides consume exactly those rounded values.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BLOCK_TOKENS = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """Geometry and policy of one PBSA attention layer."""

    name: str
    heads: int
    head_dim: int
    frame_h: int
    frame_w: int
    tile_h: int
    tile_w: int
    chunk_frames: int      # frames per query chunk
    hist_frames: int       # frames of KV history before the chunk (single-step workloads)
    capacity: int          # persistent capacity C, sinks included
    window_frames: int     # local window W, in frames
    topk: int              # local top-k per query block
    gamma: float           # EMA factor of the memory update
    dtype: str             # "f32" or "bf16"
    seed: int
    block_offset_std: float = 0.0   # std of the per-block shared offset (0: none)
    layers: int = 1
    steps: int = 1                  # denoising steps per chunk sharing the persistent memory
    total_frames: int = 0           # rollouts: latent frames in the whole video
    ar_rho: float = 0.0             # rollouts: AR(1) factor of block offsets across frames
    batch: int = 1

    @property
    def blocks_per_frame(self) -> int:
        return (self.frame_h // self.tile_h) * (self.frame_w // self.tile_w)

    @property
    def tokens_per_frame(self) -> int:
        return self.frame_h * self.frame_w

    @property
    def n_sink(self) -> int:
        return self.blocks_per_frame

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


TINY = Workload(
    name="tiny_f32", heads=1, head_dim=64, frame_h=16, frame_w=16, tile_h=8, tile_w=8,
    chunk_frames=1, hist_frames=6, capacity=8, window_frames=2, topk=4, gamma=0.9,
    dtype="f32", seed=0)

DECODE_5S = Workload(
    name="decode_5s_last_chunk_bf16", heads=12, head_dim=128, frame_h=32, frame_w=48,
    tile_h=8, tile_w=8, chunk_frames=3, hist_frames=18, capacity=96, window_frames=6,
    topk=32, gamma=0.9, dtype="bf16", seed=1, block_offset_std=0.5)

ROLLOUT_5S = dataclasses.replace(
    DECODE_5S, name="rollout_5s_30layers_bf16", hist_frames=0, layers=30, steps=4,
    total_frames=21, seed=2)

ROLLOUT_1MIN = dataclasses.replace(
    DECODE_5S, name="rollout_1min_30layers_bf16", hist_frames=0, layers=30, steps=1,
    total_frames=241, ar_rho=0.98, seed=3)

TRAIN_FWD_BWD = Workload(
    name="train_fwd_bwd_bf16_b2", heads=12, head_dim=128, frame_h=32, frame_w=48,
    tile_h=8, tile_w=8, chunk_frames=3, hist_frames=0, capacity=0, window_frames=0,
    topk=16, gamma=0.9, dtype="bf16", seed=4, total_frames=9, batch=2)

WORKLOADS = {w.name: w for w in (TINY, DECODE_5S, ROLLOUT_5S, ROLLOUT_1MIN, TRAIN_FWD_BWD)}


def _gen(device: str | torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def stream_seed(*parts: int) -> int:
    """A fixed integer mix of (workload seed, tensor tag, indices) into one seed."""
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h ^= (int(p) + 0x9E3779B97F4A7C15 + ((h << 6) & 0xFFFFFFFFFFFFFFFF) + (h >> 2))
        h &= 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFF_FFFF_FFFF_FFFF


def tokens(w: Workload, n_frames: int, seed: int, *, device="cpu",
           offset_std: float | None = None, dtype: torch.dtype | None = None) -> torch.Tensor:
    """Raster-order token tensor ``[n_frames*frame_h*frame_w, heads, head_dim]``.

    Values are N(0,1), plus (if ``offset_std`` > 0) one N(0, offset_std^2) vector per
    (head, 64-token tile) shared by all tokens of that tile, so that tiles have
    distinguishable means.  Returned in the workload dtype (fp32 or bf16).
    """
    offset_std = w.block_offset_std if offset_std is None else offset_std
    g = _gen(device, seed)
    T = n_frames * w.tokens_per_frame
    x = torch.randn((T, w.heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    if offset_std > 0:
        ty, tx = w.frame_h // w.tile_h, w.frame_w // w.tile_w
        off = torch.randn((n_frames, ty, 1, tx, 1, w.heads, w.head_dim), generator=g,
                          device=device, dtype=torch.float32) * offset_std
        x = (x.view(n_frames, ty, w.tile_h, tx, w.tile_w, w.heads, w.head_dim) + off).view(
            T, w.heads, w.head_dim)
    return x.to(dtype or w.torch_dtype)


def ar1_offsets(w: Workload, n_frames: int, seed: int, *, device="cpu") -> torch.Tensor:
    """AR(1) tile offsets ``[n_frames, ty, tx, heads, d]``, stationary with std ``block_offset_std``.

    o_0 ~ N(0, s^2);  o_t = rho * o_{t-1} + sqrt(1 - rho^2) * e_t,  e_t ~ N(0, s^2).
    """
    g = _gen(device, seed)
    ty, tx = w.frame_h // w.tile_h, w.frame_w // w.tile_w
    s, rho = w.block_offset_std, w.ar_rho
    e = torch.randn((n_frames, ty, tx, w.heads, w.head_dim), generator=g, device=device) * s
    out = torch.empty_like(e)
    out[0] = e[0]
    c = math.sqrt(1.0 - rho * rho)
    for t in range(1, n_frames):
        out[t] = rho * out[t - 1] + c * e[t]
    return out


def tokens_with_offsets(w: Workload, offsets: torch.Tensor, seed: int, *, device="cpu") -> torch.Tensor:
    """N(0,1) tokens for ``offsets.shape[0]`` frames plus the given per-tile offsets."""
    g = _gen(device, seed)
    n_frames, ty, tx = offsets.shape[:3]
    T = n_frames * w.tokens_per_frame
    x = torch.randn((T, w.heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    x = (x.view(n_frames, ty, w.tile_h, tx, w.tile_w, w.heads, w.head_dim)
         + offsets.to(device)[:, :, None, :, None]).view(T, w.heads, w.head_dim)
    return x.to(w.torch_dtype)


def single_step(w: Workload, *, device="cpu"):
    """Q of one chunk and K, V of the ``hist_frames`` frames before it (single-step workloads)."""
    q = tokens(w, w.chunk_frames, stream_seed(w.seed, 1), device=device)
    k = tokens(w, w.hist_frames, stream_seed(w.seed, 2), device=device)
    v = tokens(w, w.hist_frames, stream_seed(w.seed, 3), device=device)
    return q, k, v


def rollout_chunks(w: Workload) -> list[tuple[int, int]]:
    """(first frame, n frames) of each chunk of a rollout.

    With ``ar_rho`` set (the 1-minute workload) frame 0 is a chunk of its own and the
    remaining frames come in chunks of ``chunk_frames``; otherwise all chunks have
    ``chunk_frames`` frames.
    """
    out, f = [], 0
    if w.ar_rho > 0:
        out.append((0, 1))
        f = 1
    while f < w.total_frames:
        n = min(w.chunk_frames, w.total_frames - f)
        out.append((f, n))
        f += n
    return out


def train_inputs(w: Workload, *, device="cpu"):
    """Q, K, V, dO of the trainable-path workload: ``[batch, T, heads, d]`` each, N(0,1)."""
    T = w.total_frames * w.tokens_per_frame
    outs = []
    for tag in range(4):
        g = _gen(device, stream_seed(w.seed, 10 + tag))
        outs.append(torch.randn((w.batch, T, w.heads, w.head_dim), generator=g, device=device)
                    .to(w.torch_dtype))
    return tuple(outs)


def train_lists(w: Workload, seed: int, n_frames: int | None = None, batch: int | None = None):
    """Block lists of the trainable-path workload, with the batch folded into the frame axis.

    Query block r of batch b (global block id b*F*bpf + r, F = frames per sequence) attends:
    its own chunk's blocks; and, for chunks after the first, the sink blocks (frame 0 of its
    sequence) plus ``topk`` blocks drawn uniformly (seeded) from the earlier non-sink blocks
    of its sequence -- masks with the structure of the trainable path but random contents,
    for structural tests of the attention kernels (the method's own masks are computed by
    the library from the coarse scores).  Pool slot = global block id.  Returns a list over
    heads of lists over query blocks of slot lists.
    """
    F = n_frames or w.total_frames
    B = batch or w.batch
    bpf, cf = w.blocks_per_frame, w.chunk_frames
    g = _gen("cpu", seed)
    out = []
    for h in range(w.heads):
        rows = []
        for b in range(B):
            base = b * F * bpf
            for r in range(F * bpf):
                c = (r // bpf) // cf
                own = list(range(base + c * cf * bpf, base + min((c + 1) * cf, F) * bpf))
                if c == 0:
                    rows.append(own)
                    continue
                earlier = list(range(base + bpf, base + c * cf * bpf))
                k = min(w.topk, len(earlier))
                pick = torch.randperm(len(earlier), generator=g)[:k].tolist()
                rows.append(list(range(base, base + bpf)) + sorted(earlier[i] for i in pick) + own)
        out.append(rows)
    return out
