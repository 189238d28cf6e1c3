"""Per-chunk sparsity of a rollout: chunk-aware growth, as a local top-k schedule.  Host logic.

The related *Light Forcing* method (papernotes.org notes, "方法详解", CAG) keeps the first
chunk(s) of an autoregressive rollout dense, as visual anchors, and gives each later chunk i
the sparsity s_i = s_base - alpha_i * beta, where alpha_i weighs the chunk (the noise level at
which it arrives) and beta is fixed by a FLOP budget: over the sparse chunks,
    sum_i (1 - s_base + alpha_i beta) Lq_i Lk_i d = (1 - s_target) sum_i Lq_i Lk_i d,
i.e. beta = (s_base - s_target) sum_i L_i / sum_i alpha_i L_i with L_i = Lq_i Lk_i d.

For PBSA a chunk's density (1 - s_i) is the share of its history blocks each query block
attends; the persistent blocks are always attended, so the local top-k is what remains of
that share, within the window: k_i = clamp(round((1 - s_i) * history blocks) - persistent, 0,
window blocks).  ``PBSALayerCache.set_topk`` applies it chunk by chunk.
"""
from __future__ import annotations

import math


def chunk_sparsity(q_tokens, k_tokens, head_dim: int, s_base: float, s_target: float, alpha,
                   n_dense: int = 1) -> tuple[float, list[float]]:
    """(beta, per-chunk sparsity): 0 for the first ``n_dense`` chunks, s_base - alpha_i beta after."""
    weights = [float(q) * float(k) * head_dim for q, k in zip(q_tokens, k_tokens)]
    sparse = list(range(n_dense, len(weights)))
    total = math.fsum(weights[i] for i in sparse)
    weighted = math.fsum(float(alpha[i]) * weights[i] for i in sparse)
    beta = (s_base - s_target) * total / weighted if weighted else 0.0
    return beta, [s_base - float(alpha[i]) * beta if i >= n_dense else 0.0 for i in range(len(weights))]


def chunk_topk(sparsity: float, hist_blocks: int, persistent_blocks: int, local_blocks: int) -> int:
    """Local top-k that tops the persistent blocks up to a (1 - sparsity) share of the history."""
    kept = math.floor((1.0 - sparsity) * hist_blocks + 0.5)
    return min(local_blocks, max(0, kept - persistent_blocks))


def rollout_topk(chunks, frame_tokens: int, blocks_per_frame: int, head_dim: int, capacity: int,
                 window_frames: int, s_base: float, s_target: float, alpha=None, n_dense: int = 1):
    """Local top-k per chunk of a rollout.

    ``chunks``: (first frame, frames) per chunk.  Query tokens = the chunk's; key tokens = its
    history (the frames before it).  ``alpha`` defaults to a linear decay from 1 (first sparse
    chunk) to 0 (last chunk): earlier chunks keep more of their history.  Returns (k per chunk,
    sparsity per chunk, beta).
    """
    n = len(chunks)
    if alpha is None:
        span = max(1, n - n_dense - 1)
        alpha = [1.0 - (i - n_dense) / span if i >= n_dense else 1.0 for i in range(n)]
    q_tok = [nf * frame_tokens for _, nf in chunks]
    k_tok = [f0 * frame_tokens for f0, _ in chunks]
    beta, sparsity = chunk_sparsity(q_tok, k_tok, head_dim, s_base, s_target, alpha, n_dense)
    ks = []
    for (f0, _), s in zip(chunks, sparsity):
        local_frames = f0 - max(1, f0 - window_frames) if f0 > 0 else 0
        middle_frames = max(1, f0 - window_frames) - 1 if f0 > 0 else 0
        persistent = min(capacity, blocks_per_frame * (1 + middle_frames)) if f0 > 0 else 0
        ks.append(chunk_topk(s, f0 * blocks_per_frame, persistent, local_frames * blocks_per_frame))
    return ks, sparsity, beta
