"""CPU oracle for Persistent Block-Sparse Attention (PBSA).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this module.  The product (the CUDA library and its Python binding)
never calls it, and it shares no code with the product: it is a plain, slow,
float64 restatement of what the method computes.

Source of the method: *Sparse Forcing: Native Trainable Sparse Attention for
Real-time Autoregressive Diffusion Video Generation*, as explained on
gist.science (English page, section 2 "Methodology", parts B "Structured Memory
Decomposition" and C "Persistent Block-Sparse Attention (PBSA)"; Chinese page,
section 2.2 "核心机制"; Portuguese page, "Arquitetura Proposta").  The pages give
the method in prose only, so the open points are fixed as follows (each is a
reading, not a quotation):

* block representative = mean of the block's 64 token vectors (mean pooling, as
  the related *Light Forcing* notes on papernotes.org, "HSA" design, state for
  their token compression);
* coarse score of query block r against KV block b = scale * <qbar_r, kbar_b>,
  scale = 1/sqrt(d);
* top-k local selection: the k largest scores, ties to the lower global block id;
* fine attention: one softmax over the union of the persistent blocks and the
  query block's selected local blocks (the "hybrid mask");
* memory update ("Top-C retention"): pool = persistent set plus evicted blocks;
  p_r = softmax of the coarse scores of query block r over the pool; a_b = mean_r
  p_{r,b}; EMA s_b <- gamma*s_b + (1-gamma)*a_b (s_b <- a_b when first seen);
  keep the sinks plus the top-(C - #sinks) other blocks by EMA, ties to the lower id.

Parity pins (tests/test_oracle.py): closed-form block means, brute-force and
permutation checks of the selection, reduction of the attention to dense
softmax attention (a library routine) when every block is selected, softmax
row sums, closed-form memory-update values (with scale 1 and with the scale
1/sqrt(d)), invariants of the persistent set, the EMA carried between a
rollout's updates, central finite differences for the backward pass, a hand-built
trainable-path case whose top-k is known by construction, and hand values of the two
near-tie gaps (``kth_gap``, ``ema_boundary_gap``).
tests/test_oracle_mutants.py plants one plausible mistake at a time in a copy of
this module and checks that some pin fails for each.
"""
from __future__ import annotations

import numpy as np

BT = 64  # tokens per block


# --------------------------------------------------------------------------- geometry
def block_token_rows(frame_h: int, frame_w: int, tile_h: int, tile_w: int, gid: int) -> np.ndarray:
    """Raster token indices of global block ``gid``, in the block's own row order.

    Blocks are 1 frame x (tile_h x tile_w) tokens; global id = frame*bpf + tile_row*(W/tile_w)
    + tile_col; inside a block token (ly, lx) is row ly*tile_w + lx.
    (English page, 2.E: the latent space is "blockified" into spatiotemporal blocks.)
    """
    tpr = frame_w // tile_w
    bpf = (frame_h // tile_h) * tpr
    f, rem = divmod(gid, bpf)
    ty, tx = divmod(rem, tpr)
    rows = []
    for ly in range(tile_h):
        for lx in range(tile_w):
            y, x = ty * tile_h + ly, tx * tile_w + lx
            rows.append(f * frame_h * frame_w + y * frame_w + x)
    return np.asarray(rows, dtype=np.int64)


def block_tokens(x: np.ndarray, geom: dict, gid: int, first_frame: int = 0) -> np.ndarray:
    """Tokens ``[64, H, d]`` of block ``gid`` taken from raster tensor ``x`` that starts at ``first_frame``."""
    bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
    local = gid - first_frame * bpf
    rows = block_token_rows(geom["frame_h"], geom["frame_w"], geom["tile_h"], geom["tile_w"], local)
    return np.asarray(x, dtype=np.float64)[rows]


# --------------------------------------------------------------------------- a1: representatives
def block_reps(x: np.ndarray, geom: dict, n_frames: int) -> np.ndarray:
    """Mean-pooled representatives ``[H, n_frames*bpf, d]`` (float64) of raster ``x[T, H, d]``.

    (Chinese page 2.2 "块化压缩": one compressed representative vector per block.)
    """
    bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
    H, d = x.shape[1], x.shape[2]
    out = np.zeros((H, n_frames * bpf, d), dtype=np.float64)
    for b in range(n_frames * bpf):
        out[:, b, :] = block_tokens(x, geom, b).mean(axis=0)
    return out


# --------------------------------------------------------------------------- a2: scores + top-k
def coarse_scores(q_reps: np.ndarray, k_reps: np.ndarray, scale: float) -> np.ndarray:
    """``scale * <qbar_r, kbar_b>`` for all pairs: ``[nq, nb]`` float64."""
    return scale * (np.asarray(q_reps, np.float64) @ np.asarray(k_reps, np.float64).T)


def topk_select(scores: np.ndarray, gids, k: int) -> list[int]:
    """Positions of the ``k`` best candidates, best first: score descending, then gid ascending.

    (English page 2.C "Local Sparsity": top-K relevant blocks within the local window.)
    A full sort; ``k`` larger than the candidate count takes them all.
    """
    order = sorted(range(len(gids)), key=lambda i: (-float(scores[i]), int(gids[i])))
    return order[:k]


def kth_gap(scores: np.ndarray, gids, k: int) -> float:
    """|score of the k-th best - score of the (k+1)-th best| (inf when there is no (k+1)-th)."""
    order = topk_select(scores, gids, len(gids))
    if k <= 0 or k >= len(order):
        return float("inf")
    return abs(float(scores[order[k - 1]]) - float(scores[order[k]]))


# --------------------------------------------------------------------------- hierarchical selection
def hsa_select(q_rep, cand_reps, cand_gids, bpf: int, top_frames: int, n_recent: int, k: int,
               scale: float):
    """Two-level (frame, then block) choice of the local blocks one query block attends.

    The hierarchical sparse attention of *Light Forcing* (papernotes.org notes, "方法详解",
    HSA, steps (1)-(3)), used as the selection policy over PBSA's local window:
      1. token compression: a frame's representative is the mean of its tokens, i.e. the mean
         of its block representatives (every block holds the same number of tokens);
      2. frame level: p(t) = scale * <qbar, frame rep of t>; the chosen frames are the
         always-on ones (here the ``n_recent`` latest candidate frames: the sinks already sit in
         the persistent memory, and the current chunk is not attended at inference) plus the
         ``top_frames`` best other frames (score descending, the earlier frame on ties);
      3. block level: o(b) = scale * <qbar, kbar_b> over the blocks of the chosen frames, the
         ``k`` best (score descending, the lower gid on ties).
    Candidates come in whole frames: candidate c belongs to frame slot c // bpf, frame slots in
    time order.  Returns (candidate positions best first, frame-level gap, block-level gap); a
    gap is |score at the cut - score just past it| (inf when nothing is cut).
    """
    reps = np.asarray(cand_reps, np.float64)
    q = np.asarray(q_rep, np.float64)
    n = reps.shape[0]
    nf = n // bpf
    frame_rep = reps.reshape(nf, bpf, -1).mean(axis=1)
    p = scale * (frame_rep @ q)
    always = list(range(max(0, nf - n_recent), nf))
    others = sorted((t for t in range(nf) if t not in always), key=lambda t: (-float(p[t]), t))
    chosen = set(always) | set(others[:max(0, top_frames)])
    frame_gap = float("inf")
    if 0 < top_frames < len(others):
        frame_gap = abs(float(p[others[top_frames - 1]]) - float(p[others[top_frames]]))
    elig = [c for c in range(n) if c // bpf in chosen]
    o = scale * (reps[elig] @ q)
    gids = [int(cand_gids[c]) for c in elig]
    pos = topk_select(o, gids, k)
    return [elig[i] for i in pos], frame_gap, kth_gap(o, gids, k)


# --------------------------------------------------------------------------- per-chunk sparsity
def cag_sparsity(lq, lk, d: int, s_base: float, s_target: float, alpha, n_dense: int = 1):
    """Chunk-aware growth of the related *Light Forcing* method (papernotes.org notes,
    "方法详解", CAG): the first ``n_dense`` chunks keep dense attention, chunk i after them gets
    sparsity s_i = s_base - alpha_i * beta, and beta makes the attention FLOPs of those chunks
    equal the target:
        sum_i (1 - s_base + alpha_i beta) lq_i lk_i d = (1 - s_target) sum_i lq_i lk_i d.
    ``lq``, ``lk``: query and key token counts per chunk; ``alpha``: each chunk's weight
    (the noise level at which it arrives, on the pages).  Returns (beta, [s_i] per chunk).
    """
    n = len(lq)
    L = [float(lq[i]) * float(lk[i]) * d for i in range(n)]
    tail = range(n_dense, n)
    num = (s_base - s_target) * sum(L[i] for i in tail)
    den = sum(float(alpha[i]) * L[i] for i in tail)
    beta = num / den if den != 0.0 else 0.0
    return beta, [0.0 if i < n_dense else s_base - float(alpha[i]) * beta for i in range(n)]


def cag_topk(sparsity: float, n_hist_blocks: int, n_persistent: int, n_local: int) -> int:
    """Local top-k of a chunk whose attention keeps a (1 - sparsity) share of its history blocks,
    the persistent blocks counted first: clamp(round((1 - s) * n_hist) - n_persistent, 0, n_local)."""
    keep = int(np.floor((1.0 - sparsity) * n_hist_blocks + 0.5))
    return max(0, min(n_local, keep - n_persistent))


# --------------------------------------------------------------------------- a3: fine attention
def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Softmax attention of query rows over key/value rows; returns (out [n, d], lse [n]).

    out_i = sum_j softmax_j(scale * q_i . k_j) v_j ; lse_i = log sum_j exp(scale * q_i . k_j).
    An empty key set gives out = 0 and lse = -inf.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1])), np.full(q.shape[0], -np.inf)
    logits = scale * (q @ k.T)
    m = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - m)
    s = e.sum(axis=1, keepdims=True)
    out = (e / s) @ v
    lse = (m + np.log(s))[:, 0]
    return out, lse


def attention_bwd(q, k, v, do, scale: float):
    """Gradients of ``attention`` (textbook): returns dq, dk, dv in float64.

    P = softmax(scale*QK^T); dV = P^T dO; dP = dO V^T; dS = P*(dP - rowsum(dO*O));
    dQ = scale*dS K; dK = scale*dS^T Q.
    (English page 2.D: the same sparse cache is used in training, so the sparse
    attention needs its gradient.)
    """
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    logits = scale * (q @ k.T)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    D = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - D)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


# --------------------------------------------------------------------------- a4: memory update
def memory_update(q_reps: np.ndarray, pool_reps: np.ndarray, pool_gids, prev_ema, is_sink,
                  scale: float, gamma: float, capacity: int):
    """Top-C retention of one head.  Returns (ema [nb] float64, keep [nb] bool, a [nb]).

    ``prev_ema[b]`` is NaN for a block seen for the first time.  Sinks are scored
    (they take part in the softmax) and always kept; the other places go to the
    top-(C - #sinks) non-sink blocks by EMA, ties to the lower global id.
    (English page 2.C "Dynamic Update"; Chinese page 2.2 "粗粒度评分与更新".)
    """
    s = coarse_scores(q_reps, pool_reps, scale)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    a = p.mean(axis=0)
    prev = np.asarray(prev_ema, np.float64)
    ema = np.where(np.isnan(prev), a, gamma * prev + (1.0 - gamma) * a)
    sink = np.asarray(is_sink, bool)
    keep = sink.copy()
    free = capacity - int(sink.sum())
    cand = [i for i in range(len(pool_gids)) if not sink[i]]
    order = sorted(cand, key=lambda i: (-float(np.float32(ema[i])), int(pool_gids[i])))
    for i in order[:max(free, 0)]:
        keep[i] = True
    return ema, keep, a


def ema_boundary_gap(ema: np.ndarray, pool_gids, is_sink, capacity: int) -> float:
    """Relative gap between the last kept and the first dropped non-sink EMA (inf if none dropped)."""
    sink = np.asarray(is_sink, bool)
    free = capacity - int(sink.sum())
    vals = sorted((float(ema[i]) for i in range(len(pool_gids)) if not sink[i]), reverse=True)
    if free <= 0 or free >= len(vals):
        return float("inf")
    return abs(vals[free - 1] - vals[free]) / max(abs(vals[free - 1]), 1e-30)


# --------------------------------------------------------------------------- workload plans
def frame_blocks(frames, bpf: int) -> list[int]:
    """Global ids of all blocks of the given frames, ascending."""
    return [f * bpf + j for f in sorted(frames) for j in range(bpf)]


def window_frames(hist: int, window: int) -> list[int]:
    """Local window after ``hist`` committed frames: the last ``window`` frames, frame 0 excluded.

    (English page 2.B: the local window L_t is a sliding window of recent blocks; frame 0
    holds the sinks, which live in the persistent memory instead.)
    """
    return list(range(max(1, hist - window), hist))


def single_step_plan(q, k, geom: dict, hist: int, chunk: int, capacity: int, window: int,
                     topk: int, gamma: float, k_chunk=None, q_reps=None, k_reps=None):
    """Selections of one chunk decode over a history of ``hist`` frames (one layer, all heads).

    Persistent memory is bootstrapped by one update (no prior EMA) over the sinks and every
    middle block, scored by this chunk's query representatives; then each query block
    selects its top-k local blocks; then, if ``k_chunk`` (the chunk's keys) is given, the
    post-chunk update runs with the blocks that the chunk pushes out of the window.
    Returns a dict of per-head lists of global ids.
    """
    bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
    scale = geom["scale"]
    H = q.shape[1]
    qr = block_reps(q, geom, chunk) if q_reps is None else q_reps
    kr = block_reps(k, geom, hist) if k_reps is None else k_reps
    sinks = frame_blocks([0], bpf)
    local = frame_blocks(window_frames(hist, window), bpf)
    middle = frame_blocks(range(1, max(1, hist - window)), bpf)
    out = {"sinks": sinks, "local": local, "middle": middle, "P": [], "P_ema": [],
           "sel": [], "sel_gap": [], "boot_gap": [], "P2": [], "P2_gap": []}
    for h in range(H):
        pool = sinks + middle
        ema, keep, _ = memory_update(qr[h], kr[h][pool], pool, [np.nan] * len(pool),
                                     [g < bpf for g in pool], scale, gamma, capacity)
        P = [g for g, kp in zip(pool, keep) if kp]
        out["P"].append(P)
        out["P_ema"].append({g: float(e) for g, e, kp in zip(pool, ema, keep) if kp})
        out["boot_gap"].append(ema_boundary_gap(ema, pool, [g < bpf for g in pool], capacity))
        sc = coarse_scores(qr[h], kr[h][local], scale).astype(np.float32)
        sel_h, gap_h = [], []
        for r in range(qr.shape[1]):
            pos = topk_select(sc[r], local, topk)
            sel_h.append([local[i] for i in pos])
            gap_h.append(kth_gap(sc[r], local, topk))
        out["sel"].append(sel_h)
        out["sel_gap"].append(gap_h)
        if k_chunk is not None:
            evicted = frame_blocks(range(max(1, hist - window),
                                         max(1, hist + chunk - window)), bpf)
            pool2 = P + evicted
            prev = [out["P_ema"][h][g] for g in P] + [np.nan] * len(evicted)
            ema2, keep2, _ = memory_update(qr[h], kr[h][pool2], pool2, prev,
                                           [g < bpf for g in pool2], scale, gamma, capacity)
            out["P2"].append(sorted(g for g, kp in zip(pool2, keep2) if kp))
            out["P2_gap"].append(ema_boundary_gap(ema2, pool2, [g < bpf for g in pool2], capacity))
    return out


def attend_gids(q, k, v, geom: dict, h: int, r: int, gids, q_first_frame: int = 0):
    """Fine attention of query block ``r`` (global id ``q_first_frame*bpf + r``) of head ``h``
    over the tokens of the KV blocks ``gids`` (one joint softmax: the hybrid mask).
    ``k``/``v`` are raster tensors whose frame 0 is global frame 0.
    Returns (out [64, d], lse [64]) in float64."""
    bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
    qb = block_tokens(q, geom, q_first_frame * bpf + r, q_first_frame)[:, h, :]
    if len(gids) == 0:
        return attention(qb, np.zeros((0, qb.shape[1])), np.zeros((0, v.shape[2])), geom["scale"])
    kk = np.concatenate([block_tokens(k, geom, g)[:, h, :] for g in gids])
    vv = np.concatenate([block_tokens(v, geom, g)[:, h, :] for g in gids])
    return attention(qb, kk, vv, geom["scale"])


class RolloutOracle:
    """Persistent-memory state machine of one layer over an autoregressive rollout.

    State per head: the persistent set P (global id -> EMA).  For each chunk: if nothing
    has been committed yet the chunk attends its own blocks only; otherwise each query
    block attends P plus its top-k blocks of the local window.  When the chunk is
    finished it is committed: its frames enter the window, the frames that leave the
    window form the eviction set E, and the memory update runs over P + E (plus the
    sinks when frame 0 is committed), scored by the chunk's last-step query
    representatives.  (English page 2.B-2.C; Chinese page 2.1: P_t is shared across the
    diffusion steps of a chunk.)
    """

    def __init__(self, geom: dict, heads: int, capacity: int, window: int, topk: int,
                 gamma: float):
        self.geom, self.H, self.C, self.W, self.k, self.gamma = geom, heads, capacity, window, topk, gamma
        self.bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
        self.hist = 0
        self.P = [dict() for _ in range(heads)]
        self.kreps = {}            # gid -> [H, d]
        self.last_gap = []
        self.last_pool_ema = []    # per head: {gid: EMA} of every pool entry of the last update

    def local(self) -> list[int]:
        return frame_blocks(window_frames(self.hist, self.W), self.bpf)

    def select(self, q_reps: np.ndarray):
        """Per head, per query block: (attended gids, k-th gap).  None when history is empty."""
        if self.hist == 0:
            return None
        local = self.local()
        out = []
        for h in range(self.H):
            P = sorted(self.P[h])
            kr = np.stack([self.kreps[g][h] for g in local]) if local else np.zeros((0, q_reps.shape[2]))
            sc = coarse_scores(q_reps[h], kr, self.geom["scale"]).astype(np.float32)
            rows = []
            for r in range(q_reps.shape[1]):
                pos = topk_select(sc[r], local, self.k) if local else []
                rows.append((P + [local[i] for i in pos], kth_gap(sc[r], local, self.k)))
            out.append(rows)
        return out

    def commit(self, first_frame: int, n_frames: int, k_reps_chunk: np.ndarray,
               q_reps_last: np.ndarray, prev_state=None):
        """Commit a finished chunk and run the memory update.  ``prev_state`` (optional,
        per head {gid: ema}) replaces P before the update, to check one step from a given state."""
        if prev_state is not None:
            self.P = [dict(p) for p in prev_state]
        old_win = set(window_frames(self.hist, self.W))
        for j in range(k_reps_chunk.shape[1]):
            self.kreps[first_frame * self.bpf + j] = k_reps_chunk[:, j, :]
        new_hist = first_frame + n_frames
        new_win = set(window_frames(new_hist, self.W))
        entering = {f for f in range(first_frame, new_hist) if f != 0}
        evicted = frame_blocks((old_win | entering) - new_win, self.bpf)
        new_sinks = frame_blocks([0], self.bpf) if first_frame == 0 else []
        self.last_gap = []
        self.last_pool_ema = []
        for h in range(self.H):
            pool = sorted(self.P[h]) + new_sinks + evicted
            prev = [self.P[h].get(g, np.nan) for g in pool]
            reps = np.stack([self.kreps[g][h] for g in pool])
            sink = [g < self.bpf for g in pool]
            ema, keep, _ = memory_update(q_reps_last[h], reps, pool, prev, sink,
                                         self.geom["scale"], self.gamma, self.C)
            self.P[h] = {g: float(e) for g, e, kp in zip(pool, ema, keep) if kp}
            self.last_gap.append(ema_boundary_gap(ema, pool, sink, self.C))
            self.last_pool_ema.append({g: float(e) for g, e in zip(pool, ema)})
        self.hist = new_hist
        return evicted


def train_masks(q, k, geom: dict, batch_frames: int, chunk: int, topk: int):
    """Fixed block masks of the trainable path, per (batch, head, query block): global ids.

    Chunk 0 attends its own blocks.  A later chunk attends the sinks (frame 0), its top-k
    blocks among the earlier non-sink blocks, and its own chunk's blocks (a sequence whose
    length is not a whole number of chunks ends with a shorter chunk).  ``q``/``k``
    are ``[B, T, H, d]``.  Returns masks[b][h][r] (r over all query blocks of the sequence)
    and the k-th gaps.
    """
    bpf = (geom["frame_h"] // geom["tile_h"]) * (geom["frame_w"] // geom["tile_w"])
    B, H = q.shape[0], q.shape[2]
    masks, gaps = [], []
    for b in range(B):
        qr = block_reps(q[b], geom, batch_frames)
        kr = block_reps(k[b], geom, batch_frames)
        mb, gb = [], []
        for h in range(H):
            mh, gh = [], []
            for r in range(batch_frames * bpf):
                c = (r // bpf) // chunk
                own = frame_blocks(range(c * chunk, min((c + 1) * chunk, batch_frames)), bpf)
                if c == 0:
                    mh.append(own)
                    gh.append(float("inf"))
                    continue
                earlier = frame_blocks(range(1, c * chunk), bpf)
                sc = coarse_scores(qr[h][r:r + 1], kr[h][earlier], geom["scale"])[0].astype(np.float32)
                pos = topk_select(sc, earlier, topk)
                mh.append(frame_blocks([0], bpf) + sorted(earlier[i] for i in pos) + own)
                gh.append(kth_gap(sc, earlier, topk))
            mb.append(mh)
            gb.append(gh)
        masks.append(mb)
        gaps.append(gb)
    return masks, gaps
