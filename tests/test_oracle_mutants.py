"""The oracle's pins have teeth: a plausible mistake planted in the oracle (a dropped term, a
wrong sign, index or axis, an off-by-one count, a reversed tie rule) makes at least one pin of
tests/test_oracle.py fail.  Each mutant is the oracle's own source with one textual change,
executed as a separate module and patched in for the pins it should trip.  CPU only; the
mistakes are planted in a copy of the oracle, never in the CUDA path."""
import inspect
import types

import pytest

import test_oracle as T
from oracle import pbsa_oracle as O

SRC = inspect.getsource(O)

PINS = {
    "block_reps": lambda: (T.test_block_reps_closed_form(8, 8), T.test_block_reps_closed_form(4, 16)),
    "block_rows": T.test_block_rows_cover_frame_once,
    "topk_ties": T.test_topk_ties_go_to_lower_id,
    "topk_brute": T.test_topk_brute_force_and_permutation,
    "dense": T.test_all_blocks_selected_is_dense_attention,
    "softmax": T.test_softmax_rows_sum_to_one_and_convex_hull,
    "empty": T.test_empty_key_set,
    "bwd_fd": T.test_backward_finite_differences,
    "mu_closed": T.test_memory_update_closed_form,
    "mu_scaled": T.test_memory_update_closed_form_with_the_attention_scale,
    "mu_inv": T.test_memory_update_invariants,
    "mu_ties": T.test_memory_update_equal_ema_ties_to_lower_id,
    "rollout": T.test_rollout_windows_and_capacity_5s,
    "rollout_ema": T.test_rollout_carries_the_ema_between_updates,
    "single_step": T.test_single_step_partition_5s,
    "train_masks": T.test_train_masks_shape,
    "train_select": T.test_train_masks_selection_hand_built,
    "kth_gap": T.test_kth_gap_hand_values,
    "ema_gap": T.test_ema_boundary_gap_hand_values,
    "hsa_mean": T.test_hsa_frames_ranked_by_mean_not_by_best_block,
    "hsa_flat": lambda: [T.test_hsa_reduces_to_flat_topk(s) for s in (0, 1, 2)],
    "hsa_brute": T.test_hsa_brute_force_small,
    "cag_budget": T.test_cag_meets_the_flop_budget,
    "cag_special": T.test_cag_special_cases,
    "cag_topk": T.test_cag_topk_mapping,
}

# (what the mistake is, oracle text, mistaken text, pins expected to catch it)
MUTANTS = [
    ("block rows: tile row and column swapped", "ty, tx = divmod(rem, tpr)", "tx, ty = divmod(rem, tpr)",
     ["block_reps", "block_rows"]),
    ("block rows: frame stride dropped", "rows.append(f * frame_h * frame_w + y * frame_w + x)",
     "rows.append(y * frame_w + x)", ["block_reps", "block_rows"]),
    ("block mean over 63 tokens", "out[:, b, :] = block_tokens(x, geom, b).mean(axis=0)",
     "out[:, b, :] = block_tokens(x, geom, b).sum(axis=0) / 63.0", ["block_reps"]),
    ("coarse score without the scale", "return scale * (np.asarray(q_reps, np.float64) @",
     "return (np.asarray(q_reps, np.float64) @", ["mu_closed", "mu_scaled", "mu_inv"]),
    ("coarse score with the wrong sign", "return scale * (np.asarray(q_reps, np.float64) @",
     "return -scale * (np.asarray(q_reps, np.float64) @", ["mu_closed", "mu_scaled", "mu_inv"]),
    ("top-k ties to the higher id", "key=lambda i: (-float(scores[i]), int(gids[i])))",
     "key=lambda i: (-float(scores[i]), -int(gids[i])))", ["topk_ties", "topk_brute"]),
    ("top-k keeps one block too few", "    return order[:k]\n", "    return order[:max(0, k - 1)]\n",
     ["topk_ties", "topk_brute"]),
    ("attention logits without the scale", "    logits = scale * (q @ k.T)\n    m = logits.max(axis=1, keepdims=True)",
     "    logits = (q @ k.T)\n    m = logits.max(axis=1, keepdims=True)", ["dense"]),
    ("attention softmax over the query axis", "    e = np.exp(logits - m)\n    s = e.sum(axis=1, keepdims=True)",
     "    e = np.exp(logits - m)\n    s = e.sum(axis=0, keepdims=True)", ["dense", "softmax"]),
    ("log-sum-exp without the maximum", "    lse = (m + np.log(s))[:, 0]", "    lse = np.log(s)[:, 0]", ["dense"]),
    ("backward: rowsum(dO*O) term dropped", "    ds = p * (dp - D)\n    dq", "    ds = p * dp\n    dq", ["bwd_fd"]),
    ("backward: dK from dS instead of dS^T", "    dk = scale * (ds.T @ q)", "    dk = scale * (ds @ q)", ["bwd_fd"]),
    ("backward: dV from P instead of P^T", "    dv = p.T @ do", "    dv = p @ do", ["bwd_fd"]),
    ("EMA weights swapped", "gamma * prev + (1.0 - gamma) * a)", "(1.0 - gamma) * prev + gamma * a)",
     ["mu_closed"]),
    ("attention share averaged over the pool instead of the rows", "    a = p.mean(axis=0)\n    prev",
     "    a = p.mean(axis=1).mean() * np.ones(p.shape[1])\n    prev", ["mu_closed", "mu_inv"]),
    ("first observation damped like a repeat", "ema = np.where(np.isnan(prev), a,",
     "ema = np.where(np.isnan(prev), (1.0 - gamma) * a,", ["mu_closed"]),
    ("sinks not forced into the persistent set", "    keep = sink.copy()\n    free = capacity - int(sink.sum())\n    cand = [i for i in range(len(pool_gids)) if not sink[i]]",
     "    keep = np.zeros_like(sink)\n    free = capacity\n    cand = list(range(len(pool_gids)))", ["mu_inv", "mu_closed"]),
    ("retention ties to the higher id", "order = sorted(cand, key=lambda i: (-float(np.float32(ema[i])), int(pool_gids[i])))",
     "order = sorted(cand, key=lambda i: (-float(np.float32(ema[i])), -int(pool_gids[i])))", ["mu_ties"]),
    ("window includes frame 0", "    return list(range(max(1, hist - window), hist))",
     "    return list(range(max(0, hist - window), hist))", ["rollout"]),
    ("two-level selection ranks frames by their best block", "    frame_rep = reps.reshape(nf, bpf, -1).mean(axis=1)\n    p = scale * (frame_rep @ q)",
     "    p = scale * (reps @ q).reshape(nf, bpf).max(axis=1)", ["hsa_mean"]),
    ("two-level selection keeps the oldest frames always on", "always = list(range(max(0, nf - n_recent), nf))",
     "always = list(range(0, min(nf, n_recent)))", ["hsa_flat", "hsa_brute"]),
    ("chunk-aware growth with the wrong sign", "s_base - float(alpha[i]) * beta for i in range(n)]",
     "s_base + float(alpha[i]) * beta for i in range(n)]", ["cag_budget"]),
    ("chunk top-k ignores the persistent blocks", "return max(0, min(n_local, keep - n_persistent))",
     "return max(0, min(n_local, keep))", ["cag_topk", "cag_special"]),
    ("rollout: the sinks never enter the persistent memory",
     "new_sinks = frame_blocks([0], self.bpf) if first_frame == 0 else []", "new_sinks = []", ["rollout"]),
    ("rollout: the EMA restarts at every update", "prev = [self.P[h].get(g, np.nan) for g in pool]",
     "prev = [np.nan for g in pool]", ["rollout_ema"]),
    ("single step: middle frames start at frame 0", "middle = frame_blocks(range(1, max(1, hist - window)), bpf)",
     "middle = frame_blocks(range(0, max(1, hist - window)), bpf)", ["single_step", "dense"]),
    ("attended query block indexed as if the chunk began at frame 0",
     "qb = block_tokens(q, geom, q_first_frame * bpf + r, q_first_frame)",
     "qb = block_tokens(q, geom, q_first_frame * bpf + r, 0)", ["dense"]),
    ("training masks: own chunk is one frame", "own = frame_blocks(range(c * chunk, min((c + 1) * chunk, batch_frames)), bpf)",
     "own = frame_blocks(range(c * chunk, c * chunk + 1), bpf)", ["train_masks"]),
    ("training masks: a short last chunk runs past the sequence",
     "own = frame_blocks(range(c * chunk, min((c + 1) * chunk, batch_frames)), bpf)",
     "own = frame_blocks(range(c * chunk, (c + 1) * chunk), bpf)", ["train_masks"]),
    ("training masks: sinks missing from later chunks", "mh.append(frame_blocks([0], bpf) + sorted(earlier[i] for i in pos) + own)",
     "mh.append(sorted(earlier[i] for i in pos) + own)", ["train_masks"]),
    ("training masks: every row scored with the chunk's first query block",
     "sc = coarse_scores(qr[h][r:r + 1], kr[h][earlier]", "sc = coarse_scores(qr[h][c * chunk * bpf:c * chunk * bpf + 1], kr[h][earlier]",
     ["train_select"]),
    ("training masks: keys of the other batch item", "kr = block_reps(k[b], geom, batch_frames)",
     "kr = block_reps(k[B - 1 - b], geom, batch_frames)", ["train_select"]),
    ("training masks: own chunk among the candidates", "earlier = frame_blocks(range(1, c * chunk), bpf)",
     "earlier = frame_blocks(range(1, (c + 1) * chunk), bpf)", ["train_select"]),
    ("training masks: sinks among the candidates", "earlier = frame_blocks(range(1, c * chunk), bpf)",
     "earlier = frame_blocks(range(0, c * chunk), bpf)", ["train_select"]),
    ("k-th gap taken one place early", "return abs(float(scores[order[k - 1]]) - float(scores[order[k]]))",
     "return abs(float(scores[order[k - 2]]) - float(scores[order[k - 1]]))", ["kth_gap"]),
    ("k-th gap of zero when nothing is cut", "    if k <= 0 or k >= len(order):\n        return float(\"inf\")",
     "    if k <= 0 or k >= len(order):\n        return 0.0", ["kth_gap"]),
    ("EMA boundary gap absolute instead of relative",
     "return abs(vals[free - 1] - vals[free]) / max(abs(vals[free - 1]), 1e-30)",
     "return abs(vals[free - 1] - vals[free])", ["ema_gap"]),
    ("EMA boundary gap ranks the sinks too", "vals = sorted((float(ema[i]) for i in range(len(pool_gids)) if not sink[i]), reverse=True)",
     "vals = sorted((float(ema[i]) for i in range(len(pool_gids))), reverse=True)", ["ema_gap"]),
    ("EMA boundary gap one place late", "return abs(vals[free - 1] - vals[free]) / max(abs(vals[free - 1]), 1e-30)",
     "return abs(vals[free] - vals[min(free + 1, len(vals) - 1)]) / max(abs(vals[free]), 1e-30)", ["ema_gap"]),
]


def _mutant(old: str, new: str) -> types.ModuleType:
    assert SRC.count(old) == 1, f"the planted mistake must replace exactly one spot: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(SRC.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("what,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_a_planted_mistake_fails_a_pin(what, old, new, pins, monkeypatch):
    mod = _mutant(old, new)
    for name, val in vars(mod).items():
        if getattr(val, "__module__", None) == "oracle_mutant":
            monkeypatch.setattr(O, name, val)
    caught = []
    for pin in pins:
        try:
            PINS[pin]()
        except Exception:   # an assertion, or the mistake breaking a shape
            caught.append(pin)
    assert caught, f"no pin caught: {what}"


def test_the_unmutated_oracle_passes_the_same_pins():
    for pin in sorted({p for m in MUTANTS for p in m[3]}):
        PINS[pin]()
