"""Pins of the CPU oracle against the mathematics (closed forms, brute force, library
routines, invariants).  No GPU needed."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import pbsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def geom(fh=16, fw=24, th=8, tw=8, d=8):
    return {"frame_h": fh, "frame_w": fw, "tile_h": th, "tile_w": tw, "scale": 1.0 / math.sqrt(d)}


# ------------------------------------------------------------------ representatives
@pytest.mark.parametrize("th,tw", [(8, 8), (4, 16), (16, 4)])
def test_block_reps_closed_form(th, tw):
    g = geom(16, 32, th, tw)
    n_frames, H, d = 2, 3, 4
    fh, fw = g["frame_h"], g["frame_w"]
    x = np.zeros((n_frames * fh * fw, H, d))
    for f in range(n_frames):
        for y in range(fh):
            for xx in range(fw):
                t = f * fh * fw + y * fw + xx
                for h in range(H):
                    x[t, h, :] = f * 1000 + y * fw + xx + 0.5 * h + 0.25 * np.arange(d)
    reps = O.block_reps(x, g, n_frames)
    tpr, bpf = fw // tw, (fh // th) * (fw // tw)
    assert reps.shape == (H, n_frames * bpf, d)
    for b in range(n_frames * bpf):
        f, rem = divmod(b, bpf)
        ty, tx = divmod(rem, tpr)
        # mean of y over the tile rows and of x over the tile columns
        my, mx = ty * th + (th - 1) / 2, tx * tw + (tw - 1) / 2
        for h in range(H):
            want = f * 1000 + my * fw + mx + 0.5 * h + 0.25 * np.arange(d)
            np.testing.assert_allclose(reps[h, b], want, rtol=0, atol=1e-9)


def test_block_rows_cover_frame_once():
    g = geom(32, 48)
    seen = np.concatenate([O.block_token_rows(32, 48, 8, 8, b) for b in range(2 * 24)])
    assert sorted(seen.tolist()) == list(range(2 * 32 * 48))


# ------------------------------------------------------------------ selection
def test_topk_ties_go_to_lower_id():
    scores = np.zeros(10, np.float32)
    gids = [17, 3, 9, 11, 4, 8, 30, 1, 2, 5]
    got = [gids[i] for i in O.topk_select(scores, gids, 4)]
    assert got == [1, 2, 3, 4]


def test_topk_brute_force_and_permutation():
    rng = np.random.default_rng(0)
    for trial in range(50):
        n, k = int(rng.integers(1, 9)), int(rng.integers(1, 6))
        sc = rng.integers(-3, 3, n).astype(np.float32)  # many exact ties
        gids = rng.permutation(100)[:n].tolist()
        sel = {gids[i] for i in O.topk_select(sc, gids, k)}
        # brute force: the chosen set is the lexicographically best k-subset under
        # (score desc, gid asc) -- every chosen one beats every unchosen one
        best = None
        for comb in itertools.combinations(range(n), min(k, n)):
            key = sorted(((-float(sc[i]), gids[i]) for i in comb))
            if best is None or key < best[0]:
                best = (key, {gids[i] for i in comb})
        assert sel == best[1]
        perm = rng.permutation(n)
        sel2 = {gids[perm[i]] for i in O.topk_select(sc[perm], [gids[j] for j in perm], k)}
        assert sel2 == sel


# ------------------------------------------------------------------ attention
def _sdpa64(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)[0, 0].numpy()


def test_all_blocks_selected_is_dense_attention():
    g = geom(16, 16, 8, 8, d=64)
    rng = np.random.default_rng(1)
    hist, chunk, H, d = 6, 1, 2, 64
    q = rng.standard_normal((chunk * 256, H, d))
    k = rng.standard_normal((hist * 256, H, d))
    v = rng.standard_normal((hist * 256, H, d))
    # capacity holds sinks + every middle block, top-k takes the whole window
    plan = O.single_step_plan(q, k, g, hist, chunk, capacity=4 + 12, window=2, topk=8, gamma=0.9)
    for h in range(H):
        for r in range(4):
            gids = plan["P"][h] + plan["sel"][h][r]
            assert sorted(gids) == list(range(24))
            out, lse = O.attend_gids(q, k, v, g, h, r, gids, q_first_frame=hist)
            qb = O.block_tokens(q, g, hist * 4 + r, hist)[:, h]
            ref = _sdpa64(qb, k[:, h], v[:, h], g["scale"])
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
            logits = g["scale"] * qb @ k[:, h].T
            np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(logits), 1).numpy(),
                                       rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one_and_convex_hull():
    rng = np.random.default_rng(2)
    n, m = 5, 12
    q = rng.standard_normal((n, 7)) * 3
    k = rng.standard_normal((m, 7)) * 3
    eye = np.eye(m)
    p, _ = O.attention(q, k, eye, 0.5)          # V = identity -> out is the softmax matrix
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    assert (p > 0).all()
    v = rng.standard_normal((m, 3))
    out, _ = O.attention(q, k, v, 0.5)
    assert (out <= v.max(axis=0) + 1e-12).all() and (out >= v.min(axis=0) - 1e-12).all()
    perm = rng.permutation(m)
    out2, _ = O.attention(q, k[perm], v[perm], 0.5)
    np.testing.assert_allclose(out, out2, atol=1e-13)


def test_empty_key_set():
    out, lse = O.attention(np.ones((3, 4)), np.zeros((0, 4)), np.zeros((0, 4)), 1.0)
    assert (out == 0).all() and np.isneginf(lse).all()


# ------------------------------------------------------------------ backward
def test_backward_finite_differences():
    rng = np.random.default_rng(3)
    n, m, d = 4, 6, 5
    q, k, v, do = (rng.standard_normal(s) for s in ((n, d), (m, d), (m, d), (n, d)))
    scale = 0.7
    dq, dk, dv = O.attention_bwd(q, k, v, do, scale)
    f = lambda q_, k_, v_: float((O.attention(q_, k_, v_, scale)[0] * do).sum())
    eps = 1e-6
    for name, a, g_ in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            ap, am = a.copy(), a.copy()
            ap[idx] += eps
            am[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = ap, am
            num[idx] = (f(args_p["q"], args_p["k"], args_p["v"])
                        - f(args_m["q"], args_m["k"], args_m["v"])) / (2 * eps)
        np.testing.assert_allclose(g_, num, rtol=1e-6, atol=1e-8)


# ------------------------------------------------------------------ memory update
def test_memory_update_closed_form():
    fx = json.load(open(os.path.join(GOLDEN, "memory_update_closed_form.json")))
    prev = [np.nan if p is None else p for p in fx["prev_ema"]]
    ema, keep, a = O.memory_update(np.array(fx["q_reps"]), np.array(fx["pool_reps"]), fx["pool_gids"],
                                   prev, fx["is_sink"], 1.0, fx["gamma"], fx["capacity"])
    np.testing.assert_allclose(a, fx["expected_a"], atol=1e-15)
    np.testing.assert_allclose(ema, fx["expected_ema"], atol=1e-15)
    assert keep.tolist() == fx["expected_keep"]


def test_memory_update_closed_form_with_the_attention_scale():
    """d = 4: the scale 1/2 enters the softmax (the d = 1 fixture above cannot see it)."""
    fx = json.load(open(os.path.join(GOLDEN, "memory_update_closed_form_scaled.json")))
    d = len(fx["q_reps"][0])
    assert fx["scale"] == 1.0 / math.sqrt(d)
    prev = [np.nan if p is None else p for p in fx["prev_ema"]]
    ema, keep, a = O.memory_update(np.array(fx["q_reps"]), np.array(fx["pool_reps"]), fx["pool_gids"],
                                   prev, fx["is_sink"], fx["scale"], fx["gamma"], fx["capacity"])
    np.testing.assert_allclose(a, fx["expected_a"], atol=1e-15)
    np.testing.assert_allclose(ema, fx["expected_ema"], atol=1e-15)
    assert keep.tolist() == fx["expected_keep"]


def test_memory_update_invariants():
    rng = np.random.default_rng(4)
    for trial in range(30):
        nq, nb, d = int(rng.integers(1, 6)), int(rng.integers(2, 30)), 8
        n_sink = int(rng.integers(0, min(nb, 5) + 1))
        C = int(rng.integers(n_sink, nb + 3))
        qr, pr = rng.standard_normal((nq, d)), rng.standard_normal((nb, d))
        gids = rng.permutation(1000)[:nb].tolist()
        sink = [i < n_sink for i in range(nb)]
        prev = np.where(rng.random(nb) < 0.5, np.nan, rng.random(nb) * 0.1)
        ema, keep, a = O.memory_update(qr, pr, gids, prev, sink, 0.3, 0.9, C)
        assert abs(a.sum() - 1.0) < 1e-12
        assert keep.sum() <= C and all(keep[i] for i in range(n_sink))
        if C >= nb:
            assert keep.all()
        dropped = [ema[i] for i in range(nb) if not keep[i]]
        kept_ns = [ema[i] for i in range(nb) if keep[i] and not sink[i]]
        if dropped and kept_ns:
            assert min(kept_ns) >= max(dropped)
    # a constant score stream is a fixed point of the EMA
    qr, pr = rng.standard_normal((3, 8)), rng.standard_normal((5, 8))
    _, _, a = O.memory_update(qr, pr, list(range(5)), [np.nan] * 5, [False] * 5, 0.3, 0.9, 5)
    ema, _, _ = O.memory_update(qr, pr, list(range(5)), a, [False] * 5, 0.3, 0.9, 5)
    np.testing.assert_allclose(ema, a, atol=1e-15)


def test_memory_update_equal_ema_ties_to_lower_id():
    pr = np.zeros((4, 2))
    ema, keep, _ = O.memory_update(np.ones((1, 2)), pr, [9, 7, 8, 6], [np.nan] * 4,
                                   [False] * 4, 1.0, 0.9, 2)
    assert {g for g, kp in zip([9, 7, 8, 6], keep) if kp} == {6, 7}


# ------------------------------------------------------------------ workload plans
def test_rollout_windows_and_capacity_5s():
    """5 s rollout shapes: 24 blocks/frame, chunks of 3 frames, W = 6, C = 96."""
    g = geom(32, 48, 8, 8, d=4)
    ro = O.RolloutOracle(g, heads=1, capacity=96, window=6, topk=32, gamma=0.9)
    rng = np.random.default_rng(5)
    local_sizes, p_sizes, evicted = [], [], []
    for c in range(7):
        f0 = 3 * c
        local_sizes.append(len(ro.local()))
        q = rng.standard_normal((1, 72, 4))
        sel = ro.select(q)
        if c == 0:
            assert sel is None
        else:
            assert len(sel[0][0][0]) == len(ro.P[0]) + min(32, len(ro.local()))
        ev = ro.commit(f0, 3, rng.standard_normal((1, 72, 4)), q)
        evicted.append(sorted({b // 24 for b in ev}))
        p_sizes.append(len(ro.P[0]))
        assert set(range(24)) <= set(ro.P[0]) and len(ro.P[0]) <= 96
    assert local_sizes == [0, 48, 120, 144, 144, 144, 144]
    assert evicted == [[], [], [1, 2], [3, 4, 5], [6, 7, 8], [9, 10, 11], [12, 13, 14]]
    assert p_sizes[:3] == [24, 24, 72] and all(p == 96 for p in p_sizes[3:])


def test_rollout_carries_the_ema_between_updates():
    """A block kept by two consecutive updates ends with EMA gamma * (its EMA before) + (1 - gamma)
    * a, a its attention share in the second update (that update's value with no history)."""
    g = geom(32, 48, 8, 8, d=4)
    ro = O.RolloutOracle(g, heads=1, capacity=96, window=6, topk=32, gamma=0.9)
    rng = np.random.default_rng(9)
    for c in range(4):
        ro.commit(3 * c, 3, rng.standard_normal((1, 72, 4)), rng.standard_normal((1, 72, 4)))
    before = dict(ro.P[0])
    q = rng.standard_normal((1, 72, 4))
    evicted = ro.commit(12, 3, rng.standard_normal((1, 72, 4)), q)
    pool = sorted(before) + evicted
    reps = np.stack([ro.kreps[gg][0] for gg in pool])
    _, _, a = O.memory_update(q[0], reps, pool, [np.nan] * len(pool), [gg < 24 for gg in pool],
                              g["scale"], 0.9, 96)
    carried = [gg for gg in before if gg in ro.P[0]]
    assert len(carried) >= 24
    for gg in carried:
        want = 0.9 * before[gg] + 0.1 * a[pool.index(gg)]
        assert abs(ro.P[0][gg] - want) <= 1e-12 * max(1.0, abs(want))


def test_single_step_partition_5s():
    """Last-chunk decode of the 5 s video: 18 history frames = 24 sinks + 264 middle + 144 local."""
    g = geom(32, 48, 8, 8, d=4)
    q = np.random.default_rng(6).standard_normal((3 * 1536, 1, 4))
    k = np.random.default_rng(7).standard_normal((18 * 1536, 1, 4))
    plan = O.single_step_plan(q, k, g, 18, 3, capacity=96, window=6, topk=32, gamma=0.9,
                              k_chunk=np.zeros(1))
    assert len(plan["sinks"]) == 24 and len(plan["middle"]) == 264 and len(plan["local"]) == 144
    assert plan["local"][0] == 12 * 24 and plan["middle"][-1] == 12 * 24 - 1
    assert len(plan["P"][0]) == 96 and set(range(24)) <= set(plan["P"][0])
    assert all(len(s) == 32 and set(s) <= set(plan["local"]) for s in plan["sel"][0])
    assert len(plan["P2"][0]) == 96


def test_train_masks_shape():
    g = geom(16, 16, 8, 8, d=4)      # 4 blocks per frame
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 9 * 256, 1, 4))
    k = rng.standard_normal((1, 9 * 256, 1, 4))
    masks, _ = O.train_masks(q, k, g, 9, 3, topk=2)
    m = masks[0][0]
    assert m[0] == list(range(12))
    assert len(m[12]) == 4 + 2 + 12 and set(m[12][:4]) == set(range(4))
    assert set(m[12][4:6]) <= set(range(4, 12))
    assert set(m[30][4:6]) <= set(range(4, 24))
    # 8 frames: the last chunk holds frames 6 and 7 only
    masks, _ = O.train_masks(q[:, :8 * 256], k[:, :8 * 256], g, 8, 3, topk=2)
    m = masks[0][0]
    assert len(m) == 32 and m[31][-8:] == list(range(24, 32)) and len(m[31]) == 4 + 2 + 8


def _const_block_tokens(reps, fh, fw, th, tw, n_frames):
    """Raster tokens [n_frames*fh*fw, H, d] in which every token of block b equals reps[:, b]
    (so each block's mean is exactly reps[:, b]); block of token (f, y, x) = f*bpf +
    (y // th)*(fw // tw) + x // tw, written out here independently of the oracle."""
    H, _, d = reps.shape
    x = np.zeros((n_frames * fh * fw, H, d))
    bpf = (fh // th) * (fw // tw)
    for f in range(n_frames):
        for y in range(fh):
            for xx in range(fw):
                x[f * fh * fw + y * fw + xx] = reps[:, f * bpf + (y // th) * (fw // tw) + xx // tw]
    return x


def test_train_masks_selection_hand_built():
    """Trainable-path masks on a case whose top-2 is known by construction (4 blocks per frame,
    9 frames, 3-frame chunks, batch 2).  Every block's tokens are one constant vector, so the
    representatives are exact.  Query block r scores with e_(r mod 2) * 2 (even rows rank the
    keys by their first coordinate a, odd rows by their second b; scale 1/2 undoes the 2).
    Batch 0: a = 100 on the sinks, 50 on chunk 1's blocks 12..23, 200 on chunk 2's blocks
    24..35 (each would win if sinks, the own chunk or a later chunk were candidates), and
    a[4..11] = 1, 7, 3, 7, -2, 5, 0, 7 (a three-way tie at 7 on blocks 5, 7, 11);
    b = 100 on the sinks, 300 on chunk 2, b[4] = 9, b[8] = 8, b[20] = 10, else 0.
    Batch 1 swaps a and b (its even rows see batch 0's odd-row ranking)."""
    fh, fw, th, tw, d, F, cf, bpf = 16, 16, 8, 8, 4, 9, 3, 4
    g = {"frame_h": fh, "frame_w": fw, "tile_h": th, "tile_w": tw, "scale": 0.5}
    a = np.zeros(36)
    a[0:4], a[12:24], a[24:36] = 100, 50, 200
    a[4:12] = [1, 7, 3, 7, -2, 5, 0, 7]
    b = np.zeros(36)
    b[0:4], b[24:36] = 100, 300
    b[4], b[8], b[20] = 9, 8, 10
    kreps = np.zeros((2, 1, 36, d))
    kreps[0, 0, :, 0], kreps[0, 0, :, 1] = a, b
    kreps[1, 0, :, 0], kreps[1, 0, :, 1] = b, a
    qreps = np.zeros((2, 1, 36, d))
    for r in range(36):
        qreps[:, 0, r, r % 2] = 2.0
    q = np.stack([_const_block_tokens(qreps[i], fh, fw, th, tw, F) for i in range(2)])
    k = np.stack([_const_block_tokens(kreps[i], fh, fw, th, tw, F) for i in range(2)])
    masks, gaps = O.train_masks(q, k, g, F, cf, topk=2)
    sinks = [0, 1, 2, 3]
    own = {c: list(range(12 * c, 12 * c + 12)) for c in range(3)}
    # chosen local blocks by (batch, chunk, row parity), worked out from the tables above
    want = {(0, 1, 0): [5, 7], (0, 1, 1): [4, 8], (0, 2, 0): [12, 13], (0, 2, 1): [20, 4],
            (1, 1, 0): [4, 8], (1, 1, 1): [5, 7], (1, 2, 0): [20, 4], (1, 2, 1): [12, 13]}
    # |2nd best - 3rd best|: 7 - 7; 8 - 0; 50 - 50; 9 - 8
    want_gap = {(0, 1, 0): 0.0, (0, 1, 1): 8.0, (0, 2, 0): 0.0, (0, 2, 1): 1.0,
                (1, 1, 0): 8.0, (1, 1, 1): 0.0, (1, 2, 0): 1.0, (1, 2, 1): 0.0}
    for bb in range(2):
        for r in range(36):
            c = r // 12
            m = masks[bb][0][r]
            if c == 0:
                assert m == own[0] and gaps[bb][0][r] == float("inf")
                continue
            key = (bb, c, r % 2)
            assert m[:4] == sinks and m[-12:] == own[c]
            assert sorted(m[4:-12]) == sorted(want[key]), (bb, r, m)
            assert gaps[bb][0][r] == pytest.approx(want_gap[key]), (bb, r)


def test_kth_gap_hand_values():
    """Scores 3, 1, 2.5, 2.5, -1 (gids 10..14) in ranking order: 3 | 2.5 (gid 12) | 2.5 (gid 13)
    | 1 | -1.  The gap at k is |k-th - (k+1)-th|; none when k is 0 or takes every candidate."""
    sc = np.array([3.0, 1.0, 2.5, 2.5, -1.0], np.float32)
    gids = [10, 11, 12, 13, 14]
    assert [O.kth_gap(sc, gids, k) for k in range(6)] == [float("inf"), 0.5, 0.0, 1.5, 2.0, float("inf")]


def test_ema_boundary_gap_hand_values():
    """EMA 0.5 (sink), 0.30, 0.12, 0.20, 0.03: the non-sink values ranked are 0.30, 0.20, 0.12,
    0.03 and C - 1 of them are kept; the gap is (last kept - first dropped) / last kept."""
    ema = np.array([0.5, 0.30, 0.12, 0.20, 0.03])
    gids = [0, 11, 12, 13, 14]
    sink = [True, False, False, False, False]
    got = {C: O.ema_boundary_gap(ema, gids, sink, C) for C in range(1, 6)}
    assert got[1] == float("inf") and got[5] == float("inf")
    assert got[2] == pytest.approx(0.1 / 0.3, rel=1e-12)
    assert got[3] == pytest.approx(0.08 / 0.20, rel=1e-12)
    assert got[4] == pytest.approx(0.09 / 0.12, rel=1e-12)


# ------------------------------------------------------------------ hierarchical (frame -> block) selection
def test_hsa_frames_ranked_by_mean_not_by_best_block():
    """Hand-built case: frame 0 holds the single best block but the lowest mean, frame 1 the
    best mean; frame 2 is the always-on latest frame.  With one extra frame the selection is
    frame 1's blocks then frame 2's, and frame 0's best block is left out."""
    bpf, scale = 2, 1.0
    q = np.array([1.0, 0.0])
    block_score = [10.0, -9.0, 2.0, 2.0, 0.0, 0.0]     # frame means 0.5, 2.0, 0.0
    reps = np.array([[s, 7.0] for s in block_score])
    gids = [100, 101, 102, 103, 104, 105]
    pos, fgap, bgap = O.hsa_select(q, reps, gids, bpf, top_frames=1, n_recent=1, k=3, scale=scale)
    assert pos == [2, 3, 4]                 # scores 2, 2 (lower gid first), then 0 (gid 104 < 105)
    assert fgap == pytest.approx(1.5)       # frame 1 (2.0) vs frame 0 (0.5)
    assert bgap == 0.0                      # 4th best ties with the 3rd (0 vs 0)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_hsa_reduces_to_flat_topk(seed):
    """Every frame chosen (enough extra frames, or every frame always-on) is the flat top-k."""
    rng = np.random.default_rng(seed)
    bpf, nf, d, k = 4, 6, 8, 7
    q = rng.normal(size=d)
    reps = rng.normal(size=(nf * bpf, d))
    gids = rng.permutation(1000)[:nf * bpf]
    flat = O.topk_select(O.coarse_scores(q[None], reps, 0.3)[0], gids, k)
    for top_frames, n_recent in [(nf, 1), (nf - 1, 1), (0, nf), (3, nf)]:
        pos, _, _ = O.hsa_select(q, reps, gids, bpf, top_frames, n_recent, k, 0.3)
        assert pos == flat


def test_hsa_brute_force_small():
    """Against an exhaustive restatement: frame sets by frame-mean score, then the best blocks."""
    rng = np.random.default_rng(5)
    bpf, nf, d = 3, 5, 4
    for trial in range(20):
        q = rng.normal(size=d)
        reps = rng.normal(size=(nf * bpf, d))
        gids = list(range(nf * bpf))
        top_frames, n_recent, k = int(rng.integers(0, nf)), int(rng.integers(0, 3)), int(rng.integers(1, 8))
        pos, _, _ = O.hsa_select(q, reps, gids, bpf, top_frames, n_recent, k, 1.0)
        fmean = [float(np.mean([reps[t * bpf + b] @ q for b in range(bpf)])) for t in range(nf)]
        always = set(range(max(0, nf - n_recent), nf))
        others = [t for t in range(nf) if t not in always]
        # the best subset of other frames of size top_frames by total mean score (ties unlikely)
        best = max(itertools.combinations(others, min(top_frames, len(others))),
                   key=lambda c: sum(fmean[t] for t in c), default=())
        frames = always | set(best)
        cands = sorted((c for c in range(nf * bpf) if c // bpf in frames), key=lambda c: -(reps[c] @ q))
        assert pos == cands[:k]
        # selected blocks lie in chosen frames, the latest n_recent frames are always available
        assert all(c // bpf in frames for c in pos)


# ------------------------------------------------------------------ per-chunk sparsity (chunk-aware growth)
def test_cag_meets_the_flop_budget():
    """beta solves the budget equation exactly; the dense chunks stay dense."""
    lq = [4608] * 7
    lk = [0, 4608, 9216, 13824, 18432, 23040, 27648]
    alpha = [1.0, 1.0, 0.8, 0.6, 0.4, 0.2, 0.0]
    s_base, s_target, d = 0.9, 0.8, 128
    beta, s = O.cag_sparsity(lq, lk, d, s_base, s_target, alpha, n_dense=1)
    lhs = sum((1 - s_base + alpha[i] * beta) * lq[i] * lk[i] * d for i in range(1, 7))
    rhs = (1 - s_target) * sum(lq[i] * lk[i] * d for i in range(1, 7))
    assert lhs == pytest.approx(rhs, rel=1e-12)
    assert s[0] == 0.0 and beta > 0
    # the attended share (1 - s_i) of every later chunk averages, FLOP-weighted, to 1 - s_target
    w = [lq[i] * lk[i] for i in range(1, 7)]
    assert sum((1 - s[i]) * w[i - 1] for i in range(1, 7)) / sum(w) == pytest.approx(1 - s_target, rel=1e-12)
    # larger alpha -> less sparse
    assert all(s[i] <= s[i + 1] for i in range(1, 6))


def test_cag_special_cases():
    lq, lk = [10, 10, 10], [0, 20, 40]
    beta, s = O.cag_sparsity(lq, lk, 8, 0.7, 0.7, [0.3, 0.5, 0.9])
    assert beta == 0.0 and s == [0.0, 0.7, 0.7]              # target = base: no growth
    beta, s = O.cag_sparsity(lq, lk, 8, 0.9, 0.6, [1.0, 0.5, 0.5])
    assert s[1] == pytest.approx(0.6) and s[2] == pytest.approx(0.6)   # uniform alpha: every chunk at the target


def test_cag_topk_mapping():
    assert O.cag_topk(0.0, 288, 96, 144) == 144          # dense: every local block
    assert O.cag_topk(0.5, 288, 96, 144) == 48           # 144 kept - 96 persistent
    assert O.cag_topk(0.9, 288, 96, 144) == 0            # the persistent blocks already exceed the share
    assert O.cag_topk(0.75, 100, 10, 200) == 15          # round(25) - 10
