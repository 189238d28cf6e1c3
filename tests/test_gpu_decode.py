"""End-to-end GPU parity of a chunk decode and of rollouts (through PBSALayerCache and the
C-ABI) against the oracle's own plan computed from the same raw Q/K/V."""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import inputs as I
from oracle import pbsa_oracle as O
from tests._util import (EMA_NEAR_TIE_REL, F32_MAX_ABS, NEAR_TIE, assert_bf16_close, block_rows, f64,
                         geom_dict)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def layer_cfg(w, staging=0, hsa=None, own_chunk=False, max_topk=-1):
    top, recent = hsa if hsa is not None else (-1, 1)
    return P.LayerConfig(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.capacity,
                         w.window_frames, w.chunk_frames, w.topk, w.gamma, w.dtype, staging,
                         hsa_top_frames=top, hsa_recent=recent, own_chunk=own_chunk, max_topk=max_topk)


def _decode_single_step(w, sample_units=None, hsa=None, own_chunk=False):
    """One chunk decode against the oracle's plan.  ``hsa`` = (top_frames, recent frames)
    selects with the two-level policy (through the one-launch blockify + selection);
    otherwise the flat top-k through the two-call path."""
    q, k, v = I.single_step(w)
    kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
    vc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 5))
    bpf = w.blocks_per_frame
    cache = P.PBSALayerCache(layer_cfg(w, (w.hist_frames - w.window_frames) * bpf, hsa, own_chunk))
    qd = q.to(DEV)
    q_reps = cache.query_reps(qd)
    cache.prefill(k.to(DEV), v.to(DEV), w.hist_frames, q_reps)
    P_gpu = cache.persistent_gids()
    lse = torch.zeros((w.heads, qd.shape[0]), device=DEV)
    if own_chunk:   # the step's K, V (here the chunk's committed ones) are attended as well
        o = cache.decode_step(qd, kc.to(DEV), vc.to(DEV), lse=lse)
        kv_slot, kv_cnt = cache.kv_slot, cache.kv_cnt
    else:
        if hsa is None:
            kv_slot, kv_cnt, ld = cache.select(q_reps)
        else:
            _, kv_slot, kv_cnt, ld = cache.query_select(qd)
        o = cache.attend(qd, kv_slot, kv_cnt, ld, lse=lse)
    s2g = cache.slot_to_gid()
    slot_gid = cache.slot_gid.cpu()
    kv_slot, kv_cnt, o, lse = kv_slot.cpu(), kv_cnt.cpu(), o.cpu(), lse.cpu()
    assert P.pbsa_get_device_error(cache.ws) == 0
    cache.commit(kc.to(DEV), vc.to(DEV))
    P2_gpu = cache.persistent_gids()
    assert P.pbsa_get_device_error(cache.ws) == 0

    q64, k64, v64 = f64(q), f64(k), f64(v)
    own = list(range(w.hist_frames * bpf, (w.hist_frames + w.chunk_frames) * bpf)) if own_chunk else []
    if own_chunk:   # K, V of the history followed by the chunk's
        k64, v64 = np.concatenate([k64, f64(kc)]), np.concatenate([v64, f64(vc)])
    gd = geom_dict(w)
    plan = O.single_step_plan(q64, k64, gd, w.hist_frames, w.chunk_frames, w.capacity,
                              w.window_frames, w.topk, w.gamma, k_chunk=f64(kc))
    if hsa is not None:   # replace the flat selections by the two-level ones
        qr64, kr64, local = O.block_reps(q64, gd, w.chunk_frames), O.block_reps(k64, gd, w.hist_frames), plan["local"]
        for h in range(w.heads):
            for r in range(qr64.shape[1]):
                pos, fgap, bgap = O.hsa_select(qr64[h, r], kr64[h][local], local, bpf, hsa[0], hsa[1], w.topk, gd["scale"])
                plan["sel"][h][r] = [local[i] for i in pos]
                plan["sel_gap"][h][r] = min(fgap, bgap)
    nq = w.chunk_frames * bpf
    units = [(h, r) for h in range(w.heads) for r in range(nq)]
    if sample_units is not None:
        units = [units[i] for i in np.random.default_rng(0).choice(len(units), sample_units, replace=False)]
    compared = 0
    for h in range(w.heads):
        boot_exact = plan["boot_gap"][h] > EMA_NEAR_TIE_REL
        if boot_exact:
            assert P_gpu[h] == set(plan["P"][h])
        assert len(P_gpu[h]) == w.capacity and set(range(bpf)) <= P_gpu[h]
        pers_slot_gid = {s: int(slot_gid[h, s]) for s in range(w.capacity) if slot_gid[h, s] >= 0}
        for r in range(nq):
            n = int(kv_cnt[h, r])
            slots = kv_slot[h, r, :n].tolist()
            own_s2g = {int(x): own[i] for i, x in enumerate(cache._frames_dst(w.hist_frames, w.chunk_frames).cpu())} \
                if own_chunk else {}
            gids = [pers_slot_gid[s] if s < w.capacity else (own_s2g[s] if s in own_s2g else s2g[s]) for s in slots]
            if own_chunk:
                assert gids[len(gids) - len(own):] == own
                gids = gids[:len(gids) - len(own)]
            sel = set(gids[len(pers_slot_gid):])
            if plan["sel_gap"][h][r] > NEAR_TIE:
                assert sel == set(plan["sel"][h][r]), (h, r)
            if (h, r) in units and boot_exact and plan["sel_gap"][h][r] > NEAR_TIE:
                want, wlse = O.attend_gids(q64, k64, v64, gd, h, r, plan["P"][h] + plan["sel"][h][r] + own,
                                           q_first_frame=w.hist_frames)
                rows = block_rows(w, r)
                if w.dtype == "f32":
                    np.testing.assert_allclose(f64(o[rows, h]), want, rtol=0, atol=F32_MAX_ABS)
                else:
                    assert_bf16_close(f64(o[rows, h]), want, f"h{h} r{r}")
                np.testing.assert_allclose(f64(lse[h, rows]), wlse, rtol=0, atol=2e-3)
                compared += 1
        if plan["P2_gap"][h] > EMA_NEAR_TIE_REL and boot_exact:
            assert P2_gpu[h] == set(plan["P2"][h])
    assert compared >= len(units) // 2


def test_decode_tiny_f32():
    _decode_single_step(I.TINY)


def test_decode_5s_last_chunk_bf16():
    """All 864 (head, query block) units of the 5 s last-chunk decode: selections, O and LSE."""
    _decode_single_step(I.DECODE_5S)


def test_decode_5s_last_chunk_hierarchical_selection():
    _decode_single_step(I.DECODE_5S, sample_units=24, hsa=(3, 1))


def test_decode_tiny_hierarchical_selection():
    _decode_single_step(I.TINY, hsa=(0, 1))


def test_decode_5s_last_chunk_own_chunk():
    _decode_single_step(I.DECODE_5S, sample_units=24, own_chunk=True)


def test_decode_tiny_own_chunk():
    _decode_single_step(I.TINY, own_chunk=True)


def _unit_kv(store, gd, bpf, h, gids):
    """Keys and values (float64 [64 * len(gids), d]) of head h's blocks ``gids`` from the per-frame
    raster store {frame: (k, v)}."""
    ks, vs = [], []
    for g in gids:
        kf, vf = store[g // bpf]
        rows = O.block_token_rows(gd["frame_h"], gd["frame_w"], gd["tile_h"], gd["tile_w"], g % bpf)
        ks.append(f64(kf[rows, h]))
        vs.append(f64(vf[rows, h]))
    return np.concatenate(ks), np.concatenate(vs)


def _adopt_near_tie(ro, h, got, w):
    """The oracle's update of head h ended in a near tie at the top-(C - S) EMA boundary, so either
    side of it is a correct persistent set.  Check that the GPU's set differs from the oracle's only
    by blocks whose EMA lies at the boundary (relative 2x the near-tie band), then continue the
    oracle from the GPU's set, with the oracle's own EMA values.  Returns the number of swaps."""
    pool_ema = ro.last_pool_ema[h]
    want = set(ro.P[h])
    assert len(got) == len(want) and set(range(w.blocks_per_frame)) <= got and got <= set(pool_ema)
    kept_ns = [pool_ema[g] for g in want if g >= w.blocks_per_frame]
    edge = min(kept_ns)
    for g in got ^ want:
        assert abs(pool_ema[g] - edge) <= 2 * EMA_NEAR_TIE_REL * edge, (h, g, pool_ema[g], edge)
    ro.P[h] = {g: pool_ema[g] for g in got}
    return len(got - want)


def _rollout(w, n_chunks, sample_every=3, k_schedule=None):
    """Layer-0 rollout: GPU cache vs the oracle state machine, chunk by chunk, for every head.
    Per chunk: the attended sets of every (head, query block) outside near ties, the persistent
    set of every head after the memory update, O of one query block per head on the sampled
    chunks, and the cache's device memory (flat).  Where the update's boundary is a near tie the
    oracle adopts the GPU's (checked) choice and goes on.  The host keeps only the frames some
    head can still attend.  ``k_schedule``: a local top-k per chunk (set on both sides)."""
    bpf = w.blocks_per_frame
    cache = P.PBSALayerCache(layer_cfg(w, max_topk=w.window_frames * bpf if k_schedule else -1))
    ro = O.RolloutOracle(geom_dict(w), w.heads, w.capacity, w.window_frames, w.topk, w.gamma)
    gd = geom_dict(w)
    offsets = ([I.ar1_offsets(w, w.total_frames, I.stream_seed(w.seed, 99, t)) for t in range(3)]
               if w.ar_rho > 0 else None)
    store = {}          # frame -> (k, v) raster bf16 on the host, while some head may attend it
    kv_bytes0 = cache.kv_bytes
    live_bytes = []
    swaps = sampled = 0
    chunks = I.rollout_chunks(w)[:n_chunks]
    for c, (f0, nf) in enumerate(chunks):
        assert nf == w.chunk_frames or c == 0
        if k_schedule is not None:
            cache.set_topk(k_schedule[c])
            ro.k = k_schedule[c]
        wc = dataclasses.replace(w, chunk_frames=nf)
        for s in range(w.steps):
            seeds = [I.stream_seed(w.seed, c, s, t) for t in range(3)]
            if offsets is not None:
                q, k, v = (I.tokens_with_offsets(w, off[f0:f0 + nf], sd) for off, sd in zip(offsets, seeds))
            else:
                q, k, v = (I.tokens(wc, nf, sd) for sd in seeds)
            o = cache.decode_step(q.to(DEV), k.to(DEV), v.to(DEV)).cpu()
            q64 = f64(q)
            q_reps = O.block_reps(q64, gd, nf)
            sel = ro.select(q_reps)
            if sel is None and s == w.steps - 1:
                # empty history: the chunk attends its own blocks (this step's K, V)
                own = list(range(f0 * bpf, (f0 + nf) * bpf))
                r = c % q_reps.shape[1]
                for h in range(w.heads):
                    want, _ = O.attend_gids(q64, f64(k), f64(v), gd, h, r, own, q_first_frame=f0)
                    assert_bf16_close(f64(o[block_rows(wc, r), h]), want, f"own c{c} h{h}")
            if sel is not None:
                kv_slot, kv_cnt = cache.kv_slot.cpu(), cache.kv_cnt.cpu()
                s2g = cache.slot_to_gid()
                sg = cache.slot_gid.cpu()
                r_sample = (c * 7 + s) % q_reps.shape[1]
                for h in range(w.heads):
                    pers = {int(x) for x in sg[h] if x >= 0}
                    assert pers == set(ro.P[h]), (c, s, h)
                    for r in range(q_reps.shape[1]):
                        gids_want, gap = sel[h][r]
                        n = int(kv_cnt[h, r])
                        slots = kv_slot[h, r, :n].tolist()
                        got = [int(sg[h, x]) if x < w.capacity else s2g[x] for x in slots]
                        assert len(set(got)) == len(got) and pers <= set(got)
                        if gap > NEAR_TIE:
                            assert set(got) == set(gids_want), (c, s, h, r)
                        else:
                            assert len(got) == len(gids_want) and set(got) - pers <= set(ro.local())
                        if c % sample_every == 0 and r == r_sample:
                            kk, vv = _unit_kv(store, gd, bpf, h, sorted(got))
                            want, _ = O.attention(q64[block_rows(wc, r), h], kk, vv, w.scale)
                            assert_bf16_close(f64(o[block_rows(wc, r), h]), want, f"c{c} h{h} r{r}")
                            sampled += 1
        cache.commit(k.to(DEV), v.to(DEV))
        assert P.pbsa_get_device_error(cache.ws) == 0
        for i in range(nf):
            rows = slice(i * w.tokens_per_frame, (i + 1) * w.tokens_per_frame)
            store[f0 + i] = (k[rows].clone(), v[rows].clone())
        ro.commit(f0, nf, O.block_reps(f64(k), gd, nf), q_reps)
        got_P = cache.persistent_gids()
        for h in range(w.heads):
            assert len(got_P[h]) <= w.capacity and set(range(bpf)) <= got_P[h]
            if ro.last_gap[h] > EMA_NEAR_TIE_REL:
                assert got_P[h] == set(ro.P[h]), (c, h)
            elif got_P[h] != set(ro.P[h]):
                swaps += _adopt_near_tie(ro, h, got_P[h], w)
        # the host keeps the frames still in a persistent set or in the window
        keep = {g // bpf for h in range(w.heads) for g in ro.P[h]} | {g // bpf for g in ro.local()}
        for f in [f for f in store if f not in keep]:
            del store[f]
        # KV memory stays flat: the same cache size, and no device memory that grows per chunk
        assert cache.kv_bytes == kv_bytes0
        del o, q, k, v
        torch.cuda.synchronize()
        live_bytes.append(torch.cuda.memory_allocated())
    assert sampled >= w.heads * (len(chunks) // sample_every) // 2
    steady = live_bytes[min(8, len(live_bytes) - 1):]   # once the index-list memo is full
    assert max(steady) == min(steady), live_bytes
    return swaps


def test_decode_step_is_deterministic():
    """The 5 s chunk decode (fused selection, attention, overlapped memory-update plan and commit,
    copies) run twice from the same state gives bit-identical lists, O and cache."""
    w = I.DECODE_5S
    q, k, v = I.single_step(w)
    kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
    vc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 5))
    bpf = w.blocks_per_frame
    cache = P.PBSALayerCache(layer_cfg(w, (w.hist_frames - w.window_frames) * bpf))
    qd, kcd, vcd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    cache.prefill(k.to(DEV), v.to(DEV), w.hist_frames, cache.query_reps(qd))
    step = P.ChunkDecodeStep(cache)
    snap = step.snapshot()
    runs = []
    for _ in range(2):
        step.restore(snap)
        o = torch.empty_like(qd)
        step.run(qd, kcd, vcd, o)
        torch.cuda.synchronize()
        runs.append([o.clone(), step.kv_slot.clone(), step.kv_cnt.clone()] +
                    [getattr(cache, n).clone() for n in ("slot_gid", "slot_ema", "k_pool", "v_pool", "k_reps")])
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    assert P.pbsa_get_device_error(cache.ws) == 0


def test_rollout_overlapped_commit_matches_serial():
    """Each chunk committed right after its last-step attention with the overlap (the write of
    the chunk and the memory update's plan as programmatic dependents of attend) gives the same
    outputs and the same cache, bit for bit, as the same kernels run in series."""
    w = I.ROLLOUT_5S
    caches = [P.PBSALayerCache(layer_cfg(w)) for _ in range(2)]   # [serial, overlapped]
    for c, (f0, nf) in enumerate(I.rollout_chunks(w)):
        wc = dataclasses.replace(w, chunk_frames=nf)
        for s in range(w.steps):
            q, k, v = (I.tokens(wc, nf, I.stream_seed(w.seed, c, s, t)).to(DEV) for t in range(3))
            outs = []
            for i, ca in enumerate(caches):
                outs.append(ca.decode_step(q, k, v))
                if s == w.steps - 1:
                    ca.commit(k, v, overlap=i == 1, split=i == 0)
            torch.cuda.synchronize()
            assert torch.equal(outs[0], outs[1]), (c, s)
        a, b = caches
        for name in ("slot_gid", "slot_ema", "k_pool", "v_pool", "k_reps", "p_list", "p_cnt"):
            assert torch.equal(getattr(a, name), getattr(b, name)), (c, name)
        for ca in caches:
            assert P.pbsa_get_device_error(ca.ws) == 0


def test_rollout_5s_layer0():
    _rollout(I.ROLLOUT_5S, n_chunks=7)


def test_rollout_5s_layer0_chunk_topk_schedule():
    """The 5 s rollout with a per-chunk local top-k from the chunk-aware-growth schedule."""
    from block_sparse_attention_pbsa_b200 import schedule as S
    w = I.ROLLOUT_5S
    ks, _, _ = S.rollout_topk(I.rollout_chunks(w), w.tokens_per_frame, w.blocks_per_frame, w.head_dim,
                              w.capacity, w.window_frames, 0.7, 0.5)
    assert len(set(ks[1:])) > 2       # the schedule really varies
    _rollout(w, n_chunks=7, k_schedule=ks)


@pytest.mark.slow
def test_rollout_1min_layer0_every_chunk():
    """The 1-minute rollout (241 frames: frame 0, then 80 chunks of 3 frames; AR(1) tile offsets,
    so the persistent sets churn), layer 0, all 81 chunks: attended sets, persistent sets after
    every update, sampled O, and flat KV memory, against the oracle state machine."""
    w = I.ROLLOUT_1MIN
    assert len(I.rollout_chunks(w)) == 81
    _rollout(w, n_chunks=81, sample_every=2)


def test_chunk_decode_step_needs_a_history():
    """The first chunk attends its own blocks (decode_step + commit); a step object refuses it."""
    w = I.ROLLOUT_5S
    cache = P.PBSALayerCache(layer_cfg(w))
    with pytest.raises(ValueError):
        P.ChunkDecodeStep(cache)


def test_pipelined_host_step_matches_the_graph_step():
    """ChunkDecodeStep.run_pipelined (one graph with the transfers: the selection and attention
    behind the upload of Q, as a whole or frame by frame, O downloaded behind them, the memory
    update ahead of the commit of K and V) gives the same O and the same cache, bit for bit,
    as the single-graph step on the same inputs."""
    w = I.DECODE_5S
    q, k, v = I.single_step(w)
    kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
    vc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 5))
    bpf = w.blocks_per_frame
    cache = P.PBSALayerCache(layer_cfg(w, (w.hist_frames - w.window_frames) * bpf))
    qd, kcd, vcd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    cache.prefill(k.to(DEV), v.to(DEV), w.hist_frames, cache.query_reps(qd))
    step = P.ChunkDecodeStep(cache)
    snap = step.snapshot()
    o = torch.empty_like(qd)
    step.run(qd, kcd, vcd, o)
    want_o = o.cpu()
    names = ("slot_gid", "slot_ema", "k_pool", "v_pool", "k_reps", "p_list", "p_cnt")
    want = [getattr(cache, n).cpu() for n in names]
    step.restore(snap)
    qb, kb, vb, ob = (torch.empty_like(t) for t in (qd, kcd, vcd, o))
    qh, kh, vh = (t.pin_memory() for t in (q, kc, vc))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    for parts in (1, 3):
        step.restore(snap)
        step.capture_pipeline(qb, kb, vb, ob, qh, kh, vh, oh, parts=parts)
        for _ in range(2):
            step.restore(snap)
            oh.zero_()
            step.run_pipelined(qh, kh, vh, oh)
            torch.cuda.synchronize()
            assert torch.equal(oh, want_o), parts
            for n, t in zip(names, want):
                assert torch.equal(getattr(cache, n).cpu(), t), (parts, n)
    assert P.pbsa_get_device_error(cache.ws) == 0


@pytest.mark.parametrize("world", [3, 5])
def test_head_sharded_caches_match_the_whole_layer(world):
    """The layer split by heads over ``world`` ranks (each rank its heads' cache, inputs and
    kernels; here the ranks run one after another on one GPU, with no waits between them):
    over five chunks of the 5 s rollout the ranks' outputs and caches equal the whole layer's
    heads, bit for bit."""
    from block_sparse_attention_pbsa_b200 import shard
    w = I.ROLLOUT_5S
    full = P.PBSALayerCache(layer_cfg(w))
    parts = [P.PBSALayerCache(shard.local_config(layer_cfg(w), world, r)) for r in range(world)]
    for c, (f0, nf) in enumerate(I.rollout_chunks(w)[:5]):
        wc = dataclasses.replace(w, chunk_frames=nf)
        for s in range(2):
            q, k, v = (I.tokens(wc, nf, I.stream_seed(w.seed, c, s, t)).to(DEV) for t in range(3))
            o = full.decode_step(q, k, v)
            for r, ca in enumerate(parts):
                h0, h1 = shard.head_range(w.heads, world, r)
                qs, ks, vs = (shard.head_slice(t, w.heads, world, r) for t in (q, k, v))
                assert torch.equal(ca.decode_step(qs, ks, vs), o[:, h0:h1]), (c, s, r)
                if s == 1:
                    ca.commit(ks, vs)
            if s == 1:
                full.commit(k, v)
        for r, ca in enumerate(parts):
            h0, h1 = shard.head_range(w.heads, world, r)
            for name in ("slot_gid", "slot_ema", "k_pool", "v_pool", "k_reps", "p_list", "p_cnt"):
                assert torch.equal(getattr(ca, name), getattr(full, name)[h0:h1]), (c, r, name)
            assert P.pbsa_get_device_error(ca.ws) == 0


def test_rollout_resumes_from_a_checkpoint():
    """A 5 s rollout checkpointed after its fourth chunk (state copied to the host) and resumed in
    a fresh cache gives the same outputs and the same cache, bit for bit, over the remaining
    chunks as the uninterrupted rollout."""
    w = I.ROLLOUT_5S
    chunks = I.rollout_chunks(w)
    inputs = {}

    def step(ca, c, s):
        f0, nf = chunks[c]
        wc = dataclasses.replace(w, chunk_frames=nf)
        if (c, s) not in inputs:
            inputs[c, s] = [I.tokens(wc, nf, I.stream_seed(w.seed, c, s, t)).to(DEV) for t in range(3)]
        q, k, v = inputs[c, s]
        o = ca.decode_step(q, k, v)
        if s == 1:
            ca.commit(k, v)
        return o

    full = P.PBSALayerCache(layer_cfg(w))
    for c in range(4):
        for s in range(2):
            step(full, c, s)
    ckpt = full.state_dict()
    assert all(t.device.type == "cpu" for t in ckpt.values() if isinstance(t, torch.Tensor))
    resumed = P.PBSALayerCache(layer_cfg(w))
    resumed.load_state_dict(ckpt)
    for c in range(4, len(chunks)):
        for s in range(2):
            assert torch.equal(step(full, c, s), step(resumed, c, s)), (c, s)
    for name in P.PBSALayerCache._STATE:
        assert torch.equal(getattr(full, name), getattr(resumed, name)), name
    assert resumed.hist == full.hist
    with pytest.raises(ValueError):
        P.PBSALayerCache(dataclasses.replace(layer_cfg(w), capacity=48)).load_state_dict(ckpt)
    assert P.pbsa_get_device_error(full.ws) == 0 and P.pbsa_get_device_error(resumed.ws) == 0
