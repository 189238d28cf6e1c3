#!/usr/bin/env python
"""PBSA chunk-decode benchmark on B200.

One step = one chunk decode of one attention layer on the 5 s-video last-chunk workload
(12 heads, d=128, 32x48-token frames in 64-token blocks, 3-frame chunk = 72 query blocks,
18 history frames, C=96 persistent blocks, 6-frame window, top-32 local blocks), i.e.
every row of the hot path: blockify(Q) -> coarse score + top-k -> block-sparse attention
(tcgen05) -> commit of the chunk's K/V (blockify into the ring) -> persistent-memory
update.  Inputs are resident in HBM before timing; L2 is flushed between timed steps;
each step is timed with CUDA events on its stream.  The state the step mutates is
restored (outside the timed region) so every step does identical work.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pbsa|reference]

N > 1 (torchrun, one rank per GPU): every rank decodes its own independent layer (weak
scaling, no collective on the data path); the step time is the max over ranks.
``--impl reference`` times the CPU oracle on the host cores on a bounded sample of the
same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "PBSA ms/chunk-decode and selected-block TFLOP/s (% of B200 bf16 peak), 1 GPU"
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                for n, v in zip(names, r[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def profiled_traffic(record: str, source: str):
    """DRAM bytes per launch from the ncu counters recorded beside the profile summaries
    (``profiles/<record>``: a small JSON with the kernel source's sha256 prefix), or None when
    the kernel source has changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            rec = json.load(f)
        sha = hashlib.sha256(open(os.path.join(ROOT, source), "rb").read()).hexdigest()[:16]
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256") != sha:
        return None
    return int(rec["dram_bytes_per_launch"])


def workload_config(w):
    return {"workload": w.name, "heads": w.heads, "head_dim": w.head_dim,
            "frame_tokens": f"{w.frame_h}x{w.frame_w}", "block": f"1 frame x {w.tile_h}x{w.tile_w}",
            "chunk_frames": w.chunk_frames, "query_blocks": w.chunk_frames * w.blocks_per_frame,
            "hist_frames": w.hist_frames, "capacity": w.capacity, "window_frames": w.window_frames,
            "topk": w.topk, "kv_blocks_per_query_block": w.capacity + w.topk,
            "l2": "flushed (256 MiB write) before every timed step"}


# ----------------------------------------------------------------------------- CPU oracle arm
def oracle_sample(w, q, k, v, units: int, seed: int = 0):
    """Time the oracle, single-threaded (BLAS pools limited to one thread), on a bounded sample of
    one chunk decode; returns (seconds extrapolated to the full step, description, threads)."""
    from threadpoolctl import threadpool_info, threadpool_limits
    from oracle import pbsa_oracle as O
    gd = {"frame_h": w.frame_h, "frame_w": w.frame_w, "tile_h": w.tile_h, "tile_w": w.tile_w, "scale": w.scale}
    q64, k64, v64 = (t.double().numpy() for t in (q, k, v))
    nq = w.chunk_frames * w.blocks_per_frame
    with threadpool_limits(limits=1):
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        t0 = time.perf_counter()
        plan = O.single_step_plan(q64, k64, gd, w.hist_frames, w.chunk_frames, w.capacity, w.window_frames,
                                  w.topk, w.gamma)
        t_plan = time.perf_counter() - t0
        rng = np.random.default_rng(seed)
        pick = rng.choice(w.heads * nq, size=units, replace=False)
        t0 = time.perf_counter()
        for u in pick:
            h, r = divmod(int(u), nq)
            O.attend_gids(q64, k64, v64, gd, h, r, plan["P"][h] + plan["sel"][h][r], q_first_frame=w.hist_frames)
        t_att = (time.perf_counter() - t0) / units
    full = t_plan + t_att * w.heads * nq
    desc = (f"single-threaded oracle: selection/update plan for all {w.heads} heads (timed whole, {t_plan:.2f}s) + "
            f"fine attention of {units} of {w.heads * nq} (head, query block) units timed and extrapolated "
            f"to all of them ({t_att * 1e3:.1f} ms per unit)")
    return full, desc, threads


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    from block_sparse_attention_pbsa_b200 import inputs as I
    q, k, v = I.single_step(w)
    flops = 4.0 * 64 * 64 * w.head_dim * w.heads * w.chunk_frames * w.blocks_per_frame * (w.capacity + w.topk)
    units = 24
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, 4)
    times = []
    desc, threads = "", 1
    for s in range(args.steps):
        t, desc, threads = oracle_sample(w, q, k, v, units, seed=s)
        times.append(t)
    t = statistics.mean(times)
    value = flops / t / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- PBSA arm
def algorithmic_bytes(w, ncopy: int):
    """Bytes each kernel group must move at minimum (per step)."""
    H, d, bpf = w.heads, w.head_dim, w.blocks_per_frame
    nq = w.chunk_frames * bpf
    tok = nq * 64 * H * d * 2                      # one chunk's raster tensor, bf16
    reps_q = H * nq * d * 4
    nwin = w.window_frames * bpf
    return {
        # fused blockify(Q) + score + top-k: Q read once, q reps written, window reps read,
        # lists written, persistent prefix read
        "blockify_score_select": tok + reps_q + H * nwin * d * 4 + H * nq * (w.capacity + w.topk) * 4
        + H * w.capacity * 4,
        "commit_blockify_kv": 2 * (tok + tok) + 2 * reps_q,
        # plan: q reps + pool reps read, slot tables and lists (the score matrix stays on chip)
        "memory_update_plan": reps_q + H * (w.capacity + w.chunk_frames * bpf) * d * 4
        + H * w.capacity * 4 * 4,
        # apply: K, V blocks and k_reps rows of every promoted block, read and written
        "memory_update_apply": ncopy * 2 * (2 * 64 * d * 2 + d * 4),
    }


def run_train(P, I, dev, steps: int, peaks, batch: int | None = None):
    """Trainable-path workload (batch 2 x 9 frames, 12 heads, 3-frame chunks; every query block
    of a later chunk attends the 24 sinks + its top-16 earlier blocks by coarse score + its own
    chunk): the masks (pbsa_blockify_train_select), the forward (pbsa_attend) and the backward
    (pbsa_attend_bwd), each timed with CUDA events, L2 flushed before each; inputs resident in HBM.
    ``batch`` overrides the workload's batch (a smaller case for profiler captures)."""
    w = I.TRAIN_FWD_BWD if batch is None else dataclasses.replace(I.TRAIN_FWD_BWD, batch=batch)
    frames, batch = w.total_frames, w.batch
    qf = batch * frames
    q4, k4, v4, do4 = I.train_inputs(w, device=dev)
    shape = (qf * w.tokens_per_frame, w.heads, w.head_dim)
    q, k, v, do = (t.reshape(shape) for t in (q4, k4, v4, do4))
    nq = qf * w.blocks_per_frame
    g = P.make_geom(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, "bf16")
    slots = nq
    ld = w.n_sink + w.topk + w.chunk_frames * w.blocks_per_frame
    kp = torch.empty((w.heads, slots, 64, w.head_dim), dtype=torch.bfloat16, device=dev)
    vp = torch.empty_like(kp)
    k_reps = torch.empty((w.heads, slots, w.head_dim), device=dev)
    q_reps = torch.empty((w.heads, nq, w.head_dim), device=dev)
    kv = torch.empty((w.heads, nq, ld), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.heads, nq), dtype=torch.int32, device=dev)
    ws = torch.zeros(max(P.pbsa_workspace_bytes(g, 64, 64), P.pbsa_bwd_workspace_bytes(g, qf, slots, ld)),
                     dtype=torch.uint8, device=dev)
    P.pbsa_blockify_kv(g, k, v, qf, k_reps, None, slots, None, kp, vp, slots, ws=ws)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, q.shape[0]), device=dev)
    dq = torch.empty_like(q)
    dk, dv = torch.empty_like(kp), torch.empty_like(vp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sel_ms, fwd_ms, bwd_ms = [], [], []
    for it in range(steps + 2):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        flush.fill_(0)
        e[0].record()
        P.pbsa_blockify_train_select(g, q, qf, q_reps, k_reps, slots, frames, w.chunk_frames, 1, w.topk,
                                     kv, cnt, ld, None, ws)
        e[1].record()
        flush.fill_(1)
        e[2].record()
        P.pbsa_attend(g, q, qf, kp, vp, slots, kv, cnt, ld, o, lse, ws)
        e[3].record()
        flush.fill_(2)
        e[4].record()
        P.pbsa_attend_bwd(g, q, qf, kp, vp, slots, kv, cnt, ld, o, do, lse, dq, dk, dv, ws)
        e[5].record()
        torch.cuda.synchronize(dev)
        if it >= 2:
            sel_ms.append(e[0].elapsed_time(e[1]))
            fwd_ms.append(e[2].elapsed_time(e[3]))
            bwd_ms.append(e[4].elapsed_time(e[5]))
    _check_device(P, ws, "in the training workload")
    fwd_flops = 4.0 * 64 * 64 * w.head_dim * float(cnt.sum().item())
    bwd_flops = 2.5 * fwd_flops
    sm, fm, bm = statistics.mean(sel_ms), statistics.mean(fwd_ms), statistics.mean(bwd_ms)
    sel_bytes = q.numel() * 2 + q_reps.numel() * 4 + k_reps.numel() * 4 + kv.numel() * 4
    sel_floor = same_bytes_copy_ms(dev, sel_bytes, flush)
    return {"workload": w.name, "batch": w.batch, "query_blocks": nq, "heads": w.heads, "steps": steps,
            "masks": "24 sinks + top-16 by coarse score among the earlier non-sink blocks + own chunk "
                     "(pbsa_blockify_train_select)",
            "select_ms": sm, "select_algorithmic_bytes": sel_bytes,
            "select_frac_hbm": sel_bytes / (sm * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "select_same_bytes_copy_ms": sel_floor, "select_frac_of_same_bytes_copy": sel_floor / sm,
            "fwd_ms": fm, "bwd_ms": bm, "fwd_flops": fwd_flops, "bwd_flops": bwd_flops,
            "fwd_tflops": fwd_flops / (fm * 1e-3) / 1e12, "bwd_tflops": bwd_flops / (bm * 1e-3) / 1e12,
            "fwd_frac_of_bf16_peak": fwd_flops / (fm * 1e-3) / 1e12 / peaks["bf16"],
            "bwd_frac_of_bf16_peak": bwd_flops / (bm * 1e-3) / 1e12 / peaks["bf16"],
            "launches_per_iteration": 1 + 1 + 5,
            "note": "bwd FLOPs counted as 2.5x the forward's (5 GEMM-sized contractions vs 2); "
                    "the dK/dV pass computes S and dP once per pair and stores the dS tiles "
                    "(bf16, 8 KB per pair) that the dQ pass reads back"}


def run_rollout(P, I, dev, w, max_chunks=None, k_schedule=None, label=None):
    """A whole rollout through the layer caches: ``w.layers`` layers, ``w.steps`` denoising
    steps per chunk sharing the persistent memory, the memory update once per finished chunk.

    Inputs are fresh N(0,1) tokens per (chunk, step, layer, tensor) plus per-tile offsets
    (i.i.d. per chunk, or an AR(1) drift across frames for ``w.ar_rho`` > 0), drawn on the
    device before each chunk's timed region.  Each chunk (all layers and steps, then the
    commits) is timed with CUDA events around eager launches on one stream.
    """
    H, d, bpf = w.heads, w.head_dim, w.blocks_per_frame
    cfg = P.LayerConfig(H, d, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.capacity, w.window_frames,
                        w.chunk_frames, w.topk, w.gamma, w.dtype, 0,
                        max_topk=w.window_frames * bpf if k_schedule is not None else -1)
    torch.cuda.synchronize(dev)
    base_alloc = torch.cuda.memory_allocated(dev)
    caches = [P.PBSALayerCache(cfg, dev) for _ in range(w.layers)]
    kv_alloc = torch.cuda.memory_allocated(dev) - base_alloc
    chunks = I.rollout_chunks(w)[:max_chunks]
    ty, tx = w.frame_h // w.tile_h, w.frame_w // w.tile_w
    gen = torch.Generator(device=dev)
    gen.manual_seed(I.stream_seed(w.seed, 7000))
    s_off = w.block_offset_std
    ar = None
    if w.ar_rho > 0:   # AR(1) tile offsets per (layer, tensor), stepped once per frame
        ar = torch.randn((w.layers, 3, ty, tx, H, d), generator=gen, device=dev) * s_off
    c_ar = math.sqrt(max(0.0, 1.0 - w.ar_rho ** 2))

    def draw(nf):
        """[steps][layers] lists of (q, k, v) for a chunk of nf frames."""
        nonlocal ar
        if ar is not None:
            offs = []
            for _ in range(nf):
                ar = w.ar_rho * ar + c_ar * s_off * torch.randn(ar.shape, generator=gen, device=dev)
                offs.append(ar)
            off = torch.stack(offs, 2)                                 # [L, 3, nf, ty, tx, H, d]
        out = []
        for _ in range(w.steps):
            if ar is None:
                off = torch.randn((w.layers, 3, nf, ty, tx, H, d), generator=gen, device=dev) * s_off
            x = torch.randn((w.layers, 3, nf, ty, w.tile_h, tx, w.tile_w, H, d), generator=gen, device=dev)
            x = (x + off[:, :, :, :, None, :, None]).view(w.layers, 3, nf * w.tokens_per_frame, H, d)
            x = x.to(torch.bfloat16)
            out.append([(x[l, 0], x[l, 1], x[l, 2]) for l in range(w.layers)])
        return out

    stream = torch.cuda.current_stream(dev)
    per_chunk, flops_chunk, o = [], [], None
    peak_alloc = peak_caches = 0
    for c, (f0, nf) in enumerate(chunks):
        if k_schedule is not None:
            for ca in caches:
                ca.set_topk(k_schedule[c])
        inp = draw(nf)
        if o is None or o.shape[0] != nf * w.tokens_per_frame:
            o = torch.empty((nf * w.tokens_per_frame, H, d), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        harness = torch.cuda.memory_allocated(dev) - base_alloc - kv_alloc   # this chunk's inputs, o
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cnt_layer0 = None
        for s in range(w.steps):
            for l in range(w.layers):
                q, k, v = inp[s][l]
                attended_history = caches[l].hist > 0
                caches[l].decode_step(q, k, v, o=o)
                if s == w.steps - 1:
                    # each layer commits right after its last-step attention: the write of the
                    # chunk and the memory update's plan overlap that attention's last wave
                    caches[l].commit(k, v, overlap=True)
                    if l == 0 and attended_history:
                        cnt_layer0 = caches[0].kv_cnt.clone()
        e1.record(stream)
        e1.synchronize()
        per_chunk.append(e0.elapsed_time(e1))
        peak_alloc = max(peak_alloc, torch.cuda.max_memory_allocated(dev) - base_alloc)
        peak_caches = max(peak_caches, torch.cuda.max_memory_allocated(dev) - base_alloc - harness)
        blocks = int(cnt_layer0.sum().item()) if cnt_layer0 is not None else H * (nf * bpf) ** 2
        flops_chunk.append(4.0 * 64 * 64 * d * blocks * w.steps * w.layers)
        del inp
        _check_device(P, caches[0].ws, f"in rollout chunk {c}")
    kv_bytes = sum(ca.kv_bytes for ca in caches)
    dense = 2 * w.layers * H * w.total_frames * w.tokens_per_frame * d * 2
    steady = [i for i in range(len(chunks)) if i >= min(4, len(chunks) - 1)]
    ms_steady = statistics.mean(per_chunk[i] for i in steady)
    tf_steady = sum(flops_chunk[i] for i in steady) / (sum(per_chunk[i] for i in steady) * 1e-3) / 1e12
    total_ms, total_flops = sum(per_chunk), sum(flops_chunk)
    return {
        "workload": w.name + (f" ({label})" if label else ""), "layers": w.layers, "steps_per_chunk": w.steps,
        "chunks": len(chunks), "local_topk_per_chunk": list(k_schedule) if k_schedule is not None else w.topk,
        "ms_total": total_ms, "selected_tflop_total": total_flops / 1e12,
        "ms_per_chunk": [round(x, 3) for x in per_chunk],
        "ms_per_chunk_steady": ms_steady, "steady_chunks": f"{steady[0]}..{steady[-1]}",
        "selected_tflops_steady": tf_steady,
        "kv_cache_bytes": {"pbsa_all_layers": kv_bytes, "dense_all_frames_all_layers": dense,
                           "ratio": kv_bytes / dense, "allocated_by_caches": kv_alloc,
                           "peak_allocated_during_chunks": peak_alloc,
                           "peak_during_chunks_minus_harness_inputs": peak_caches,
                           "measured_ratio": peak_caches / dense},
        "timing": "CUDA events around each chunk's eager launches (all layers x steps; each layer commits "
                  "right after its last-step attention)",
        "inputs": "device-drawn N(0,1) + per-tile offsets" + (" (AR(1) drift)" if w.ar_rho > 0 else ""),
    }


def run_variant(P, I, dev, w, steps: int, **cfg_changes):
    """The chunk decode of ``run_pbsa`` under a different layer policy (e.g. the hierarchical
    selection), on the same inputs: graph-captured, L2 flushed before each step, in-graph events."""
    q, k, v = I.single_step(w)
    kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
    vc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 5))
    bpf = w.blocks_per_frame
    cfg = P.LayerConfig(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.capacity,
                        w.window_frames, w.chunk_frames, w.topk, w.gamma, w.dtype,
                        (w.hist_frames - w.window_frames) * bpf, **cfg_changes)
    torch.cuda.synchronize(dev)
    alloc0 = torch.cuda.memory_allocated(dev)
    cache = P.PBSALayerCache(cfg, dev)
    cache_alloc = torch.cuda.memory_allocated(dev) - alloc0      # every device buffer the cache owns
    cache_staging = 2 * cache.k_pool[:, cache.stage_base:].numel() * cache.k_pool.element_size()
    qd, kcd, vcd = q.to(dev), kc.to(dev), vc.to(dev)
    cache.prefill(k.to(dev), v.to(dev), w.hist_frames, cache.query_reps(qd))
    step = P.ChunkDecodeStep(cache)
    o = torch.empty_like(qd)
    snap = step.snapshot()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(2):
        step.restore(snap)
        step.run(qd, kcd, vcd, o)
    torch.cuda.synchronize(dev)
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    graph = step.capture(qd, kcd, vcd, o, ends=ends)
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(7)]
    graph_parts = step.capture(qd, kcd, vcd, o, marks=marks)
    if cfg.own_chunk:   # the chunk's K, V are written before the selection
        spans = {"commit_blockify_kv": (0, 1), "blockify_select": (1, 2), "attend": (2, 3),
                 "memory_update_plan": (4, 5), "memory_update_apply": (5, 6)}
    else:
        spans = {"blockify_select": (0, 2), "attend": (2, 3), "commit_blockify_kv": (3, 4),
                 "memory_update_plan": (4, 5), "memory_update_apply": (5, 6)}
    runs = {g: [] for g in spans}
    total = []
    for s in range(steps + 3):
        for gr in (graph, graph_parts):
            step.restore(snap)
            flush.fill_(1)
            gr.replay()
            torch.cuda.synchronize(dev)
        if s >= 3:
            for g, (a, b) in spans.items():
                runs[g].append(marks[a].elapsed_time(marks[b]))
            total.append(ends[0].elapsed_time(ends[1]))
    _check_device(P, cache.ws, "in a variant run")
    flops = step.flops()
    per = {g: statistics.mean(x) for g, x in runs.items()}
    ms = statistics.mean(total)
    del graph, graph_parts
    return {"policy": cfg_changes, "ms_per_chunk_decode": ms, "kernels_ms": per,
            "selected_flops": flops, "value_tflops": flops / (ms * 1e-3) / 1e12,
            "attend_tflops": flops / (per["attend"] * 1e-3) / 1e12}


def run_hbm_at_scale(P, I, dev, peaks, reps: int = 10):
    """The HBM-bound kernels at sizes where bandwidth, not launch and first-byte latency, decides:
    the commit of K and V over an 18-frame history (the prefill's size, 340 MB moved), and the
    memory update's copies for 30 layers x 12 heads folded into 360 heads, 72 promotions each
    (1.7 GB moved).  CUDA events around a graph of the one kernel, L2 flushed before each replay."""
    w = I.DECODE_5S
    H, d, bpf = w.heads, w.head_dim, w.blocks_per_frame
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {}

    def timed(fn):
        fn()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.graph(graph, stream=side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        ts = []
        for i in range(reps + 2):
            flush.fill_(i & 255)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            e1.synchronize()
            if i >= 2:
                ts.append(e0.elapsed_time(e1))
        del graph
        return statistics.median(ts)

    # commit of K and V, 18 frames
    g = P.make_geom(H, d, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, w.dtype)
    nf = 18
    kx = torch.randn((nf * w.tokens_per_frame, H, d), device=dev).to(torch.bfloat16)
    vx = torch.randn_like(kx)
    slots = nf * bpf
    k_pool = torch.empty((H, slots, 64, d), dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty_like(k_pool)
    k_reps = torch.empty((H, slots, d), device=dev)
    ws = torch.zeros(P.pbsa_workspace_bytes(g, 72, 168), dtype=torch.uint8, device=dev)
    ms = timed(lambda: P.pbsa_blockify_kv(g, kx, vx, nf, k_reps, None, slots, None, k_pool, v_pool, slots, ws=ws))
    nbytes = 2 * (2 * kx.numel() * 2) + k_reps.numel() * 4
    out["commit_blockify_kv_18_frames"] = {"ms": ms, "algorithmic_bytes": nbytes,
                                           "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                                           "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del kx, vx, k_pool, v_pool, k_reps

    # the memory update's copies, 360 heads x 72 promotions
    Hs, C, S, nc = 30 * H, w.capacity, bpf, 72
    gs = P.make_geom(Hs, d, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, w.dtype)
    pool = C + nc
    k_pool = torch.randn((Hs, pool, 64, d), device=dev).to(torch.bfloat16)
    v_pool = torch.randn_like(k_pool)
    k_reps = torch.randn((Hs, pool, d), device=dev) * 0.35
    q_reps = torch.randn((Hs, 72, d), device=dev) * 0.3
    slot_gid = torch.full((Hs, C), -1, dtype=torch.int32, device=dev)
    slot_gid[:, :S] = torch.arange(S, dtype=torch.int32, device=dev)      # sinks only: every
    slot_ema = torch.zeros((Hs, C), device=dev)                            # candidate is promoted
    cs = (torch.arange(nc, dtype=torch.int32, device=dev) + C).repeat(Hs, 1).contiguous()
    cg = (torch.arange(nc, dtype=torch.int32, device=dev) + 1000).repeat(Hs, 1).contiguous()
    wss = torch.zeros(P.pbsa_workspace_bytes(gs, 72, C + nc), dtype=torch.uint8, device=dev)
    P.pbsa_memory_update_plan(gs, q_reps, 72, k_reps, pool, slot_gid, slot_ema, C, S, cs, cg, nc, w.gamma, ws=wss)
    torch.cuda.synchronize(dev)
    promoted = int((slot_gid >= 1000).sum().item())
    ms = timed(lambda: P.pbsa_memory_update_apply(gs, k_reps, k_pool, v_pool, pool, C, nc, ws=wss))
    nbytes = promoted * 2 * (2 * 64 * d * 2 + d * 4)
    out["memory_update_apply_360_heads"] = {"ms": ms, "promoted_blocks": promoted, "algorithmic_bytes": nbytes,
                                            "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                                            "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    _check_device(P, wss, "in the memory update at scale")
    _check_device(P, ws, "in the commit at scale")
    del k_pool, v_pool
    return out


def rank_workload(w, rank: int):
    """Weak scaling: every rank decodes its own independent layer (same shapes, its own seed)."""
    import dataclasses
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, device, world: int) -> float:
    """The slowest rank's value (time-like numbers are reported as the max over ranks)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def same_bytes_copy_ms(dev, nbytes: int, flush, reps: int = 10) -> float:
    """Device time of a plain device-to-device copy that moves ``nbytes`` (half read, half
    written), L2 flushed before each: the floor, at this size, that launch and first-byte
    latency leave for any kernel moving the same bytes.  Median of ``reps``."""
    half = max(16, (nbytes // 2) // 16 * 16)
    src = torch.empty(half, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    ts = []
    for i in range(reps + 2):
        flush.fill_(i & 255)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src)
        e1.record()
        e1.synchronize()
        if i >= 2:
            ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def sum_over_ranks(x: float, device, world: int) -> float:
    """The whole job's total of a per-rank quantity (e.g. the FLOPs of one step)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def _check_device(P, ws, when: str):
    """Raise with the workspace's device error word (code, info, kernel id) if one is set."""
    torch.cuda.synchronize()
    word = ws[:16].view(torch.int32).tolist()
    if P.pbsa_get_device_error(ws) != 0:
        raise RuntimeError(f"device error {when}: code={word[0]} info={word[1]} kernel={word[2]}")


def run_pbsa(args, w, rank, world, local_rank):
    import block_sparse_attention_pbsa_b200 as P
    from block_sparse_attention_pbsa_b200 import inputs as I

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    heads_split = args.shard == "heads" and world > 1
    # weak scaling: every rank its own independent layer; head split (strong scaling): the one
    # layer's heads partitioned over the ranks, each rank its heads' cache and inputs
    wr = w if heads_split else rank_workload(w, rank)
    q, k, v = I.single_step(wr)
    kc = I.tokens(wr, wr.chunk_frames, I.stream_seed(wr.seed, 4))
    vc = I.tokens(wr, wr.chunk_frames, I.stream_seed(wr.seed, 5))
    bpf = w.blocks_per_frame
    cfg = P.LayerConfig(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.capacity,
                        w.window_frames, w.chunk_frames, w.topk, w.gamma, w.dtype,
                        (w.hist_frames - w.window_frames) * bpf)
    if heads_split:
        from block_sparse_attention_pbsa_b200 import shard
        q, k, v, kc, vc = (shard.head_slice(t, w.heads, world, rank) for t in (q, k, v, kc, vc))
        cfg = shard.local_config(cfg, world, rank)
    torch.cuda.synchronize(dev)
    alloc0 = torch.cuda.memory_allocated(dev)
    cache = P.PBSALayerCache(cfg, dev)
    cache_alloc = torch.cuda.memory_allocated(dev) - alloc0      # every device buffer the cache owns
    cache_staging = 2 * cache.k_pool[:, cache.stage_base:].numel() * cache.k_pool.element_size()
    qd, kcd, vcd = q.to(dev), kc.to(dev), vc.to(dev)
    cache.prefill(k.to(dev), v.to(dev), w.hist_frames, cache.query_reps(qd))
    step = P.ChunkDecodeStep(cache)
    o = torch.empty_like(qd)
    snap = step.snapshot()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    # warm-up (sets kernel attributes), then capture the whole step in one CUDA graph
    for _ in range(2):
        step.restore(snap)
        step.run(qd, kcd, vcd, o, stream=stream)
    torch.cuda.synchronize(dev)
    # the timed step: events only around the whole step, so the commit of K, V may overlap
    # the tail of attend (programmatic dependent launch); a second graph with events between
    # the kernel groups gives the per-kernel breakdown
    ends = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    graph = step.capture(qd, kcd, vcd, o, ends=ends)
    marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(7)]
    graph_parts = step.capture(qd, kcd, vcd, o, marks=marks)
    torch.cuda.synchronize(dev)

    def one(gr):
        step.restore(snap)
        flush.fill_(1)
        gr.replay()

    for _ in range(max(args.warmup, 3)):
        one(graph)
        one(graph_parts)
    _check_device(P, cache.ws, "during warm-up")
    flops = step.flops()

    step_runs = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        for s in range(args.steps):
            one(graph)
            torch.cuda.synchronize(dev)
            step_runs.append(ends[0].elapsed_time(ends[1]))
    if world > 1:
        torch.distributed.barrier()
    # kernel groups by the in-graph marks they lie between (marks 1 and 2 are adjacent: the
    # fused blockify + select is one kernel); outside the timed region
    spans = {"blockify_score_select": (0, 2), "attend": (2, 3), "commit_blockify_kv": (3, 4),
             "memory_update_plan": (4, 5), "memory_update_apply": (5, 6)}
    groups = list(spans)
    per_runs = {g: [] for g in groups}
    parts_total = []
    for s in range(args.steps):
        one(graph_parts)
        torch.cuda.synchronize(dev)
        for g, (a, b) in spans.items():
            per_runs[g].append(marks[a].elapsed_time(marks[b]))
        parts_total.append(marks[0].elapsed_time(marks[6]))
    per = {g: statistics.mean(v) for g, v in per_runs.items()}
    step_ms = statistics.mean(step_runs)
    step_ms_max = max_over_ranks(step_ms, dev, world)
    # number of block copies the memory update made (for its algorithmic bytes)
    step.restore(snap)
    graph.replay()
    torch.cuda.synchronize(dev)
    ncopy = int((cache.slot_gid != snap[0]).sum().item())
    _check_device(P, cache.ws, "during the timed steps")

    # ---- end to end through the public API: pinned host inputs -> HBM -> step -> host output,
    # with the transfers overlapped with the step's kernels (ChunkDecodeStep.run_pipelined)
    qh, kh, vh = (t.pin_memory() for t in (q, kc, vc))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    step.restore(snap)
    step.capture_pipeline(qd, kcd, vcd, o, qh, kh, vh, oh)
    e2e_ms = []
    for s in range(max(1, args.steps // 2) + 1):
        step.restore(snap)
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step.run_pipelined(qh, kh, vh, oh)
        e1.record(stream)
        e1.synchronize()
        if s > 0:
            e2e_ms.append(e0.elapsed_time(e1))
    if not torch.equal(oh, o.cpu()):
        raise RuntimeError("the pipelined end-to-end step returned a different O")
    e2e_ms_max = max_over_ranks(statistics.mean(e2e_ms), dev, world)
    # the transfers alone (the same pinned buffers and bytes, no kernels): the upload of Q, K, V
    # and the download of O, each timed on its own.  The step overlaps the download of one
    # part with the upload of the next, so the upload is the floor it approaches once its
    # kernels hide behind the transfers.
    def copies_ms(pairs):
        ts = []
        for s in range(4):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for dst, src in pairs:
                dst.copy_(src, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if s > 0:
                ts.append(e0.elapsed_time(e1))
        return max_over_ranks(statistics.mean(ts), dev, world)
    h2d_ms = copies_ms(((qd, qh), (kcd, kh), (vcd, vh)))
    d2h_ms = copies_ms(((oh, o),))
    job_flops = sum_over_ranks(flops, dev, world)    # every rank's layer, or the shared layer's heads

    if rank != 0:
        return
    ab = algorithmic_bytes(w, ncopy)
    kernels = {g: {"ms": per[g]} for g in groups}
    for g, b in ab.items():
        floor = same_bytes_copy_ms(dev, b, flush)
        kernels[g].update({"algorithmic_bytes": b, "achieved_gbs": b / (per[g] * 1e-3) / 1e9,
                           "frac_hbm": b / (per[g] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                           "same_bytes_copy_ms": floor, "frac_of_same_bytes_copy": floor / per[g]})
    att_tflops = flops / (per["attend"] * 1e-3) / 1e12
    kernels["attend"].update({"flops": flops, "achieved_tflops": att_tflops})
    value = job_flops / (step_ms_max * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (q, kc, vc))
    d2h = o.numel() * o.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": step_ms_max, "ms_per_chunk_decode": step_ms_max,
        "higher_is_better": True, "scaling": "strong" if heads_split else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(w),
                   "parallelism": (f"the layer's {w.heads} heads split over {world} GPUs (no exchange in the step)"
                                   if heads_split else f"{world} independent layer decodes (one per GPU)")},
        "roofline": {"bound": "tensor", "kernel": "pbsa_attend (attend_tc_kernel)", "achieved": att_tflops,
                     "peak": peaks["bf16"], "unit": "TFLOP/s", "frac": att_tflops / peaks["bf16"],
                     "peak_source": f"{peaks['source']} burst bf16 (cuBLAS)",
                     "frac_of_sustained": att_tflops / peaks["bf16_sustained"],
                     "traffic": profiled_traffic("attend_tc_decode_5s.counters.json",
                                                 "block_sparse_attention_pbsa_b200/csrc/attend_tc.cu"),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "step_frac_of_bf16_peak": value / world / peaks["bf16"],
        "kernels": kernels,
        "ms_per_step_groups_serialised": statistics.mean(parts_total),
        "kv_cache_bytes": {"pbsa_per_layer": cache.kv_bytes,
                           "allocated_by_cache_measured": cache_alloc,
                           "allocated_minus_prefill_staging": cache_alloc - cache_staging,
                           "dense_21_frames_per_layer": 2 * w.heads * 21 * w.tokens_per_frame * w.head_dim * 2,
                           "note": "measured = torch.cuda.memory_allocated() around the cache's construction: "
                                   "K/V pools, key representatives, slot tables, lists, workspace; the staging "
                                   "area only serves the one-time prefill of a mid-video history"},
        "e2e": {"value": job_flops / (e2e_ms_max * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms_max, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "h2d_alone_ms": h2d_ms, "d2h_alone_ms": d2h_ms, "h2d_alone_frac_of_step": h2d_ms / e2e_ms_max},
        "gpu_launches": step.LAUNCHES * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_train:
        line["train"] = run_train(P, I, dev, 5, peaks)
    line["kernels_at_scale"] = run_hbm_at_scale(P, I, dev, peaks)
    line["variants"] = [run_variant(P, I, dev, w, max(5, args.steps // 2), hsa_top_frames=3, hsa_recent=1),
                        run_variant(P, I, dev, w, max(5, args.steps // 2), own_chunk=True)]
    if not args.no_rollout:
        from block_sparse_attention_pbsa_b200 import schedule as S
        w5 = I.ROLLOUT_5S
        ks, _, _ = S.rollout_topk(I.rollout_chunks(w5), w5.tokens_per_frame, w5.blocks_per_frame, w5.head_dim,
                                  w5.capacity, w5.window_frames, 0.7, 0.5)
        line["rollouts"] = [run_rollout(P, I, dev, w5), run_rollout(P, I, dev, I.ROLLOUT_1MIN),
                            run_rollout(P, I, dev, w5, k_schedule=ks,
                                        label="per-chunk top-k, chunk-aware growth s_base 0.7 -> s_target 0.5")]
    if world == 1 and not args.no_cpu_baseline:
        t, desc, threads = oracle_sample(w, q, k, v, units=24)
        line["cpu_baseline"] = {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": threads,
                                "kind": "oracle", "sample": desc, "ms_per_step": t * 1e3}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["pbsa", "reference"], default="pbsa")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-train", action="store_true", help="skip the forward+backward training workload")
    ap.add_argument("--train-only", action="store_true", help="only the training workload (for profiling)")
    ap.add_argument("--train-batch", type=int, default=None,
                    help="with --train-only: sequences in the training batch (default: the workload's 2)")
    ap.add_argument("--no-rollout", action="store_true", help="skip the 30-layer 5 s and 1-minute rollouts")
    ap.add_argument("--shard", choices=["layers", "heads"], default="layers",
                    help="N > 1: every rank its own layer (weak scaling, the default) or one layer's heads "
                         "split over the ranks (strong scaling)")
    args = ap.parse_args()
    from block_sparse_attention_pbsa_b200 import inputs as I
    w = I.DECODE_5S
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    if args.train_only:
        import block_sparse_attention_pbsa_b200 as P
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        print(json.dumps(run_train(P, I, dev, args.steps, load_peaks(), args.train_batch)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_pbsa(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
