"""GPU parity of the backward pass (pbsa_attend_bwd) against the oracle's textbook
gradients, under fixed seeded block lists with the structure of the trainable path (random
selections: structural cases such as odd query-block pairs and unattended slots).  The
trainable-path workload under the method's own masks is in test_gpu_train.py."""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import inputs as I
from oracle import pbsa_oracle as O
from tests._util import BF16_MAX_ABS, BF16_MEAN_ABS, assert_bf16_close, block_rows, f64, geom_dict

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(w, frames, batch, extra_slots=0, seed=0):
    gq, gk, gv, gd = (torch.Generator().manual_seed(seed * 10 + i) for i in range(4))
    shape = (batch * frames * w.tokens_per_frame, w.heads, w.head_dim)
    q, k, v, do = (torch.randn(shape, generator=g_).to(torch.bfloat16) for g_ in (gq, gk, gv, gd))
    lists = I.train_lists(w, seed + 7, n_frames=frames, batch=batch)
    nq = batch * frames * w.blocks_per_frame
    slots = nq + extra_slots
    ld = max(len(l) for row in lists for l in row)
    kv = torch.zeros((w.heads, nq, ld), dtype=torch.int32)
    cnt = torch.zeros((w.heads, nq), dtype=torch.int32)
    for h in range(w.heads):
        for r in range(nq):
            kv[h, r, :len(lists[h][r])] = torch.tensor(lists[h][r], dtype=torch.int32)
            cnt[h, r] = len(lists[h][r])
    return q, k, v, do, lists, kv, cnt, ld, slots


def _gpu(w, q, k, v, do, kv, cnt, ld, slots, q_frames):
    g = P.make_geom(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, "bf16")
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    kp = torch.zeros((w.heads, slots, 64, w.head_dim), dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV)
    ws = torch.zeros(max(P.pbsa_workspace_bytes(g, 64, 64),
                         P.pbsa_bwd_workspace_bytes(g, q_frames, slots, ld)), dtype=torch.uint8, device=DEV)
    P.pbsa_blockify(g, kd, q_frames, reps, slots, None, kp, slots, ws)
    P.pbsa_blockify(g, vd, q_frames, reps, slots, None, vp, slots, ws)
    kvd, cntd = kv.to(DEV), cnt.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty((w.heads, qd.shape[0]), device=DEV)
    P.pbsa_attend(g, qd, q_frames, kp, vp, slots, kvd, cntd, ld, o, lse, ws)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kp, float("nan"))
    dv = torch.full_like(vp, float("nan"))
    P.pbsa_attend_bwd(g, qd, q_frames, kp, vp, slots, kvd, cntd, ld, o, dod, lse, dq, dk, dv, ws)
    torch.cuda.synchronize()
    word = ws[:16].view(torch.int32).tolist()
    assert P.pbsa_get_device_error(ws) == 0, word
    return dq.cpu(), dk.cpu(), dv.cpu()


def _oracle_unit(w, q64, k64, v64, do64, h, r, slots):
    gd = geom_dict(w)
    rows = block_rows(w, r)
    kk = np.concatenate([O.block_tokens(k64, gd, s)[:, h] for s in slots])
    vv = np.concatenate([O.block_tokens(v64, gd, s)[:, h] for s in slots])
    dq, dk, dv = O.attention_bwd(q64[rows, h], kk, vv, do64[rows, h], w.scale)
    return rows, dq, dk, dv


def _rel_close(got, want, what):
    """bf16 absolute bounds, plus a relative bound so small gradients are still checked."""
    assert_bf16_close(got, want, what)
    rms = float(np.sqrt(np.mean(want ** 2))) + 1e-30
    rel = float(np.sqrt(np.mean((got - want) ** 2))) / rms
    assert rel < 2e-2, f"{what}: relative rms error {rel:.3e}"


@pytest.mark.parametrize("fh,fw,frames,batch,topk,extra", [
    (16, 32, 6, 2, 4, 3),      # 96 query blocks, unattended extra slots
    (8, 24, 3, 1, 2, 0),       # 9 query blocks and 9 slots: odd pairs
])
def test_bwd_small(fh, fw, frames, batch, topk, extra):
    w = dataclasses.replace(I.TRAIN_FWD_BWD, heads=2, frame_h=fh, frame_w=fw, total_frames=frames,
                            batch=batch, topk=topk)
    q, k, v, do, lists, kv, cnt, ld, slots = _setup(w, frames, batch, extra)
    q_frames = batch * frames
    dq, dk, dv = _gpu(w, q, k, v, do, kv, cnt, ld, slots, q_frames)
    q64, k64, v64, do64 = (f64(t) for t in (q, k, v, do))
    nq = q_frames * w.blocks_per_frame
    for h in range(w.heads):
        want_dk = np.zeros((slots, 64, w.head_dim))
        want_dv = np.zeros((slots, 64, w.head_dim))
        for r in range(nq):
            rows, gq, gk, gv = _oracle_unit(w, q64, k64, v64, do64, h, r, lists[h][r])
            _rel_close(f64(dq[rows, h]), gq, f"dq h{h} r{r}")
            for i, s in enumerate(lists[h][r]):
                want_dk[s] += gk[i * 64:(i + 1) * 64]
                want_dv[s] += gv[i * 64:(i + 1) * 64]
        _rel_close(f64(dk[h]), want_dk, f"dk h{h}")
        _rel_close(f64(dv[h]), want_dv, f"dv h{h}")
        if extra:
            assert (dk[h, nq:] == 0).all() and (dv[h, nq:] == 0).all()


def test_bwd_edge_lists_and_determinism():
    """Hand-built lists around the dS tiles the two passes exchange: query blocks with empty
    lists (alone and next to a non-empty partner in either half of a pair), a row filled to
    kv_ld with its slots in descending order (the highest tile positions), the pool's last
    slot; gradients against the oracle, dQ of an empty row exactly zero, and two runs bit for
    bit equal."""
    w = dataclasses.replace(I.TRAIN_FWD_BWD, heads=2, frame_h=16, frame_w=32, total_frames=2, batch=1)
    frames, q_frames = 2, 2
    nq = frames * w.blocks_per_frame                # 16 query blocks
    slots, ld = nq + 8, 12                          # 8 pool slots beyond the query frames
    gq, gk, gv, gd = (torch.Generator().manual_seed(90 + i) for i in range(4))
    shape = (frames * w.tokens_per_frame, w.heads, w.head_dim)
    q, do = (torch.randn(shape, generator=g_).to(torch.bfloat16) for g_ in (gq, gd))
    kv_frames = slots // w.blocks_per_frame          # keys and values for every slot
    kshape = (kv_frames * w.tokens_per_frame, w.heads, w.head_dim)
    k, v = (torch.randn(kshape, generator=g_).to(torch.bfloat16) for g_ in (gk, gv))
    rng = np.random.default_rng(5)
    lists = []
    for h in range(w.heads):
        rows = []
        for r in range(nq):
            if r in (0, 1, 5, 10):               # pair 0 both empty; 5 (B of pair 2); 10 (A of pair 5)
                rows.append([])
            elif r == 7:                          # full row, descending, includes the last slot
                rows.append(sorted(rng.choice(slots - 1, ld - 1, replace=False).tolist() + [slots - 1],
                                   reverse=True))
            else:
                rows.append(rng.choice(slots, int(rng.integers(1, ld)), replace=False).tolist())
        lists.append(rows)
    kv = torch.zeros((w.heads, nq, ld), dtype=torch.int32)
    cnt = torch.zeros((w.heads, nq), dtype=torch.int32)
    for h in range(w.heads):
        for r in range(nq):
            kv[h, r, :len(lists[h][r])] = torch.tensor(lists[h][r], dtype=torch.int32)
            cnt[h, r] = len(lists[h][r])
    g = P.make_geom(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, "bf16")
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    kp = torch.zeros((w.heads, slots, 64, w.head_dim), dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV)
    ws = torch.zeros(max(P.pbsa_workspace_bytes(g, 64, 64),
                         P.pbsa_bwd_workspace_bytes(g, q_frames, slots, ld)), dtype=torch.uint8, device=DEV)
    P.pbsa_blockify(g, kd, kv_frames, reps, slots, None, kp, slots, ws)
    P.pbsa_blockify(g, vd, kv_frames, reps, slots, None, vp, slots, ws)
    kvd, cntd = kv.to(DEV), cnt.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty((w.heads, qd.shape[0]), device=DEV)
    P.pbsa_attend(g, qd, q_frames, kp, vp, slots, kvd, cntd, ld, o, lse, ws)
    runs = []
    for _ in range(2):
        dq = torch.full_like(qd, float("nan"))
        dk = torch.full_like(kp, float("nan"))
        dv = torch.full_like(vp, float("nan"))
        P.pbsa_attend_bwd(g, qd, q_frames, kp, vp, slots, kvd, cntd, ld, o, dod, lse, dq, dk, dv, ws)
        torch.cuda.synchronize()
        assert P.pbsa_get_device_error(ws) == 0
        runs.append((dq.cpu(), dk.cpu(), dv.cpu()))
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a, b)
    dq, dk, dv = runs[0]
    q64, k64, v64, do64 = (f64(t) for t in (q, k, v, do))
    for h in range(w.heads):
        want_dk = np.zeros((slots, 64, w.head_dim))
        want_dv = np.zeros((slots, 64, w.head_dim))
        for r in range(nq):
            rows = block_rows(w, r)
            if not lists[h][r]:
                assert (dq[rows, h] == 0).all(), f"dq of the empty row h{h} r{r}"
                continue
            rows, gq_, gk_, gv_ = _oracle_unit(w, q64, k64, v64, do64, h, r, lists[h][r])
            _rel_close(f64(dq[rows, h]), gq_, f"dq h{h} r{r}")
            for i, s in enumerate(lists[h][r]):
                want_dk[s] += gk_[i * 64:(i + 1) * 64]
                want_dv[s] += gv_[i * 64:(i + 1) * 64]
        _rel_close(f64(dk[h]), want_dk, f"dk h{h}")
        _rel_close(f64(dv[h]), want_dv, f"dv h{h}")
