"""GPU parity of the trainable path with the method's own masks: pbsa_blockify_train_select
(sinks + top-k by coarse score among the earlier non-sink blocks + the own chunk) against the
oracle's train_masks, then pbsa_attend and pbsa_attend_bwd under those masks against the
oracle's textbook attention and gradients."""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import inputs as I
from oracle import pbsa_oracle as O
from tests._util import NEAR_TIE, assert_bf16_close, block_rows, f64, geom_dict

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rel_close(got, want, what):
    """bf16 absolute bounds, plus a relative bound so small gradients are still checked."""
    assert_bf16_close(got, want, what)
    rms = float(np.sqrt(np.mean(want ** 2))) + 1e-30
    rel = float(np.sqrt(np.mean((got - want) ** 2))) / rms
    assert rel < 2e-2, f"{what}: relative rms error {rel:.3e}"


def _geom(w):
    return P.make_geom(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, w.dtype)


def gpu_train_lists(w, g, qd, k_reps, pool_slots, n_seq, seq_frames, k, sink_frames=1, ws=None):
    """The method's masks on the GPU: (q_reps, kv_slot, kv_cnt, kv_ld, scores)."""
    bpf, H, d = w.blocks_per_frame, w.heads, w.head_dim
    qf = n_seq * seq_frames
    nq = qf * bpf
    ld = sink_frames * bpf + k + min(w.chunk_frames, seq_frames) * bpf
    q_reps = torch.zeros((H, nq, d), device=DEV)
    kv = torch.full((H, nq, ld), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((H, nq), dtype=torch.int32, device=DEV)
    sc = torch.zeros((H, nq, max(k, 1)), device=DEV)
    P.pbsa_blockify_train_select(g, qd, qf, q_reps, k_reps, pool_slots, seq_frames, w.chunk_frames, sink_frames,
                                 k, kv, cnt, ld, sc, ws)
    return q_reps, kv, cnt, ld, sc


def check_lists_against_oracle(w, q, k, kv, cnt, sc, n_seq, seq_frames, topk, sink_frames=1):
    """Every row: sinks, then the top-k, then the own chunk.  With frame 0 as the sinks the
    expected rows are the oracle's ``train_masks`` (sets outside near ties, by its k-th gaps);
    the selected scores are checked against the oracle's coarse scores to 2e-5.  q, k: raster
    CPU tensors of all sequences.  Returns the number of rows compared exactly."""
    bpf, H, tpf = w.blocks_per_frame, w.heads, w.tokens_per_frame
    T = seq_frames * tpf
    gd = geom_dict(w)
    q4 = f64(q).reshape(n_seq, T, H, w.head_dim)
    k4 = f64(k).reshape(n_seq, T, H, w.head_dim)
    nb = seq_frames * bpf
    S = sink_frames * bpf
    masks = gaps = None
    if sink_frames == 1:
        masks, gaps = O.train_masks(q4, k4, gd, seq_frames, w.chunk_frames, topk)
    kv, cnt, sc = kv.cpu(), cnt.cpu(), sc.cpu()
    exact = 0
    for s in range(n_seq):
        qr = O.block_reps(q4[s], gd, seq_frames)
        kr = O.block_reps(k4[s], gd, seq_frames)
        for h in range(H):
            for r in range(nb):
                c = (r // bpf) // w.chunk_frames
                own = O.frame_blocks(range(c * w.chunk_frames, min((c + 1) * w.chunk_frames, seq_frames)), bpf)
                row = kv[h, s * nb + r, :int(cnt[h, s * nb + r])].tolist()
                row = [x - s * nb for x in row]          # slots of sequence s -> its own block ids
                if c == 0:
                    assert row == own, (s, h, r)
                    if masks is not None:
                        assert row == masks[s][h][r]
                    continue
                earlier = O.frame_blocks(range(sink_frames, c * w.chunk_frames), bpf)
                sc32 = O.coarse_scores(qr[h][r:r + 1], kr[h][earlier], w.scale)[0].astype(np.float32)
                pos = O.topk_select(sc32, earlier, topk)
                kk = len(pos)
                assert len(row) == S + kk + len(own), (s, h, r, len(row))
                assert row[:S] == list(range(S)) and row[S + kk:] == own, (s, h, r)
                got = row[S:S + kk]
                np.testing.assert_allclose(sc[h, s * nb + r, :kk].numpy(), sc32[pos], rtol=0, atol=2e-5)
                if masks is not None:
                    want, gap = set(masks[s][h][r][S:S + kk]), gaps[s][h][r]
                    assert masks[s][h][r][:S] == row[:S] and masks[s][h][r][S + kk:] == own
                else:
                    want, gap = {earlier[i] for i in pos}, O.kth_gap(sc32, earlier, topk)
                if gap > NEAR_TIE:
                    assert set(got) == want, (s, h, r)
                    exact += 1
                else:   # a near tie: either block may be taken, but only candidates, once each
                    assert len(set(got)) == kk and set(got) <= set(earlier)
    return exact


CASES = {
    # name: (workload changes, sequences, frames per sequence, top-k, sink frames)
    "bf16_8_blocks_per_frame": (dict(heads=2, frame_h=16, frame_w=32), 2, 9, 4, 1),
    "f32_ragged_last_chunk": (dict(heads=1, head_dim=64, frame_h=16, frame_w=16, dtype="f32"), 2, 8, 3, 1),
    "bf16_no_sinks": (dict(heads=1, frame_h=16, frame_w=32, chunk_frames=2), 1, 6, 5, 0),
    "bf16_k_above_candidates": (dict(heads=2, frame_h=16, frame_w=32), 1, 6, 20, 1),
    # 264 candidates in the last chunk: past the 8-block kernel's 256
    "bf16_long_sequence": (dict(heads=1), 1, 15, 16, 1),
    # three sequences of two frames each: every sequence is a single, shorter-than-a-chunk chunk
    "f32_sequences_shorter_than_a_chunk": (dict(heads=2, head_dim=64, frame_h=16, frame_w=16, dtype="f32"),
                                           3, 2, 4, 1),
    # 5 blocks per frame (an odd count: groups of 8 query blocks end inside a frame)
    "bf16_odd_blocks_per_frame": (dict(heads=1, frame_h=8, frame_w=40), 2, 7, 6, 1),
}


@pytest.mark.parametrize("case", list(CASES))
def test_train_select(case):
    changes, n_seq, F, k, sink = CASES[case]
    w = dataclasses.replace(I.TRAIN_FWD_BWD, block_offset_std=0.5, **changes)
    g = _geom(w)
    bpf, H, d = w.blocks_per_frame, w.heads, w.head_dim
    qf = n_seq * F
    q = I.tokens(w, qf, I.stream_seed(w.seed, 41, qf))
    k_tok = I.tokens(w, qf, I.stream_seed(w.seed, 42, qf))
    pool = qf * bpf + 3
    k_reps = torch.zeros((H, pool, d), device=DEV)
    ws = torch.zeros(P.pbsa_workspace_bytes(g, 64, 64), dtype=torch.uint8, device=DEV)
    P.pbsa_blockify(g, k_tok.to(DEV), qf, k_reps, pool, ws=ws)
    qd = q.to(DEV)
    q_reps, kv, cnt, ld, sc = gpu_train_lists(w, g, qd, k_reps, pool, n_seq, F, k, sink, ws)
    assert P.pbsa_get_device_error(ws) == 0
    q_sep = torch.zeros_like(q_reps)
    P.pbsa_blockify(g, qd, qf, q_sep, qf * bpf, ws=ws)
    assert torch.equal(q_reps, q_sep)          # the fused pooling is blockify's, bit for bit
    np.testing.assert_allclose(f64(q_reps), O.block_reps(f64(q), geom_dict(w), qf), rtol=0, atol=2e-6)
    exact = check_lists_against_oracle(w, q, k_tok, kv, cnt, sc, n_seq, F, k, sink)
    n_later = n_seq * H * (F * bpf - min(w.chunk_frames, F) * bpf)
    assert exact >= n_later // 2


@pytest.mark.slow
def test_train_workload_masks_forward_backward():
    """The trainable-path workload (batch 2 x 9 frames x 1536 tokens, 12 heads, 3-frame chunks,
    24 sinks + top-16 + own chunk): the masks of every (sequence, head, query block) against the
    oracle's; then, under those masks, O and LSE of every query block and dQ, dK, dV of every
    block for two heads against the oracle's attention and textbook gradients."""
    w = I.TRAIN_FWD_BWD
    g = _geom(w)
    B, F, H, d, bpf = w.batch, w.total_frames, w.heads, w.head_dim, w.blocks_per_frame
    q4, k4, v4, do4 = I.train_inputs(w)
    qf = B * F
    q, k, v, do = (t.reshape(qf * w.tokens_per_frame, H, d) for t in (q4, k4, v4, do4))
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    nq = qf * bpf
    kp = torch.zeros((H, nq, 64, d), dtype=torch.bfloat16, device=DEV)
    vp = torch.zeros_like(kp)
    k_reps = torch.zeros((H, nq, d), device=DEV)
    ld0 = w.n_sink + w.topk + w.chunk_frames * bpf
    ws = torch.zeros(max(P.pbsa_workspace_bytes(g, 64, 64), P.pbsa_bwd_workspace_bytes(g, qf, nq, ld0)),
                     dtype=torch.uint8, device=DEV)
    P.pbsa_blockify_kv(g, kd, vd, qf, k_reps, None, nq, None, kp, vp, nq, ws=ws)
    _, kv, cnt, ld, sc = gpu_train_lists(w, g, qd, k_reps, nq, B, F, w.topk, 1, ws)
    assert ld == ld0
    o = torch.empty_like(qd)
    lse = torch.empty((H, qd.shape[0]), device=DEV)
    P.pbsa_attend(g, qd, qf, kp, vp, nq, kv, cnt, ld, o, lse, ws)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kp, float("nan"))
    dv = torch.full_like(vp, float("nan"))
    P.pbsa_attend_bwd(g, qd, qf, kp, vp, nq, kv, cnt, ld, o, dod, lse, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert P.pbsa_get_device_error(ws) == 0

    # the masks: every row of every head and sequence
    # (iid N(0,1) tokens give block representatives of std 1/8, so the top-16 boundary of about
    # one row in eight lies within 1e-4: those rows are checked for validity only)
    exact = check_lists_against_oracle(w, q, k, kv, cnt, sc, B, F, w.topk)
    assert exact >= B * H * 2 * 3 * bpf * 3 // 4

    # attention and gradients of two heads, every query block, under the GPU's (checked) masks
    kv_c, cnt_c = kv.cpu(), cnt.cpu()
    q64, k64, v64, do64 = (f64(t) for t in (q, k, v, do))
    gd = geom_dict(w)
    o_c, lse_c, dq_c, dk_c, dv_c = o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()
    for h in (0, 7):
        want_dk = np.zeros((nq, 64, d))
        want_dv = np.zeros((nq, 64, d))
        for r in range(nq):
            slots = kv_c[h, r, :int(cnt_c[h, r])].tolist()
            rows = block_rows(w, r)
            kk = np.concatenate([O.block_tokens(k64, gd, s)[:, h] for s in slots])
            vv = np.concatenate([O.block_tokens(v64, gd, s)[:, h] for s in slots])
            want_o, want_lse = O.attention(q64[rows, h], kk, vv, w.scale)
            assert_bf16_close(f64(o_c[rows, h]), want_o, f"o h{h} r{r}")
            np.testing.assert_allclose(f64(lse_c[h, rows]), want_lse, rtol=0, atol=2e-3)
            gq, gk, gv = O.attention_bwd(q64[rows, h], kk, vv, do64[rows, h], w.scale)
            _rel_close(f64(dq_c[rows, h]), gq, f"dq h{h} r{r}")
            for i, s in enumerate(slots):
                want_dk[s] += gk[i * 64:(i + 1) * 64]
                want_dv[s] += gv[i * 64:(i + 1) * 64]
        _rel_close(f64(dk_c[h]), want_dk, f"dk h{h}")
        _rel_close(f64(dv_c[h]), want_dv, f"dv h{h}")
