"""GPU parity of each C-ABI entry point against the CPU oracle, on seeded inputs.

Inputs are synthetic tensors built on the host (never outputs of the CUDA path); both
sides consume the same values (bf16 inputs are rounded once and up-converted for the
oracle).
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import inputs as I
from oracle import pbsa_oracle as O
from tests._util import (F32_MAX_ABS, NEAR_TIE, EMA_NEAR_TIE_REL, assert_bf16_close, block_rows,
                         f64, geom_dict)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def geom_for(w):
    return P.make_geom(w.heads, w.head_dim, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, w.dtype)


def ws_for(g, nq=64, pool=64):
    return torch.zeros(P.pbsa_workspace_bytes(g, nq, pool), dtype=torch.uint8, device=DEV)


def check_no_device_error(ws):
    assert P.pbsa_get_device_error(ws) == 0


# ----------------------------------------------------------------------------- blockify
@pytest.mark.parametrize("w", [I.TINY, I.DECODE_5S, dataclasses.replace(I.DECODE_5S, tile_h=4, tile_w=16)])
def test_blockify_reps_and_pool(w):
    g = geom_for(w)
    n_frames = 2
    x = I.tokens(w, n_frames, 11)
    nb = n_frames * w.blocks_per_frame
    slots = nb + 5
    dst = torch.randperm(slots, generator=torch.Generator().manual_seed(3))[:nb].to(torch.int32)
    reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV)
    pool = torch.zeros((w.heads, slots, 64, w.head_dim), dtype=x.dtype, device=DEV)
    ws = ws_for(g)
    P.pbsa_blockify(g, x.to(DEV), n_frames, reps, slots, dst.to(DEV), pool, slots, ws)
    check_no_device_error(ws)
    want = O.block_reps(f64(x), geom_dict(w), n_frames)
    got = f64(reps)
    for b in range(nb):
        s = int(dst[b])
        np.testing.assert_allclose(got[:, s], want[:, b], rtol=0, atol=2e-6)
        rows = O.block_token_rows(w.frame_h, w.frame_w, w.tile_h, w.tile_w, b)
        assert torch.equal(pool[:, s].cpu(), x[rows].permute(1, 0, 2))


@pytest.mark.parametrize("w,n_frames,with_v_reps", [(I.TINY, 3, True), (I.DECODE_5S, 7, False),
                                                     (I.DECODE_5S, 1, True),
                                                     (dataclasses.replace(I.DECODE_5S, tile_h=4, tile_w=16), 2, True)])
def test_blockify_kv_one_launch(w, n_frames, with_v_reps):
    """pbsa_blockify_kv: K and V of several frames in one launch (many units per CTA of the
    persistent grid), against the oracle's means and the raster rows of every block."""
    g = geom_for(w)
    k, v = I.tokens(w, n_frames, 21), I.tokens(w, n_frames, 22)
    nb = n_frames * w.blocks_per_frame
    slots = nb + 7
    dst = torch.randperm(slots, generator=torch.Generator().manual_seed(5))[:nb].to(torch.int32)
    k_reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV)
    v_reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV) if with_v_reps else None
    k_pool = torch.zeros((w.heads, slots, 64, w.head_dim), dtype=k.dtype, device=DEV)
    v_pool = torch.zeros_like(k_pool)
    ws = ws_for(g)
    P.pbsa_blockify_kv(g, k.to(DEV), v.to(DEV), n_frames, k_reps, v_reps, slots, dst.to(DEV), k_pool, v_pool,
                       slots, ws=ws)
    check_no_device_error(ws)
    want_k = O.block_reps(f64(k), geom_dict(w), n_frames)
    want_v = O.block_reps(f64(v), geom_dict(w), n_frames)
    got_k = f64(k_reps)
    got_v = f64(v_reps) if with_v_reps else None
    kp, vp = k_pool.cpu(), v_pool.cpu()
    for b in range(nb):
        s = int(dst[b])
        np.testing.assert_allclose(got_k[:, s], want_k[:, b], rtol=0, atol=2e-6)
        if with_v_reps:
            np.testing.assert_allclose(got_v[:, s], want_v[:, b], rtol=0, atol=2e-6)
        rows = O.block_token_rows(w.frame_h, w.frame_w, w.tile_h, w.tile_w, b)
        assert torch.equal(kp[:, s], k[rows].permute(1, 0, 2))
        assert torch.equal(vp[:, s], v[rows].permute(1, 0, 2))
    # slots that no block maps to stay untouched
    unused = sorted(set(range(slots)) - set(dst.tolist()))
    assert not kp[:, unused].any() and not vp[:, unused].any() and not k_reps[:, unused].any()
    # the K representatives equal pbsa_blockify's bit for bit (one summation order)
    k_reps1 = torch.zeros_like(k_reps)
    P.pbsa_blockify(g, k.to(DEV), n_frames, k_reps1, slots, dst.to(DEV), None, 0, ws)
    assert torch.equal(k_reps1, k_reps)


def test_blockify_kv_bad_slot_is_reported_and_skipped():
    """A destination slot outside the pool is recorded in the workspace's error word (index error,
    the bad slot) and that block is skipped; every other block is written as usual."""
    w = I.DECODE_5S
    g = geom_for(w)
    k, v = I.tokens(w, 1, 31), I.tokens(w, 1, 32)
    nb = w.blocks_per_frame
    slots = nb + 2
    dst = torch.arange(nb, dtype=torch.int32)
    dst[5] = slots + 100                               # outside the pool
    k_reps = torch.zeros((w.heads, slots, w.head_dim), device=DEV)
    k_pool = torch.zeros((w.heads, slots, 64, w.head_dim), dtype=k.dtype, device=DEV)
    v_pool = torch.zeros_like(k_pool)
    ws = ws_for(g)
    P.pbsa_blockify_kv(g, k.to(DEV), v.to(DEV), 1, k_reps, None, slots, dst.to(DEV), k_pool, v_pool, slots, ws=ws)
    torch.cuda.synchronize()
    word = ws[:16].view(torch.int32).tolist()
    assert word[0] == 5 and word[1] == slots + 100
    kp = k_pool.cpu()
    for b in range(nb):
        if b == 5:
            continue
        rows = O.block_token_rows(w.frame_h, w.frame_w, w.tile_h, w.tile_w, b)
        assert torch.equal(kp[:, b], k[rows].permute(1, 0, 2))
    assert not kp[:, 5].any() and not kp[:, nb:].any()   # nothing landed in unlisted slots


def test_bounded_wait_expires_is_reported_and_the_context_stays_usable():
    """The bounded mbarrier wait every kernel uses gives up after its limit: a wait on a barrier
    nothing arrives on (20 ms limit) returns, the error word reads PBSA_ERR_TIMEOUT, and the
    next kernel on the same context runs correctly."""
    import time
    w = I.TINY
    g = geom_for(w)
    ws = ws_for(g)
    t0 = time.perf_counter()
    P.pbsa_selftest_wait_timeout(ws, 20000)
    assert P.pbsa_get_device_error(ws) == 4            # PBSA_ERR_TIMEOUT (and the word is cleared)
    assert time.perf_counter() - t0 >= 0.019
    assert P.pbsa_get_device_error(ws) == 0
    x = I.tokens(w, 1, 41)
    reps = torch.zeros((w.heads, w.blocks_per_frame, w.head_dim), device=DEV)
    P.pbsa_blockify(g, x.to(DEV), 1, reps, w.blocks_per_frame, None, None, 0, ws)
    check_no_device_error(ws)
    np.testing.assert_allclose(f64(reps), O.block_reps(f64(x), geom_dict(w), 1), rtol=0, atol=2e-6)


# ----------------------------------------------------------------------------- score + select
def _selection_case(seed, H=3, nq=9, pool=200, ncand=144, d=128, k=32, prefix=20, dup=False):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn((H, nq, d), generator=gen) * 0.3 + torch.randn((H, 1, d), generator=gen) * 0.2
    kr = torch.randn((H, pool, d), generator=gen) * 0.3
    if dup:
        kr[:] = kr[:, :1]
    cs = torch.stack([torch.randperm(pool, generator=gen)[:ncand] for _ in range(H)]).to(torch.int32)
    cg = torch.stack([torch.randperm(5000, generator=gen)[:ncand] for _ in range(H)]).to(torch.int32)
    ps = torch.randint(0, pool, (H, prefix), generator=gen, dtype=torch.int32)
    pc = torch.tensor([prefix - h for h in range(H)], dtype=torch.int32)
    return q, kr, cs, cg, ps, pc


@pytest.mark.parametrize("dup", [False, True])
@pytest.mark.parametrize("ncand,k", [(144, 32), (48, 32), (20, 32), (300, 16), (0, 8)])
def test_score_select(ncand, k, dup):
    H, nq, d, pool, prefix = 3, 9, 128, 400, 20
    w = dataclasses.replace(I.DECODE_5S, heads=H)
    g = geom_for(w)
    q, kr, cs, cg, ps, pc = _selection_case(7 + ncand, H, nq, pool, ncand, d, k, prefix, dup)
    out_ld = prefix + k + 3
    out = torch.full((H, nq, out_ld), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((H, nq), dtype=torch.int32, device=DEV)
    sc = torch.zeros((H, nq, max(k, 1)), device=DEV)
    ws = ws_for(g)
    P.pbsa_score_select(g, q.to(DEV), nq, kr.to(DEV), pool, cs.to(DEV) if ncand else None,
                        cg.to(DEV) if ncand else None, ncand, k, ps.to(DEV), pc.to(DEV), prefix, out,
                        cnt, out_ld, sc, ws)
    check_no_device_error(ws)
    out, cnt, sc = out.cpu(), cnt.cpu(), sc.cpu()
    kk = min(k, ncand)
    checked = 0
    for h in range(H):
        for r in range(nq):
            p = int(pc[h])
            assert int(cnt[h, r]) == p + kk
            assert out[h, r, :p].tolist() == ps[h, :p].tolist()
            if ncand == 0:
                continue
            s64 = O.coarse_scores(f64(q[h, r:r + 1]), f64(kr[h][cs[h].long()]), w.scale)[0]
            s32 = s64.astype(np.float32)
            want_pos = O.topk_select(s32, cg[h].tolist(), k)
            got_slots = out[h, r, p:p + kk].tolist()
            np.testing.assert_allclose(sc[h, r, :kk].numpy(), s32[want_pos], rtol=0, atol=1e-5)
            if dup or O.kth_gap(s32, cg[h].tolist(), k) > NEAR_TIE:
                assert set(got_slots) == {int(cs[h, i]) for i in want_pos}
                checked += 1
            else:
                assert len(set(got_slots)) == kk and set(got_slots) <= set(cs[h].tolist())
    assert ncand == 0 or checked >= H * nq // 2


# ----------------------------------------------------------------------------- fused blockify + select
@pytest.mark.parametrize("wname,ncand,k,dup", [("decode", 144, 32, False), ("decode", 48, 32, False),
                                               ("decode", 300, 16, False), ("decode", 144, 32, True),
                                               ("decode", 0, 8, False), ("tiny", 8, 4, False),
                                               ("tile4x16", 20, 32, False),
                                               # either side of the 8-block kernel's 256-candidate limit
                                               ("decode", 256, 32, False), ("decode", 257, 32, False)])
def test_blockify_score_select(wname, ncand, k, dup):
    """pbsa_blockify_score_select: q reps = the oracle's block means (and bit-identical to
    pbsa_blockify), selection = the oracle's top-k of its own coarse scores outside near ties."""
    base = {"decode": dataclasses.replace(I.DECODE_5S, heads=3), "tiny": I.TINY,
            "tile4x16": dataclasses.replace(I.DECODE_5S, heads=2, tile_h=4, tile_w=16)}[wname]
    w = base
    g = geom_for(w)
    H, d, n_frames = w.heads, w.head_dim, 2
    nq = n_frames * w.blocks_per_frame
    x = I.tokens(w, n_frames, 21 + ncand)
    gen = torch.Generator().manual_seed(5 + ncand)
    pool, prefix = 400, 20
    kr = torch.randn((H, pool, d), generator=gen) * 0.3
    if dup:
        kr[:] = kr[:, :1]
    cs = torch.stack([torch.randperm(pool, generator=gen)[:ncand] for _ in range(H)]).to(torch.int32)
    cg = torch.stack([torch.randperm(5000, generator=gen)[:ncand] for _ in range(H)]).to(torch.int32)
    ps = torch.randint(0, pool, (H, prefix), generator=gen, dtype=torch.int32)
    pc = torch.tensor([prefix - h for h in range(H)], dtype=torch.int32)
    out_ld = prefix + k + 3
    out = torch.full((H, nq, out_ld), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((H, nq), dtype=torch.int32, device=DEV)
    sc = torch.zeros((H, nq, max(k, 1)), device=DEV)
    qr = torch.zeros((H, nq, d), device=DEV)
    ws = ws_for(g)
    xd = x.to(DEV)
    P.pbsa_blockify_score_select(g, xd, n_frames, qr, kr.to(DEV), pool, cs.to(DEV) if ncand else None,
                                 cg.to(DEV) if ncand else None, ncand, k, ps.to(DEV), pc.to(DEV), prefix,
                                 out, cnt, out_ld, sc, ws)
    check_no_device_error(ws)
    qr_sep = torch.zeros_like(qr)
    P.pbsa_blockify(g, xd, n_frames, qr_sep, nq, ws=ws)
    assert torch.equal(qr, qr_sep)
    want_q = O.block_reps(f64(x), geom_dict(w), n_frames)
    np.testing.assert_allclose(f64(qr), want_q, rtol=0, atol=2e-6)
    out, cnt, sc = out.cpu(), cnt.cpu(), sc.cpu()
    kk = min(k, ncand)
    checked = 0
    for h in range(H):
        for r in range(nq):
            p = int(pc[h])
            assert int(cnt[h, r]) == p + kk
            assert out[h, r, :p].tolist() == ps[h, :p].tolist()
            if ncand == 0:
                continue
            s64 = O.coarse_scores(want_q[h, r:r + 1], f64(kr[h][cs[h].long()]), w.scale)[0]
            s32 = s64.astype(np.float32)
            want_pos = O.topk_select(s32, cg[h].tolist(), k)
            got_slots = out[h, r, p:p + kk].tolist()
            np.testing.assert_allclose(sc[h, r, :kk].numpy(), s32[want_pos], rtol=0, atol=2e-5)
            if dup or O.kth_gap(s32, cg[h].tolist(), k) > NEAR_TIE:
                assert set(got_slots) == {int(cs[h, i]) for i in want_pos}
                checked += 1
            else:
                assert len(set(got_slots)) == kk and set(got_slots) <= set(cs[h].tolist())
    assert ncand == 0 or checked >= H * nq // 2


@pytest.mark.parametrize("wname,nf,top_frames,n_recent,k", [
    ("decode", 6, 3, 1, 32), ("decode", 6, 0, 1, 32), ("decode", 6, 5, 1, 32), ("decode", 6, 2, 0, 16),
    ("decode", 12, 4, 2, 40), ("tiny", 4, 1, 1, 4)])
def test_blockify_hsa_select(wname, nf, top_frames, n_recent, k):
    """pbsa_blockify_hsa_select against the oracle's two-level (frame, then block) selection;
    sets compared where neither cut-off is a near tie."""
    w = {"decode": dataclasses.replace(I.DECODE_5S, heads=3), "tiny": I.TINY}[wname]
    g = geom_for(w)
    H, d, bpf, n_frames = w.heads, w.head_dim, w.blocks_per_frame, 2
    nq = n_frames * bpf
    ncand = nf * bpf
    x = I.tokens(w, n_frames, 41 + nf + top_frames)
    gen = torch.Generator().manual_seed(9 + nf + 10 * top_frames + n_recent)
    pool, prefix = ncand + 50, 12
    # window reps: one offset per frame so that frames differ, plus block noise
    kr = torch.randn((H, pool, d), generator=gen) * 0.3
    frame_off = torch.randn((H, nf, d), generator=gen) * 0.3
    cs = torch.stack([torch.randperm(pool, generator=gen)[:ncand] for _ in range(H)]).to(torch.int32)
    for h in range(H):
        for c in range(ncand):
            kr[h, int(cs[h, c])] += frame_off[h, c // bpf]
    first_frame = 3
    cg = torch.tensor([[(first_frame + c // bpf) * bpf + c % bpf for c in range(ncand)]] * H, dtype=torch.int32)
    ps = torch.randint(0, pool, (H, prefix), generator=gen, dtype=torch.int32)
    pc = torch.tensor([prefix - h for h in range(H)], dtype=torch.int32)
    out_ld = prefix + k + 3
    out = torch.full((H, nq, out_ld), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((H, nq), dtype=torch.int32, device=DEV)
    qr = torch.zeros((H, nq, d), device=DEV)
    ws = ws_for(g)
    P.pbsa_blockify_hsa_select(g, x.to(DEV), n_frames, qr, kr.to(DEV), pool, cs.to(DEV), cg.to(DEV), ncand,
                               top_frames, n_recent, k, ps.to(DEV), pc.to(DEV), prefix, out, cnt, out_ld, None, ws)
    check_no_device_error(ws)
    want_q = O.block_reps(f64(x), geom_dict(w), n_frames)
    np.testing.assert_allclose(f64(qr), want_q, rtol=0, atol=2e-6)
    out, cnt = out.cpu(), cnt.cpu()
    nchosen = min(nf, n_recent + top_frames) * bpf
    checked = 0
    for h in range(H):
        reps_h = f64(kr[h][cs[h].long()])
        for r in range(nq):
            p = int(pc[h])
            kk = min(k, nchosen)
            assert int(cnt[h, r]) == p + kk
            assert out[h, r, :p].tolist() == ps[h, :p].tolist()
            pos, fgap, bgap = O.hsa_select(want_q[h, r], reps_h, cg[h].tolist(), bpf, top_frames, n_recent,
                                           k, w.scale)
            got = out[h, r, p:p + kk].tolist()
            assert len(set(got)) == kk and set(got) <= set(cs[h].tolist())
            if fgap > NEAR_TIE and bgap > NEAR_TIE:
                assert set(got) == {int(cs[h, c]) for c in pos}, (h, r)
                checked += 1
    assert checked >= H * nq // 2


# ----------------------------------------------------------------------------- attend
def _attend_case(w, q_frames, slots, lists, seed):
    gen = torch.Generator().manual_seed(seed)
    dt = w.torch_dtype
    q = (torch.randn((q_frames * w.tokens_per_frame, w.heads, w.head_dim), generator=gen)).to(dt)
    kp = torch.randn((w.heads, slots, 64, w.head_dim), generator=gen)
    kp = (kp + torch.randn((w.heads, slots, 1, w.head_dim), generator=gen) * 0.5).to(dt)
    vp = torch.randn((w.heads, slots, 64, w.head_dim), generator=gen).to(dt)
    nq = q_frames * w.blocks_per_frame
    ld = max(1, max(len(l) for row in lists for l in row))
    kv = torch.zeros((w.heads, nq, ld), dtype=torch.int32)
    cnt = torch.zeros((w.heads, nq), dtype=torch.int32)
    for h in range(w.heads):
        for r in range(nq):
            kv[h, r, :len(lists[h][r])] = torch.tensor(lists[h][r], dtype=torch.int32)
            cnt[h, r] = len(lists[h][r])
    return q, kp, vp, kv, cnt, ld


def _run_attend(w, q, q_frames, kp, vp, kv, cnt, ld):
    g = geom_for(w)
    o = torch.full(q.shape, float("nan"), dtype=q.dtype, device=DEV)
    lse = torch.zeros((w.heads, q.shape[0]), device=DEV)
    ws = ws_for(g)
    P.pbsa_attend(g, q.to(DEV), q_frames, kp.to(DEV), vp.to(DEV), kp.shape[1], kv.to(DEV), cnt.to(DEV),
                  ld, o, lse, ws)
    check_no_device_error(ws)
    return o.cpu(), lse.cpu()


def _oracle_unit(w, q, kp, vp, h, r, slots):
    rows = block_rows(w, r)
    kk = f64(kp[h][list(slots)].reshape(-1, w.head_dim)) if slots else np.zeros((0, w.head_dim))
    vv = f64(vp[h][list(slots)].reshape(-1, w.head_dim)) if slots else np.zeros((0, w.head_dim))
    return rows, O.attention(f64(q[rows, h]), kk, vv, w.scale)


def _lists(rng, H, nq, slots, shared, local, empty_every=0):
    out = []
    for h in range(H):
        pers = rng.choice(slots, size=shared, replace=False).tolist()
        rest = [s for s in range(slots) if s not in pers]
        rows = []
        for r in range(nq):
            if empty_every and r % empty_every == empty_every - 1:
                rows.append([])
                continue
            nl = int(rng.integers(0, local + 1))
            rows.append(pers + rng.choice(rest, size=nl, replace=False).tolist())
        out.append(rows)
    return out


def test_attend_f32_tiny():
    w = I.TINY
    rng = np.random.default_rng(0)
    slots = 24
    lists = _lists(rng, w.heads, 4, slots, 8, 4, empty_every=4)
    lists[0][0] = list(range(24))
    q, kp, vp, kv, cnt, ld = _attend_case(w, 1, slots, lists, 5)
    o, lse = _run_attend(w, q, 1, kp, vp, kv, cnt, ld)
    for r in range(4):
        rows, (want, wlse) = _oracle_unit(w, q, kp, vp, 0, r, lists[0][r])
        np.testing.assert_allclose(f64(o[rows, 0]), want, rtol=0, atol=F32_MAX_ABS)
        if lists[0][r]:
            np.testing.assert_allclose(f64(lse[0, rows]), wlse, rtol=0, atol=F32_MAX_ABS)
        else:
            assert np.isneginf(f64(lse[0, rows])).all()


@pytest.mark.parametrize("fh,fw,q_frames,shared,local,empty", [
    (8, 24, 1, 10, 6, 0),      # 3 query blocks: odd count, last CTA has one half
    (16, 16, 2, 20, 9, 5),     # empty lists and ragged counts
    (32, 48, 1, 96, 32, 0),    # the decode shape: 96 shared + 32 local
    (8, 8, 1, 1, 0, 0),        # a single block
])
def test_attend_bf16(fh, fw, q_frames, shared, local, empty):
    w = dataclasses.replace(I.DECODE_5S, heads=2, frame_h=fh, frame_w=fw)
    nq = q_frames * w.blocks_per_frame
    slots = max(shared + local + 7, 40)
    rng = np.random.default_rng(fh * 100 + fw)
    lists = _lists(rng, w.heads, nq, slots, shared, local, empty)
    q, kp, vp, kv, cnt, ld = _attend_case(w, q_frames, slots, lists, fh + fw)
    o, lse = _run_attend(w, q, q_frames, kp, vp, kv, cnt, ld)
    for h in range(w.heads):
        for r in range(nq):
            rows, (want, wlse) = _oracle_unit(w, q, kp, vp, h, r, lists[h][r])
            assert_bf16_close(f64(o[rows, h]), want, f"h{h} r{r}")
            if lists[h][r]:
                np.testing.assert_allclose(f64(lse[h, rows]), wlse, rtol=0, atol=2e-3)
            else:
                assert np.isneginf(f64(lse[h, rows])).all()


def test_attend_bf16_running_max_grows():
    """Key magnitudes grow geometrically along every (sorted) list, so each row's running
    maximum jumps by more than 2^8 at many steps of both softmax streams and both S buffers:
    the path that rescales the O accumulator, against the oracle."""
    w = dataclasses.replace(I.DECODE_5S, heads=2, frame_h=16, frame_w=16)
    q_frames, slots = 2, 48
    nq = q_frames * w.blocks_per_frame
    rng = np.random.default_rng(7)
    lists = [[sorted(rng.choice(slots, size=int(rng.integers(9, 41)), replace=False).tolist()) for _ in range(nq)]
             for _ in range(w.heads)]
    q, kp, vp, kv, cnt, ld = _attend_case(w, q_frames, slots, lists, 11)
    kp = (kp.float() * (1.12 ** torch.arange(slots, dtype=torch.float32)).view(1, slots, 1, 1)).to(kp.dtype)
    o, lse = _run_attend(w, q, q_frames, kp, vp, kv, cnt, ld)
    jumps = 0
    for h in range(w.heads):
        for r in range(nq):
            rows, (want, wlse) = _oracle_unit(w, q, kp, vp, h, r, lists[h][r])
            assert_bf16_close(f64(o[rows, h]), want, f"h{h} r{r}")
            np.testing.assert_allclose(f64(lse[h, rows]), wlse, rtol=1e-5, atol=2e-3)
            # how often the running maximum (log2 units) grew by more than 8 along the list
            lg = w.scale / np.log(2.0) * f64(q[rows, h]) @ f64(kp[h][lists[h][r]]).reshape(-1, w.head_dim).T
            bm = lg.reshape(len(rows), len(lists[h][r]), 64).max(axis=2)
            run = np.maximum.accumulate(bm, axis=1)
            jumps += int((bm[:, 1:] > run[:, :-1] + 8).sum())
    assert jumps > 100


def test_attend_bf16_short_lists():
    """Merged lists of 0 to 5 steps (128 keys each): fewer steps than the kernel's three S
    buffers, exactly three, and more, so the first S of each buffer, the last PV and the
    hand-offs between the two softmax streams are exercised at each count.  The two query
    blocks of a pair attend disjoint blocks (one sometimes nothing), so the merged list, its
    masks and the odd last step differ from either list."""
    w = dataclasses.replace(I.DECODE_5S, heads=2, frame_h=8, frame_w=64)   # 8 query blocks, 4 pairs
    nq, slots = w.blocks_per_frame, 40
    rng = np.random.default_rng(23)
    # (|A|, |B|) per pair, disjoint lists: merged lengths 0, 1, 2, 3, 5, 6, 7, 9 -> 0 to 5 steps
    sizes = [(0, 0), (1, 0), (1, 1), (2, 1), (3, 2), (0, 6), (4, 3), (5, 4)]
    lists = []
    for h in range(w.heads):
        rows = []
        for p in range(nq // 2):
            na, nb = sizes[h * (nq // 2) + p]
            perm = rng.permutation(slots).tolist()
            rows += [perm[:na], perm[na:na + nb]]
        lists.append(rows)
    q, kp, vp, kv, cnt, ld = _attend_case(w, 1, slots, lists, 29)
    o, lse = _run_attend(w, q, 1, kp, vp, kv, cnt, ld)
    for h in range(w.heads):
        for r in range(nq):
            rows, (want, wlse) = _oracle_unit(w, q, kp, vp, h, r, lists[h][r])
            assert_bf16_close(f64(o[rows, h]), want, f"h{h} r{r}")
            if lists[h][r]:
                np.testing.assert_allclose(f64(lse[h, rows]), wlse, rtol=0, atol=2e-3)
            else:
                assert np.isneginf(f64(lse[h, rows])).all()


@pytest.mark.parametrize("case", ["pool_above_bitmap", "merged_list_at_capacity"])
def test_attend_bf16_list_merge_limits(case):
    """The pair's list merge at its limits: a pool of more slots than the membership bitmaps
    cover (the quadratic merge, slots above 8192 in the lists), and two disjoint lists of the
    maximum length 512 (a merged list of 1024 entries)."""
    w = dataclasses.replace(I.DECODE_5S, heads=1, frame_h=8, frame_w=16)   # 2 query blocks
    rng = np.random.default_rng(3)
    if case == "pool_above_bitmap":
        slots = 8300
        shared = rng.choice(np.arange(8100, slots), size=12, replace=False).tolist()
        lists = [[shared + rng.choice(slots, size=n, replace=False).tolist() for n in (20, 9)]]
    else:
        slots = 1024
        perm = rng.permutation(slots).tolist()
        lists = [[perm[:512], perm[512:]]]
    q, kp, vp, kv, cnt, ld = _attend_case(w, 1, slots, lists, 17)
    o, lse = _run_attend(w, q, 1, kp, vp, kv, cnt, ld)
    for r in range(2):
        rows, (want, wlse) = _oracle_unit(w, q, kp, vp, 0, r, lists[0][r])
        assert_bf16_close(f64(o[rows, 0]), want, f"r{r}")
        np.testing.assert_allclose(f64(lse[0, rows]), wlse, rtol=0, atol=2e-3)


def test_attend_bf16_bad_slot_is_reported():
    w = dataclasses.replace(I.DECODE_5S, heads=1, frame_h=8, frame_w=16)
    lists = [[[0, 1, 999], [2, 3]]]
    q, kp, vp, kv, cnt, ld = _attend_case(w, 1, 8, lists, 1)
    g = geom_for(w)
    ws = ws_for(g)
    o = torch.zeros(q.shape, dtype=q.dtype, device=DEV)
    P.pbsa_attend(g, q.to(DEV), 1, kp.to(DEV), vp.to(DEV), 8, kv.to(DEV), cnt.to(DEV), ld, o, None, ws)
    assert P.pbsa_get_device_error(ws) == 5
    assert P.pbsa_get_device_error(ws) == 0   # cleared by the read
    # the bad entry is skipped: the row equals attention over the two valid blocks
    rows, (want, _) = _oracle_unit(w, q, kp, vp, 0, 0, [0, 1])
    assert_bf16_close(f64(o.cpu()[rows, 0]), want)


def test_invalid_arguments_are_rejected_on_host():
    w = I.DECODE_5S
    g = geom_for(w)
    x = torch.zeros((w.tokens_per_frame, w.heads, w.head_dim), dtype=torch.bfloat16, device=DEV)
    reps = torch.zeros((w.heads, 24, w.head_dim), device=DEV)
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_blockify(g, x, 0, reps, 24)
    assert e.value.code == 1
    bad = P.make_geom(12, 128, 32, 48, 8, 7, w.scale, "bf16")
    with pytest.raises(P.PBSAError):
        P.pbsa_blockify(bad, x, 1, reps, 24)


# ----------------------------------------------------------------------------- memory update
@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("n_pers,ncand,C,nq", [(70, 72, 96, 72), (24, 48, 96, 72), (96, 72, 96, 72), (0, 264, 96, 72),
                                               (3, 5, 8, 72),
                                               # either side of the one-launch limits: 256 pool entries, 128 query blocks
                                               (96, 160, 96, 72), (96, 161, 96, 72), (70, 72, 96, 128),
                                               (70, 72, 96, 129)])
def test_memory_update(n_pers, ncand, C, nq, split):
    _check_memory_update(n_pers, ncand, C, nq, split)


def _check_memory_update(n_pers, ncand, C, nq, split, gamma=0.9):
    """pbsa_memory_update, or (split) pbsa_memory_update_plan + pbsa_memory_update_apply --
    one CTA per head for pools of up to 256 entries, the two-launch score kernel above -- against
    the oracle: kept sets (outside EMA near-ties), EMA values, promoted copies, persistent list."""
    H, d, S = 3, 128, min(24, C // 2)
    w = dataclasses.replace(I.DECODE_5S, heads=H)
    g = geom_for(w)
    gen = torch.Generator().manual_seed(n_pers * 1000 + ncand)
    pool = C + ncand + 10
    qr = torch.randn((H, nq, d), generator=gen) * 0.3 + torch.randn((H, 1, d), generator=gen) * 0.3
    kr = torch.randn((H, pool, d), generator=gen) * 0.35
    kp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    vp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    sgid = torch.full((H, C), -1, dtype=torch.int32)
    sema = torch.zeros((H, C))
    cs = torch.zeros((H, ncand), dtype=torch.int32)
    cg = torch.zeros((H, ncand), dtype=torch.int32)
    for h in range(H):
        pslots = torch.randperm(C, generator=gen)[:n_pers]
        gids = torch.randperm(4000, generator=gen)[:n_pers + ncand] + S
        ns = min(S, n_pers) if n_pers else 0
        for i, s in enumerate(pslots.tolist()):
            sgid[h, s] = i if i < ns else int(gids[i])        # the first ns are sinks (gid < S)
            sema[h, s] = float(torch.rand((), generator=gen)) * 0.02
        cs[h] = torch.randperm(pool - C, generator=gen)[:ncand].to(torch.int32) + C
        cg[h] = gids[n_pers:n_pers + ncand].to(torch.int32)
        if n_pers == 0 and ncand >= S:
            cg[h, :S] = torch.arange(S, dtype=torch.int32)   # sinks arriving as candidates
    kr_d, kp_d, vp_d = kr.to(DEV), kp.to(DEV), vp.to(DEV)
    cs_d, cg_d = (cs.to(DEV), cg.to(DEV)) if ncand else (None, None)
    sgid_d, sema_d = sgid.to(DEV), sema.to(DEV)
    plist = torch.full((H, C), -5, dtype=torch.int32, device=DEV)
    pcnt = torch.zeros((H,), dtype=torch.int32, device=DEV)
    ws = torch.zeros(P.pbsa_workspace_bytes(g, nq, C + ncand), dtype=torch.uint8, device=DEV)
    if split:
        P.pbsa_memory_update_plan(g, qr.to(DEV), nq, kr_d, pool, sgid_d, sema_d, C, S, cs_d, cg_d, ncand,
                                  gamma, plist, pcnt, ws=ws)
        P.pbsa_memory_update_apply(g, kr_d, kp_d, vp_d, pool, C, ncand, ws=ws)
    else:
        P.pbsa_memory_update(g, qr.to(DEV), nq, kr_d, kp_d, vp_d, pool, sgid_d, sema_d, C, S, cs_d,
                             cg_d, ncand, gamma, plist, pcnt, ws)
    check_no_device_error(ws)
    new_gid, new_ema = sgid_d.cpu(), sema_d.cpu()
    for h in range(H):
        ent = [(s, int(sgid[h, s]), float(sema[h, s])) for s in range(C) if sgid[h, s] >= 0]
        ent += [(int(cs[h, i]), int(cg[h, i]), np.nan) for i in range(ncand)]
        slots_, gids_, prev = zip(*ent)
        sink = [gg < S for gg in gids_]
        ema, keep, a = O.memory_update(f64(qr[h]), f64(kr[h][list(slots_)]), gids_, prev, sink, w.scale, gamma, C)
        want = {gg for gg, kp_ in zip(gids_, keep) if kp_}
        got = {int(x) for x in new_gid[h] if x >= 0}
        assert len(got) <= C and {gg for gg in gids_ if gg < S} <= got
        if O.ema_boundary_gap(ema, gids_, sink, C) > EMA_NEAR_TIE_REL:
            assert got == want
        ema_of = dict(zip(gids_, ema))
        src_of = dict(zip(gids_, slots_))
        for s in range(C):
            gg = int(new_gid[h, s])
            if gg < 0:
                continue
            np.testing.assert_allclose(float(new_ema[h, s]), ema_of[gg], rtol=2e-5, atol=1e-9)
            src = src_of[gg]
            if src != s:   # promoted: K, V, k_reps copied into slot s
                assert src >= C
                assert torch.equal(kp_d[h, s].cpu(), kp[h, src]) and torch.equal(vp_d[h, s].cpu(), vp[h, src])
                assert torch.equal(kr_d[h, s].cpu(), kr[h, src])
        valid = [s for s in range(C) if new_gid[h, s] >= 0]
        assert int(pcnt[h]) == len(valid) and plist[h, :len(valid)].cpu().tolist() == valid


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("n_pers,ncand,C,gamma", [
    (70, 72, 96, 0.0),     # the EMA is the chunk's attention alone
    (70, 72, 96, 1.0),     # the EMA of a block seen before never moves
    (20, 30, 96, 0.9),     # capacity above the entries: everything is kept, no eviction
    (70, 0, 96, 0.9),      # no candidates: re-scoring and EMA only
])
def test_memory_update_degenerate(n_pers, ncand, C, gamma, split):
    """The update at its degenerate points, against the oracle (same checks as above)."""
    _check_memory_update(n_pers, ncand, C, 72, split, gamma)


@pytest.mark.parametrize("split", [False, True])
def test_memory_update_bad_candidate_slot_is_reported_and_dropped(split):
    """A candidate whose slot lies outside the staging range is reported (PBSA_ERR_DEVICE_INDEX)
    and left out of the softmax and the ranking: the result is the oracle's over the others."""
    H, d, nq, C, S, ncand = 1, 128, 24, 16, 4, 12
    w = dataclasses.replace(I.DECODE_5S, heads=H)
    g = geom_for(w)
    gen = torch.Generator().manual_seed(99)
    pool = C + ncand + 4
    qr = torch.randn((H, nq, d), generator=gen) * 0.3
    kr = torch.randn((H, pool, d), generator=gen) * 0.35
    kp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    vp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    sgid = torch.full((H, C), -1, dtype=torch.int32)
    sema = torch.zeros((H, C))
    for s_ in range(10):                       # 4 sinks + 6 earlier blocks
        sgid[0, s_] = s_ if s_ < S else 100 + s_
        sema[0, s_] = 0.01 * (s_ % 3)
    cs = (torch.arange(ncand, dtype=torch.int32) + C).view(H, ncand).clone()
    cg = (torch.arange(ncand, dtype=torch.int32) + 500).view(H, ncand).clone()
    cs[0, 3] = pool + 7                        # out of range
    kr_d, kp_d, vp_d, sgid_d, sema_d = (t.to(DEV) for t in (kr, kp, vp, sgid, sema))
    plist = torch.full((H, C), -5, dtype=torch.int32, device=DEV)
    pcnt = torch.zeros((H,), dtype=torch.int32, device=DEV)
    ws = torch.zeros(P.pbsa_workspace_bytes(g, nq, C + ncand), dtype=torch.uint8, device=DEV)
    if split:
        P.pbsa_memory_update_plan(g, qr.to(DEV), nq, kr_d, pool, sgid_d, sema_d, C, S, cs.to(DEV), cg.to(DEV),
                                  ncand, 0.9, plist, pcnt, ws=ws)
        P.pbsa_memory_update_apply(g, kr_d, kp_d, vp_d, pool, C, ncand, ws=ws)
    else:
        P.pbsa_memory_update(g, qr.to(DEV), nq, kr_d, kp_d, vp_d, pool, sgid_d, sema_d, C, S, cs.to(DEV),
                             cg.to(DEV), ncand, 0.9, plist, pcnt, ws)
    assert P.pbsa_get_device_error(ws) == 5
    ent = [(s_, int(sgid[0, s_]), float(sema[0, s_])) for s_ in range(C) if sgid[0, s_] >= 0]
    ent += [(int(cs[0, i]), int(cg[0, i]), np.nan) for i in range(ncand) if i != 3]
    slots_, gids_, prev = zip(*ent)
    sink = [gg < S for gg in gids_]
    ema, keep, _ = O.memory_update(f64(qr[0]), f64(kr[0][list(slots_)]), gids_, prev, sink, w.scale, 0.9, C)
    got = {int(x) for x in sgid_d.cpu()[0] if x >= 0}
    assert int(cg[0, 3]) not in got
    if O.ema_boundary_gap(ema, gids_, sink, C) > EMA_NEAR_TIE_REL:
        assert got == {gg for gg, k_ in zip(gids_, keep) if k_}
    ema_of = dict(zip(gids_, ema))
    new_ema = sema_d.cpu()
    for s_ in range(C):
        gg = int(sgid_d[0, s_])
        if gg >= 0:
            np.testing.assert_allclose(float(new_ema[0, s_]), ema_of[gg], rtol=2e-5, atol=1e-9)
