"""pbsa_memory_update_noalloc: the memory update for callers that cannot allocate device
memory (its scratch is a fixed array inside the library instead of a caller workspace).

Checked through the C-ABI against the workspace entry point pbsa_memory_update on the
same inputs, for two updates in a row (the second starts from the state the first left):
identical persistent sets, EMA values within the memory-update tolerance of the parity
tests, identical promoted K/V/representative copies and persistent-slot lists.  This file
is collected last so that a run stopping at the first failure has run everything else.
"""
import dataclasses

import pytest
import torch

import block_sparse_attention_pbsa_b200 as P
from block_sparse_attention_pbsa_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _state(seed, H, C, S, pool, d):
    gen = torch.Generator().manual_seed(seed)
    kr = torch.randn((H, pool, d), generator=gen) * 0.35
    kp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    vp = torch.randn((H, pool, 64, d), generator=gen).to(torch.bfloat16)
    sgid = torch.full((H, C), -1, dtype=torch.int32)
    sema = torch.zeros((H, C))
    for h in range(H):
        sgid[h, :S] = torch.arange(S, dtype=torch.int32)
        sema[h, :S] = torch.rand(S, generator=gen) * 0.02
    return [t.to(DEV) for t in (kr, kp, vp, sgid, sema)]


def _cands(seed, H, C, pool, ncand, first_gid):
    gen = torch.Generator().manual_seed(seed)
    cs = torch.stack([torch.randperm(pool - C, generator=gen)[:ncand] + C for _ in range(H)]).to(torch.int32)
    cg = (torch.arange(ncand, dtype=torch.int32) + first_gid).repeat(H, 1)
    return cs.to(DEV), cg.to(DEV)


@pytest.mark.parametrize("ncand", [72, 264])
def test_noalloc_matches_workspace_update_twice(ncand):
    # 72 candidates: the one-launch update (its scratch holds the error word); 264: the pool of
    # 360 entries takes the two-launch path, whose column partial sums, per-head completion
    # counts and copy list all live in the scratch
    H, d, nq, C, S = 12, 128, 72, 96, 24
    pool = C + 3 * ncand
    w = dataclasses.replace(I.DECODE_5S, heads=H)
    g = P.make_geom(H, d, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, "bf16")
    a = _state(1, H, C, S, pool, d)                  # updated by pbsa_memory_update
    b = [t.clone() for t in a]                       # updated by pbsa_memory_update_noalloc
    ws = torch.zeros(P.pbsa_workspace_bytes(g, nq, C + ncand), dtype=torch.uint8, device=DEV)
    lists = {k: (torch.zeros((H, C), dtype=torch.int32, device=DEV), torch.zeros(H, dtype=torch.int32, device=DEV))
             for k in "ab"}
    for call in range(2):
        gen = torch.Generator().manual_seed(100 + call)
        qr = (torch.randn((H, nq, d), generator=gen) * 0.3).to(DEV)
        cs, cg = _cands(200 + call, H, C, pool, ncand, first_gid=1000 * (call + 1))
        kr, kp, vp, sgid, sema = a
        P.pbsa_memory_update(g, qr, nq, kr, kp, vp, pool, sgid, sema, C, S, cs, cg, ncand, 0.9,
                             lists["a"][0], lists["a"][1], ws)
        kr, kp, vp, sgid, sema = b
        P.pbsa_memory_update_noalloc(g, qr, nq, kr, kp, vp, pool, sgid, sema, C, S, cs, cg, ncand, 0.9,
                                     lists["b"][0], lists["b"][1])
        torch.cuda.synchronize()
        assert P.pbsa_get_device_error(ws) == 0
        assert P.pbsa_memory_update_noalloc_error() == 0
        assert torch.equal(a[3], b[3]), f"call {call}: persistent sets differ"
        assert (a[3] >= 0).sum() > S, "the update promoted nothing; the check would be vacuous"
        torch.testing.assert_close(a[4], b[4], rtol=2e-5, atol=1e-9)
        for x, y in zip(a[:3], b[:3]):
            assert torch.equal(x, y), f"call {call}: pool contents differ"
        assert torch.equal(lists["a"][1], lists["b"][1])
        for h in range(H):
            n = int(lists["a"][1][h])
            assert torch.equal(lists["a"][0][h, :n], lists["b"][0][h, :n])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    H, d, C = 12, 128, 96
    g = P.make_geom(H, d, 32, 48, 8, 8, d ** -0.5, "bf16")
    nq, ncand = 4000, 1000                            # needs ~200 MB of scratch
    # the call is rejected on the host before any launch, so small buffers suffice
    kr = torch.zeros((H, 1, d), device=DEV)
    kp = torch.zeros((H, 1, 64, d), dtype=torch.bfloat16, device=DEV)
    qr = torch.zeros((H, 1, d), device=DEV)
    sgid = torch.full((H, C), -1, dtype=torch.int32, device=DEV)
    sema = torch.zeros((H, C), device=DEV)
    cs = torch.zeros((H, ncand), dtype=torch.int32, device=DEV)
    with pytest.raises(P.PBSAError) as e:
        P.pbsa_memory_update_noalloc(g, qr, nq, kr, kp, kp, C + ncand, sgid, sema, C, 24, cs, cs,
                                     ncand, 0.9)
    assert e.value.code == 2


def test_noalloc_reports_a_bad_candidate_slot_through_its_error_query():
    """Callers of the scratch-free update hold no workspace, so its device error word is read
    with pbsa_memory_update_noalloc_error: a candidate whose slot lies outside the pool is
    reported (PBSA_ERR_DEVICE_INDEX) and left out, like the workspace update does, and reading
    the word clears it.  The result equals the workspace update's on the same inputs."""
    H, d, nq, C, S, ncand = 2, 128, 24, 16, 4, 12
    w = dataclasses.replace(I.DECODE_5S, heads=H)
    g = P.make_geom(H, d, w.frame_h, w.frame_w, w.tile_h, w.tile_w, w.scale, "bf16")
    pool = C + ncand + 4
    a = _state(7, H, C, S, pool, d)
    b = [t.clone() for t in a]
    cs = (torch.arange(ncand, dtype=torch.int32) + C).repeat(H, 1)
    cs[1, 5] = pool + 9                               # out of range: checked and skipped on the device
    cg = (torch.arange(ncand, dtype=torch.int32) + 500).repeat(H, 1)
    cs, cg = cs.to(DEV), cg.to(DEV)
    qr = (torch.randn((H, nq, d), generator=torch.Generator().manual_seed(8)) * 0.3).to(DEV)
    ws = torch.zeros(P.pbsa_workspace_bytes(g, nq, C + ncand), dtype=torch.uint8, device=DEV)
    kr, kp, vp, sgid, sema = a
    P.pbsa_memory_update(g, qr, nq, kr, kp, vp, pool, sgid, sema, C, S, cs, cg, ncand, 0.9, ws=ws)
    kr, kp, vp, sgid, sema = b
    P.pbsa_memory_update_noalloc(g, qr, nq, kr, kp, vp, pool, sgid, sema, C, S, cs, cg, ncand, 0.9)
    assert P.pbsa_get_device_error(ws) == 5
    assert P.pbsa_memory_update_noalloc_error() == 5
    assert P.pbsa_memory_update_noalloc_error() == 0       # read once, cleared
    assert torch.equal(a[3], b[3]) and 505 not in b[3][1].tolist()
    torch.testing.assert_close(a[4], b[4], rtol=2e-5, atol=1e-9)
