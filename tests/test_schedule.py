"""The per-chunk top-k schedule (chunk-aware growth) of the package against the oracle's
restatement of the same rule.  Host logic: no GPU needed."""
import numpy as np
import pytest

from block_sparse_attention_pbsa_b200 import inputs as I
from block_sparse_attention_pbsa_b200 import schedule as S
from oracle import pbsa_oracle as O


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_sparsity_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 12))
    lq = rng.integers(64, 5000, size=n).tolist()
    lk = rng.integers(0, 50000, size=n).tolist()
    alpha = rng.uniform(0.0, 1.0, size=n).tolist()
    s_base = float(rng.uniform(0.5, 0.95))
    s_target = float(rng.uniform(0.3, s_base))
    n_dense = int(rng.integers(0, 2))
    beta, s = S.chunk_sparsity(lq, lk, 128, s_base, s_target, alpha, n_dense)
    beta_o, s_o = O.cag_sparsity(lq, lk, 128, s_base, s_target, alpha, n_dense)
    assert beta == pytest.approx(beta_o, rel=1e-12, abs=1e-15)
    np.testing.assert_allclose(s, s_o, rtol=1e-12, atol=1e-15)


def test_topk_matches_oracle():
    for s in np.linspace(0.0, 1.0, 21):
        for hist, pers, local in [(288, 96, 144), (72, 24, 48), (100, 10, 200), (24, 24, 0)]:
            assert S.chunk_topk(float(s), hist, pers, local) == O.cag_topk(float(s), hist, pers, local)


@pytest.mark.parametrize("w", [I.ROLLOUT_5S, I.ROLLOUT_1MIN])
def test_rollout_schedule(w):
    """Per chunk: the oracle's mapping of the oracle's sparsity, with the persistent and window
    block counts of the oracle's rollout state machine."""
    chunks = I.rollout_chunks(w)
    ks, sparsity, beta = S.rollout_topk(chunks, w.tokens_per_frame, w.blocks_per_frame, w.head_dim,
                                        w.capacity, w.window_frames, 0.7, 0.5)
    n = len(chunks)
    alpha = [1.0 - (i - 1) / max(1, n - 2) if i >= 1 else 1.0 for i in range(n)]
    beta_o, s_o = O.cag_sparsity([nf * w.tokens_per_frame for _, nf in chunks],
                                 [f0 * w.tokens_per_frame for f0, _ in chunks], w.head_dim, 0.7, 0.5, alpha)
    np.testing.assert_allclose(sparsity, s_o, rtol=1e-12, atol=1e-15)
    bpf = w.blocks_per_frame
    for (f0, _), s, k in zip(chunks, s_o, ks):
        local = len(O.window_frames(f0, w.window_frames)) * bpf if f0 > 0 else 0
        middle = len(range(1, max(1, f0 - w.window_frames))) if f0 > 0 else 0
        pers = min(w.capacity, bpf * (1 + middle)) if f0 > 0 else 0
        assert k == O.cag_topk(s, f0 * bpf, pers, local)
        assert 0 <= k <= local
