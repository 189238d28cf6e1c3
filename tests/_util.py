"""Test helpers: tolerance checks and small conversions (no method arithmetic)."""
from __future__ import annotations

import numpy as np
import torch

# Attention outputs / gradients with bf16 inputs and fp32 accumulation vs the float64 oracle.
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
# fp32 path vs the float64 oracle.
F32_MAX_ABS = 1e-5
# Selection: index sets must match exactly where the k-th and (k+1)-th scores differ by more.
NEAR_TIE = 1e-4
# Memory update: relative gap below which the top-(C-S) EMA boundary counts as a near tie.
EMA_NEAR_TIE_REL = 1e-4


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_bf16_close(got, want, what=""):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= BF16_MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= BF16_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"


def geom_dict(w) -> dict:
    return {"frame_h": w.frame_h, "frame_w": w.frame_w, "tile_h": w.tile_h, "tile_w": w.tile_w,
            "scale": w.scale}


def block_rows(w, r: int) -> np.ndarray:
    """Raster rows of query block r of a chunk (frame r // bpf of the chunk)."""
    tpr = w.frame_w // w.tile_w
    f, rem = divmod(r, w.blocks_per_frame)
    ty, tx = divmod(rem, tpr)
    return np.array([f * w.tokens_per_frame + (ty * w.tile_h + ly) * w.frame_w + tx * w.tile_w + lx
                     for ly in range(w.tile_h) for lx in range(w.tile_w)])
