"""Shared helpers for the GPU parity tests: tolerances and comparisons.

Tolerances (the contract for bf16 inputs with fp32 accumulation; the page
"FlexAttention 是什么，以及 DFlash2 之谜的完整侦破", section 4, experiment 1,
measured a 0.0071 maximum deviation for FA2 bf16 against an fp32 reference):
  max |dO| <= 2e-2, mean |dO| <= 2e-3, max |dLSE| <= 1e-3 (rows with keys);
  rows with no visible key must give O == 0 exactly and LSE == -inf.
"""
import numpy as np
import torch

MAX_ABS_O = 2e-2
MEAN_ABS_O = 2e-3
MAX_ABS_LSE = 1e-3


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """o_gpu/lse_gpu: torch tensors (any device); o_ref/lse_ref: float64 numpy.

    Shapes: [..., d] and [...] with the same leading shape.
    """
    o = o_gpu.detach().float().cpu().double().numpy().reshape(o_ref.shape)
    lse = lse_gpu.detach().float().cpu().double().numpy().reshape(lse_ref.shape)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: fully-masked rows differ"
    if empty.any():
        assert np.all(o[empty] == 0.0), f"{what}: fully-masked rows must give O = 0"
    keep = ~empty
    if not keep.any():
        return {}
    assert np.isfinite(o[keep]).all() and np.isfinite(lse[keep]).all(), f"{what}: non-finite"
    d_o = np.abs(o[keep] - o_ref[keep])
    d_l = np.abs(lse[keep] - lse_ref[keep])
    stats = {"max_abs_o": float(d_o.max()), "mean_abs_o": float(d_o.mean()),
             "max_abs_lse": float(d_l.max())}
    assert stats["max_abs_o"] <= MAX_ABS_O, f"{what}: {stats}"
    assert stats["mean_abs_o"] <= MEAN_ABS_O, f"{what}: {stats}"
    assert stats["max_abs_lse"] <= MAX_ABS_LSE, f"{what}: {stats}"
    return stats


def to_dev(*ts, device="cuda"):
    return [None if t is None else t.to(device).contiguous() for t in ts]


def sample_rows(B, H, L, n_per_head, seed=0, must=()):
    """Flat row indices (b*H + h)*L + i: tile edges, the last rows and random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    edges = [0, 1, 126, 127, 128, 129, L - 2, L - 1]
    for b in range(B):
        for h in range(H):
            base = (b * H + h) * L
            for i in edges + list(must):
                if 0 <= i < L:
                    rows.add(base + i)
            for i in rng.integers(0, L, size=n_per_head):
                rows.add(base + int(i))
    return np.array(sorted(rows), dtype=np.int64)
