"""Shared comparison helpers for the GPU parity tests."""
import numpy as np
import torch

# Tolerance of the workloads (bf16 inputs, fp32 accumulation): element-wise
# max |delta| <= 1e-2 and mean |delta| <= 1e-3 against the fp64 oracle.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
# Block statistics are compared with this band: a block whose oracle statistic
# lies within it of the threshold may be decided either way.
NEAR_BAND = 1e-3


def assert_close(gpu, ref, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what="output"):
    g = gpu.detach().float().cpu().double().numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: non-finite pattern differs"
    d = np.abs(g[fin] - r[fin]) if fin.any() else np.zeros(1)
    assert d.max() <= max_abs, f"{what}: max |delta| = {d.max():.3g} > {max_abs}"
    assert d.mean() <= mean_abs, f"{what}: mean |delta| = {d.mean():.3g} > {mean_abs}"
    return float(d.max()), float(d.mean())


def compare_masks(gpu_mask, ora_mask, ora_stat, tau):
    """Block masks must agree except for blocks whose oracle statistic is within
    NEAR_BAND of the threshold; returns (n_blocks, n_near_disagreements, override)
    where override (int8, -1/0/1) replays the GPU's decisions on those blocks."""
    g = np.asarray(gpu_mask)
    o = np.asarray(ora_mask)
    diff = g != o
    H = o.shape[1]
    tau_b = np.asarray(tau, dtype=np.float64).reshape(1, H, 1, 1)
    near = np.abs(np.asarray(ora_stat) - tau_b) <= NEAR_BAND
    bad = diff & ~near
    assert not bad.any(), f"{int(bad.sum())} block decisions differ outside the near-threshold band"
    # never a listed/unlisted disagreement
    assert np.array_equal(g == 0, o == 0)
    override = np.full(o.shape, -1, np.int8)
    override[diff] = (g[diff] == 2).astype(np.int8)
    return int((o != 0).sum()), int(diff.sum()), override
