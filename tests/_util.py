"""Shared helpers of the GPU parity tests (comparison rules only)."""
import numpy as np

MARGIN = 1e-5   # decisions whose oracle margin exceeds this (relative) must agree exactly


def max_abs_rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


def check_decisions(gpu, want, margin, what, thr=MARGIN, max_low_margin=None):
    """Integer decisions decided by floating point: every position whose oracle
    margin is above thr must match exactly; below-threshold mismatches are
    counted and returned (they are legitimate rounding-order ties)."""
    gpu = np.asarray(gpu)
    want = np.asarray(want)
    margin = np.broadcast_to(np.asarray(margin, np.float64), want.shape)
    bad = (gpu != want)
    hard = bad & (margin > thr)
    assert not hard.any(), f"{what}: {int(hard.sum())} mismatches above margin {thr} at {np.nonzero(hard)}"
    low = int(bad.sum())
    if max_low_margin is not None:
        assert low <= max_low_margin, f"{what}: {low} low-margin mismatches"
    return low


def to_np(t):
    return t.detach().cpu().numpy()
