"""Comparison helpers shared by the parity tests (no attention arithmetic here)."""
from __future__ import annotations

import numpy as np

# bf16 outputs with fp32 accumulation against the fp64 oracle on the same bf16 inputs
MAX_ABS_TOL = 1e-2
REL_L2_TOL = 4e-3
# routing lists must agree except where a score lies this close to the k-th score
TIE_REL_TOL = 1e-4


def f64(t):
    import torch
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rel_l2(got, want):
    got, want = f64(got), f64(want)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def assert_close_out(got, want, what=""):
    got, want = f64(got), f64(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx = float(np.abs(got - want).max()) if got.size else 0.0
    rl = rel_l2(got, want)
    assert mx <= MAX_ABS_TOL and rl <= REL_L2_TOL, f"{what}: max-abs {mx:.3e}, rel-L2 {rl:.3e}"
    return mx, rl


def rows_agree_up_to_ties(gpu_cols, orc_cols, orc_scores_row, k_top, forced=()):
    """True if the selected sets are equal, or differ only in blocks whose oracle score
    is within TIE_REL_TOL (relative) of the oracle's k-th largest score. ``forced``
    blocks (padded ones) must be in both sets; the threshold is then the
    (k_top - len(forced))-th largest score among the other blocks."""
    g, o = set(int(x) for x in gpu_cols), set(int(x) for x in orc_cols)
    fset = set(int(x) for x in forced)
    if not (fset <= g and fset <= o):
        return False
    if g == o:
        return True
    s = np.asarray(orc_scores_row, dtype=np.float64)
    free = np.asarray([s[j] for j in range(len(s)) if j not in fset])
    kth = np.sort(free)[::-1][k_top - len(fset) - 1]
    tol = TIE_REL_TOL * max(abs(kth), 1e-30)
    return all(abs(s[j] - kth) <= tol for j in g ^ o)
