"""Choose k% and p% so that the hybrid mask reaches a target block sparsity.

The pages tune k% and p% by hand for a target sparsity (paper.rainbus.top
summary, 局限与改进 and 独立分析的弱点: manual calibration). This host-side
helper automates it: Top-k is fixed at half the kept budget, k = (1 - target)/2,
and p is bisected until the realised sparsity lies within `tol` of the target.
Realised sparsity is non-increasing in p (Top-p sets are nested), so the
bisection is well defined. The count function is supplied by the caller (the
GPU mask kernel in the bench, the oracle in CPU tests).
"""

from __future__ import annotations

from typing import Callable


def calibrate_p(kept_blocks: Callable[[float, float], int], total_blocks: int, target: float,
                k_frac: float | None = None, tol: float = 0.0025, iters: int = 40):
    """Return (k_frac, p_frac, realised_sparsity).

    kept_blocks(k, p) -> number of kept blocks over all rows of the problem.
    """
    if not 0.0 < target < 1.0:
        raise ValueError("target sparsity must lie in (0, 1)")
    k = (1.0 - target) / 2.0 if k_frac is None else k_frac

    def sparsity(p):
        return 1.0 - kept_blocks(k, p) / float(total_blocks)

    s_lo = sparsity(0.0)            # Top-k alone: the sparsest the pair can be
    if s_lo <= target + tol:
        return k, 0.0, s_lo
    lo, hi = 0.0, 1.0
    best = (abs(s_lo - target), 0.0, s_lo)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        s = sparsity(mid)
        if abs(s - target) < best[0]:
            best = (abs(s - target), mid, s)
        if abs(s - target) <= tol:
            return k, mid, s
        if s > target:
            lo = mid                # too sparse: keep more mass
        else:
            hi = mid
    return k, best[1], best[2]
