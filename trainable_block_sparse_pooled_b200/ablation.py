"""Mask strategies compared by row type: Top-k alone, Top-p alone, and the hybrid.

The pages argue that Top-k fails on rows whose attention is spread out (a fixed
count of blocks misses most of the mass), that Top-p fails on rows dominated by
an attention sink (one or two blocks already reach the threshold), and that the
union of the two avoids both failures (paper.rainbus.top summary, 问题与动机
limitation L1 and 核心创新点; chatpaper.ai abstract (i)). Their error figures
come from real attention maps of Wan2.1. This module runs the same comparison
through this library's own kernels on seeded synthetic inputs, with each
strategy set to the same block sparsity.

Error of a mask on one query row r: the L1 distance between the block-sparse
attention row (softmax over the kept columns only) and the full attention row,

    || P_sparse,r - P_full,r ||_1 = 2 (1 - tau_r),

where tau_r is the full row's probability mass on the kept columns (kept
entries are scaled by 1 / tau_r, dropped ones lose all of their mass). Since
LSE_sparse,r = LSE_full,r + ln tau_r, the forward's LSE through the sparse mask
and through the all-kept mask give tau_r exactly.
"""

from __future__ import annotations

import json
import sys

from . import binding as b
from .calibrate import calibrate_p

STRATEGIES = ("topk", "topp", "hybrid")


def strategy_params(spa, q, k, strategy: str, target: float):
    """(k_frac, p_frac, realised block sparsity) of one strategy at `target`.

    topk: p = 0 and k = 1 - target; topp: k = 0 (one block per row, the least
    Top-k allows) and p bisected; hybrid: k = (1 - target) / 2 and p bisected.
    """
    total = spa.B * spa.H * spa.Tm * spa.Tn

    def kept(kk, pp):
        return spa.block_mask(q, k, kk, pp).kept_blocks()

    if strategy == "topk":
        kf = 1.0 - target
        return kf, 0.0, 1.0 - kept(kf, 0.0) / total
    if strategy == "topp":
        return calibrate_p(kept, total, target, k_frac=0.0)
    if strategy == "hybrid":
        return calibrate_p(kept, total, target)
    raise ValueError(f"unknown strategy {strategy!r}")


def row_l1(lse_sparse, lse_full):
    """Per-row L1 distance 2 (1 - exp(LSE_sparse - LSE_full)), clipped to [0, 2]."""
    return (2.0 * (1.0 - (lse_sparse - lse_full).exp())).clamp(0.0, 2.0)


def parity_row_type(qblock: int) -> str:
    """Row type of the mixed-rows inputs: even q-blocks near-uniform, odd skewed."""
    return "uniform" if qblock % 2 == 0 else "skewed"


def row_type_errors(spa, q, k, v, target: float, row_type=parity_row_type, strategies=STRATEGIES):
    """{strategy: {"k_frac", "p_frac", "sparsity", <row type>: mean row L1, ...}}.

    `row_type` maps a q-block index to a label; each label's value is the mean
    of `row_l1` over the token rows of the q-blocks it labels (all heads).
    """
    torch = spa.torch
    full = spa.block_mask(q, k, 1.0, 0.0)
    _, lse_full = spa.fwd(q, k, v, full, want_o_lo=False)
    qblock = torch.arange(spa.N, device=q.device) // b.BQ
    labels = {}
    for i in range(spa.Tm):
        labels.setdefault(row_type(i), []).append(i)
    rows = {lab: torch.isin(qblock, torch.tensor(ids, device=q.device)) for lab, ids in labels.items()}
    out = {}
    for st in strategies:
        kf, pf, sp = strategy_params(spa, q, k, st, target)
        m = spa.block_mask(q, k, kf, pf)
        _, lse = spa.fwd(q, k, v, m, want_o_lo=False)
        e = row_l1(lse, lse_full)
        res = {"k_frac": kf, "p_frac": pf, "sparsity": sp}
        for lab, sel in rows.items():
            res[lab] = float(e[..., sel].mean().item())
        out[st] = res
    spa.check()
    return out


def main(argv=None):
    """Row-type comparison on the 1.3B layer shape (mixed-rows inputs): one JSON
    line per (target sparsity, strategy)."""
    import argparse

    from . import synth

    ap = argparse.ArgumentParser(description=main.__doc__)
    ap.add_argument("--targets", default="0.8,0.9,0.95", help="comma-separated target block sparsities")
    ap.add_argument("--heads", type=int, default=12)
    ap.add_argument("--seed", type=int, default=2)
    args = ap.parse_args(argv)
    B, H, N, d = 1, args.heads, 32760, 128
    q, k, v = synth.mixed_rows(B=B, H=H, N=N, d=d, seed=args.seed, device="cuda")
    spa = b.Spa2(B, H, N, d)
    for t in (float(x) for x in args.targets.split(",")):
        for st, res in row_type_errors(spa, q, k, v, t).items():
            print(json.dumps({"ablation": "row_type_l1", "workload": f"mixed rows B{B} H{H} N{N} d{d}",
                              "target_sparsity": t, "strategy": st, **res}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
