"""Row-type comparison of the mask strategies, on the CPU with the oracle.

Pins (paper.rainbus.top summary, 问题与动机 limitation L1 and 核心创新点;
chatpaper.ai abstract (i)):
  * the error metric: the L1 distance between the block-sparse and the full
    attention row equals 2 (1 - exp(LSE_sparse - LSE_full)), checked against the
    attention rows written out token by token;
  * the pages' ordering on near-uniform and sink-skewed rows at equal block
    sparsity: Top-p beats Top-k on uniform rows, Top-k beats Top-p on skewed
    rows, and the hybrid avoids the failure of each.
"""

import numpy as np
import pytest
import torch

import oracle.spa2_oracle as O
from trainable_block_sparse_pooled_b200 import ablation, synth
from trainable_block_sparse_pooled_b200.calibrate import calibrate_p

BQ, BKV = 128, 64


def _f64(x):
    return x.float().double().numpy()


def test_row_l1_identity_against_explicit_attention_rows():
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=520, d=64, seed=3)
    Q, K, V = _f64(q), _f64(k), _f64(v)
    N, d = Q.shape[-2], Q.shape[-1]
    _, _, mask = O.block_mask(Q, K, BQ, BKV, 0.1, 0.3)
    Tm, Tn = mask.shape[-2:]
    full = np.ones_like(mask)
    _, lse_s = O.masked_attn_fwd(Q, K, V, mask, BQ, BKV)
    _, lse_f = O.masked_attn_fwd(Q, K, V, full, BQ, BKV)
    got = ablation.row_l1(torch.from_numpy(lse_s), torch.from_numpy(lse_f)).numpy()[0, 0]
    # attention rows written out: softmax over all columns, and over the kept ones
    s = (Q[0, 0] @ K[0, 0].T) / np.sqrt(d)
    p_full = np.exp(s - s.max(axis=1, keepdims=True))
    p_full /= p_full.sum(axis=1, keepdims=True)
    keep = O.token_mask(mask[0, 0], N, BQ, BKV)
    s_kept = np.where(keep, s, -np.inf)
    p_sparse = np.exp(s_kept - s_kept.max(axis=1, keepdims=True))
    p_sparse /= p_sparse.sum(axis=1, keepdims=True)
    want = np.abs(p_sparse - p_full).sum(axis=1)
    assert 0 < mask.sum() < Tm * Tn
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def _oracle_errors(Q, K, V, target):
    """Oracle counterpart of ablation.row_type_errors on one head."""
    Tm, Tn = O.block_counts(Q.shape[-2], BQ, BKV)
    total = Tm * Tn

    def mask_of(kf, pf):
        return O.block_mask(Q, K, BQ, BKV, kf, pf)[2]

    def kept(kf, pf):
        return int(mask_of(kf, pf).sum())

    params = {
        "topk": (1.0 - target, 0.0),
        "topp": calibrate_p(kept, total, target, k_frac=0.0)[:2],
        "hybrid": calibrate_p(kept, total, target)[:2],
    }
    _, lse_f = O.masked_attn_fwd(Q, K, V, np.ones((1, 1, Tm, Tn), bool), BQ, BKV)
    qblock = np.arange(Q.shape[-2]) // BQ
    out = {}
    for st, (kf, pf) in params.items():
        m = mask_of(kf, pf)
        _, lse = O.masked_attn_fwd(Q, K, V, m, BQ, BKV)
        e = ablation.row_l1(torch.from_numpy(lse), torch.from_numpy(lse_f)).numpy()[0, 0]
        out[st] = {"sparsity": 1.0 - m.sum() / total, "uniform": e[qblock % 2 == 0].mean(),
                   "skewed": e[qblock % 2 == 1].mean()}
    return out


@pytest.mark.parametrize("target", [0.8, 0.9])
def test_row_type_ordering_on_mixed_rows(target):
    q, k, v = synth.mixed_rows(B=1, H=1, N=4096, d=128, seed=4, grid=(4, 32, 32))
    res = _oracle_errors(_f64(q), _f64(k), _f64(v), target)
    for st in ablation.STRATEGIES:
        assert abs(res[st]["sparsity"] - target) <= 0.02, (st, res[st]["sparsity"])
    tk, tp, hy = res["topk"], res["topp"], res["hybrid"]
    assert tp["uniform"] < tk["uniform"]        # spread-out rows: a fixed count misses mass
    assert tk["skewed"] < tp["skewed"]          # sink rows: the threshold is met too early
    assert hy["uniform"] < tk["uniform"]        # the hybrid avoids both failures
    assert hy["skewed"] < tp["skewed"]


class _OracleSpa2:
    """CPU stand-in for binding.Spa2 with the oracle behind block_mask / fwd, so
    that ablation.row_type_errors' own logic (strategy parameters, row labels,
    means) runs without a GPU. Test infrastructure only."""

    class _Mask:
        def __init__(self, dense):
            self.dense = dense

        def kept_blocks(self):
            return int(self.dense.sum())

    def __init__(self, Q, K, V):
        self.torch = torch
        self.Q, self.K, self.V = Q, K, V
        self.B, self.H, self.N, self.d = Q.shape
        self.Tm, self.Tn = O.block_counts(self.N, BQ, BKV)

    def block_mask(self, q, k, k_frac, p_frac):
        return self._Mask(O.block_mask(self.Q, self.K, BQ, BKV, k_frac, p_frac)[2])

    def fwd(self, q, k, v, mask, want_o_lo=True):
        _, lse = O.masked_attn_fwd(self.Q, self.K, self.V, mask.dense, BQ, BKV)
        return None, torch.from_numpy(lse)

    def check(self):
        pass


def test_row_type_errors_aggregation_matches_direct_computation():
    q, k, v = synth.mixed_rows(B=1, H=1, N=4096, d=128, seed=4, grid=(4, 32, 32))
    Q, K, V = _f64(q), _f64(k), _f64(v)
    spa = _OracleSpa2(Q, K, V)
    got = ablation.row_type_errors(spa, torch.zeros(0), torch.zeros(0), torch.zeros(0), 0.9)
    want = _oracle_errors(Q, K, V, 0.9)
    for st in ablation.STRATEGIES:
        assert got[st]["sparsity"] == pytest.approx(want[st]["sparsity"], abs=1e-12)
        for lab in ("uniform", "skewed"):
            assert got[st][lab] == pytest.approx(want[st][lab], abs=1e-9), (st, lab)
