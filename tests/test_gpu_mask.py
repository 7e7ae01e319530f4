"""GPU parity of the mask path (pooling, pooled softmax, hybrid selection, CSC)
against the float64 oracle, through the C ABI."""

import os

import numpy as np
import pytest
import torch

import oracle
from tests._parity import csc_to_dense, csr_to_dense, f64
from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import synth

pytestmark = pytest.mark.gpu

# P-bar (GPU fp32 vs oracle fp64): max-abs 1e-5 (P-bar <= 1). fp32 pooling and
# dot products move a logit by ~1e-6 of its size, and P-bar moves by at most a
# quarter of the logit error (dP/ds = P (1 - P) <= 1/4).
PBAR_RTOL, PBAR_ATOL = 0.0, 1e-5


def _mask_case(q, k, kf, pf):
    B, H, N, d = q.shape
    s = b.Spa2(B, H, N, d, with_pbar=True, with_bitmap=True)
    m = s.block_mask(q, k, kf, pf)
    s.check(b.OP_MASK)
    return s, m


def _check_mask(q, k, kf, pf, min_agree=0.95):
    B, H, N, d = q.shape
    s, m = _mask_case(q, k, kf, pf)
    pbar_gpu = m.pbar.cpu().numpy()
    pbar64, _, mask_oracle = oracle.block_mask(f64(q), f64(k), 128, 64, kf, pf)
    np.testing.assert_allclose(pbar_gpu, pbar64, rtol=PBAR_RTOL, atol=PBAR_ATOL)
    # selection: bit-exact on identical (the GPU's) float32 P-bar
    want = oracle.select_blocks(pbar_gpu, kf, pf)
    got = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(m.bitmap.cpu().numpy().astype(bool), want)
    np.testing.assert_array_equal(csc_to_dense(m.col_cnt.cpu().numpy(), m.col_idx.cpu().numpy(), s.Tm), want)
    # the oracle's own float64 mask: near-ties may flip, so only an agreement rate
    agree = (got == mask_oracle).mean()
    assert agree >= min_agree, agree
    return m


def test_pr1_mask():
    q, k, _ = synth.gaussian_with_sinks(B=1, H=2, N=512, d=64, seed=0, device="cuda")
    _check_mask(q, k, 0.20, 0.60)


@pytest.mark.parametrize("N,d,kf,pf", [(1000, 128, 0.1, 0.5), (1000, 64, 0.3, 0.0), (77, 128, 0.0, 0.9),
                                       (4000, 128, 0.05, 0.9), (2500, 64, 1.0, 0.0), (700, 128, 0.0, 1.0)])
def test_ragged_masks(N, d, kf, pf):
    q, k, _ = synth.gaussian_with_sinks(B=2, H=3, N=N, d=d, seed=N + d, device="cuda")
    m = _check_mask(q, k, kf, pf)
    if kf >= 1.0:
        assert (m.row_cnt.cpu().numpy() == (N + 63) // 64).all()


def test_smoothed_field_mask_small_grid():
    q, k, _ = synth.smoothed_field(B=1, H=2, N=8192, d=128, seed=3, device="cuda")
    _check_mask(q, k, 0.025, 0.5)


def _golden_rows():
    path = os.path.join(os.path.dirname(__file__), "golden", "pages_rows.txt")
    from tests.test_oracle_selection import _golden
    assert os.path.exists(path)
    return _golden()


@pytest.mark.parametrize("rec", _golden_rows(), ids=lambda r: r[0])
def test_select_pages_rows(rec):
    _name, row, kf, pf, kept, _K, _R = rec
    pbar = torch.tensor(row, dtype=torch.float32, device="cuda").view(1, 1, 1, -1)
    m = b.select_blocks(pbar, kf, pf)
    n = int(m.row_cnt[0, 0, 0])
    assert m.row_idx[0, 0, 0, :n].cpu().tolist() == kept


def _hard_rows(rng, Tn, nrows):
    rows = []
    for r in range(nrows):
        kind = r % 6
        if kind == 0:
            x = rng.dirichlet(np.full(Tn, 0.3))
        elif kind == 1:                         # exact ties everywhere
            x = np.full(Tn, 1.0 / Tn)
        elif kind == 2:                         # planted tie groups
            x = rng.dirichlet(np.full(Tn, 1.0))
            x[rng.integers(0, Tn, Tn // 3)] = x[0]
        elif kind == 3:                         # sink + near-uniform tail
            x = np.full(Tn, 0.4 / max(Tn - 1, 1)); x[rng.integers(Tn)] = 0.6
        elif kind == 4:                         # one-hot (Top-p reaches p with one block)
            x = np.zeros(Tn); x[rng.integers(Tn)] = 1.0
        else:                                   # tiny values below 2^-32 mixed in
            x = rng.dirichlet(np.full(Tn, 0.05)); x[x < 1e-9] = 1e-12
        rows.append(x.astype(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("Tn", [1, 7, 32, 33, 512, 1182, 2048])
def test_select_bit_exact_hard_rows(Tn):
    rng = np.random.default_rng(Tn)
    rows = _hard_rows(rng, Tn, 36).reshape(2, 3, 6, Tn)
    pbar = torch.tensor(rows, device="cuda")
    for kf, pf in [(0.0, 0.0), (0.025, 0.5), (0.05, 0.9), (0.2, 0.6), (0.5, 1.0), (1.0, 0.3), (0.0, 0.95)]:
        m = b.select_blocks(pbar, kf, pf)
        got = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), Tn)
        np.testing.assert_array_equal(got, oracle.select_blocks(rows, kf, pf), err_msg=f"k={kf} p={pf}")
        np.testing.assert_array_equal(csc_to_dense(m.col_cnt.cpu().numpy(), m.col_idx.cpu().numpy(), 6), got)


@pytest.mark.slow
def test_wan13b_mask_sampled_rows():
    """Full 1.3B layer shape (B1 H12 N32760 d128): P-bar of every row against the
    oracle's pooled softmax, selection bit-exact on 96 sampled rows."""
    q, k, _ = synth.smoothed_field(B=1, H=12, N=32760, d=128, seed=1, device="cuda")
    s, m = _mask_case(q, k, 0.025, 0.6)
    pbar_gpu = m.pbar.cpu().numpy()
    pbar64 = oracle.pooled_attention(oracle.pool_blocks(f64(q), 128), oracle.pool_blocks(f64(k), 64), 128)
    np.testing.assert_allclose(pbar_gpu, pbar64, rtol=PBAR_RTOL, atol=PBAR_ATOL)
    rng = np.random.default_rng(0)
    cnt, idx = m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy()
    for _ in range(96):
        h, i = int(rng.integers(12)), int(rng.integers(s.Tm))
        want = oracle.select_row(pbar_gpu[0, h, i], 0.025, 0.6)
        assert list(idx[0, h, i, :cnt[0, h, i]]) == list(want)
    # the last (ragged, 56-row) kv block and 120-row q block are handled
    assert s.Tm == 256 and s.Tn == 512
