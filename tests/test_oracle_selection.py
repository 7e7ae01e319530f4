"""Pins for the oracle's pooling, pooled softmax and hybrid selection.

Each test checks the oracle against something other than itself: the rows the
SpargeAttention2 pages print (tests/golden/pages_rows.txt), closed forms, and
brute force over every subset of a small row.
"""

import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_rows.txt")


def _parse_row(text):
    vals = []
    for part in text.split(","):
        part = part.strip()
        if " x " in part:
            v, n = part.split(" x ")
            vals += [float(v)] * int(n)
        else:
            vals.append(float(part))
    return np.array(vals, dtype=np.float32)


def _golden():
    recs = []
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, _src, row, k, p, kept, K, R = [x.strip() for x in line.split(" | ")]
            recs.append((name, _parse_row(row), float(k), float(p),
                         [int(x) for x in kept.split(",")], int(K), int(R)))
    return recs


@pytest.mark.parametrize("rec", _golden(), ids=lambda r: r[0])
def test_pages_rows(rec):
    _name, row, k, p, kept, K, R = rec
    order = oracle.spa2_oracle.rank_order(row)
    assert oracle.topk_count(k, row.shape[0]) == K
    assert oracle.topp_count(row, order, p) == R
    assert list(oracle.select_row(row, k, p)) == kept


def test_topp_inclusive_vs_exclusive():
    # The sink row: a ">" stop rule would also keep the 0.2 block; the page's
    # "Top-p(60%) selects only the sink" fixes the inclusive reading.
    row = np.array([0.6, 0.2, 0.1, 0.1], dtype=np.float32)
    assert list(oracle.select_row(row, 0.0, 0.6)) == [0]
    # a threshold just above the sink's mass needs the next block too
    assert list(oracle.select_row(row, 0.0, np.nextafter(np.float32(0.6), np.float32(1)))) == [0, 1]


def test_topk_rounding_is_half_up():
    # 0.2f * 10 = 2.0000000298; ceil would give 3, the pages' example says 2
    assert oracle.topk_count(0.2, 10) == 2
    assert oracle.topk_count(0.25, 10) == 3      # 2.5 rounds up
    assert oracle.topk_count(0.0, 10) == 1       # never an empty row
    assert oracle.topk_count(1.0, 10) == 10
    assert oracle.topk_count(0.05, 512) == 26    # 25.6 -> 26


def _q(v):
    return int(math.floor(float(np.float32(v)) * 2 ** 32))


def _brute_topk(row, K):
    # maximum quantised mass over all K-subsets; ties -> lexicographically smallest ids
    best = None
    for sub in itertools.combinations(range(len(row)), K):
        m = sum(_q(row[j]) for j in sub)
        key = (-m, sub)
        if best is None or key < best:
            best = key
    return set(best[1])


def _brute_topp(row, p):
    thr = int(math.floor(float(np.float32(p)) * 2 ** 32))
    n = len(row)
    for c in range(n + 1):
        for sub in itertools.combinations(range(n), c):
            if sum(_q(row[j]) for j in sub) >= thr:
                return c
    return n


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_small_rows(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 11))
    alpha = float(rng.choice([0.2, 1.0, 5.0]))
    row = rng.dirichlet(np.full(n, alpha)).astype(np.float32)
    if seed % 5 == 0:   # plant exact ties
        row[: n // 2] = row[0]
    k = float(rng.choice([0.0, 0.1, 0.2, 0.35, 0.5]))
    p = float(rng.choice([0.0, 0.3, 0.6, 0.9, 0.95]))
    K = oracle.topk_count(k, n)
    order = oracle.spa2_oracle.rank_order(row)
    R = oracle.topp_count(row, order, p)
    topk_set = _brute_topk(row, K)
    assert set(order[:K]) == topk_set
    assert R == _brute_topp(row, p)
    # the union: Top-k set U (a minimum-cardinality Top-p set taken in rank order)
    kept = set(oracle.select_row(row, k, p))
    assert kept == topk_set | set(order[:R])
    assert len(kept) == max(K, R)


@pytest.mark.parametrize("seed", range(10))
def test_monotone_in_k_and_p(seed):
    rng = np.random.default_rng(100 + seed)
    row = rng.dirichlet(np.full(64, 0.5)).astype(np.float32)
    prev = set()
    for k in np.linspace(0, 1, 11):
        cur = set(oracle.select_row(row, k, 0.3))
        assert prev <= cur
        prev = cur
    assert prev == set(range(64))
    prev = set()
    for p in np.linspace(0, 1, 11):
        cur = set(oracle.select_row(row, 0.05, p))
        assert prev <= cur
        prev = cur
    assert prev == set(range(64))     # p = 1 on a full-support row keeps all


def test_pool_closed_forms():
    # ramp rows x_r = r: the mean of rows [lo, hi) is (lo + hi - 1) / 2, ragged tail included
    N, d = 300, 4
    X = np.repeat(np.arange(N, dtype=np.float64)[:, None], d, axis=1)[None, None]
    P = oracle.pool_blocks(X, 128)
    assert P.shape == (1, 1, 3, d)
    np.testing.assert_array_equal(P[0, 0, :, 0], [63.5, 191.5, (256 + 299) / 2])
    # block-constant rows pool to the constant
    c = np.random.default_rng(0).normal(size=(3, d))
    Y = np.concatenate([np.tile(c[t], (min(64, 150 - 64 * t), 1)) for t in range(3)])[None, None]
    np.testing.assert_allclose(oracle.pool_blocks(Y, 64)[0, 0], c, rtol=0, atol=1e-13)


def test_pooled_attention_two_blocks_is_logistic():
    # two key blocks: P-bar row = (sigma(s0 - s1), sigma(s1 - s0)) with s = q.k / sqrt(d)
    d = 16
    a = 1.7
    Qbar = np.zeros((1, d)); Qbar[0, 0] = a
    Kbar = np.zeros((2, d)); Kbar[0, 0] = 2.0; Kbar[1, 1] = 5.0
    P = oracle.pooled_attention(Qbar, Kbar, d)
    s0 = a * 2.0 / 4.0
    assert abs(P[0, 0] - 1.0 / (1.0 + math.exp(-s0))) < 1e-15
    # identical key blocks give a uniform row; every row sums to 1
    Kb = np.tile(np.random.default_rng(1).normal(size=(1, d)), (7, 1))
    np.testing.assert_allclose(oracle.pooled_attention(np.random.default_rng(2).normal(size=(3, d)), Kb, d),
                               np.full((3, 7), 1 / 7), atol=1e-15)


def test_block_mask_end_to_end_small():
    # k = 100% keeps every block; k tiny with p = 0 keeps exactly one block per row,
    # the arg-max of the pooled logits (brute force over blocks)
    rng = np.random.default_rng(3)
    Q = rng.normal(size=(1, 2, 200, 8)); K = rng.normal(size=(1, 2, 200, 8))
    _, _, m = oracle.block_mask(Q, K, 128, 64, 1.0, 0.0)
    assert m.all()
    _, p32, m = oracle.block_mask(Q, K, 128, 64, 0.0, 0.0)
    assert (m.sum(-1) == 1).all()
    Qb = np.stack([Q[..., :128, :].mean(-2), Q[..., 128:, :].mean(-2)], axis=-2)
    Kb = np.stack([K[..., j * 64:min(200, j * 64 + 64), :].mean(-2) for j in range(4)], axis=-2)
    logits = np.einsum("bhid,bhjd->bhij", Qb, Kb)
    np.testing.assert_array_equal(m.argmax(-1), logits.argmax(-1))
