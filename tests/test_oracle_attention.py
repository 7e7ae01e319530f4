"""Pins for the oracle's masked attention forward and backward.

Checked against library routines (torch scaled_dot_product_attention and
autograd in float64, scipy logsumexp), the pages' error decomposition, and
central finite differences of the oracle's own forward.
"""

import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle


def _inputs(seed, B=1, H=2, N=200, d=16):
    rng = np.random.default_rng(seed)
    Q, K, V, dO = (rng.normal(size=(B, H, N, d)) for _ in range(4))
    return Q, K, V, dO


def _random_mask(seed, B, H, Tm, Tn, dens=0.4):
    rng = np.random.default_rng(seed)
    m = rng.random((B, H, Tm, Tn)) < dens
    m[..., 0] |= ~m.any(-1)         # no empty row
    return m


def _sdpa(Q, K, V, tok_mask, scale):
    q, k, v = (torch.tensor(x, dtype=torch.float64) for x in (Q, K, V))
    am = torch.tensor(tok_mask)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=am, scale=scale)


def _tok_masks(mask, N, bq, bkv):
    B, H = mask.shape[:2]
    return np.stack([np.stack([oracle.token_mask(mask[b, h], N, bq, bkv) for h in range(H)])
                     for b in range(B)])


def test_dense_equals_sdpa():
    Q, K, V, _ = _inputs(0)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = np.ones((B, H, Tm, Tn), dtype=bool)
    O, LSE = oracle.masked_attn_fwd(Q, K, V, mask, 128, 64)
    ref = _sdpa(Q, K, V, np.ones((B, H, N, N), bool), 1 / math.sqrt(d)).numpy()
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    s = np.einsum("bhnd,bhmd->bhnm", Q, K) / math.sqrt(d)
    np.testing.assert_allclose(LSE, logsumexp(s, axis=-1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_block_mask_equals_sdpa_token_mask(seed):
    Q, K, V, _ = _inputs(seed, N=333)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = _random_mask(seed, B, H, Tm, Tn)
    scale = 0.3
    O, LSE = oracle.masked_attn_fwd(Q, K, V, mask, 128, 64, scale)
    tm = _tok_masks(mask, N, 128, 64)
    np.testing.assert_allclose(O, _sdpa(Q, K, V, tm, scale).numpy(), rtol=0, atol=1e-12)
    s = np.einsum("bhnd,bhmd->bhnm", Q, K) * scale
    s = np.where(tm, s, -np.inf)
    np.testing.assert_allclose(LSE, logsumexp(s, axis=-1), rtol=0, atol=1e-12)


def test_error_decomposition():
    # SpargeAttention2 (paper.rainbus.top), 技术新颖性: O_full - O_sparse =
    # (p (.) (1 - m) + (1 - 1/tau) (p (.) m)) V with tau the kept mass of row p.
    Q, K, V, _ = _inputs(7, N=256)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = _random_mask(8, B, H, Tm, Tn, 0.5)
    O_sp, _ = oracle.masked_attn_fwd(Q, K, V, mask, 128, 64)
    O_full, _ = oracle.masked_attn_fwd(Q, K, V, np.ones_like(mask), 128, 64)
    s = np.einsum("bhnd,bhmd->bhnm", Q, K) / math.sqrt(d)
    p = np.exp(s - s.max(-1, keepdims=True)); p /= p.sum(-1, keepdims=True)
    m = _tok_masks(mask, N, 128, 64).astype(np.float64)
    tau = (p * m).sum(-1, keepdims=True)
    e = np.einsum("bhnm,bhmd->bhnd", p * (1 - m) + (1 - 1 / tau) * (p * m), V)
    np.testing.assert_allclose(O_full - O_sp, e, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [4, 5])
def test_backward_equals_autograd(seed):
    Q, K, V, dO = _inputs(seed, N=300)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = _random_mask(seed, B, H, Tm, Tn)
    scale = 1 / math.sqrt(d)
    dQ, dK, dV = oracle.masked_attn_bwd(Q, K, V, mask, dO, 128, 64)
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.tensor(_tok_masks(mask, N, 128, 64)), scale=scale)
    o.backward(torch.tensor(dO))
    np.testing.assert_allclose(dQ, q.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, k.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, v.grad.numpy(), rtol=0, atol=1e-11)


def test_backward_finite_differences():
    # d/dX sum(O * dO) by central differences of the oracle forward, tiny case
    Q, K, V, dO = _inputs(9, B=1, H=1, N=20, d=4)
    bq, bkv = 8, 4
    Tm, Tn = oracle.block_counts(20, bq, bkv)
    mask = _random_mask(9, 1, 1, Tm, Tn, 0.5)
    dQ, dK, dV = oracle.masked_attn_bwd(Q, K, V, mask, dO, bq, bkv)
    h = 1e-6

    def f(Qx, Kx, Vx):
        return float((oracle.masked_attn_fwd(Qx, Kx, Vx, mask, bq, bkv)[0] * dO).sum())

    rng = np.random.default_rng(0)
    for X, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        for _ in range(6):
            idx = (0, 0, int(rng.integers(20)), int(rng.integers(4)))
            args = [Q.copy(), K.copy(), V.copy()]
            args[which][idx] += h
            fp = f(*args)
            args[which][idx] -= 2 * h
            fm = f(*args)
            assert abs((fp - fm) / (2 * h) - G[idx]) < 1e-6


def test_attn_flops_counts_valid_rows_and_cols():
    N, bq, bkv, d = 200, 128, 64, 8
    Tm, Tn = oracle.block_counts(N, bq, bkv)
    mask = np.ones((Tm, Tn), bool)
    assert oracle.attn_flops(mask, N, bq, bkv, d) == 4 * d * N * N


@pytest.mark.parametrize("N,bq,bkv", [(1000, 128, 64), (333, 128, 64), (77, 64, 128), (2049, 256, 128)])
def test_attn_flops_equals_brute_token_count(N, bq, bkv):
    """Forward flops = 4 d per kept (query token, key token) pair: a random
    ragged block mask expanded token by token and counted element by element."""
    d = 128
    Tm, Tn = oracle.block_counts(N, bq, bkv)
    mask = _random_mask(N + bq, 2, 3, Tm, Tn, 0.3)
    brute = sum(int(oracle.token_mask(mask[b, h], N, bq, bkv).sum()) for b in range(2) for h in range(3))
    assert oracle.attn_flops(mask, N, bq, bkv, d) == 4.0 * d * brute
    # a mask that differs in one block changes the count by that block's token pairs
    m2 = mask.copy()
    m2[0, 0, Tm - 1, Tn - 1] ^= True
    rows, cols = N - (Tm - 1) * bq, N - (Tn - 1) * bkv
    delta = 4.0 * d * rows * cols * (1 if m2[0, 0, Tm - 1, Tn - 1] else -1)
    assert oracle.attn_flops(m2, N, bq, bkv, d) == oracle.attn_flops(mask, N, bq, bkv, d) + delta


def test_sampled_backward_matches_full_backward():
    Q, K, V, dO = _inputs(11, N=450)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = _random_mask(11, B, H, Tm, Tn, 0.4)
    scale = 1 / math.sqrt(d)
    dQ, dK, dV = oracle.masked_attn_bwd(Q, K, V, mask, dO, 128, 64)
    sq, skv = oracle.masked_attn_bwd_blocks(Q, K, V, mask, dO, 128, 64, scale, 0, 1, [1, 3], [0, 6])
    for i, g in sq.items():
        np.testing.assert_allclose(g, dQ[0, 1, i * 128:i * 128 + g.shape[0]], atol=1e-12)
    for j, (gk, gv) in skv.items():
        np.testing.assert_allclose(gk, dK[0, 1, j * 64:j * 64 + gk.shape[0]], atol=1e-12)
        np.testing.assert_allclose(gv, dV[0, 1, j * 64:j * 64 + gv.shape[0]], atol=1e-12)


def test_row_contributions_sum_to_full_backward():
    Q, K, V, dO = _inputs(12, N=400)
    B, H, N, d = Q.shape
    Tm, Tn = oracle.block_counts(N, 128, 64)
    mask = _random_mask(12, B, H, Tm, Tn, 0.5)
    scale = 1 / math.sqrt(d)
    dQ, dK, dV = oracle.masked_attn_bwd(Q, K, V, mask, dO, 128, 64)
    q1, k1, v1 = oracle.masked_attn_bwd_rows(Q, K, V, mask, dO, 128, 64, scale, 0, 1, [0, 2])
    q2, k2, v2 = oracle.masked_attn_bwd_rows(Q, K, V, mask, dO, 128, 64, scale, 0, 1, [1, 3])
    np.testing.assert_allclose(k1 + k2, dK[0, 1], atol=1e-12)
    np.testing.assert_allclose(v1 + v2, dV[0, 1], atol=1e-12)
    for i, g in {**q1, **q2}.items():
        np.testing.assert_allclose(g, dQ[0, 1, i * 128:i * 128 + g.shape[0]], atol=1e-12)
