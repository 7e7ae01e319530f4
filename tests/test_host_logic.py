"""Host-side logic that needs no GPU: sparsity calibration (against the oracle's
mask as the counting function) and the bench's flop / byte accounting."""

import numpy as np

import oracle
from trainable_block_sparse_pooled_b200 import calibrate, synth


def test_calibration_hits_target_with_oracle_counts():
    q, k, _ = synth.smoothed_field(B=1, H=2, N=8192, d=64, seed=0, grid=(8, 32, 32))
    Qb = oracle.pool_blocks(q.float().numpy().astype(np.float64), 128)
    Kb = oracle.pool_blocks(k.float().numpy().astype(np.float64), 64)
    pbar32 = oracle.pooled_attention(Qb, Kb, 64).astype(np.float32)
    total = pbar32.shape[0] * pbar32.shape[1] * pbar32.shape[2] * pbar32.shape[3]

    def kept(kf, pf):
        return int(oracle.select_blocks(pbar32, kf, pf).sum())

    kf, pf, s = calibrate.calibrate_p(kept, total, 0.90, tol=0.01)
    assert abs(kf - 0.05) < 1e-12
    assert abs(s - 0.90) <= 0.01
    assert abs((1 - kept(kf, pf) / total) - s) < 1e-12


def test_calibration_returns_topk_only_when_target_is_loose():
    kf, pf, s = calibrate.calibrate_p(lambda k, p: 10, 100, 0.95)
    assert pf == 0.0 and abs(s - 0.9) < 1e-12


def test_code_digest_ignores_comments_but_not_code():
    import bench
    src = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    same = "// header\nint f(int x) {\n\n  return x + 1;  // plus one\n}\n"
    changed = "int f(int x) {\n  return x + 2;  // add one\n}\n"
    assert bench.code_text_digest(src) == bench.code_text_digest(same)
    assert bench.code_text_digest(src) != bench.code_text_digest(changed)



def test_calibration_bisection_property():
    """For any kept-count curve that grows continuously in p (here a + (1 - a) p^g
    of a million blocks), the bisection lands within its tolerance of every
    target that Top-k alone overshoots."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=200, deadline=None)
    @given(a=st.floats(0.001, 0.5), g=st.floats(0.2, 5.0), target=st.floats(0.05, 0.95))
    def check(a, g, target):
        total = 1_000_000

        def kept(k, p):
            return int(total * (a + (1.0 - a) * p ** g))

        kf, pf, s = calibrate.calibrate_p(kept, total, target)
        assert 0.0 <= pf <= 1.0
        assert s == 1.0 - kept(kf, pf) / total
        if 1.0 - a > target + 0.0025:
            assert abs(s - target) <= 0.0025
        else:
            assert pf == 0.0

    check()


def test_bench_kept_flops_equals_oracle_attn_flops():
    """bench.kept_flops (the numerator of every TFLOP/s figure) counts, from the
    CSR form of a mask, what oracle.attn_flops counts from its dense form."""
    import torch

    import bench
    from trainable_block_sparse_pooled_b200 import binding as b

    rng = np.random.default_rng(3)
    for N, bq, bkv in ((1000, 128, 64), (32760, 128, 64), (333, 128, 64), (5000, 256, 128), (700, 64, 128)):
        Tm, Tn = oracle.block_counts(N, bq, bkv)
        dense = rng.random((2, 3, Tm, Tn)) < 0.2
        dense[..., rng.integers(Tn)] = True                       # no empty row
        cnt = dense.sum(-1).astype(np.int32)
        idx = np.full((2, 3, Tm, Tn), -1, dtype=np.int32)         # unused tail entries hold garbage
        for pos in np.ndindex(cnt.shape):
            ids = np.flatnonzero(dense[pos])
            idx[pos][:ids.size] = ids
        m = b.Mask(torch.tensor(cnt), torch.tensor(idx), None, None)
        assert bench.kept_flops(m, N, 128, bq, bkv) == oracle.attn_flops(dense, N, bq, bkv, 128)
