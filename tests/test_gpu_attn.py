"""GPU parity of the block-sparse attention forward (O, LSE) and backward
(dQ, dK, dV) against the float64 oracle, under the GPU's own block mask,
through the C ABI. Tolerance: max-abs 2e-2 and relative L1 1e-2."""

import numpy as np
import pytest
import torch

import oracle
from tests._parity import Accum, AccumBf16, assert_close, assert_close_bf16_out, csr_to_dense, f64
from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import synth

pytestmark = pytest.mark.gpu


def _run(q, k, v, kf, pf, dout=None, mask=None):
    B, H, N, d = q.shape
    s = b.Spa2(B, H, N, d)
    m = s.block_mask(q, k, kf, pf) if mask is None else mask
    o, lse = s.fwd(q, k, v, m)
    grads = None
    if dout is not None:
        grads = s.bwd(q, k, v, o, lse, dout, m)
    s.check()
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    return s, m, dense, o, lse, grads


def _o32(s, o):
    """O carried to ~16 mantissa bits: the bf16 output plus its bf16 residual."""
    return f64(o) + f64(s.o_lo)


def _check_fwd(q, k, v, dense, o, lse, s=None):
    O, LSE = oracle.masked_attn_fwd(f64(q), f64(k), f64(v), dense, 128, 64)
    if s is not None:
        assert_close(_o32(s, o), O, "O (o + o_lo)")
    assert_close_bf16_out(f64(o), O, "O (bf16)")
    assert_close(lse.cpu().numpy(), LSE, "LSE")


def _check_bwd(q, k, v, dense, dout, grads):
    dQ, dK, dV = oracle.masked_attn_bwd(f64(q), f64(k), f64(v), dense, f64(dout), 128, 64)
    assert_close(f64(grads[0]), dQ, "dQ")
    assert_close(f64(grads[1]), dK, "dK")
    assert_close(f64(grads[2]), dV, "dV")


def test_pr1_fwd_bwd():
    """B=1 H=2 N=512 d=64, N(0,1) with 2 sinks, k=20% p=60%, forward + backward."""
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=512, d=64, seed=0, device="cuda")
    dout = synth.normal_like(q.shape, seed=1, device="cuda")
    s, _, dense, o, lse, grads = _run(q, k, v, 0.2, 0.6, dout)
    _check_fwd(q, k, v, dense, o, lse, s)
    _check_bwd(q, k, v, dense, dout, grads)


@pytest.mark.parametrize("N,d,kf,pf", [(1000, 128, 0.1, 0.5), (1000, 64, 0.2, 0.3), (130, 128, 0.0, 0.7),
                                       (2049, 128, 0.05, 0.9), (333, 64, 1.0, 0.0)])
def test_ragged_fwd_bwd(N, d, kf, pf):
    q, k, v = synth.gaussian_with_sinks(B=2, H=2, N=N, d=d, seed=N, device="cuda")
    dout = synth.normal_like(q.shape, seed=N + 1, device="cuda")
    s, _, dense, o, lse, grads = _run(q, k, v, kf, pf, dout)
    _check_fwd(q, k, v, dense, o, lse, s)
    _check_bwd(q, k, v, dense, dout, grads)


@pytest.mark.parametrize("d", [128, 64])
def test_bf16_gradients_within_tolerance_plus_output_rounding(d):
    """bf16 gradient outputs: the stated tolerance plus half a bf16 ulp of each
    expected value (the representation error of the output format itself).
    N = 1000 leaves a ragged last q-block (104 rows) and kv-block (40 rows)."""
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=1000, d=d, seed=12, device="cuda")
    dout = synth.normal_like(q.shape, seed=13, device="cuda")
    s = b.Spa2(1, 2, 1000, d)
    m = s.block_mask(q, k, 0.1, 0.6)
    o, lse = s.fwd(q, k, v, m)
    g16 = s.bwd(q, k, v, o, lse, dout, m, grad_dtype=b.DTYPE_BF16)
    s.check()
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    ref = oracle.masked_attn_bwd(f64(q), f64(k), f64(v), dense, f64(dout), 128, 64)
    for name, g, e in zip(("dQ", "dK", "dV"), g16, ref):
        assert g.dtype == torch.bfloat16
        half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(e), 1e-30))) - 8)
        err = np.abs(f64(g) - e)
        assert (err <= 2e-2 + half_ulp).all(), f"{name}: worst excess {(err - 2e-2 - half_ulp).max():.3e}"
        assert err.sum() / np.abs(e).sum() <= 1e-2, name


def test_dense_k100_equals_full_attention():
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=640, d=128, seed=5, device="cuda")
    s, m, dense, o, lse, _ = _run(q, k, v, 1.0, 0.0)
    assert dense.all()
    ref = torch.nn.functional.scaled_dot_product_attention(q.double().cpu(), k.double().cpu(), v.double().cpu())
    assert_close(_o32(s, o), ref.numpy(), "O vs SDPA")
    assert_close_bf16_out(f64(o), ref.numpy(), "O (bf16) vs SDPA")


def test_uncovered_kv_block_gets_zero_grads():
    """A kv-block no q-block keeps: dK = dV = 0 there (CSC column is empty)."""
    B, H, N, d = 1, 1, 640, 128
    q, k, v = synth.gaussian_with_sinks(B=B, H=H, N=N, d=d, seed=9, device="cuda")
    dout = synth.normal_like(q.shape, seed=10, device="cuda")
    Tm, Tn = b.block_counts(N)
    rng = np.random.default_rng(0)
    pbar = rng.dirichlet(np.ones(Tn), size=(B, H, Tm)).astype(np.float32)
    pbar[..., 3] = 0.0
    mask = b.select_blocks(torch.tensor(pbar, device="cuda"), 0.2, 0.5)
    assert int(mask.col_cnt[0, 0, 3]) == 0
    s, _, dense, o, lse, grads = _run(q, k, v, 0, 0, dout, mask=mask)
    assert not dense[..., 3].any()
    assert torch.count_nonzero(grads[1][0, 0, 192:256]) == 0
    assert torch.count_nonzero(grads[2][0, 0, 192:256]) == 0
    _check_fwd(q, k, v, dense, o, lse, s)
    _check_bwd(q, k, v, dense, dout, grads)


def test_forward_is_deterministic():
    q, k, v = synth.gaussian_with_sinks(B=1, H=4, N=3000, d=128, seed=2, device="cuda")
    s = b.Spa2(1, 4, 3000, 128)
    m = s.block_mask(q, k, 0.05, 0.8)
    o1, l1 = s.fwd(q, k, v, m)
    o2, l2 = s.fwd(q, k, v, m)
    s.check()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_mixed_rows_fwd_bwd_small():
    """Mixed-rows recipe (near-uniform even q-blocks, +6-logit skewed odd q-blocks,
    k=5% p=90%) on the 8x32x32 grid, whole heads, forward and backward."""
    q, k, v = synth.mixed_rows(B=1, H=2, N=8192, d=128, seed=4, device="cuda", grid=(8, 32, 32))
    dout = synth.normal_like(q.shape, seed=5, device="cuda")
    s, m, dense, o, lse, grads = _run(q, k, v, 0.05, 0.9, dout)
    cnt = m.row_cnt.cpu().numpy()[0]
    assert cnt[:, 0::2].mean() > cnt[:, 1::2].mean()      # uniform rows keep more blocks
    _check_fwd(q, k, v, dense, o, lse, s)
    _check_bwd(q, k, v, dense, dout, grads)


@pytest.mark.slow
def test_wan13b_fwd_sampled_qblocks():
    """1.3B layer (B1 H12 N32760 d128, smoothed field + 4 sinks) at k=2.5% p=60%:
    16 seeded q-blocks per head plus the last (120-row) q-block, every head."""
    q, k, v = synth.smoothed_field(B=1, H=12, N=32760, d=128, seed=1, device="cuda")
    s, m, dense, o, lse, _ = _run(q, k, v, 0.025, 0.6)
    rng = np.random.default_rng(0)
    qf, kf_, vf = f64(q), f64(k), f64(v)
    o32, o16 = _o32(s, o), f64(o)
    l64 = lse.cpu().numpy()
    acc_o, acc_o16, acc_l = Accum("O (o + o_lo)"), AccumBf16("O (bf16)"), Accum("LSE")
    for h in range(12):
        blocks = sorted(set(rng.integers(0, s.Tm - 1, 16).tolist()) | {s.Tm - 1})
        ref = oracle.masked_attn_fwd_rows(qf, kf_, vf, dense, 128, 64, 1 / np.sqrt(128), 0, h, blocks)
        for i, (Oi, Li) in ref.items():
            rows = slice(i * 128, i * 128 + Oi.shape[0])
            acc_o.add(o32[0, h, rows], Oi)
            acc_o16.add(o16[0, h, rows], Oi)
            acc_l.add(l64[0, h, rows], Li)
    acc_o.check()
    acc_o16.check()
    acc_l.check()


def _calibrated_layer(q, k, target):
    """Spa2 + mask of the layer at `target` block sparsity (k = (1 - target) / 2,
    p bisected with the GPU's own mask), as the bench calibrates it."""
    from trainable_block_sparse_pooled_b200 import calibrate
    B, H, N, d = q.shape
    s = b.Spa2(B, H, N, d)
    m = s.new_mask()

    def kept(kf, pf):
        s.block_mask(q, k, kf, pf, m)
        return m.kept_blocks()

    kf, pf, sp = calibrate.calibrate_p(kept, B * H * s.Tm * s.Tn, target)
    assert abs(sp - target) <= 0.0025
    s.block_mask(q, k, kf, pf, m)
    return s, m, kf, pf


@pytest.mark.slow
def test_wan13b_bench_operating_point():
    """The exact configuration bench.py times: the 1.3B layer (B1 H12 N32760 d128)
    from the smoothed-field generator with seed 0, dO from seed 1000, k = 2.5% and
    p calibrated to 95% block sparsity, forward + fp32-gradient backward.
    Forward: O (bf16 and o + o_lo) and LSE of 16 seeded q-blocks plus the ragged
    last one in every head. Backward: dQ of 8 sampled q-blocks (the ragged last one
    included) and dK, dV of 8 sampled kv-blocks (the ragged last one included) in
    heads 0, 5 and 11."""
    import bench
    wl = bench.WORKLOADS["wan2.1-1.3b-layer"]
    q, k, v, dout = bench.make_inputs(wl, seed=0, device="cuda")
    s, m, kf, pf = _calibrated_layer(q, k, 0.95)
    assert abs(kf - 0.025) < 1e-12
    o, lse = s.fwd(q, k, v, m)
    grads = s.bwd(q, k, v, o, lse, dout, m)
    s.check()
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    qf, kf_, vf, df = f64(q), f64(k), f64(v), f64(dout)
    o32, o16, l64 = _o32(s, o), f64(o), lse.cpu().numpy()
    dq, dk, dv = (f64(g) for g in grads)
    sc = 1 / np.sqrt(128)
    rng = np.random.default_rng(2024)
    acc = {n: (AccumBf16(n) if n == "O (bf16)" else Accum(n))
           for n in ("O (o + o_lo)", "O (bf16)", "LSE", "dQ", "dK", "dV")}
    for h in range(12):
        blocks = sorted(set(rng.integers(0, s.Tm - 1, 16).tolist()) | {s.Tm - 1})
        ref = oracle.masked_attn_fwd_rows(qf, kf_, vf, dense, 128, 64, sc, 0, h, blocks)
        for i, (Oi, Li) in ref.items():
            rows = slice(i * 128, i * 128 + Oi.shape[0])
            acc["O (o + o_lo)"].add(o32[0, h, rows], Oi)
            acc["O (bf16)"].add(o16[0, h, rows], Oi)
            acc["LSE"].add(l64[0, h, rows], Li)
    for h in (0, 5, 11):
        qb = sorted(set(rng.integers(0, s.Tm - 1, 7).tolist()) | {s.Tm - 1})
        kb = sorted(set(rng.integers(0, s.Tn - 1, 7).tolist()) | {s.Tn - 1})
        sq, skv = oracle.masked_attn_bwd_blocks(qf, kf_, vf, dense, df, 128, 64, sc, 0, h, qb, kb)
        for i, g in sq.items():
            acc["dQ"].add(dq[0, h, i * 128:i * 128 + g.shape[0]], g)
        for j, (gk, gv) in skv.items():
            acc["dK"].add(dk[0, h, j * 64:j * 64 + gk.shape[0]], gk)
            acc["dV"].add(dv[0, h, j * 64:j * 64 + gv.shape[0]], gv)
    for a in acc.values():
        a.check()


@pytest.mark.slow
def test_wan13b_bwd_sampled_blocks():
    """1.3B shape, mixed rows, k=5% p=90%, forward + backward:
    dQ of 8 sampled q-blocks and dK, dV of 8 sampled kv-blocks (the last, ragged,
    one included) in heads 0 and 11, against the oracle."""
    q, k, v = synth.mixed_rows(B=1, H=12, N=32760, d=128, seed=2, device="cuda")
    dout = synth.normal_like(q.shape, seed=3, device="cuda")
    s, m, dense, o, lse, grads = _run(q, k, v, 0.05, 0.9, dout)
    rng = np.random.default_rng(1)
    qf, kf_, vf, df = f64(q), f64(k), f64(v), f64(dout)
    dq, dk, dv = (f64(g) for g in grads)
    acc = {n: Accum(n) for n in ("dQ", "dK", "dV")}
    for h in (0, 11):
        qb = sorted(set(rng.integers(0, s.Tm, 8).tolist()))
        kb = sorted(set(rng.integers(0, s.Tn - 1, 7).tolist()) | {s.Tn - 1})
        sq, skv = oracle.masked_attn_bwd_blocks(qf, kf_, vf, dense, df, 128, 64, 1 / np.sqrt(128), 0, h, qb, kb)
        for i, g in sq.items():
            acc["dQ"].add(dq[0, h, i * 128:i * 128 + g.shape[0]], g)
        for j, (gk, gv) in skv.items():
            acc["dK"].add(dk[0, h, j * 64:j * 64 + gk.shape[0]], gk)
            acc["dV"].add(dv[0, h, j * 64:j * 64 + gv.shape[0]], gv)
    for a in acc.values():
        a.check()


@pytest.mark.slow
def test_wan14b_fwd_bwd_sampled():
    """14B layer (B1 H40 N75600 d128, smoothed field + 4 sinks, 591 x 1182 blocks) at
    95% block sparsity (k = 2.5%, p calibrated): O and LSE of 16 seeded q-blocks plus
    the ragged last one in heads 0, 17 and 39; dQ of 6 q-blocks and dK, dV of 6
    kv-blocks plus the ragged last one in heads 0 and 39."""
    B, H, N, d = 1, 40, 75600, 128
    q, k, v = synth.smoothed_field(B=B, H=H, N=N, d=d, seed=5, device="cuda")
    dout = synth.normal_like(q.shape, seed=6, device="cuda")
    s, m, _, _ = _calibrated_layer(q, k, 0.95)
    o, lse = s.fwd(q, k, v, m)
    grads = s.bwd(q, k, v, o, lse, dout, m)
    s.check()
    heads = [0, 17, 39]
    dense_all = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    dense = dense_all[:, heads]
    sl = lambda t: f64(t[:, heads])  # noqa: E731
    qf, kf_, vf, df = sl(q), sl(k), sl(v), sl(dout)
    o32 = f64(o[:, heads]) + f64(s.o_lo[:, heads])
    l64 = lse[:, heads].cpu().numpy()
    dq, dk, dv = (sl(g) for g in grads)
    rng = np.random.default_rng(7)
    acc = {n: Accum(n) for n in ("O (o + o_lo)", "LSE", "dQ", "dK", "dV")}
    for hi, h in enumerate(heads):
        blocks = sorted(set(rng.integers(0, s.Tm - 1, 16).tolist()) | {s.Tm - 1})
        ref = oracle.masked_attn_fwd_rows(qf, kf_, vf, dense, 128, 64, 1 / np.sqrt(d), 0, hi, blocks)
        for i, (Oi, Li) in ref.items():
            rows = slice(i * 128, i * 128 + Oi.shape[0])
            acc["O (o + o_lo)"].add(o32[0, hi, rows], Oi)
            acc["LSE"].add(l64[0, hi, rows], Li)
        if h in (0, 39):
            qb = sorted(set(rng.integers(0, s.Tm, 6).tolist()))
            kb = sorted(set(rng.integers(0, s.Tn - 1, 6).tolist()) | {s.Tn - 1})
            sq, skv = oracle.masked_attn_bwd_blocks(qf, kf_, vf, dense, df, 128, 64, 1 / np.sqrt(d), 0, hi, qb, kb)
            for i, g in sq.items():
                acc["dQ"].add(dq[0, hi, i * 128:i * 128 + g.shape[0]], g)
            for j, (gk, gv) in skv.items():
                acc["dK"].add(dk[0, hi, j * 64:j * 64 + gk.shape[0]], gk)
                acc["dV"].add(dv[0, hi, j * 64:j * 64 + gv.shape[0]], gv)
    for a in acc.values():
        a.check()


@pytest.mark.parametrize("bq,bkv", [(64, 64), (64, 128), (128, 128), (256, 64), (256, 128)])
@pytest.mark.parametrize("N,d", [(1000, 128), (777, 64)])
def test_block_sizes_mask_fwd_bwd(bq, bkv, N, d):
    """Block sizes other than (128, 64) (per-layer block sizes): pooled softmax and
    selection (bit-exact on the GPU's own P-bar) with the oracle's block
    partition, CSC, then O, LSE, dQ, dK, dV against the oracle under that mask.
    N = 1000 and 777 leave ragged last blocks of every size (777 with b_q = 64
    leaves the last 128-row query tile half empty)."""
    from tests._parity import csc_to_dense
    B, H = 1, 2
    q, k, v = synth.gaussian_with_sinks(B=B, H=H, N=N, d=d, seed=bq * 7 + bkv + N, device="cuda")
    dout = synth.normal_like(q.shape, seed=N + bq + bkv, device="cuda")
    s = b.Spa2(B, H, N, d, bq=bq, bkv=bkv, with_pbar=True)
    kf, pf = 0.15, 0.5
    m = s.block_mask(q, k, kf, pf)
    o, lse = s.fwd(q, k, v, m)
    grads = s.bwd(q, k, v, o, lse, dout, m)
    s.check()
    Tm, Tn = oracle.block_counts(N, bq, bkv)
    assert (s.Tm, s.Tn) == (Tm, Tn)
    pbar = m.pbar.cpu().numpy()
    pbar64 = oracle.pooled_attention(oracle.pool_blocks(f64(q), bq), oracle.pool_blocks(f64(k), bkv), d)
    np.testing.assert_allclose(pbar, pbar64, rtol=0, atol=1e-5)
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), Tn)
    np.testing.assert_array_equal(dense, oracle.select_blocks(pbar, kf, pf))
    np.testing.assert_array_equal(csc_to_dense(m.col_cnt.cpu().numpy(), m.col_idx.cpu().numpy(), Tm), dense)
    O, LSE = oracle.masked_attn_fwd(f64(q), f64(k), f64(v), dense, bq, bkv)
    assert_close(_o32(s, o), O, "O (o + o_lo)")
    assert_close_bf16_out(f64(o), O, "O (bf16)")
    assert_close(lse.cpu().numpy(), LSE, "LSE")
    dQ, dK, dV = oracle.masked_attn_bwd(f64(q), f64(k), f64(v), dense, f64(dout), bq, bkv)
    assert_close(f64(grads[0]), dQ, "dQ")
    assert_close(f64(grads[1]), dK, "dK")
    assert_close(f64(grads[2]), dV, "dV")


def test_block_size_64_rows_with_disjoint_halves():
    """b_q = 64 where the two query blocks sharing a 128-row tile keep disjoint
    kv-blocks (from a hand-made P-bar): every tile entry excludes one half, and
    the rows of each half must see only their own block's keys."""
    B, H, N, d = 1, 1, 512, 128
    q, k, v = synth.gaussian_with_sinks(B=B, H=H, N=N, d=d, seed=77, device="cuda")
    dout = synth.normal_like(q.shape, seed=78, device="cuda")
    Tm, Tn = oracle.block_counts(N, 64, 64)                      # 8 x 8
    pbar = np.full((B, H, Tm, Tn), 1e-4, dtype=np.float32)
    for i in range(Tm):                                          # even blocks keep kv 0..3, odd ones 4..7
        cols = range(0, 4) if i % 2 == 0 else range(4, 8)
        for j in cols:
            pbar[0, 0, i, j] = 0.2
    mask = b.select_blocks(torch.tensor(pbar, device="cuda"), 0.5, 0.0)
    s = b.Spa2(B, H, N, d, bq=64, bkv=64)
    o, lse = s.fwd(q, k, v, mask)
    grads = s.bwd(q, k, v, o, lse, dout, mask)
    s.check()
    dense = csr_to_dense(mask.row_cnt.cpu().numpy(), mask.row_idx.cpu().numpy(), Tn)
    assert dense[0, 0, 0, :4].all() and not dense[0, 0, 0, 4:].any() and dense[0, 0, 1, 4:].all()
    O, LSE = oracle.masked_attn_fwd(f64(q), f64(k), f64(v), dense, 64, 64)
    assert_close(_o32(s, o), O, "O (o + o_lo)")
    assert_close(lse.cpu().numpy(), LSE, "LSE")
    dQ, dK, dV = oracle.masked_attn_bwd(f64(q), f64(k), f64(v), dense, f64(dout), 64, 64)
    assert_close(f64(grads[0]), dQ, "dQ")
    assert_close(f64(grads[1]), dK, "dK")
    assert_close(f64(grads[2]), dV, "dV")
