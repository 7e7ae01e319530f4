"""Shared comparison helpers for the GPU parity tests."""

import numpy as np

# BASELINE tolerance for attention outputs and gradients (bf16 inputs, fp32
# accumulation): max-abs 2e-2 and relative L1 1e-2, element by element.
MAX_ABS = 2e-2
REL_L1 = 1e-2


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(actual, expected, what, max_abs=MAX_ABS, rel_l1=REL_L1):
    a = np.asarray(actual, dtype=np.float64)
    e = np.asarray(expected, dtype=np.float64)
    assert a.shape == e.shape, (what, a.shape, e.shape)
    assert np.isfinite(a).all(), f"{what}: non-finite values"
    err = np.abs(a - e)
    ma = float(err.max()) if err.size else 0.0
    rl1 = float(err.sum() / max(np.abs(e).sum(), 1e-300))
    assert ma <= max_abs and rl1 <= rel_l1, f"{what}: max_abs={ma:.3e} (<= {max_abs}) rel_l1={rl1:.3e} (<= {rel_l1})"
    return ma, rl1


def bf16_half_ulp(x):
    """Half a bf16 ulp of |x| (the rounding error of storing x as bf16)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 8)


def assert_close_bf16_out(actual, expected, what, max_abs=MAX_ABS, rel_l1=REL_L1):
    """bf16 outputs: the stated tolerance plus half a bf16 ulp of each expected value."""
    a = np.asarray(actual, dtype=np.float64)
    e = np.asarray(expected, dtype=np.float64)
    assert a.shape == e.shape, (what, a.shape, e.shape)
    err = np.abs(a - e)
    excess = err - (max_abs + bf16_half_ulp(e))
    rl1 = float(err.sum() / max(np.abs(e).sum(), 1e-300))
    assert excess.max() <= 0 and rl1 <= rel_l1, f"{what}: worst excess {excess.max():.3e} rel_l1={rl1:.3e}"


class Accum:
    """Max-abs per element and relative L1 over several sampled blocks of one tensor."""

    def __init__(self, what):
        self.what, self.err, self.ref, self.ma = what, 0.0, 0.0, 0.0

    def add(self, actual, expected):
        a = np.asarray(actual, dtype=np.float64)
        e = np.asarray(expected, dtype=np.float64)
        assert a.shape == e.shape and np.isfinite(a).all()
        d = np.abs(a - e)
        self.ma = max(self.ma, float(d.max()))
        self.err += float(d.sum())
        self.ref += float(np.abs(e).sum())

    def check(self, max_abs=MAX_ABS, rel_l1=REL_L1):
        rl1 = self.err / max(self.ref, 1e-300)
        assert self.ma <= max_abs and rl1 <= rel_l1, f"{self.what}: max_abs={self.ma:.3e} rel_l1={rl1:.3e}"
        return self.ma, rl1


class AccumBf16(Accum):
    """Accum for a bf16 output: per element |err| <= max_abs + half a bf16 ulp of
    the expected value (the output format's own rounding), and the same
    relative-L1 bound as every other output, summed over all sampled blocks."""

    def __init__(self, what):
        super().__init__(what)
        self.excess = -np.inf

    def add(self, actual, expected):
        super().add(actual, expected)
        e = np.asarray(expected, dtype=np.float64)
        d = np.abs(np.asarray(actual, dtype=np.float64) - e)
        self.excess = max(self.excess, float((d - bf16_half_ulp(e)).max()))

    def check(self, max_abs=MAX_ABS, rel_l1=REL_L1):
        rl1 = self.err / max(self.ref, 1e-300)
        assert self.excess <= max_abs and rl1 <= rel_l1, \
            f"{self.what}: max excess over half an ulp={self.excess:.3e} rel_l1={rl1:.3e}"
        return self.excess, rl1


def csr_to_dense(row_cnt, row_idx, Tn):
    """bool [.., Tm, Tn] from CSR numpy arrays; checks ids ascending and in range."""
    cnt = np.asarray(row_cnt)
    idx = np.asarray(row_idx)
    out = np.zeros(cnt.shape + (Tn,), dtype=bool)
    for pos in np.ndindex(cnt.shape):
        n = int(cnt[pos])
        ids = idx[pos][:n]
        assert 1 <= n <= Tn
        assert (np.diff(ids) > 0).all() and ids.min() >= 0 and ids.max() < Tn
        out[pos][ids] = True
    return out


def csc_to_dense(col_cnt, col_idx, Tm):
    cnt = np.asarray(col_cnt)
    idx = np.asarray(col_idx)
    out = np.zeros(cnt.shape + (Tm,), dtype=bool)
    for pos in np.ndindex(cnt.shape):
        n = int(cnt[pos])
        ids = idx[pos][:n]
        assert 0 <= n <= Tm
        if n:
            assert (np.diff(ids) > 0).all() and ids.min() >= 0 and ids.max() < Tm
        out[pos][ids] = True
    return np.swapaxes(out, -1, -2)
