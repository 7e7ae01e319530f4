"""spa2_block_mask_noalloc (the block mask with its scratch in a fixed device
array instead of a caller workspace) against spa2_block_mask, through the C ABI.

The two entry points run the same kernels, so every output must match exactly.
Two calls in a row, with different inputs and then a different shape, check
that nothing left in the shared scratch leaks into the next result.
"""

import ctypes

import pytest
import torch

from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import synth

SCRATCH_BYTES = 64 << 20  # SPA2_NOALLOC_MASK_SCRATCH_BYTES


def _filled_mask(s: b.Spa2) -> b.Mask:
    m = s.new_mask()
    for t in (m.row_cnt, m.row_idx, m.col_cnt, m.col_idx):
        t.fill_(-1)
    m.pbar.fill_(-1.0)
    m.bitmap.fill_(7)
    return m


def _noalloc(s: b.Spa2, q, k, kf, pf, m: b.Mask, status: torch.Tensor) -> None:
    cm = m.c()
    rc = b.spa2_block_mask_noalloc(q.data_ptr(), k.data_ptr(), s.B, s.H, s.N, s.d, b.BQ, b.BKV, float(kf),
                                   float(pf), cm, status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == b.OK, b.status_string(rc)


def _assert_same(got: b.Mask, want: b.Mask) -> None:
    for name in ("row_cnt", "row_idx", "col_cnt", "col_idx", "pbar", "bitmap"):
        g, w = getattr(got, name), getattr(want, name)
        assert torch.equal(g, w), name


def _one_shape(B, H, N, d, kf, pf, seeds, gen=synth.gaussian_with_sinks):
    s = b.Spa2(B, H, N, d, with_pbar=True, with_bitmap=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for seed in seeds:                       # two calls in a row on one stream
        q, k, _ = gen(B=B, H=H, N=N, d=d, seed=seed, device="cuda")
        want = s.block_mask(q, k, kf, pf, _filled_mask(s))
        s.check(b.OP_MASK)
        got = _filled_mask(s)
        _noalloc(s, q, k, kf, pf, got, status)
        rc = b.spa2_stream_status(status.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == b.OK, b.status_string(rc)
        _assert_same(got, want)


@pytest.mark.gpu
def test_noalloc_matches_block_mask_wan_layer():
    # one attention layer of the 1.3B video model: 12 heads, 32760 tokens, d=128
    assert b.spa2_workspace_bytes(b.OP_MASK, 1, 12, 32760, 128) <= SCRATCH_BYTES
    _one_shape(1, 12, 32760, 128, 0.025, 0.7, seeds=(11, 12), gen=synth.smoothed_field)


@pytest.mark.gpu
def test_noalloc_ragged_shapes_in_a_row():
    _one_shape(2, 3, 1000, 64, 0.1, 0.5, seeds=(1, 2))
    _one_shape(1, 2, 77, 128, 0.0, 0.9, seeds=(3, 4))   # a smaller shape after a larger one


def test_noalloc_refuses_oversize_shapes():
    """Scratch beyond the fixed size is refused before anything is launched."""
    B, H, N, d = 4, 40, 131072, 128
    need = b.spa2_workspace_bytes(b.OP_MASK, B, H, N, d)
    assert need > SCRATCH_BYTES
    dummy = ctypes.c_void_p(16)              # never dereferenced: the size check comes first
    m = b.spa2_mask(16, 16, 16, 16, None, None)
    rc = b.spa2_block_mask_noalloc(dummy, dummy, B, H, N, d, b.BQ, b.BKV, 0.1, 0.5, m, None, None)
    assert rc == b.ERR_WORKSPACE
