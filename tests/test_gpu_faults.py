"""Device-side failure detection, exercised without faulting the GPU: a bounded
wait that runs out, and masks whose counts or ids fail the kernels' own bounds
checks. Each case must end with a status code and leave the context usable."""

import pytest
import torch

from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import synth

pytestmark = pytest.mark.gpu


def _small_pass():
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=256, d=64, seed=0, device="cuda")
    s = b.Spa2(1, 1, 256, 64)
    m = s.block_mask(q, k, 0.3, 0.5)
    o, _ = s.fwd(q, k, v, m)
    s.check()
    assert torch.isfinite(o.float()).all()


def test_bounded_wait_times_out_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    try:
        assert b.spa2_debug_set_wait_limit_ns(1_000_000) == b.OK     # 1 ms
        assert b.spa2_debug_timeout_probe(ws.data_ptr(), 256, stream) == b.OK
        assert b.spa2_stream_status(ws.data_ptr(), stream) == b.ERR_DEVICE_TIMEOUT
        # the status word was cleared by the read
        assert b.spa2_stream_status(ws.data_ptr(), stream) == b.OK
    finally:
        b.spa2_debug_set_wait_limit_ns(0)
    _small_pass()


def test_bad_row_count_is_reported():
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=512, d=128, seed=1, device="cuda")
    s = b.Spa2(1, 2, 512, 128)
    m = s.block_mask(q, k, 0.3, 0.5)
    s.check()
    m.row_cnt[0, 1, 2] = 0            # a q-block with no kv-block is invalid
    s.fwd(q, k, v, m)
    with pytest.raises(b.Spa2Error) as e:
        s.check(b.OP_FWD)
    assert e.value.code == b.ERR_DEVICE_BOUNDS
    _small_pass()


def test_bad_kv_id_aborts_the_tile_cleanly():
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=512, d=128, seed=2, device="cuda")
    s = b.Spa2(1, 2, 512, 128)
    m = s.block_mask(q, k, 0.5, 0.5)
    s.check()
    n = int(m.row_cnt[0, 0, 1])
    m.row_idx[0, 0, 1, n - 1] = 10_000    # outside [0, T_n)
    s.fwd(q, k, v, m)
    with pytest.raises(b.Spa2Error) as e:
        s.check(b.OP_FWD)
    assert e.value.code == b.ERR_DEVICE_BOUNDS
    _small_pass()


def test_bad_column_count_is_reported_by_backward():
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=512, d=64, seed=3, device="cuda")
    dout = synth.normal_like(q.shape, seed=4, device="cuda")
    s = b.Spa2(1, 1, 512, 64)
    m = s.block_mask(q, k, 0.3, 0.5)
    o, lse = s.fwd(q, k, v, m)
    s.check()
    m.col_cnt[0, 0, 0] = 99           # more than T_m = 4
    s.bwd(q, k, v, o, lse, dout, m)
    with pytest.raises(b.Spa2Error) as e:
        s.check(b.OP_BWD)
    assert e.value.code == b.ERR_DEVICE_BOUNDS
    _small_pass()


def test_v_outside_fp16_range_is_reported():
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=256, d=128, seed=5, device="cuda")
    v = v.clone()
    v[0, 0, 17, 3] = 1e6
    s = b.Spa2(1, 1, 256, 128)
    m = s.block_mask(q, k, 0.5, 0.5)
    o, _ = s.fwd(q, k, v, m)
    with pytest.raises(b.Spa2Error) as e:
        s.check(b.OP_FWD)
    assert e.value.code == b.ERR_RANGE
    assert torch.isfinite(o.float()).all()      # clamped, never inf
    _small_pass()
