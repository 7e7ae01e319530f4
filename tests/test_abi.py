"""Host-side checks of the C ABI: the library loads without a GPU, exports
every symbol include/spa2.h declares, and rejects bad arguments before it
launches anything (no compute calls are made here)."""

import ctypes

import pytest

from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import build


@pytest.fixture(scope="module")
def L():
    build.build()
    return b.lib()


def test_exports_every_header_symbol(L):
    names = b.header_symbols()
    assert {"spa2_block_mask", "spa2_select_blocks", "spa2_sparse_attn_fwd", "spa2_sparse_attn_bwd"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    # and the binding wraps each of them under the same name
    for n in names:
        assert n in b._SIGS, n


def test_version_and_status_strings(L):
    assert b.spa2_abi_version() == 1
    for code in range(8):
        assert b.status_string(code)
    assert b.status_string(99) == "unknown status"


def test_workspace_sizes(L):
    B, H, N, d = 1, 12, 32760, 128
    Tm, Tn = 256, 512
    m = b.spa2_workspace_bytes(b.OP_MASK, B, H, N, d)
    assert m >= 256 + B * H * (Tm + Tn) * d * 4 + B * H * Tm * 16 * 4   # Qbar, Kbar^T, kept-bit words
    assert b.spa2_workspace_bytes(b.OP_FWD, B, H, N, d) == 256 + B * H * N * d * 2   # status + fp16 V
    al = lambda n: -(-n // 256) * 256  # noqa: E731
    # status word, D (fp32 per row), fp16 copies of dO and Q, the order of the dK/dV
    # pass's columns (one int per kv column), each 256-byte aligned
    assert b.spa2_workspace_bytes(b.OP_BWD, B, H, N, d) == (256 + al(B * H * N * 4) + 2 * al(B * H * N * d * 2)
                                                          + al(B * H * Tn * 4))
    assert b.spa2_workspace_bytes(b.OP_BWD, 1, 2, 1000, 64) == (256 + al(2 * 1000 * 4) + 2 * al(2 * 1000 * 64 * 2)
                                                              + al(2 * 16 * 4))
    assert b.spa2_workspace_bytes(b.OP_SELECT, 2, 3, 5, 40, 0, 0) == 256 + 256   # 2*3*5*2 words = 240 B
    # unsupported shapes report 0
    assert b.spa2_workspace_bytes(b.OP_MASK, 1, 1, 100, 96) == 0
    assert b.spa2_workspace_bytes(b.OP_MASK, 1, 1, 100, 128, 32, 64) == 0
    assert b.spa2_workspace_bytes(b.OP_MASK, 1, 1, 100, 128, 128, 256) == 0
    for bq in (64, 128, 256):
        for bkv in (64, 128):
            assert b.spa2_workspace_bytes(b.OP_FWD, 1, 2, 1000, 128, bq, bkv) > 0
    # tile lists are extra workspace only for sizes other than (128, 64)
    assert b.spa2_workspace_bytes(b.OP_FWD, 1, 2, 1000, 128, 64, 128) > b.spa2_workspace_bytes(b.OP_FWD, 1, 2, 1000, 128)
    assert b.spa2_workspace_bytes(b.OP_MASK, 1, 1, 0, 128) == 0


def test_argument_errors_are_synchronous(L):
    m = b.spa2_mask()
    # null tensors
    assert b.spa2_block_mask(None, None, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m, None, 0, None) == b.ERR_INVALID_ARG
    fake = 1 << 20            # never dereferenced: validation fails first
    m = b.spa2_mask(fake, fake, None, None, None, None)
    # unsupported head dim / block sizes / fractions
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 96, 128, 64, 0.1, 0.5, m, fake, 1 << 30, None) == b.ERR_UNSUPPORTED
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 96, 64, 0.1, 0.5, m, fake, 1 << 30, None) == b.ERR_UNSUPPORTED
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, 1.5, 0.5, m, fake, 1 << 30, None) == b.ERR_UNSUPPORTED
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, float("nan"), 0.5, m, fake, 1 << 30,
                             None) == b.ERR_UNSUPPORTED
    # misaligned tensor
    assert b.spa2_block_mask(fake + 2, fake, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m, fake, 1 << 30,
                             None) == b.ERR_INVALID_ARG
    # workspace missing / too small / misaligned
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m, None, 0, None) == b.ERR_WORKSPACE
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m, fake, 300, None) == b.ERR_WORKSPACE
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m, fake + 16, 1 << 30,
                             None) == b.ERR_WORKSPACE
    # half a CSC
    m2 = b.spa2_mask(fake, fake, fake, None, None, None)
    assert b.spa2_block_mask(fake, fake, 1, 1, 128, 128, 128, 64, 0.1, 0.5, m2, fake, 1 << 30,
                             None) == b.ERR_INVALID_ARG
    # forward / backward
    assert b.spa2_sparse_attn_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 64, m, 0.0, fake, None, None, fake, 256,
                                  None) == b.ERR_INVALID_ARG                        # no lse
    assert b.spa2_sparse_attn_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 64, m, 0.0, fake, fake + 8, fake, fake,
                                  256, None) == b.ERR_INVALID_ARG                   # misaligned o_lo
    assert b.spa2_sparse_attn_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 64, m, -1.0, fake, None, fake, fake, 256,
                                  None) == b.ERR_UNSUPPORTED
    assert b.spa2_sparse_attn_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 64, m, 0.0, fake, None, fake, fake, 255,
                                  None) == b.ERR_WORKSPACE
    assert b.spa2_sparse_attn_bwd(fake, fake, fake, fake, None, fake, fake, 1, 1, 128, 128, 128, 64, m, 0.0, fake,
                                  fake, fake, b.DTYPE_F32, fake, 1 << 30, None) == b.ERR_INVALID_ARG  # no CSC
    mc = b.spa2_mask(fake, fake, fake, fake, None, None)
    assert b.spa2_sparse_attn_bwd(fake, fake, fake, fake, None, fake, fake, 1, 1, 128, 128, 128, 64, mc, 0.0, fake,
                                  fake, fake, b.DTYPE_F32, fake, 1000, None) == b.ERR_WORKSPACE
    assert b.spa2_sparse_attn_bwd(fake, fake, fake, fake, None, fake, fake, 1, 1, 128, 128, 128, 64, mc, 0.0, fake,
                                  fake, fake, 7, fake, 1 << 30, None) == b.ERR_UNSUPPORTED      # bad grad dtype
    assert b.spa2_select_blocks(fake, 1, 1, 4, 5000, 0.1, 0.5, m, fake, 1 << 30, None) == b.ERR_UNSUPPORTED
    assert b.spa2_debug_timeout_probe(None, 0, None) == b.ERR_WORKSPACE
    assert b.spa2_debug_set_wait_limit_ns(0) == b.OK


def test_stream_status_without_ws(L):
    assert b.spa2_stream_status(None, None) == b.ERR_WORKSPACE


def test_timing_symbols_without_a_gpu(L):
    """The per-kernel timing aid: names for every kernel kind, and a read with
    nothing recorded returns zero launches without touching a device."""
    n = b.spa2_kernel_count()
    names = [b.spa2_kernel_name(i) for i in range(n)]
    assert len(set(names)) == n and "fwd_kernel" in names and "bwd_dkdv_kernel" in names
    assert b.spa2_kernel_name(n) == "unknown"
    assert b.spa2_timing_read() == {}
    assert b.spa2_timing_enable(False) == b.OK
