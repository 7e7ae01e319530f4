"""`torch.autograd` front end of the sparse attention path.

sparse_attention(q, k, v, k_frac, p_frac) builds the hybrid Top-k + Top-p block
mask of (q, k) (paper.rainbus.top summary, 方法步骤详情 steps 1-3), runs the
block-sparse forward (step 4) and, when a gradient is requested, the backward
through the same mask, which the method holds constant (its trainable part is
the attention itself: chatpaper.ai abstract (ii)). Every step runs in the
libspa2 kernels; this module only marshals arguments through the C ABI
(`binding.Spa2`) and caches the per-shape workspaces.

A mask can also be built once with `block_mask(q, k, k_frac, p_frac)` and
passed as `sparse_attention(..., mask=m)` to later calls of the same shape
(other diffusion steps or layers), which then skip pooling and selection.

Device-side errors (a bounds check that failed on a bad mask, V outside the
fp16 range, a wait that timed out) are reported without synchronising the
stream: after every call the status words are copied, in stream order, into
pinned host memory; the next call on that shape and stream raises `Spa2Error`
once such a copy has landed with an error in it, and `check_errors()` waits for
every pending copy and raises.

Workspaces are cached per (shape, device, CUDA stream): calls on different
streams never share scratch memory.
"""

from __future__ import annotations

from collections import deque

import torch

from . import binding as b

_cache: dict = {}


class _StatusWatch:
    """Stream-ordered, non-blocking copies of one Spa2's status words."""

    SLOTS = 16

    def __init__(self, spa: b.Spa2):
        self.spa = spa
        self.host = torch.zeros(self.SLOTS, 3, dtype=torch.int32).pin_memory()
        self.pending: deque = deque()      # (slot, event, ops) in launch order
        self.next = 0

    def after(self, ops):
        """Queue a copy of the status words of `ops` behind the work just launched."""
        if len(self.pending) == self.SLOTS:
            self._finish(self.pending.popleft(), wait=True)
        slot = self.next
        self.next = (self.next + 1) % self.SLOTS
        for col, op in enumerate(ops):
            self.host[slot, col:col + 1].copy_(self.spa.ws[op][:4].view(torch.int32), non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self.pending.append((slot, ev, tuple(ops)))

    def poll(self):
        """Raise the first error among copies that have landed (never waits)."""
        while self.pending and self.pending[0][1].query():
            self._finish(self.pending.popleft(), wait=False)

    def drain(self):
        """Wait for every pending copy, then raise the first error among them."""
        while self.pending:
            self._finish(self.pending.popleft(), wait=True)

    def _finish(self, item, wait):
        slot, ev, ops = item
        if wait:
            ev.synchronize()
        for col, op in enumerate(ops):
            code = int(self.host[slot, col])
            if code != b.OK:
                self.pending.clear()
                raise b.Spa2Error(code, f"device status of sparse_attention (op {op})")


def _spa(B, H, N, d, device, bq=b.BQ, bkv=b.BKV) -> b.Spa2:
    stream = torch.cuda.current_stream(device).cuda_stream
    key = (B, H, N, d, bq, bkv, str(device), stream)
    s = _cache.get(key)
    if s is None:
        s = _cache[key] = b.Spa2(B, H, N, d, device=device, bq=bq, bkv=bkv)
        s.watch = _StatusWatch(s)
    s.watch.poll()
    return s


def check_errors():
    """Wait for every pending status copy of every cached workspace and raise
    `Spa2Error` if any call of sparse_attention / block_mask recorded a
    device-side error."""
    for s in list(_cache.values()):
        s.watch.drain()


class SparseAttentionFunction(torch.autograd.Function):
    """O = block-sparse attention of (q, k, v) under the hybrid mask of (q, k).

    q, k, v: [B, H, N, d] bf16 CUDA tensors (d in {64, 128}); gradients come back
    in bf16. The mask of the last call is kept on the function's context (and
    returned by `sparse_attention(..., return_mask=True)`).
    """

    @staticmethod
    def forward(ctx, q, k, v, k_frac: float, p_frac: float, scale: float = 0.0, mask: b.Mask | None = None,
                bq: int = b.BQ, bkv: int = b.BKV):
        if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
            raise TypeError("sparse_attention expects bf16 q, k, v")
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        B, H, N, d = q.shape
        s = _spa(B, H, N, d, q.device, bq, bkv)
        ops = [b.OP_FWD]
        if mask is None:
            mask = s.block_mask(q, k, k_frac, p_frac)
            ops.insert(0, b.OP_MASK)
        elif tuple(mask.row_cnt.shape) != (B, H, s.Tm) or tuple(mask.row_idx.shape) != (B, H, s.Tm, s.Tn) \
                or mask.col_cnt is None or mask.row_cnt.device != q.device:
            raise ValueError("mask does not belong to a problem of this shape and device")
        o, lse = s.fwd(q, k, v, mask, scale)
        s.watch.after(ops)
        ctx.save_for_backward(q, k, v, o, lse, s.o_lo)
        ctx.mask, ctx.scale, ctx.spa = mask, scale, s
        row_cnt = mask.row_cnt.clone()  # the kept-block counts (a copy: a reused mask serves many calls)
        ctx.mark_non_differentiable(row_cnt)
        return o, row_cnt

    @staticmethod
    def backward(ctx, do, _row_cnt_grad):
        q, k, v, o, lse, o_lo = ctx.saved_tensors
        ctx.spa.watch.poll()
        dq, dk, dv = ctx.spa.bwd(q, k, v, o, lse, do.contiguous(), ctx.mask, ctx.scale, o_lo=o_lo,
                                 grad_dtype=b.DTYPE_BF16)
        ctx.spa.watch.after([b.OP_BWD])
        return dq, dk, dv, None, None, None, None, None, None


def block_mask(q, k, k_frac: float, p_frac: float, bq: int = b.BQ, bkv: int = b.BKV) -> b.Mask:
    """The hybrid block mask of (q, k) alone (CSR and CSC on the device), for
    reuse through `sparse_attention(..., mask=...)`."""
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise TypeError("block_mask expects bf16 q, k")
    q, k = q.contiguous(), k.contiguous()
    B, H, N, d = q.shape
    s = _spa(B, H, N, d, q.device, bq, bkv)
    m = s.block_mask(q, k, k_frac, p_frac)
    s.watch.after([b.OP_MASK])
    return m


def sparse_attention(q, k, v, k_frac: float = 0.0, p_frac: float = 0.0, scale: float = 0.0,
                     return_mask: bool = False, mask: b.Mask | None = None, bq: int = b.BQ, bkv: int = b.BKV):
    """Differentiable hybrid block-sparse attention with query blocks of bq rows
    (64, 128 or 256) and key/value blocks of bkv rows (64 or 128).

    With `mask` (from `block_mask` on a problem of the same shape and block
    sizes) the given mask is used as is and k_frac, p_frac are ignored.
    """
    o, row_cnt = SparseAttentionFunction.apply(q, k, v, k_frac, p_frac, scale, mask, bq, bkv)
    return (o, row_cnt) if return_mask else o
