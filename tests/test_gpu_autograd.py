"""The torch.autograd front end (sparse_attention) on the GPU: gradients of a
loss through the block-sparse forward and backward kernels against the float64
oracle, and a few steps of velocity-distillation training of a small synthetic
DiT attention block (sparse student, dense teacher) that must lower the loss."""

import numpy as np
import pytest
import torch

import oracle
from tests._parity import assert_close, assert_close_bf16_out, csr_to_dense, f64
from trainable_block_sparse_pooled_b200 import binding as b
from trainable_block_sparse_pooled_b200 import synth
from trainable_block_sparse_pooled_b200.autograd import block_mask, sparse_attention

pytestmark = pytest.mark.gpu


def test_autograd_gradients_match_oracle():
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=1000, d=64, seed=21, device="cuda")
    dout = synth.normal_like(q.shape, seed=22, device="cuda")
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    o, row_cnt = sparse_attention(qg, kg, vg, 0.2, 0.6, return_mask=True)
    (o.float() * dout.float()).sum().backward()
    # the same mask, rebuilt through the C ABI (the selection is deterministic)
    s = b.Spa2(1, 2, 1000, 64)
    m = s.block_mask(q, k, 0.2, 0.6)
    s.check()
    assert torch.equal(m.row_cnt, row_cnt)
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), s.Tn)
    O, _ = oracle.masked_attn_fwd(f64(q), f64(k), f64(v), dense, 128, 64)
    dQ, dK, dV = oracle.masked_attn_bwd(f64(q), f64(k), f64(v), dense, f64(dout), 128, 64)
    assert_close_bf16_out(f64(o.detach()), O, "O (bf16)")
    for name, g, e in (("dQ", qg.grad, dQ), ("dK", kg.grad, dK), ("dV", vg.grad, dV)):
        assert g.dtype == torch.bfloat16
        assert_close_bf16_out(f64(g), e, name)


def test_reused_mask():
    """A mask built once with block_mask and passed to later calls: on the same
    inputs it reproduces the call that builds its own mask bit for bit (both
    passes are deterministic); on another step's inputs it matches the oracle
    under that same mask."""
    q, k, v = synth.gaussian_with_sinks(B=1, H=2, N=1000, d=128, seed=31, device="cuda")
    dout = synth.normal_like(q.shape, seed=32, device="cuda")
    m = block_mask(q, k, 0.2, 0.6)
    runs = []
    for kw in (dict(k_frac=0.2, p_frac=0.6), dict(mask=m)):
        qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
        o = sparse_attention(qg, kg, vg, **kw)
        (o.float() * dout.float()).sum().backward()
        runs.append((o.detach(), qg.grad, kg.grad, vg.grad))
    for a, c in zip(*runs):
        assert torch.equal(a, c)
    # another diffusion step: new q, k, v of the same shape, the mask of the first
    q2, k2, v2 = synth.gaussian_with_sinks(B=1, H=2, N=1000, d=128, seed=33, device="cuda")
    o2 = sparse_attention(q2, k2, v2, mask=m)
    dense = csr_to_dense(m.row_cnt.cpu().numpy(), m.row_idx.cpu().numpy(), m.row_idx.shape[-1])
    O2, _ = oracle.masked_attn_fwd(f64(q2), f64(k2), f64(v2), dense, 128, 64)
    assert_close_bf16_out(f64(o2), O2, "O (bf16), reused mask")
    with pytest.raises(ValueError):
        sparse_attention(q2[:, :1].contiguous(), k2[:, :1].contiguous(), v2[:, :1].contiguous(), mask=m)


class _AttnBlock(torch.nn.Module):
    """x -> softmax attention over H heads of width d -> x (random init)."""

    def __init__(self, C, H, seed):
        super().__init__()
        g = torch.Generator().manual_seed(seed)
        self.H, self.d = H, C // H
        self.qkv = torch.nn.Parameter((torch.randn(C, 3 * C, generator=g) / C ** 0.5).cuda())
        self.out = torch.nn.Parameter((torch.randn(C, C, generator=g) / C ** 0.5).cuda())

    def heads(self, x):
        B, N, C = x.shape
        q, k, v = (x @ self.qkv).split(C, dim=-1)
        f = lambda t: t.view(B, N, self.H, self.d).transpose(1, 2).contiguous().bfloat16()  # noqa: E731
        return f(q), f(k), f(v)

    def merge(self, o):
        B, H, N, d = o.shape
        return o.float().transpose(1, 2).reshape(B, N, H * d) @ self.out


def test_velocity_distillation_steps_lower_the_loss():
    """Sparse student (k = 10%, p = 50%, its own random init) distilled towards a
    frozen dense teacher of the same architecture (torch SDPA, float32) on seeded
    tokens: the loss
    || student(x) - teacher(x) ||^2 falls over a few Adam steps, and every gradient
    of the student passes through the sparse backward kernels."""
    torch.manual_seed(0)
    B, N, C, H = 1, 2048, 256, 2
    x = torch.randn(B, N, C, device="cuda")
    teacher = _AttnBlock(C, H, seed=1)
    student = _AttnBlock(C, H, seed=2)
    with torch.no_grad():
        tq, tk, tv = (t.float() for t in teacher.heads(x))
        target = teacher.merge(torch.nn.functional.scaled_dot_product_attention(tq, tk, tv))
    opt = torch.optim.Adam(student.parameters(), lr=2e-3)
    losses = []
    for _ in range(8):
        q, k, v = student.heads(x)
        y = student.merge(sparse_attention(q, k, v, 0.10, 0.50))
        loss = ((y - target) ** 2).mean()
        opt.zero_grad()
        loss.backward()
        assert all(torch.isfinite(p.grad).all() for p in student.parameters())
        opt.step()
        losses.append(loss.item())
    assert np.isfinite(losses).all()
    assert losses[-1] < 0.8 * losses[0], losses


def test_forward_only_errors_are_raised():
    """Inference without a backward: a V value outside the fp16 range is clamped
    and recorded on the device; check_errors() raises it (no backward needed),
    and later calls run clean."""
    from trainable_block_sparse_pooled_b200.autograd import check_errors
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=384, d=64, seed=41, device="cuda")
    check_errors()
    bad = v.clone()
    bad[0, 0, 5, 7] = 1e6
    with torch.no_grad():
        sparse_attention(q, k, bad, 0.3, 0.5)
    with pytest.raises(b.Spa2Error) as e:
        check_errors()
    assert e.value.code == b.ERR_RANGE
    with torch.no_grad():
        o = sparse_attention(q, k, v, 0.3, 0.5)
    check_errors()
    assert torch.isfinite(o.float()).all()


def test_workspaces_are_per_stream():
    """The same shape on two streams gets two workspace sets."""
    from trainable_block_sparse_pooled_b200 import autograd
    q, k, v = synth.gaussian_with_sinks(B=1, H=1, N=256, d=64, seed=42, device="cuda")
    side = torch.cuda.Stream()
    o1 = sparse_attention(q, k, v, 0.3, 0.5)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o2 = sparse_attention(q, k, v, 0.3, 0.5)
    torch.cuda.current_stream().wait_stream(side)
    autograd.check_errors()
    keys = [key for key in autograd._cache if key[:4] == (1, 1, 256, 64)]
    assert len({key[-1] for key in keys}) == 2
    assert torch.equal(o1, o2)
