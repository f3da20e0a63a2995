"""kda_chunk (the differentiable prefill): gradient routing on the CPU with
stand-in forward/backward callables (the GPU comparison with kda_chunk_bwd is in
test_zz_autograd_gpu.py)."""
import torch

from kimi_delta_attention_30_b200.autograd import kda_chunk

B, T, H, DK, DV = 1, 10, 2, 4, 3


class Fakes:
    """Stand-ins with chunk_fwd / chunk_bwd's signatures that record their
    arguments and return recognisable values."""

    def __init__(self):
        self.fwd_kw = self.bwd_args = self.bwd_kw = None

    def fwd(self, q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, C=64):
        self.fwd_kw = dict(init_state=init_state, cu_seqlens=cu_seqlens, C=C)
        o = torch.full(q.shape[:-1] + (v.shape[-1],), 1.5, dtype=q.dtype)
        fs = torch.full((B, H, DK, DV), 2.5)
        return o, fs

    def bwd(self, q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None, cu_seqlens=None, C=64,
            need_d_init_state=True):
        self.bwd_args = (q, k, v, log_alpha, beta, d_o)
        self.bwd_kw = dict(init_state=init_state, d_final_state=d_final_state, cu_seqlens=cu_seqlens, C=C,
                           need_d_init_state=need_d_init_state)
        grads = tuple(torch.full_like(t, float(i + 1)) for i, t in enumerate((q, k, v, log_alpha, beta)))
        d_init = torch.full((B, H, DK, DV), 7.0) if need_d_init_state else None
        return grads + (d_init,)


def _inputs(with_state=True):
    g = torch.Generator().manual_seed(0)
    mk = lambda *s: torch.randn(*s, generator=g).requires_grad_()
    q, k, la = mk(B, T, H, DK), mk(B, T, H, DK), mk(B, T, H, DK)
    v, beta = mk(B, T, H, DV), mk(B, T, H)
    s0 = mk(B, H, DK, DV) if with_state else None
    return q, k, v, la, beta, s0


def test_gradients_reach_every_input():
    f = Fakes()
    q, k, v, la, beta, s0 = _inputs()
    o, fs = kda_chunk(q, k, v, la, beta, init_state=s0, cu_seqlens=[0, 4, 10], C=128, ops=(f.fwd, f.bwd))
    assert f.fwd_kw["cu_seqlens"] == [0, 4, 10] and f.fwd_kw["C"] == 128 and f.fwd_kw["init_state"] is s0
    w = torch.randn(o.shape)
    (o * w).sum().backward()
    # the upstream gradients are what the backward receives
    assert torch.equal(f.bwd_args[5], w)
    assert torch.equal(f.bwd_kw["d_final_state"], torch.zeros_like(fs))
    assert f.bwd_kw["cu_seqlens"] == [0, 4, 10] and f.bwd_kw["C"] == 128 and f.bwd_kw["need_d_init_state"]
    for saved, x in zip(f.bwd_args[:5], (q, k, v, la, beta)):
        assert torch.equal(saved, x.detach())
    # and each gradient lands on its own input
    for i, x in enumerate((q, k, v, la, beta)):
        assert torch.equal(x.grad, torch.full_like(x, float(i + 1)))
    assert torch.equal(s0.grad, torch.full_like(s0, 7.0))


def test_final_state_gradient_and_no_initial_state():
    f = Fakes()
    q, k, v, la, beta, _ = _inputs(with_state=False)
    o, fs = kda_chunk(q, k, v, la, beta, ops=(f.fwd, f.bwd))
    wf = torch.randn(fs.shape)
    (fs * wf).sum().backward()
    assert torch.equal(f.bwd_kw["d_final_state"], wf)
    assert torch.equal(f.bwd_args[5], torch.zeros_like(o))
    assert f.bwd_kw["init_state"] is None and not f.bwd_kw["need_d_init_state"]
    assert torch.equal(q.grad, torch.full_like(q, 1.0))


def test_initial_state_without_grad_is_not_differentiated():
    f = Fakes()
    q, k, v, la, beta, s0 = _inputs()
    s0 = s0.detach()
    o, _ = kda_chunk(q, k, v, la, beta, init_state=s0, ops=(f.fwd, f.bwd))
    o.sum().backward()
    assert not f.bwd_kw["need_d_init_state"] and f.bwd_kw["init_state"] is s0
