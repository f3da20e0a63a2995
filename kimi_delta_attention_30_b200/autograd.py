"""The chunkwise prefill as a differentiable PyTorch op.

``kda_chunk`` calls the library's prefill (``kda_chunk_fwd``) in the forward
direction and its backward (``kda_chunk_bwd``, which recomputes the forward's
intermediates from the saved inputs) in the reverse direction, so a training
step can use the prefill like any other op.  This module only marshals
arguments: both directions run in the library's kernels.

The recurrence it differentiates is the delta rule with one gate per key
channel, S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
o_t = S_t^T q_t ("From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, delta-rule
and Kimi Linear paragraphs; "我终于看懂了 KDA" explainer, pwwt.cn/news/3787313,
sections 6, 8 and 9).  The essay says training needs the chunkwise parallel
form but gives no backward pass; the library's is the chain rule applied to
that form.

``ops`` replaces the (forward, backward) pair with two callables of the same
signatures as :func:`chunk_fwd` and :func:`chunk_bwd`; that is how the routing
of gradients is tested without a GPU.
"""
from __future__ import annotations

import torch


class _ChunkKDA(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, log_alpha, beta, init_state, cu_seqlens, C, ops):
        fwd, bwd = ops
        o, final_state = fwd(q, k, v, log_alpha, beta, init_state=init_state, cu_seqlens=cu_seqlens, C=C)
        ctx.save_for_backward(q, k, v, log_alpha, beta, init_state)
        ctx.cu_seqlens, ctx.C, ctx.bwd = cu_seqlens, C, bwd
        return o, final_state

    @staticmethod
    def backward(ctx, d_o, d_final_state):
        q, k, v, log_alpha, beta, init_state = ctx.saved_tensors
        need_d_init = init_state is not None and ctx.needs_input_grad[5]
        if d_o is None:
            d_o = torch.zeros(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=q.device)
        dq, dk, dv, dla, dbeta, d_init = ctx.bwd(
            q, k, v, log_alpha, beta, d_o.contiguous(), init_state=init_state,
            d_final_state=None if d_final_state is None else d_final_state.contiguous(),
            cu_seqlens=ctx.cu_seqlens, C=ctx.C, need_d_init_state=need_d_init)
        return dq, dk, dv, dla, dbeta, (d_init if need_d_init else None), None, None, None


def kda_chunk(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, C: int = 64, ops=None):
    """Differentiable prefill: returns ``(o, final_state)`` as :func:`chunk_fwd`
    does (same shapes, dtypes and ``cu_seqlens`` convention).  Gradients reach
    q, k, v, log_alpha, beta and ``init_state`` (when given and requiring grad);
    the gradient of log_alpha is zero where the kernels' floor of -100 applied."""
    if ops is None:
        from . import chunk_bwd, chunk_fwd
        ops = (chunk_fwd, chunk_bwd)
    return _ChunkKDA.apply(q, k, v, log_alpha, beta, init_state, cu_seqlens, C, ops)
