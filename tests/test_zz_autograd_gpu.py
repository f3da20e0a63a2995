"""kda_chunk (the differentiable prefill) on the GPU: the gradients autograd
delivers equal those of a direct kda_chunk_bwd call with the same upstream
gradients."""
import pytest
import torch

from kimi_delta_attention_30_b200.autograd import kda_chunk


@pytest.mark.gpu
def test_autograd_matches_chunk_bwd(cuda_ok):
    import kimi_delta_attention_30_b200 as kda
    from kda_inputs import make_prefill, to_f64
    from kda_testlib import rel_err
    inp = make_prefill("prefill", device="cuda:0", B=2, T=200, H=4, seed=91)
    leaves = [t.detach().clone().requires_grad_() for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)]
    s0 = inp.init_state.detach().clone().requires_grad_()
    o, fs = kda_chunk(*leaves, init_state=s0, C=64)
    w = torch.randn(o.shape, device=o.device).to(o.dtype)
    wf = 0.1 * torch.randn(fs.shape, device=fs.device)
    ((o.float() * w.float()).sum() + (fs * wf).sum()).backward()
    ref = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, w, init_state=inp.init_state,
                        d_final_state=wf, C=64)
    torch.cuda.synchronize()
    for got, want in zip([x.grad for x in leaves] + [s0.grad], ref):
        assert got.dtype == want.dtype and got.shape == want.shape
        # dk and dlog_alpha add per-tile terms with atomics: equal up to summation
        # order, which may move a bf16 result by one unit in the last place
        stored = "bf16" if got.dtype == torch.bfloat16 else None
        assert rel_err(to_f64(got), to_f64(want), stored_as=stored, both_stored=True) <= 1e-3
