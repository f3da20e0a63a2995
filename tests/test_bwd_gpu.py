"""GPU parity of the backward pass (``kda_chunk_bwd``) against the fp64
oracle's reverse-mode gradient (O3), itself pinned to the forward oracle by
finite differences.  Bar: max |got - ref| / rms(ref) <= 2e-2 for bf16 inputs
(gradients stored in bf16, the storage half-ulp allowed) and <= 1e-4 for fp32,
for each of dq, dk, dv, dlog alpha, dbeta and the initial-state gradient.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import kimi_delta_attention_30_b200 as kda
from kda_inputs import WORKLOADS, make_grad_outputs, make_prefill
from kda_testlib import TOL, gpu_grad_slices, oracle_backward, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init_state")


def _to(inp, dev):
    for name in ("q", "k", "v", "log_alpha", "beta"):
        setattr(inp, name, getattr(inp, name).to(dev))
    if inp.init_state is not None:
        inp.init_state = inp.init_state.to(dev)
    return inp


def _bwd(inp, d_o, dfs, C=64):
    g = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, d_o, init_state=inp.init_state,
                      d_final_state=dfs, cu_seqlens=inp.cu_seqlens, C=C)
    torch.cuda.synchronize()
    return g


def _check(inp, grads, d_o, dfs, tol, **sel):
    ref, ti, seqs, heads = oracle_backward(inp, d_o, dfs, **sel)
    got = gpu_grad_slices(grads, ti, seqs, heads)
    stored = "bf16" if inp.dtype == "bf16" else None
    errs = {}
    for name in NAMES:
        if name not in got:
            continue
        assert np.isfinite(got[name]).all(), name
        errs[name] = rel_err(got[name], ref[name], stored_as=None if name == "d_init_state" else stored)
    bad = {n: e for n, e in errs.items() if e > tol}
    assert not bad, f"gradient rel err over {tol}: {bad} (all: {errs})"
    return errs




@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_bwd_f32_small(cuda_ok, dk, dv):
    """fp32 inputs, several chunks and a ragged tail, random initial state and
    final-state gradient, tol 1e-4."""
    wl = replace(WORKLOADS["tiny_f32"], dk=dk, dv=dv)
    inp = _to(make_prefill(wl, B=2, T=200, H=2, seed=5, init_zero=False), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=5)
    _check(inp, _bwd(inp, d_o, dfs), d_o, dfs, TOL["f32"])


@pytest.mark.parametrize("C", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 64, 200, 300])
def test_bwd_bf16_ragged(cuda_ok, C, T):
    """bf16, d=128, B=2, H=3: several chunks and a ragged tail (a request for
    128-token chunks is served with 64-token chunks)."""
    inp = _to(make_prefill("prefill", B=2, T=T, H=3, seed=T), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=T)
    _check(inp, _bwd(inp, d_o, dfs, C=C), d_o, dfs, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_bwd_bf16_small_heads(cuda_ok, dk, dv):
    """bf16 with d_k or d_v of 64 (CUDA-core recompute), ragged tail."""
    wl = replace(WORKLOADS["prefill"], dk=dk, dv=dv)
    inp = _to(make_prefill(wl, B=2, T=150, H=2, seed=13), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=13)
    _check(inp, _bwd(inp, d_o, dfs), d_o, dfs, TOL["bf16"])


def test_bwd_varlen_with_empty_and_tiny_sequences(cuda_ok):
    inp = _to(make_prefill("prefill", lengths=[0, 1, 70, 0, 129, 5], H=2, seed=4), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=4)
    errs = _check(inp, _bwd(inp, d_o, dfs), d_o, dfs, TOL["bf16"])
    assert "d_init_state" in errs


def test_bwd_without_state_gradients(cuda_ok):
    """init_state None (zero), d_final_state None, no d_init_state output."""
    inp = _to(make_prefill("prefill", B=1, T=130, H=2, seed=6, init_zero=True), DEV)
    d_o, _ = make_grad_outputs(inp, seed=6, final=False)
    g = kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, d_o, need_d_init_state=False)
    torch.cuda.synchronize()
    assert g[5] is None
    _check(inp, g, d_o, None, TOL["bf16"])


def test_bwd_gate_regimes_and_special_heads(cuda_ok):
    """Near-one, near-zero and mixed gates (the varlen workload's regimes), and
    the long workload's special heads (alpha = 1; one scalar alpha per token)."""
    wl = replace(WORKLOADS["varlen"], n_seqs=0)
    inp = _to(make_prefill(wl, B=1, T=300, H=3, seed=8), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=8)
    _check(inp, _bwd(inp, d_o, dfs), d_o, dfs, TOL["bf16"])
    inp = _to(make_prefill("long", B=1, T=300, H=3, seed=9), DEV)
    d_o, dfs = make_grad_outputs(inp, seed=9)
    _check(inp, _bwd(inp, d_o, dfs), d_o, dfs, TOL["bf16"])


def test_bwd_alpha_zero_and_beta_edges(cuda_ok):
    """log alpha = -inf on whole tokens (memory cleared), beta = 0 and 1."""
    inp = make_prefill("prefill", B=1, T=200, H=2, seed=10)
    inp.log_alpha[0, 70] = float("-inf")
    inp.log_alpha[0, 150, 1] = float("-inf")
    inp.beta[0, 10] = 0.0
    inp.beta[0, 11] = 1.0
    inp = _to(inp, DEV)
    d_o, dfs = make_grad_outputs(inp, seed=10)
    g = _bwd(inp, d_o, dfs)
    _check(inp, g, d_o, dfs, TOL["bf16"])
    assert torch.all(g[3][0, 70] == 0) and torch.all(g[3][0, 150, 1] == 0)


def test_bwd_full_size_sampled(cuda_ok):
    """B=4, H=16, T=4096, d=128, bf16 (the backward benchmark's launch);
    sampled (sequence, head) pairs over all 4096 tokens."""
    inp = make_prefill("prefill", device=DEV)
    d_o, dfs = make_grad_outputs(inp, seed=1)
    g = _bwd(inp, d_o, dfs)
    for t in g:
        assert torch.isfinite(t.float()).all()
    for seqs, heads in (([0], [0, 9]), ([3], [15])):
        _check(inp, g, d_o, dfs, TOL["bf16"], seqs=seqs, heads=heads)
