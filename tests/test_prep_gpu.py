"""GPU parity of the fused input preprocessing: ``kda_chunk_fwd_prep`` and
``kda_decode_step_prep`` on raw q / k, gate logits and beta logits against
``oracle.prep`` followed by the fp64 oracle (same tolerance as the plain path:
max |got - ref| / rms(ref) <= 2e-2 for bf16 inputs, 1e-4 for fp32).

Flags that are not set leave their argument as the plain operator's input, so
those arguments come from the matching ready-made workload.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import kimi_delta_attention_30_b200 as kda
import oracle
from kda_inputs import RAW_PREP, WORKLOADS, make_decode_state, make_decode_token, make_prefill, to_f64
from kda_testlib import TOL, gpu_slices, oracle_prefill, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
L2, SP, SG = kda.PREP_QK_L2NORM, kda.PREP_GATE_SOFTPLUS, kda.PREP_BETA_SIGMOID


def _mixed_prefill(prep, **kw):
    """Raw arguments for the set flags, ready ones for the others."""
    raw = make_prefill("prefill_raw", **kw)
    ready = make_prefill("prefill", **kw)
    if not prep & L2:
        raw.q, raw.k = ready.q, ready.k
    if not prep & SP:
        raw.log_alpha = ready.log_alpha
    if not prep & SG:
        raw.beta = ready.beta
    return raw


def _to(inp, dev):
    for name in ("q", "k", "v", "log_alpha", "beta"):
        setattr(inp, name, getattr(inp, name).to(dev))
    if inp.init_state is not None:
        inp.init_state = inp.init_state.to(dev)
    return inp


def _run(inp, prep, C=64):
    o, fs = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state,
                          cu_seqlens=inp.cu_seqlens, C=C, prep=prep)
    torch.cuda.synchronize()
    return o, fs


def _check(inp, o, fs, prep, tol=TOL["bf16"], **sel):
    o_ref, fs_ref, ti, seqs, heads = oracle_prefill(inp, prep=prep, **sel)
    og, fg = gpu_slices(o, fs, ti, seqs, heads)
    assert np.isfinite(og).all() and np.isfinite(fg).all()
    eo, es = rel_err(og, o_ref, stored_as="bf16"), rel_err(fg, fs_ref)
    assert eo <= tol, f"o rel err {eo:.3e}"
    assert es <= tol, f"state rel err {es:.3e}"


# ----------------------------------------------------------------------- prefill

@pytest.mark.parametrize("prep", [L2, SP, SG, L2 | SP | SG])
@pytest.mark.parametrize("C", [64, 128])
@pytest.mark.parametrize("T", [1, 63, 200, 300])
def test_prep_prefill_ragged(cuda_ok, prep, C, T):
    """B=2, H=3, d=128 bf16, several chunks and a ragged tail, random initial state."""
    inp = _to(_mixed_prefill(prep, B=2, T=T, H=3, seed=T + 11 * prep), DEV)
    o, fs = _run(inp, prep, C=C)
    _check(inp, o, fs, prep)


def test_prep_prefill_varlen_with_empty_and_tiny_sequences(cuda_ok):
    inp = _to(make_prefill("prefill_raw", lengths=[0, 1, 70, 0, 129, 5], H=2, seed=4), DEV)
    o, fs = _run(inp, RAW_PREP)
    _check(inp, o, fs, RAW_PREP)


def test_prep_prefill_edges(cuda_ok):
    """All-zero q and k rows (normalised to zero), gate logits at +-80 and +120
    (alpha ~ 0, alpha ~ 1, and a decay past the kernels' log-alpha floor of
    -100), beta logits at +-30, and a raw k scaled by 1e3 (the norm removes it)."""
    inp = make_prefill("prefill_raw", B=1, T=200, H=2, seed=9)
    inp.q[0, 5, 0] = 0.0
    inp.k[0, 5, 0] = 0.0
    inp.k[0, 70, 1] = 0.0
    inp.k[0, 90:95] *= 1000.0
    inp.log_alpha[0, 40, 0] = 80.0
    inp.log_alpha[0, 41:60, 1] = -80.0
    inp.log_alpha[0, 130, :, :7] = 120.0
    inp.beta[0, 10] = 30.0
    inp.beta[0, 11] = -30.0
    inp = _to(inp, DEV)
    o, fs = _run(inp, RAW_PREP)
    _check(inp, o, fs, RAW_PREP)


def test_prep_scale_invariance_on_the_gpu(cuda_ok):
    """With the L2 norm fused in, raw q and k rescaled by powers of two (exact in
    bf16) give the same result: the kernels normalise, they do not take the
    inputs as given.  Bound: 1e-5 of rms plus the bf16 storage half-ulps."""
    inp = _to(make_prefill("prefill_raw", B=2, T=300, H=3, seed=21), DEV)
    o1, f1 = _run(inp, RAW_PREP)
    o1, f1 = o1.clone(), f1.clone()
    inp.q = inp.q * 0.25
    inp.k = inp.k * 8.0
    o2, f2 = _run(inp, RAW_PREP)
    assert rel_err(to_f64(o2), to_f64(o1), stored_as="bf16", both_stored=True) <= 1e-5
    assert rel_err(to_f64(f2), to_f64(f1)) <= 1e-5


def test_prep_full_prefill_b4_h16_t4096(cuda_ok):
    """B=4, H=16, T=4096, d=128, bf16 raw inputs with every flag (the fused
    prefill benchmark's launch); sampled (sequence, head) pairs, all tokens."""
    inp = make_prefill("prefill_raw", device=DEV)
    o, fs = _run(inp, RAW_PREP)
    assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    for seqs, heads in (([0], [0, 7]), ([2], [15])):
        _check(inp, o, fs, RAW_PREP, seqs=seqs, heads=heads)


def test_prep_prefill_rejected_off_the_tensor_core_path(cuda_ok):
    inp = _to(make_prefill("prefill_raw", B=1, T=64, H=1, seed=1), DEV)
    with pytest.raises(kda.KdaError):
        kda.chunk_fwd(inp.q.float(), inp.k.float(), inp.v.float(), inp.log_alpha.float(), inp.beta.float(),
                      prep=RAW_PREP)
    with pytest.raises(ValueError):
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, algo="simt", prep=RAW_PREP)


# ------------------------------------------------------------------------ decode

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("prep", [L2, SP | SG, L2 | SP | SG])
def test_prep_decode_steps_small(cuda_ok, dtype, dk, dv, prep):
    raw_wl = replace(WORKLOADS["decode_raw"], dtype=dtype, dk=dk, dv=dv)
    ready_wl = replace(WORKLOADS["decode"], dtype=dtype, dk=dk, dv=dv)
    N, H = 5, 3
    state = make_decode_state(ready_wl, N=N, H=H, seed=3)
    s_gpu = state.to(DEV).clone()
    s_ref = to_f64(state)
    for step in range(4):
        tok = make_decode_token(raw_wl, step=step, N=N, H=H, seed=3)
        ready = make_decode_token(ready_wl, step=step, N=N, H=H, seed=3)
        if not prep & L2:
            tok.q, tok.k = ready.q, ready.k
        if not prep & SP:
            tok.log_alpha = ready.log_alpha
        if not prep & SG:
            tok.beta = ready.beta
        if step == 1:
            tok.k[0, 0] = 0.0                    # all-zero key: no write, decay only
        o = kda.decode_step(tok.q.to(DEV), tok.k.to(DEV), tok.v.to(DEV), tok.log_alpha.to(DEV),
                            tok.beta.to(DEV), s_gpu, prep=prep)
        q, k, la, b = oracle.prep.preprocess(to_f64(tok.q), to_f64(tok.k), to_f64(tok.log_alpha),
                                             to_f64(tok.beta), prep)
        o_ref, s_ref = oracle.decode_step(q, k, to_f64(tok.v), la, b, s_ref)
        torch.cuda.synchronize()
        assert rel_err(to_f64(o), o_ref, stored_as=dtype) <= TOL[dtype], step
        assert rel_err(to_f64(s_gpu), s_ref) <= TOL[dtype], step


def test_prep_decode_full_size_sampled(cuda_ok):
    """256 sequences x 32 heads x 128 x 128 raw tokens with every flag (the fused
    decode benchmark's launch), 4 steps; sampled sequences vs the oracle."""
    wl = WORKLOADS["decode_raw"]
    state = make_decode_state(wl, device=DEV)
    idx = [0, 17, 128, 255]
    s_ref = to_f64(state[idx])
    for step in range(4):
        tok = make_decode_token(wl, step=step, device=DEV)
        o = kda.decode_step(tok.q, tok.k, tok.v, tok.log_alpha, tok.beta, state, prep=RAW_PREP)
        q, k, la, b = oracle.prep.preprocess(to_f64(tok.q[idx]), to_f64(tok.k[idx]), to_f64(tok.log_alpha[idx]),
                                             to_f64(tok.beta[idx]), RAW_PREP)
        o_ref, s_ref = oracle.decode_step(q, k, to_f64(tok.v[idx]), la, b, s_ref)
        torch.cuda.synchronize()
        assert rel_err(to_f64(o[idx]), o_ref, stored_as="bf16") <= 2e-2
    assert rel_err(to_f64(state[idx]), s_ref) <= 2e-2
    assert torch.isfinite(state).all()
