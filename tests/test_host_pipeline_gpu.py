"""GPU: the host-buffer prefill (kda_chunk_fwd_host), which copies groups of
sequences to the device, computes them and copies the results back with the
transfers of neighbouring groups overlapping the computation.

Each group is one kda_chunk_fwd call on that group's sequences, and a
sequence's result does not depend on the others in the batch, so the outputs
must equal the device call's on the whole batch bit for bit (and, through it,
the oracle at the usual bound, checked here as well on the whole batch)."""
from dataclasses import replace

import pytest
import torch

import kimi_delta_attention_30_b200 as kda
from kda_inputs import WORKLOADS, make_prefill
from kda_testlib import TOL, gpu_slices, oracle_prefill, parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
LENGTHS = [0, 1, 63, 64, 200, 1000, 17, 0, 640, 129]


def _host(inp):
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    return {n: pin(getattr(inp, n)) for n in ("q", "k", "v", "log_alpha", "beta", "init_state")}


def _device_call(inp):
    dev = {n: (None if t is None else t.to(DEV)) for n, t in _host(inp).items()}
    o, fs = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], init_state=dev["init_state"],
                          cu_seqlens=inp.cu_seqlens, C=inp.C)
    torch.cuda.synchronize()
    return o.cpu(), fs.cpu()


@pytest.mark.parametrize("wl", ["bf16", "f32"])
@pytest.mark.parametrize("n_groups", [1, 3, 16])
def test_host_pipeline_equals_the_device_call(wl, n_groups):
    if wl == "bf16":
        w = replace(WORKLOADS["varlen"], H=3)
    else:
        w = replace(WORKLOADS["tiny_f32"], dk=64, dv=128, H=2)
    inp = make_prefill(w, seed=7, lengths=LENGTHS)
    h = _host(inp)
    o_ref, fs_ref = _device_call(inp)
    buf = torch.empty(kda.host_buffer_size(inp.cu_seqlens, inp.q.shape[2], inp.q.shape[3], inp.v.shape[3], inp.C,
                                           inp.q.dtype, n_groups), dtype=torch.uint8, device=DEV)
    o, fs = kda.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], inp.cu_seqlens,
                               init_state=h["init_state"], C=inp.C, n_groups=n_groups, device_buffer=buf)
    assert torch.equal(o, o_ref)
    assert torch.equal(fs, fs_ref)
    assert kda.host_device_status(buf) == 0
    # and against the oracle on every sequence and head
    ref_o, ref_fs, ti, seqs, heads = oracle_prefill(inp)
    og, fg = gpu_slices(o, fs, ti, seqs, heads)
    tol = TOL["bf16" if wl == "bf16" else "f32"]
    parity(f"host pipeline {wl} groups={n_groups} o", og, ref_o, tol, stored_as=inp.dtype)
    parity(f"host pipeline {wl} groups={n_groups} state", fg, ref_fs, tol)


def test_host_pipeline_without_initial_or_final_state():
    inp = make_prefill(replace(WORKLOADS["varlen"], H=2), seed=3, lengths=[300, 5, 0, 77])
    h = _host(inp)
    o, fs = kda.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], inp.cu_seqlens, init_state=None,
                               C=64, n_groups=2, output_final_state=False)
    assert fs is None
    dev = {n: (None if t is None else t.to(DEV)) for n, t in h.items()}
    o_ref, _ = kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], init_state=None,
                             cu_seqlens=inp.cu_seqlens, C=64)
    assert torch.equal(o, o_ref.cpu())


def test_host_pipeline_from_pageable_memory():
    """Pageable (not page-locked) host tensors work too: the copies then do not
    overlap, the results are the same."""
    inp = make_prefill(replace(WORKLOADS["varlen"], H=2), seed=11, lengths=[130, 64, 1, 500])
    q, k, v, la, b = (getattr(inp, n).contiguous() for n in ("q", "k", "v", "log_alpha", "beta"))
    assert not q.is_pinned()
    o, fs = kda.chunk_fwd_host(q, k, v, la, b, inp.cu_seqlens, init_state=inp.init_state.contiguous(), C=64,
                               n_groups=3, o=torch.empty(v.shape, dtype=v.dtype),
                               final_state=torch.empty(inp.init_state.shape, dtype=torch.float32))
    o_ref, fs_ref = _device_call(inp)
    assert torch.equal(o, o_ref)
    assert torch.equal(fs, fs_ref)
