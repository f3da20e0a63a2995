"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
memory (a plugin host that passes only inputs and outputs, or a runtime whose
pool owns the whole device).  Its scratch is the library's own fixed device
array, so its results must equal those of kda_chunk_fwd with a caller-owned
workspace, call after call, whatever the previous call left in that array.

This file is collected last on purpose: if it fails, every other test has
already run.
"""
import ctypes

import pytest
import torch

import kimi_delta_attention_30_b200 as kda
from kda_inputs import make_prefill
from kda_testlib import gpu_slices, oracle_prefill, rel_err

E_SCRATCH = -11


def test_noalloc_rejects_oversized_problem_before_launch():
    """A problem whose scratch exceeds the fixed array is refused on the host
    (fake device pointers: nothing may be dereferenced or launched)."""
    lib = kda.lib()
    vp = ctypes.c_void_p
    B, T, H = 4, 4096, 16                    # needs far more than 64 MiB of scratch
    assert kda.workspace_size(B, T, H, 128, 128, 64, torch.bfloat16) > kda.NOALLOC_SCRATCH_BYTES
    st = lib.kda_chunk_fwd_noalloc(vp(0x10000), vp(0x20000), vp(0x30000), vp(0x40000), vp(0x50000), 0, None,
                                   None, 0, B, T, H, 128, 128, 64, vp(0x60000), None, None)
    assert st == E_SCRATCH
    assert "SCRATCH" in lib.kda_status_string(E_SCRATCH).decode()


def test_noalloc_limits_stated_in_the_header():
    """The per-path bounds the header states follow from the workspace sizes:
    450 tensor-core chunk-heads fit, the CUDA-core path holds about 18.7 K
    token-heads at d = 128 and 43 K at d = 64 (host computation only)."""
    lim = kda.NOALLOC_SCRATCH_BYTES
    assert kda.workspace_size(1, 1792, 16, 128, 128, 64, torch.bfloat16) <= lim < \
        kda.workspace_size(1, 1792 + 64, 16, 128, 128, 64, torch.bfloat16)
    assert kda.workspace_size(1, 18 * 1024, 1, 128, 128, 64, torch.float32) <= lim < \
        kda.workspace_size(1, 19 * 1024, 1, 128, 128, 64, torch.float32)
    assert kda.workspace_size(1, 42 * 1024, 1, 64, 64, 64, torch.float32) <= lim < \
        kda.workspace_size(1, 44 * 1024, 1, 64, 64, 64, torch.float32)


def _args(inp):
    return (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)


def _ref_and_noalloc(inp):
    kw = dict(init_state=inp.init_state, cu_seqlens=inp.cu_seqlens, C=inp.C)
    return (kda.chunk_fwd(*_args(inp), **kw), kda.chunk_fwd_noalloc(*_args(inp), **kw))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(cuda_ok):
    """Both entry points run the same deterministic kernels on the same inputs,
    so their results must agree bit for bit, whatever the shared array held
    before: the tensor-core path (bf16, d = 128) and the CUDA-core path (fp32,
    d = 64), each before and after a larger problem has used the array."""
    from dataclasses import replace
    from kda_inputs import WORKLOADS
    dev = "cuda:0"
    f32 = replace(WORKLOADS["prefill"], dtype="f32", dk=64, dv=64)
    cases = {
        "tc": make_prefill("prefill", device=dev, B=2, T=300, H=4, seed=41),
        "tc_varlen": make_prefill("varlen", device=dev, H=4, lengths=[130, 0, 257, 64], seed=42),
        "simt": make_prefill(f32, device=dev, B=2, T=300, H=3, seed=43),
        "simt_big": make_prefill(f32, device=dev, B=1, T=2048, H=16, seed=44),
        "tc_big": make_prefill("prefill", device=dev, B=1, T=1024, H=16, seed=45),
    }
    for name, inp in cases.items():
        B, T, H, dk = inp.q.shape
        need = kda.workspace_size(B, T, H, dk, inp.v.shape[-1], inp.C, inp.q.dtype, cu_seqlens=inp.cu_seqlens)
        assert 0 < need <= kda.NOALLOC_SCRATCH_BYTES, name
    # two calls in a row, then the small problems again after the large ones
    order = ["tc", "tc_varlen", "simt", "simt_big", "simt", "tc_big", "tc", "simt"]
    for name in order:
        inp = cases[name]
        (o_r, fs_r), (o, fs) = _ref_and_noalloc(inp)
        torch.cuda.synchronize()
        assert torch.equal(o, o_r), name
        assert torch.equal(fs, fs_r), name
        assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    # the status word belongs to the last call on the array: a tensor-core one here
    inp = cases["tc"]
    kda.chunk_fwd_noalloc(*_args(inp), init_state=inp.init_state, C=inp.C)
    B, T, H = inp.q.shape[:3]
    assert kda.device_status("noalloc", None, torch.bfloat16, B, T, H, 128, 128, inp.C) == 0
    # a sanity check against the oracle on the last (fp32) problem
    inp = cases["simt"]
    _, (o, fs) = _ref_and_noalloc(inp)
    torch.cuda.synchronize()
    o_ref, fs_ref, ti, seqs, heads = oracle_prefill(inp)
    og, fg = gpu_slices(o, fs, ti, seqs, heads)
    assert rel_err(og, o_ref) <= 1e-4 and rel_err(fg, fs_ref) <= 1e-4
