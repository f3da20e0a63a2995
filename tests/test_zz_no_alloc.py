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
from kda_inputs import make_prefill, to_f64
from kda_testlib import rel_err

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


def _args(inp):
    return (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point(cuda_ok):
    dev = "cuda:0"
    cases = [make_prefill("prefill", device=dev, B=2, T=300, H=4, seed=41),
             make_prefill("varlen", device=dev, H=4, lengths=[130, 0, 257, 64], seed=42)]
    for inp in cases:
        need = kda.workspace_size(inp.q.shape[0], inp.q.shape[1], inp.q.shape[2], 128, 128, inp.C,
                                  torch.bfloat16, cu_seqlens=inp.cu_seqlens)
        assert 0 < need <= kda.NOALLOC_SCRATCH_BYTES
    # two calls in a row, each leaving its own contents in the shared array
    got = [kda.chunk_fwd_noalloc(*_args(x), init_state=x.init_state, cu_seqlens=x.cu_seqlens, C=x.C)
           for x in cases]
    torch.cuda.synchronize()
    ref = [kda.chunk_fwd(*_args(x), init_state=x.init_state, cu_seqlens=x.cu_seqlens, C=x.C) for x in cases]
    torch.cuda.synchronize()
    for (o, fs), (o_r, fs_r) in zip(got, ref):
        assert rel_err(to_f64(o), to_f64(o_r), stored_as="bf16") <= 2e-2
        assert rel_err(to_f64(fs), to_f64(fs_r)) <= 2e-2
        assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    # the first problem again, after the second one used the array
    o_again, fs_again = kda.chunk_fwd_noalloc(*_args(cases[0]), init_state=cases[0].init_state, C=cases[0].C)
    torch.cuda.synchronize()
    B, T, H = cases[0].q.shape[:3]
    assert kda.device_status("noalloc", None, torch.bfloat16, B, T, H, 128, 128, cases[0].C) == 0
    assert rel_err(to_f64(o_again), to_f64(ref[0][0]), stored_as="bf16") <= 2e-2
    assert rel_err(to_f64(fs_again), to_f64(ref[0][1])) <= 2e-2
