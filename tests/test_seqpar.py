"""Sequence parallelism (one long sequence split across ranks, states handed
over through one all-gather of per-segment affine maps).

CPU: gloo ranks run the exchange with the fp64 oracle standing in for the
per-segment prefill (injected as ``fwd``), and the pieces must reproduce the
single-pass oracle.  GPU: the same split simulated on one GPU with the CUDA
prefill, against the single-call prefill and the oracle.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))


def oracle_fwd(q, k, v, log_alpha, beta, init_state=None, C=64):
    """chunk_fwd's signature on CPU torch tensors, computed by the oracle (fp64)."""
    import oracle
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f = lambda t: t.detach().to(torch.float64).reshape(B * T, *t.shape[2:]).numpy()
    s0 = None if init_state is None else init_state.detach().to(torch.float64).numpy()
    o, fs = oracle.forward(f(q), f(k), f(v), f(log_alpha), beta.detach().to(torch.float64).reshape(B * T, H).numpy(),
                           np.arange(B + 1, dtype=np.int64) * T, init_state=s0)
    return torch.from_numpy(o).reshape(B, T, H, dv), torch.from_numpy(fs)


def _inputs(T, seed, H=2, d=8, B=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, d))
    la = -np.logaddexp(0.0, rng.standard_normal((B, T, H, d)) + 2.0)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    s0 = rng.standard_normal((B, H, d, d)) * 0.1
    return [torch.from_numpy(x) for x in (q, k, v, la, beta, s0)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, T, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from kimi_delta_attention_30_b200 import seqpar
        q, k, v, la, beta, s0 = _inputs(T, seed=11)
        seg = T // world
        sl = slice(rank * seg, (rank + 1) * seg)
        o, fs = seqpar.seqpar_forward(q[:, sl], k[:, sl], v[:, sl], la[:, sl], beta[:, sl], init_state=s0,
                                      fwd=oracle_fwd)
        out[rank] = (o.numpy(), fs.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_seqpar_gloo_ranks_match_single_pass(world):
    T = 36
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), T, out), nprocs=world, join=True, start_method="spawn")
    q, k, v, la, beta, s0 = _inputs(T, seed=11)
    o_ref, fs_ref = oracle_fwd(q, k, v, la, beta, init_state=s0)
    o = np.concatenate([out[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(out[world - 1][1], fs_ref.numpy(), rtol=1e-9, atol=1e-11)


def test_segment_maps_are_the_affine_map():
    """S_end = M S_start + F for any start state (oracle on CPU)."""
    from kimi_delta_attention_30_b200 import seqpar
    q, k, v, la, beta, s0 = _inputs(20, seed=12)
    M, F = seqpar.segment_maps(q, k, v, la, beta, fwd=oracle_fwd)
    _, fs = oracle_fwd(q, k, v, la, beta, init_state=s0)
    np.testing.assert_allclose(torch.matmul(M, s0).numpy() + F.numpy(), fs.numpy(), rtol=1e-10, atol=1e-12)
    starts = seqpar.start_states([M, M], [F, F], init_state=s0)
    np.testing.assert_allclose(starts[1].numpy(), fs.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.gpu
@pytest.mark.parametrize("n_seg", [2, 4])
def test_seqpar_simulated_on_one_gpu(cuda_ok, n_seg):
    """B=2, H=3, T=1024 bf16, d=128 (tensor-core path) split into n_seg segments:
    maps on the GPU, start states chained, each segment's prefill from its start
    state; against the single call (same kernels) and the oracle on sampled heads."""
    import kimi_delta_attention_30_b200 as kda
    from kimi_delta_attention_30_b200 import seqpar
    from kda_inputs import make_prefill
    from kda_testlib import oracle_prefill, gpu_slices, rel_err
    inp = make_prefill("prefill", B=2, T=1024, H=3, seed=21, device="cuda:0")
    o1, f1 = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state)
    seg = 1024 // n_seg
    parts = [slice(i * seg, (i + 1) * seg) for i in range(n_seg)]
    take = lambda t, sl: t[:, sl].contiguous()
    maps = [seqpar.segment_maps(*(take(t, sl) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)))
            for sl in parts]
    starts = seqpar.start_states([m for m, _ in maps], [f for _, f in maps], init_state=inp.init_state)
    outs = [kda.chunk_fwd(*(take(t, sl) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)),
                          init_state=starts[i].contiguous()) for i, sl in enumerate(parts)]
    torch.cuda.synchronize()
    o2 = torch.cat([o for o, _ in outs], dim=1)
    f2 = outs[-1][1]
    assert rel_err(o2.float().cpu().numpy(), o1.float().cpu().numpy(), stored_as="bf16", both_stored=True) <= 2e-2
    assert rel_err(f2.cpu().numpy(), f1.cpu().numpy()) <= 2e-2
    o_ref, fs_ref, ti, s_, h_ = oracle_prefill(inp, heads=[0, 2])
    og, fg = gpu_slices(o2, f2, ti, s_, h_)
    assert rel_err(og, o_ref, stored_as="bf16") <= 2e-2
    assert rel_err(fg, fs_ref) <= 2e-2
