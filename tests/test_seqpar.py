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


def oracle_maps(q, k, v, log_alpha, beta, C=64):
    """segment_map's results computed by the oracle: M is the final state from
    the identity with v = 0 (the recurrence is then linear in the state), F the
    final state from a zero start."""
    B, _, H, dk = q.shape
    eye = torch.eye(dk, dtype=torch.float64).expand(B, H, dk, dk).contiguous()
    _, M = oracle_fwd(q, k, torch.zeros_like(v), log_alpha, beta, init_state=eye, C=C)
    _, F = oracle_fwd(q, k, v, log_alpha, beta, init_state=None, C=C)
    return M, F


def host_compose(Ms, Fs, init_state=None):
    """compose_states' result on the host: S_0 = init (or 0), S_{r+1} = M_r S_r + F_r."""
    S = torch.zeros_like(Fs[0]) if init_state is None else init_state.to(Fs.dtype)
    out = [S]
    for r in range(Ms.shape[0]):
        S = torch.matmul(Ms[r], S) + Fs[r]
        out.append(S)
    return torch.stack(out)


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
                                      fwd=oracle_fwd, maps=oracle_maps, compose=host_compose)
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
    M, F = seqpar.segment_maps(q, k, v, la, beta, maps=oracle_maps)
    _, fs = oracle_fwd(q, k, v, la, beta, init_state=s0)
    np.testing.assert_allclose(torch.matmul(M, s0).numpy() + F.numpy(), fs.numpy(), rtol=1e-10, atol=1e-12)
    starts = seqpar.start_states(torch.stack([M, M]), torch.stack([F, F]), init_state=s0, compose=host_compose)
    np.testing.assert_allclose(starts[1].numpy(), fs.numpy(), rtol=1e-10, atol=1e-12)


def _gpu_inputs(dtype, B=2, T=1024, H=3, seed=21, d=128):
    from dataclasses import replace
    from kda_inputs import WORKLOADS, make_prefill
    wl = replace(WORKLOADS["prefill"], dtype=dtype, dk=d, dv=d)
    return make_prefill(wl, B=B, T=T, H=H, seed=seed, device="cuda:0")


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,tol", [("bf16", 128, 2e-2), ("f32", 64, 1e-4)])
def test_segment_map_matches_oracle(cuda_ok, dtype, d, tol):
    """kda_chunk_segment_map against the oracle: M is the final state from the
    identity with v = 0, F the final state from zero (tensor-core path for bf16
    d = 128, CUDA-core path for fp32 d = 64), including a ragged, an empty and a
    one-token sequence of a packed batch."""
    import kimi_delta_attention_30_b200 as kda
    from dataclasses import replace
    from kda_inputs import WORKLOADS, make_prefill, to_f64
    from kda_testlib import parity
    wl = replace(WORKLOADS["prefill"], dtype=dtype, dk=d, dv=d)
    for inp in (_gpu_inputs(dtype, d=d), make_prefill(wl, lengths=[200, 0, 1, 130], H=2, seed=5, device="cuda:0")):
        M, F = kda.segment_map(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, cu_seqlens=inp.cu_seqlens)
        torch.cuda.synchronize()
        ss = inp.seq_start
        n_tok = int(ss[-1])
        f = lambda t: to_f64(t).reshape(n_tok, *t.shape[2:])
        N, H = M.shape[0], M.shape[1]
        eye = np.broadcast_to(np.eye(d), (N, H, d, d)).copy()
        import oracle
        _, M_ref = oracle.forward(f(inp.q), f(inp.k), np.zeros_like(f(inp.v)), f(inp.log_alpha),
                                  to_f64(inp.beta).reshape(n_tok, H), ss, init_state=eye)
        _, F_ref = oracle.forward(f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha),
                                  to_f64(inp.beta).reshape(n_tok, H), ss)
        assert parity(f"segment map M {dtype} d={d}", to_f64(M), M_ref, tol) <= tol
        assert parity(f"segment map F {dtype} d={d}", to_f64(F), F_ref, tol) <= tol


@pytest.mark.gpu
def test_compose_states_matches_matrix_chain(cuda_ok):
    """kda_compose_states against the chain S_{r+1} = M_r S_r + F_r in fp64."""
    import kimi_delta_attention_30_b200 as kda
    g = torch.Generator(device="cpu").manual_seed(3)
    for R, N, H, d, init in ((3, 2, 2, 128, True), (1, 1, 3, 64, False), (0, 2, 1, 128, True)):
        M = torch.randn((R, N, H, d, d), generator=g) / d ** 0.5
        F = torch.randn((R, N, H, d, d), generator=g)
        s0 = torch.randn((N, H, d, d), generator=g) if init else None
        out = kda.compose_states(M.cuda(), F.cuda(), None if s0 is None else s0.cuda())
        torch.cuda.synchronize()
        ref = host_compose(M.double(), F.double(), None if s0 is None else s0.double())
        assert out.shape == ref.shape
        assert torch.allclose(out.cpu().double(), ref, rtol=1e-5, atol=1e-5)


@pytest.mark.gpu
@pytest.mark.parametrize("n_seg", [2, 4])
def test_seqpar_simulated_on_one_gpu(cuda_ok, n_seg):
    """B=2, H=3, T=1024 bf16, d=128 (tensor-core path) split into n_seg segments:
    maps from kda_chunk_segment_map, start states from kda_compose_states, each
    segment's prefill from its start state; against the single call and the
    oracle on sampled heads."""
    import kimi_delta_attention_30_b200 as kda
    from kimi_delta_attention_30_b200 import seqpar
    from kda_testlib import oracle_prefill, gpu_slices, parity, rel_err
    inp = _gpu_inputs("bf16")
    o1, f1 = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state)
    seg = 1024 // n_seg
    parts = [slice(i * seg, (i + 1) * seg) for i in range(n_seg)]
    take = lambda t, sl: t[:, sl].contiguous()
    maps = [seqpar.segment_maps(*(take(t, sl) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)))
            for sl in parts]
    starts = seqpar.start_states(torch.stack([m for m, _ in maps]), torch.stack([f for _, f in maps]),
                                 init_state=inp.init_state)
    outs = [kda.chunk_fwd(*(take(t, sl) for t in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)),
                          init_state=starts[i].contiguous()) for i, sl in enumerate(parts)]
    torch.cuda.synchronize()
    o2 = torch.cat([o for o, _ in outs], dim=1)
    f2 = outs[-1][1]
    assert rel_err(o2.float().cpu().numpy(), o1.float().cpu().numpy(), stored_as="bf16", both_stored=True) <= 2e-2
    assert rel_err(f2.cpu().numpy(), f1.cpu().numpy()) <= 2e-2
    assert rel_err(starts[n_seg].cpu().numpy(), f1.cpu().numpy()) <= 2e-2
    o_ref, fs_ref, ti, s_, h_ = oracle_prefill(inp, heads=[0, 2])
    og, fg = gpu_slices(o2, f2, ti, s_, h_)
    assert parity(f"seqpar {n_seg} segments o", og, o_ref, 2e-2, stored_as="bf16") <= 2e-2
    assert parity(f"seqpar {n_seg} segments state", fg, fs_ref, 2e-2) <= 2e-2
