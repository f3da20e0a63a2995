"""Sequence parallelism: one long sequence split into contiguous segments, one
segment per rank, with the state handed over between segments.

The pages note that a fixed-size state is carried from chunk to chunk ("From
GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph); across
ranks the same state must cross every segment boundary.  Instead of passing it
rank to rank (each rank waiting for the previous one), every rank first
summarises its segment by two matrices, because the chunk chain is affine in
its start state:

    S_end = M S_start + F

* M  [H, dk, dk]: the segment's final state for the identity as initial state
  and zero values (with v = 0 the recurrence is linear in S);
* F  [H, dk, dv]: the segment's final state from a zero initial state.

One all-gather exchanges (M, F) among the ranks (H (dk^2 + dk dv) fp32 per
rank and sequence: 2 MiB at H = 16, d = 128); rank r then forms its start state
S_r = M_{r-1} S_{r-1} + F_{r-1} (S_0 is the caller's initial state) with plain
matrix products, and runs the prefill once more from S_r to produce its
outputs.  Each rank runs the prefill three times on T / N tokens (rank 0 once),
against once on T tokens for a single GPU.

The per-segment prefill is the library's ``chunk_fwd`` (CUDA); ``fwd`` may be
replaced by another callable with the same signature and return value, which is
how the exchange logic is tested on CPU ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _default_fwd(q, k, v, log_alpha, beta, init_state=None, C=64):
    from . import chunk_fwd
    return chunk_fwd(q, k, v, log_alpha, beta, init_state=init_state, C=C)


def segment_maps(q, k, v, log_alpha, beta, C: int = 64, fwd=None):
    """(M, F) of one segment: q, k, log_alpha [B, T, H, dk], v [B, T, H, dv],
    beta [B, T, H].  Returns M [B, H, dk, dk] and F [B, H, dk, dv] (fp32)."""
    fwd = fwd or _default_fwd
    B, _, H, dk = q.shape
    eye = torch.eye(dk, dtype=torch.float32, device=q.device).expand(B, H, dk, dk).contiguous()
    v0 = torch.zeros(q.shape, dtype=v.dtype, device=v.device)
    _, M = fwd(q, k, v0, log_alpha, beta, init_state=eye, C=C)
    _, F = fwd(q, k, v, log_alpha, beta, init_state=None, C=C)
    return M, F


def start_states(Ms, Fs, init_state=None):
    """Start state of every segment from the gathered maps: S_0 = init_state (or
    zero), S_{r+1} = M_r S_r + F_r.  Returns the list [S_0, ..., S_{N-1}]."""
    S = torch.zeros_like(Fs[0]) if init_state is None else init_state.to(Fs[0].dtype)
    out = [S]
    for r in range(len(Ms) - 1):
        S = torch.matmul(Ms[r], S) + Fs[r]
        out.append(S)
    return out


def seqpar_forward(q, k, v, log_alpha, beta, init_state=None, C: int = 64, group=None, fwd=None):
    """Prefill of this rank's segment of the sequences (every rank holds the same
    B sequences, segment ``rank`` of each, in rank order).  Returns this rank's
    (o, final_state); the last rank's final_state is the sequences' final state.
    ``init_state`` is used by rank 0 only."""
    fwd = fwd or _default_fwd
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        return fwd(q, k, v, log_alpha, beta, init_state=init_state, C=C)
    if rank == 0:
        o, fs = fwd(q, k, v, log_alpha, beta, init_state=init_state, C=C)
        M = torch.zeros(q.shape[0], q.shape[2], q.shape[3], q.shape[3], dtype=fs.dtype, device=fs.device)
        F = fs
    else:
        M, F = segment_maps(q, k, v, log_alpha, beta, C=C, fwd=fwd)
    # rank 0's entry is (0, S_end of rank 0), so the chain below starts from its true end state
    Ms = [torch.empty_like(M) for _ in range(world)]
    Fs = [torch.empty_like(F) for _ in range(world)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Fs, F.contiguous(), group=group)
    if rank == 0:
        return o, fs
    S = Fs[0]
    for r in range(1, rank):
        S = torch.matmul(Ms[r], S) + Fs[r]
    return fwd(q, k, v, log_alpha, beta, init_state=S.contiguous(), C=C)
