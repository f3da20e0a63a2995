"""Sequence parallelism: one long sequence split into contiguous segments, one
segment per rank, with the state handed over between segments.

The pages note that a fixed-size state is carried from chunk to chunk ("From
GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph); across
ranks the same state must cross every segment boundary.  Instead of passing it
rank to rank (each rank waiting for the previous one), every rank first
summarises its segment by two matrices, because the chunk chain is affine in
its start state:

    S_end = M S_start + F

* M  [B, H, dk, dk]: the segment's final state from the identity with the
  values' contribution left out;
* F  [B, H, dk, dv]: the segment's final state from a zero start.

Both come from one library call (``kda_chunk_segment_map``).  One all-gather
exchanges (M, F) among the ranks (H (dk^2 + dk dv) fp32 per rank and sequence:
2 MiB at H = 16, d = 128); rank r chains the maps of the ranks before it with
``kda_compose_states`` and runs the prefill from the start state that gives.
This module only marshals tensors and calls NCCL; every step of the arithmetic
runs in the library.

``fwd``, ``maps`` and ``compose`` may be replaced by callables with the same
signatures and results (the CPU tests inject the fp64 oracle and a host
composition, so the exchange logic runs on gloo ranks without a GPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _default_fwd(q, k, v, log_alpha, beta, init_state=None, C=64):
    from . import chunk_fwd
    return chunk_fwd(q, k, v, log_alpha, beta, init_state=init_state, C=C)


def _default_maps(q, k, v, log_alpha, beta, C=64):
    from . import segment_map
    return segment_map(q, k, v, log_alpha, beta, C=C)


def _default_compose(Ms, Fs, init_state=None):
    from . import compose_states
    return compose_states(Ms, Fs, init_state=init_state)


def segment_maps(q, k, v, log_alpha, beta, C: int = 64, maps=None):
    """(M, F) of one segment: q, k, log_alpha [B, T, H, dk], v [B, T, H, dv],
    beta [B, T, H].  Returns M [B, H, dk, dk] and F [B, H, dk, dv] (fp32)."""
    return (maps or _default_maps)(q, k, v, log_alpha, beta, C=C)


def start_states(Ms, Fs, init_state=None, compose=None):
    """States the segments start from, given the maps of segments 0 .. R-1 as
    [R, B, H, dk, dk] and [R, B, H, dk, dv] tensors: S_0 = init_state (or zero),
    S_{r+1} = M_r S_r + F_r.  Returns [R + 1, B, H, dk, dv]."""
    return (compose or _default_compose)(Ms.contiguous(), Fs.contiguous(), init_state)


def seqpar_forward(q, k, v, log_alpha, beta, init_state=None, C: int = 64, group=None, fwd=None, maps=None,
                   compose=None):
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
        # rank 0's entry is (0, its end state), so the chain below starts from its true end state
        M = torch.zeros(q.shape[0], q.shape[2], q.shape[3], q.shape[3], dtype=fs.dtype, device=fs.device)
        F = fs
    else:
        M, F = segment_maps(q, k, v, log_alpha, beta, C=C, maps=maps)
    Ml = [torch.empty_like(M) for _ in range(world)]
    Fl = [torch.empty_like(F) for _ in range(world)]
    dist.all_gather(Ml, M.contiguous(), group=group)
    dist.all_gather(Fl, F.contiguous(), group=group)
    Ms, Fs = torch.stack(Ml), torch.stack(Fl)
    if rank == 0:
        return o, fs
    # segments 0 .. rank-1 from a zero state (segment 0's map is (0, its end state))
    S = start_states(Ms[:rank], Fs[:rank], None, compose=compose)[rank]
    return fwd(q, k, v, log_alpha, beta, init_state=S.contiguous(), C=C)
