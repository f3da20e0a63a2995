"""Helpers shared by the tests: parity metric and oracle calls on sampled slices.

The oracle (``oracle/``) is imported here only; the CUDA binding never is.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from kda_inputs import to_f64

TOL = {"bf16": 2e-2, "f32": 1e-4}


def bf16_half_ulp(x):
    """Half the bf16 spacing at each (bf16-representable) value of x: the most
    that round-to-nearest-even moves a value when it is stored as bf16."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(ax > 0, 2.0 ** (e - 8), 2.0 ** -134)


def rel_err(got, ref, stored_as=None, both_stored=False) -> float:
    """max |got - ref| / rms(ref) over the compared elements.

    With ``stored_as="bf16"`` the GPU values were rounded once to bf16 when
    they were written (the output dtype follows the inputs); that rounding is
    not an error of the computation, so each |got - ref| is first reduced by
    the half-ulp the storage may add (and floored at 0).  With
    ``both_stored=True`` (two stored GPU outputs compared with each other) the
    half-ulp of each side is allowed."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.size == 0:
        return 0.0
    d = np.abs(got - ref)
    if stored_as == "bf16":
        allow = bf16_half_ulp(got) + (bf16_half_ulp(ref) if both_stored else 0.0)
        d = np.maximum(d - allow, 0.0)
    rms = np.sqrt(np.mean(ref ** 2))
    if rms == 0.0:
        return float(np.max(d))
    return float(np.max(d) / rms)


# (label, error with the storage allowance, error without it, bound) of every
# check made through parity(); the session summary prints them
PARITY_LOG = []


def parity(label, got, ref, tol, stored_as=None, both_stored=False) -> float:
    """rel_err with the bf16 storage allowance (the figure the bound is judged
    on), logged next to the plain max |got - ref| / rms(ref), which shows how
    much of the bound the output's own bf16 rounding uses."""
    e = rel_err(got, ref, stored_as=stored_as, both_stored=both_stored)
    raw = rel_err(got, ref) if stored_as else e
    PARITY_LOG.append((label, e, raw, tol))
    return e


def oracle_prefill(inp, heads=None, seqs=None, n_threads=0, prep=0):
    """Oracle o / final_state for the given heads and sequences of a PrefillInputs.

    ``prep`` (kda_prep flags) runs the inputs through ``oracle.prep`` first.
    Returns (o_ref [n_tok_sel, n_heads, dv], fs_ref [n_seq_sel, n_heads, dk, dv],
    token index array, seq list, head list)."""
    H = inp.q.shape[2]
    heads = list(range(H)) if heads is None else list(heads)
    ss = inp.seq_start
    seqs = list(range(len(ss) - 1)) if seqs is None else list(seqs)
    flat = lambda t: t.reshape(-1, *t.shape[2:])
    tok_idx = np.concatenate([np.arange(ss[s], ss[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    lens = [int(ss[s + 1] - ss[s]) for s in seqs]
    sub_start = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ti = torch.as_tensor(tok_idx, device=inp.q.device, dtype=torch.long)
    hi = torch.as_tensor(heads, device=inp.q.device, dtype=torch.long)

    def pick(t):
        return to_f64(flat(t).index_select(0, ti).index_select(1, hi))

    s0 = None
    if inp.init_state is not None:
        si = torch.as_tensor(seqs, device=inp.q.device, dtype=torch.long)
        s0 = to_f64(inp.init_state.index_select(0, si).index_select(1, hi))
    q, k, la, beta = oracle.prep.preprocess(pick(inp.q), pick(inp.k), pick(inp.log_alpha), pick(inp.beta), prep)
    o, fs = oracle.forward(q, k, pick(inp.v), la, beta, sub_start, init_state=s0, n_threads=n_threads)
    return o, fs, tok_idx, seqs, heads


def oracle_backward(inp, d_o, d_final=None, heads=None, seqs=None, n_threads=0):
    """Oracle gradients (dict of fp64 arrays, token-major over the selected
    sequences, heads on axis 1) for the given heads and sequences."""
    H = inp.q.shape[2]
    heads = list(range(H)) if heads is None else list(heads)
    ss = inp.seq_start
    seqs = list(range(len(ss) - 1)) if seqs is None else list(seqs)
    flat = lambda t: t.reshape(-1, *t.shape[2:])
    tok_idx = np.concatenate([np.arange(ss[s], ss[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    lens = [int(ss[s + 1] - ss[s]) for s in seqs]
    sub_start = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ti = torch.as_tensor(tok_idx, device=inp.q.device, dtype=torch.long)
    hi = torch.as_tensor(heads, device=inp.q.device, dtype=torch.long)
    si = torch.as_tensor(seqs, device=inp.q.device, dtype=torch.long)

    def pick(t):
        return to_f64(flat(t).index_select(0, ti).index_select(1, hi))

    pick_s = lambda t: None if t is None else to_f64(t.index_select(0, si).index_select(1, hi))
    g = oracle.backward(pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.log_alpha), pick(inp.beta), sub_start,
                        pick(d_o), d_final_state=pick_s(d_final), init_state=pick_s(inp.init_state),
                        n_threads=n_threads)
    return g, tok_idx, seqs, heads


def gpu_grad_slices(grads, tok_idx, seqs, heads):
    """The same slices of the GPU gradients (dq, dk, dv, dlog_alpha, dbeta,
    d_init_state) as a dict of host fp64 arrays."""
    names = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init_state")
    out = {}
    for name, t in zip(names, grads):
        if t is None:
            continue
        dev = t.device
        hi = torch.as_tensor(heads, device=dev, dtype=torch.long)
        if name == "d_init_state":
            si = torch.as_tensor(seqs, device=dev, dtype=torch.long)
            out[name] = to_f64(t.index_select(0, si).index_select(1, hi))
        else:
            ti = torch.as_tensor(tok_idx, device=dev, dtype=torch.long)
            out[name] = to_f64(t.reshape(-1, *t.shape[2:]).index_select(0, ti).index_select(1, hi))
    return out


def gpu_slices(o_gpu, fs_gpu, tok_idx, seqs, heads):
    """The same slices of the GPU outputs as host fp64 arrays."""
    dev = o_gpu.device
    ti = torch.as_tensor(tok_idx, device=dev, dtype=torch.long)
    hi = torch.as_tensor(heads, device=dev, dtype=torch.long)
    o = to_f64(o_gpu.reshape(-1, *o_gpu.shape[2:]).index_select(0, ti).index_select(1, hi))
    fs = None
    if fs_gpu is not None:
        si = torch.as_tensor(seqs, device=dev, dtype=torch.long)
        fs = to_f64(fs_gpu.index_select(0, si).index_select(1, hi))
    return o, fs
