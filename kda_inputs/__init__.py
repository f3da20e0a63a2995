"""Seeded synthetic inputs for the KDA operator.

This module only draws random numbers and shapes them; it holds none of the
operator's arithmetic.  Both the CUDA path (tests, benchmark, smoke check) and
the fp64 oracle take their inputs from here.

Workloads (sizes and value distributions):

* ``tiny_f32``   -- fp32 prefill, B=1, H=2, T=256, d_k=d_v=64, chunk 64;
  log alpha = -softplus(N(0,1)+2), zero initial state.
* ``prefill``    -- bf16 prefill, B=4, H=16, T=4096, d=128, chunk 64;
  log alpha = -softplus(N(0,1)+3), initial state N(0, 0.02^2).
* ``long``       -- bf16 prefill, B=1, H=32, T=65536, d=128, chunk 64 or 128;
  as ``prefill`` except head 0 has alpha = 1 (log alpha = 0) and head 1 has one
  scalar alpha per token broadcast over the channels.
* ``decode``     -- 256 sequences x H=32, d=128, fp32 state N(0, 0.02^2), one
  fresh bf16 token per sequence per step, 64 steps.
* ``varlen``     -- 64 packed sequences, lengths uniform in [512, 32768], H=32,
  d=128, chunk 64, beta ~ U(0,1), initial state N(0, 0.02^2); the gate regime
  depends on the head index mod 3: near one (log alpha ~ U(-1e-3, 0)), near
  zero (log alpha ~ U(-16, -8)), mixed (log alpha = -softplus(N(0, 2))).

* ``prefill_raw`` / ``decode_raw`` -- the ``prefill`` / ``decode`` sizes with
  raw (un-preprocessed) inputs: q, k ~ N(0,1) * 2 NOT normalised, the gate
  argument holds logits a ~ N(0,1) + 3 (so -softplus(a) has the ``prefill``
  gate's distribution) and beta holds logits ~ N(0,1).

Common to all: q, k ~ N(0,1), L2-normalised over d_k (in fp64), v ~ N(0,1),
beta = sigmoid(N(0,1)) unless stated; every value is drawn in fp32/fp64 and
rounded once (round-to-nearest-even) to the input dtype.  N(mu, s^2) is
variance notation.  The logistic and softplus maps used here only shape the
draws' distributions.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    dk: int
    dv: int
    dtype: str                      # "bf16" or "f32"
    C: int = 64
    B: int = 1
    T: int = 0
    gate: str = "softplus3"         # softplus2 | softplus3 | regimes
    beta_dist: str = "sigmoid"      # sigmoid | uniform
    init_std: float = 0.0           # 0 -> zero initial state
    special_heads: bool = False     # head 0: alpha = 1, head 1: scalar alpha
    n_seqs: int = 0                 # varlen: number of packed sequences
    len_range: tuple = (0, 0)       # varlen: inclusive length range
    steps: int = 0                  # decode: number of steps
    raw: bool = False               # raw q/k, gate logits and beta logits
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, H=2, T=256, dk=64, dv=64, C=64, dtype="f32", gate="softplus2"),
    "prefill": Workload("prefill", B=4, H=16, T=4096, dk=128, dv=128, C=64, dtype="bf16", init_std=0.02),
    "long": Workload("long", B=1, H=32, T=65536, dk=128, dv=128, C=64, dtype="bf16", init_std=0.02,
                     special_heads=True),
    "decode": Workload("decode", B=256, H=32, T=1, dk=128, dv=128, dtype="bf16", init_std=0.02, steps=64),
    "varlen": Workload("varlen", H=32, dk=128, dv=128, C=64, dtype="bf16", gate="regimes",
                       beta_dist="uniform", init_std=0.02, n_seqs=64, len_range=(512, 32768)),
    "prefill_raw": Workload("prefill_raw", B=4, H=16, T=4096, dk=128, dv=128, C=64, dtype="bf16",
                            init_std=0.02, raw=True),
    "decode_raw": Workload("decode_raw", B=256, H=32, T=1, dk=128, dv=128, dtype="bf16", init_std=0.02,
                           steps=64, raw=True),
}

# Raw workloads pass these kda_prep flags (QK_L2NORM | GATE_SOFTPLUS | BETA_SIGMOID).
RAW_PREP = 1 | 2 | 4


def torch_dtype(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def varlen_lengths(n_seqs: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Sequence lengths, uniform integers in [lo, hi], from a seeded numpy generator."""
    rng = np.random.default_rng([seed, 0x5EC1E])
    return rng.integers(lo, hi + 1, size=n_seqs).astype(np.int64)


def cu_seqlens_of(lengths) -> np.ndarray:
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out


def _gen(device, seed: int, stream_id: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 0x9E3779B1 + stream_id * 0x85EBCA77) & ((1 << 63) - 1))
    return g


def _normal(shape, gen, device, dtype=torch.float32):
    return torch.randn(shape, generator=gen, device=device, dtype=dtype)


def _unit_rows(shape, gen, device):
    """N(0,1) rows L2-normalised over the last dimension, computed in fp64."""
    x = _normal(shape, gen, device, torch.float64)
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def _qk(shape, wl: Workload, gen, device):
    if wl.raw:
        return _normal(shape, gen, device) * 2.0
    return _unit_rows(shape, gen, device)


def _gate(shape, wl: Workload, gen, device, head_offset: int = 0):
    """log alpha of the given shape [..., H, dk] (fp32, before rounding); for a
    raw workload the gate logits."""
    H, dk = shape[-2], shape[-1]
    if wl.raw:
        if wl.gate not in ("softplus2", "softplus3") or wl.special_heads:
            raise ValueError("raw workloads draw softplus gate logits only")
        return _normal(shape, gen, device) + (2.0 if wl.gate == "softplus2" else 3.0)
    if wl.gate in ("softplus2", "softplus3"):
        shift = 2.0 if wl.gate == "softplus2" else 3.0
        la = -torch.nn.functional.softplus(_normal(shape, gen, device) + shift)
    elif wl.gate == "regimes":
        near1 = -torch.rand(shape, generator=gen, device=device) * 1e-3
        near0 = -8.0 - 8.0 * torch.rand(shape, generator=gen, device=device)
        mixed = -torch.nn.functional.softplus(_normal(shape, gen, device) * math.sqrt(2.0))
        hid = (torch.arange(H, device=device) + head_offset) % 3
        sel = hid.view(*([1] * (len(shape) - 2)), H, 1)
        la = torch.where(sel == 0, near1, torch.where(sel == 1, near0, mixed))
    else:
        raise ValueError(wl.gate)
    if wl.special_heads:
        la[..., 0, :] = 0.0                                   # head 0: alpha = 1 (DeltaNet)
        if H > 1:
            scalar = -torch.nn.functional.softplus(_normal(shape[:-2] + (1,), gen, device) + 3.0)
            la[..., 1, :] = scalar.expand(shape[:-2] + (dk,))  # head 1: one alpha per token
    return la


def _beta(shape, wl: Workload, gen, device):
    if wl.raw:
        return _normal(shape, gen, device)
    if wl.beta_dist == "sigmoid":
        return torch.sigmoid(_normal(shape, gen, device))
    return torch.rand(shape, generator=gen, device=device)


@dataclass
class PrefillInputs:
    q: torch.Tensor            # [B, T, H, dk] (varlen: [1, total, H, dk])
    k: torch.Tensor
    v: torch.Tensor            # [B, T, H, dv]
    log_alpha: torch.Tensor    # [B, T, H, dk]
    beta: torch.Tensor         # [B, T, H]
    init_state: torch.Tensor | None   # [N, H, dk, dv] fp32
    cu_seqlens: np.ndarray | None     # [N + 1] int64 (host) or None
    C: int
    dtype: str

    @property
    def n_seqs(self) -> int:
        return self.q.shape[0] if self.cu_seqlens is None else len(self.cu_seqlens) - 1

    @property
    def seq_start(self) -> np.ndarray:
        if self.cu_seqlens is not None:
            return self.cu_seqlens.astype(np.int64)
        B, T = self.q.shape[:2]
        return np.arange(B + 1, dtype=np.int64) * T


def make_prefill(wl: Workload | str, device="cpu", seed: int = 0, *, B=None, T=None, H=None,
                 lengths=None, C=None, init_zero=None, chunk_tokens: int = 1 << 20) -> PrefillInputs:
    """Draw a prefill batch for workload ``wl`` (sizes may be overridden).

    ``lengths`` (a list of sequence lengths) switches to packed varlen layout;
    the ``varlen`` workload draws them with :func:`varlen_lengths`.  Tokens are
    drawn in slices of ``chunk_tokens`` to bound temporary memory.
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    H = wl.H if H is None else H
    C = wl.C if C is None else C
    dt = torch_dtype(wl.dtype)
    if lengths is None and wl.n_seqs:
        lengths = varlen_lengths(wl.n_seqs, *wl.len_range, seed=seed)
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = cu_seqlens_of(lengths)
        Bx, Tx, N = 1, int(cu[-1]), len(lengths)
    else:
        cu = None
        Bx = wl.B if B is None else B
        Tx = wl.T if T is None else T
        N = Bx
    dk, dv = wl.dk, wl.dv
    q = torch.empty((Bx, Tx, H, dk), dtype=dt, device=device)
    k = torch.empty_like(q)
    v = torch.empty((Bx, Tx, H, dv), dtype=dt, device=device)
    la = torch.empty((Bx, Tx, H, dk), dtype=dt, device=device)
    beta = torch.empty((Bx, Tx, H), dtype=dt, device=device)
    step = max(1, chunk_tokens // max(1, H))
    for b in range(Bx):
        for s, t0 in enumerate(range(0, Tx, step)):
            t1 = min(Tx, t0 + step)
            g = _gen(device, seed, 1 + b * 100003 + s)
            n = t1 - t0
            q[b, t0:t1] = _qk((n, H, dk), wl, g, device).to(dt)
            k[b, t0:t1] = _qk((n, H, dk), wl, g, device).to(dt)
            v[b, t0:t1] = _normal((n, H, dv), g, device).to(dt)
            la[b, t0:t1] = _gate((n, H, dk), wl, g, device).to(dt)
            beta[b, t0:t1] = _beta((n, H), wl, g, device).to(dt)
    zero = (wl.init_std == 0.0) if init_zero is None else init_zero
    s0 = None
    if not zero:
        g = _gen(device, seed, 0)
        std = wl.init_std if wl.init_std else 0.02
        s0 = _normal((N, H, dk, dv), g, device) * std
    return PrefillInputs(q, k, v, la, beta, s0, cu, C, wl.dtype)


@dataclass
class DecodeInputs:
    q: torch.Tensor            # [N, H, dk]
    k: torch.Tensor
    v: torch.Tensor            # [N, H, dv]
    log_alpha: torch.Tensor    # [N, H, dk]
    beta: torch.Tensor         # [N, H]


def make_decode_state(wl: Workload | str = "decode", device="cpu", seed: int = 0, *, N=None, H=None):
    """Initial decode state [N, H, dk, dv] fp32 ~ N(0, 0.02^2)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    N = wl.B if N is None else N
    H = wl.H if H is None else H
    g = _gen(device, seed, 0)
    return _normal((N, H, wl.dk, wl.dv), g, device) * wl.init_std


def make_decode_token(wl: Workload | str = "decode", step: int = 0, device="cpu", seed: int = 0, *,
                      N=None, H=None) -> DecodeInputs:
    """The step-th token of every sequence (fresh draw per step)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    N = wl.B if N is None else N
    H = wl.H if H is None else H
    dt = torch_dtype(wl.dtype)
    g = _gen(device, seed, 7_000_001 + step)
    q = _qk((N, H, wl.dk), wl, g, device).to(dt)
    k = _qk((N, H, wl.dk), wl, g, device).to(dt)
    v = _normal((N, H, wl.dv), g, device).to(dt)
    la = _gate((N, H, wl.dk), wl, g, device).to(dt)
    beta = _beta((N, H), wl, g, device).to(dt)
    return DecodeInputs(q, k, v, la, beta)


def make_grad_outputs(inp: PrefillInputs, seed: int = 0, final: bool = True):
    """Upstream gradients for a prefill batch: d_o ~ N(0,1) in the input dtype,
    shaped like o, and (if ``final``) d_final_state ~ N(0, 0.1^2) fp32 shaped like
    the states."""
    dev = inp.q.device
    B, T, H, _ = inp.q.shape
    dv = inp.v.shape[-1]
    dk = inp.q.shape[-1]
    g = _gen(dev, seed, 9_000_001)
    d_o = _normal((B, T, H, dv), g, dev).to(inp.q.dtype)
    dfs = _normal((inp.n_seqs, H, dk, dv), g, dev) * 0.1 if final else None
    return d_o, dfs


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16 / fp32) tensor to a host fp64 array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
