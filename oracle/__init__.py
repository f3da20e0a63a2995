"""KDA reference oracle (fp64, CPU) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it, and it imports nothing from them.

Two implementations of the same operator and its gradient, in plain C
(``kda_oracle.c``):

* :func:`forward` -- the token-by-token recurrence (decay, read, error, write,
  read-out), the definition of KDA.
* :func:`backward` -- the reverse-mode gradient of the token recurrence
  (for training), states recomputed from copies kept every 64 tokens.
* :func:`chunkform` -- the chunkwise form with the WY/UT triangular solve,
  written with pairwise decay products; it also returns the intermediates that
  the GPU kernels materialise (cumulative log decay, U, Wk, W and the start
  state of every chunk).

All arrays are numpy fp64, token-major: q, k, log_alpha ``[n_tokens, H, dk]``,
v ``[n_tokens, H, dv]``, beta ``[n_tokens, H]``; sequences are contiguous token
ranges given by ``seq_start`` (``[n_seqs + 1]`` offsets starting at 0).
States are ``[n_seqs, H, dk, dv]``.

:mod:`oracle.prep` (numpy) maps raw q / k, gate logits and beta logits to the
operator's inputs (L2 norm, -softplus, sigmoid).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from . import prep  # noqa: F401  (re-exported: oracle.prep.preprocess)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            lib.kda_ref_forward_f64.argtypes = [dp, dp, dp, dp, dp, dp, i64p, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, dp, dp, ctypes.c_int]
            lib.kda_ref_forward_f64.restype = ctypes.c_int
            lib.kda_ref_chunkform_f64.argtypes = [dp, dp, dp, dp, dp, dp, i64p, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp, dp, dp,
                                                  dp, dp, dp, ctypes.c_int]
            lib.kda_ref_chunkform_f64.restype = ctypes.c_int
            lib.kda_ref_backward_f64.argtypes = [dp, dp, dp, dp, dp, dp, i64p, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp,
                                                 ctypes.c_int]
            lib.kda_ref_backward_f64.restype = ctypes.c_int
            lib.kda_ref_max_threads.argtypes = []
            lib.kda_ref_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the oracle's OpenMP runtime uses by default."""
    return int(_load().kda_ref_max_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(q, k, v, log_alpha, beta, seq_start):
    q, k, v, log_alpha, beta = (_f64(x) for x in (q, k, v, log_alpha, beta))
    seq_start = np.ascontiguousarray(seq_start, dtype=np.int64)
    n_tok, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (n_tok, H, dk) and log_alpha.shape == (n_tok, H, dk)
    assert v.shape == (n_tok, H, dv) and beta.shape == (n_tok, H)
    assert seq_start.ndim == 1 and seq_start[0] == 0 and seq_start[-1] == n_tok
    assert np.all(np.diff(seq_start) >= 0)
    return q, k, v, log_alpha, beta, seq_start, n_tok, H, dk, dv


def forward(q, k, v, log_alpha, beta, seq_start, init_state=None, n_threads: int = 0):
    """Token recurrence (O1).  Returns ``(o [n_tokens,H,dv], final_state [N,H,dk,dv])``."""
    q, k, v, log_alpha, beta, seq_start, n_tok, H, dk, dv = _check(q, k, v, log_alpha, beta, seq_start)
    n_seqs = len(seq_start) - 1
    s0 = None if init_state is None else _f64(init_state)
    if s0 is not None:
        assert s0.shape == (n_seqs, H, dk, dv)
    o = np.zeros((n_tok, H, dv))
    fs = np.zeros((n_seqs, H, dk, dv))
    rc = _load().kda_ref_forward_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(s0),
                                     seq_start.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                     n_seqs, H, dk, dv, _ptr(o), _ptr(fs), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_ref_forward_f64 failed ({rc})")
    return o, fs


def chunkform(q, k, v, log_alpha, beta, seq_start, C: int, init_state=None,
              intermediates: bool = False, n_threads: int = 0):
    """Chunkwise WY/UT form (O2).  Returns a dict with ``o`` and ``final_state``;
    with ``intermediates=True`` also ``g``, ``u``, ``wk``, ``w`` (token-major like
    the inputs) and ``s_chunk`` (``[n_chunks, H, dk, dv]``, start state of every
    chunk, chunks ordered sequence by sequence)."""
    q, k, v, log_alpha, beta, seq_start, n_tok, H, dk, dv = _check(q, k, v, log_alpha, beta, seq_start)
    n_seqs = len(seq_start) - 1
    s0 = None if init_state is None else _f64(init_state)
    lens = np.diff(seq_start)
    n_chunks = int(np.sum((lens + C - 1) // C))
    out = {"o": np.zeros((n_tok, H, dv)), "final_state": np.zeros((n_seqs, H, dk, dv))}
    if intermediates:
        out["g"] = np.zeros((n_tok, H, dk))
        out["u"] = np.zeros((n_tok, H, dv))
        out["wk"] = np.zeros((n_tok, H, dk))
        out["w"] = np.zeros((n_tok, H, dv))
        out["s_chunk"] = np.zeros((n_chunks, H, dk, dv))
    g = out.get("g")
    rc = _load().kda_ref_chunkform_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(s0),
        seq_start.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n_seqs, H, dk, dv, int(C),
        _ptr(out["o"]), _ptr(out["final_state"]), _ptr(g), _ptr(out.get("u")), _ptr(out.get("wk")),
        _ptr(out.get("w")), _ptr(out.get("s_chunk")), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_ref_chunkform_f64 failed ({rc})")
    return out


def backward(q, k, v, log_alpha, beta, seq_start, d_o, d_final_state=None, init_state=None,
             n_threads: int = 0):
    """Reverse-mode gradient of :func:`forward` (O3) for the loss
    ``sum(d_o * o) + sum(d_final_state * final_state)``.  Returns a dict with
    ``dq, dk, dv, dlog_alpha, dbeta, d_init_state`` shaped like the inputs
    (``d_init_state`` ``[N,H,dk,dv]``, the gradient for a zero initial state when
    ``init_state`` is None)."""
    q, k, v, log_alpha, beta, seq_start, n_tok, H, dk, dv = _check(q, k, v, log_alpha, beta, seq_start)
    n_seqs = len(seq_start) - 1
    s0 = None if init_state is None else _f64(init_state)
    d_o = _f64(d_o)
    assert d_o.shape == (n_tok, H, dv)
    dfs = None if d_final_state is None else _f64(d_final_state)
    if dfs is not None:
        assert dfs.shape == (n_seqs, H, dk, dv)
    out = {"dq": np.zeros((n_tok, H, dk)), "dk": np.zeros((n_tok, H, dk)), "dv": np.zeros((n_tok, H, dv)),
           "dlog_alpha": np.zeros((n_tok, H, dk)), "dbeta": np.zeros((n_tok, H)),
           "d_init_state": np.zeros((n_seqs, H, dk, dv))}
    rc = _load().kda_ref_backward_f64(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(s0),
        seq_start.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n_seqs, H, dk, dv, _ptr(d_o), _ptr(dfs),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]), _ptr(out["dbeta"]),
        _ptr(out["d_init_state"]), int(n_threads))
    if rc != 0:
        raise RuntimeError(f"kda_ref_backward_f64 failed ({rc})")
    return out


def decode_step(q, k, v, log_alpha, beta, state, n_threads: int = 0):
    """One recurrent step for N independent sequences (one token each).

    q, k, log_alpha ``[N,H,dk]``, v ``[N,H,dv]``, beta ``[N,H]``, state
    ``[N,H,dk,dv]``.  Returns ``(o [N,H,dv], new_state)``.  This is the token
    recurrence applied to N sequences of length one.
    """
    N = np.asarray(q).shape[0]
    return forward(q, k, v, log_alpha, beta, np.arange(N + 1, dtype=np.int64), init_state=state,
                   n_threads=n_threads)


def seq_start_from(B: int, T: int, cu_seqlens=None) -> np.ndarray:
    """Token offsets of the sequences: ``cu_seqlens`` as given, else B runs of T."""
    if cu_seqlens is not None:
        return np.asarray(cu_seqlens, dtype=np.int64)
    return np.arange(B + 1, dtype=np.int64) * T
