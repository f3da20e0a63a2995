"""Python binding of the KDA C ABI (``include/kda.h``, ``libkda.so``).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI.  PyTorch supplies device memory and streams.  There
is no CPU path: tensors must live on a CUDA device, and a missing or unloadable
``libkda.so`` raises :class:`KdaError`.

Calls:

* :func:`chunk_fwd` -- chunkwise prefill (``kda_chunk_fwd``).
* :func:`decode_step` -- one recurrent step, state updated in place
  (``kda_decode_step``).
* :func:`chunk_bwd` -- gradients of the prefill for training (``kda_chunk_bwd``).

Both take ``prep`` (a bitwise OR of the ``PREP_*`` flags): raw q/k, gate
logits and beta logits are then normalised / activated inside the kernels
(``kda_chunk_fwd_prep``, ``kda_decode_step_prep``).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_BF16, KDA_F32 = 0, 1
ALGOS = {"auto": 0, "simt": 1, "tc": 2}
KDA_ERR_TIMEOUT = -9   # a bounded device-side wait gave up (kda_status in include/kda.h)
_DTYPES = {torch.bfloat16: KDA_BF16, torch.float32: KDA_F32}
# kda_prep flags (include/kda.h)
PREP_NONE, PREP_QK_L2NORM, PREP_GATE_SOFTPLUS, PREP_BETA_SIGMOID = 0, 1, 2, 4
PREP_ALL = PREP_QK_L2NORM | PREP_GATE_SOFTPLUS | PREP_BETA_SIGMOID


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _lib_or_none().kda_status_string(status).decode() if _lib_or_none() else f"status {status}"
        super().__init__(f"{what}: {msg}" if what else msg)


_lock = threading.Lock()
_lib = None


def _declare(lib):
    c_int, c_size, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.kda_status_string.argtypes = [c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_version.restype = c_int
    lib.kda_chunk_fwd_workspace_size.argtypes = [c_int] * 6 + [c_int, i32p, c_int]
    lib.kda_chunk_fwd_workspace_size.restype = c_size
    lib.kda_chunk_fwd_workspace_size_ex.argtypes = [c_int] * 6 + [c_int, i32p, c_int, c_int]
    lib.kda_chunk_fwd_workspace_size_ex.restype = c_size
    lib.kda_chunk_fwd.argtypes = [vp] * 5 + [c_int, vp, i32p, c_int] + [c_int] * 6 + [vp, vp, vp, c_size, vp]
    lib.kda_chunk_fwd.restype = c_int
    lib.kda_chunk_fwd_ex.argtypes = lib.kda_chunk_fwd.argtypes + [c_int]
    lib.kda_chunk_fwd_ex.restype = c_int
    lib.kda_chunk_simt_offsets.argtypes = [c_int] * 6 + [i32p, c_int, ctypes.POINTER(c_size)]
    lib.kda_chunk_simt_offsets.restype = c_int
    lib.kda_decode_step.argtypes = [vp] * 5 + [c_int, vp] + [c_int] * 4 + [vp, vp]
    lib.kda_decode_step.restype = c_int
    lib.kda_chunk_fwd_prep.argtypes = [vp] * 5 + [c_int, ctypes.c_uint, vp, i32p, c_int] + [c_int] * 6 + \
        [vp, vp, vp, c_size, vp]
    lib.kda_chunk_fwd_prep.restype = c_int
    lib.kda_decode_step_prep.argtypes = [vp] * 5 + [c_int, ctypes.c_uint, vp] + [c_int] * 4 + [vp, vp]
    lib.kda_decode_step_prep.restype = c_int
    lib.kda_chunk_bwd_workspace_size.argtypes = [c_int] * 6 + [i32p, c_int]
    lib.kda_chunk_bwd_workspace_size.restype = c_size
    lib.kda_chunk_bwd.argtypes = [vp] * 5 + [c_int, vp, i32p, c_int] + [c_int] * 6 + [vp, vp] + [vp] * 6 + \
        [vp, c_size, vp]
    lib.kda_chunk_bwd.restype = c_int
    lib.kda_set_timing_events.argtypes = [ctypes.POINTER(vp), c_int]
    lib.kda_set_timing_events.restype = c_int
    lib.kda_chunk_fwd_kernels.argtypes = [c_int] * 7 + [i32p, c_int, c_int, ctypes.POINTER(ctypes.c_char_p), c_int]
    lib.kda_chunk_fwd_kernels.restype = c_int
    lib.kda_chunk_fwd_noalloc.argtypes = [vp] * 5 + [c_int, vp, i32p, c_int] + [c_int] * 6 + [vp, vp, vp]
    lib.kda_chunk_fwd_noalloc.restype = c_int
    lib.kda_chunk_fwd_device_status.argtypes = [vp, c_int, i32p, c_int] + [c_int] * 6 + [c_int, vp]
    lib.kda_chunk_fwd_device_status.restype = c_int
    lib.kda_chunk_bwd_device_status.argtypes = [vp, c_int, i32p, c_int] + [c_int] * 6 + [vp]
    lib.kda_chunk_bwd_device_status.restype = c_int
    lib.kda_chunk_fwd_noalloc_device_status.argtypes = [c_int, i32p, c_int] + [c_int] * 6 + [vp]
    lib.kda_chunk_fwd_noalloc_device_status.restype = c_int
    lib.kda_chunk_segment_map.argtypes = [vp] * 5 + [c_int, i32p, c_int] + [c_int] * 6 + [vp, vp, vp, c_size, vp]
    lib.kda_chunk_segment_map.restype = c_int
    lib.kda_compose_states.argtypes = [vp, vp, vp] + [c_int] * 5 + [vp, vp]
    lib.kda_compose_states.restype = c_int
    lib.kda_set_test_wait_limit.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
    lib.kda_set_test_wait_limit.restype = c_int
    lib.kda_chunk_fwd_host_buffer_size.argtypes = [c_int, i32p, c_int] + [c_int] * 5
    lib.kda_chunk_fwd_host_buffer_size.restype = c_size
    lib.kda_chunk_fwd_host.argtypes = [vp] * 5 + [c_int, vp, i32p, c_int] + [c_int] * 4 + [vp, vp, c_int, vp,
                                                                                          c_size, vp]
    lib.kda_chunk_fwd_host.restype = c_int
    lib.kda_chunk_fwd_host_device_status.argtypes = [vp, vp]
    lib.kda_chunk_fwd_host_device_status.restype = c_int
    return lib


def _lib_or_none():
    return _lib


def lib():
    """Load ``libkda.so`` (building it first when it is missing or stale and
    nvcc is present).  Raises :class:`KdaError` when it cannot be loaded."""
    global _lib
    with _lock:
        if _lib is None:
            try:
                from . import build as _build
                if _build._stale():
                    _build.build()
            except Exception as exc:  # noqa: BLE001 - report any build problem
                if not os.path.exists(LIB_PATH):
                    raise KdaError(-8, f"libkda.so missing and could not be built ({exc})") from exc
            try:
                _lib = _declare(ctypes.CDLL(LIB_PATH))
            except OSError as exc:
                raise RuntimeError(f"cannot load {LIB_PATH}: {exc}") from exc
    return _lib


def exported_symbols():
    return ["kda_status_string", "kda_version", "kda_chunk_fwd_workspace_size",
            "kda_chunk_fwd_workspace_size_ex", "kda_chunk_fwd", "kda_chunk_fwd_ex",
            "kda_chunk_simt_offsets", "kda_decode_step", "kda_set_timing_events", "kda_chunk_fwd_kernels",
            "kda_chunk_fwd_noalloc", "kda_chunk_fwd_prep", "kda_decode_step_prep", "kda_chunk_bwd_workspace_size",
            "kda_chunk_bwd", "kda_chunk_fwd_device_status", "kda_chunk_bwd_device_status",
            "kda_chunk_fwd_noalloc_device_status", "kda_chunk_segment_map", "kda_compose_states",
            "kda_set_test_wait_limit", "kda_chunk_fwd_host_buffer_size", "kda_chunk_fwd_host",
            "kda_chunk_fwd_host_device_status"]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cu_arg(cu_seqlens):
    if cu_seqlens is None:
        return None, 0, None
    arr = np.ascontiguousarray(np.asarray(cu_seqlens), dtype=np.int32)
    return arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(arr) - 1, arr


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@contextlib.contextmanager
def _launch_on(device, stream, tensors=()):
    """Run one library call on ``device``: it is made the current device for the
    duration (the library launches on the current device), and the call's stream
    is ``stream`` or that device's current stream.  Every tensor must live on
    ``device``.  Yields ``(stream, allocated)``: tensors the wrapper allocates
    are appended to ``allocated`` and, when the stream is not the device's
    current stream, recorded on it afterwards so that the caching allocator does
    not reuse their memory while the call's kernels may still run."""
    for name, t in tensors:
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, the call runs on {device}")
    with torch.cuda.device(device):
        cur = torch.cuda.current_stream(device)
        s = cur if stream is None else stream
        if s.device != device:
            raise ValueError(f"stream belongs to {s.device}, the call runs on {device}")
        allocated = []
        yield s, allocated
        if s != cur:
            for t in allocated:
                if t is not None:
                    t.record_stream(s)


def _check_cuda(name, t, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def workspace_size(B, T, H, dk, dv, C, dtype, cu_seqlens=None, algo="auto") -> int:
    cu, n, _keep = _cu_arg(cu_seqlens)
    d = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return int(lib().kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv, C, d, cu, n, ALGOS[algo]))


def simt_offsets(B, T, H, dk, dv, C, cu_seqlens=None):
    cu, n, _keep = _cu_arg(cu_seqlens)
    out = (ctypes.c_size_t * 5)()
    st = lib().kda_chunk_simt_offsets(B, T, H, dk, dv, C, cu, n, out)
    if st != 0:
        raise KdaError(st, "kda_chunk_simt_offsets")
    return [int(x) for x in out]


def chunk_kernels(B, T, H, dk, dv, C, dtype, cu_seqlens=None, algo="auto"):
    """Names of the kernels one chunk_fwd call launches, in launch order."""
    cu, n, _keep = _cu_arg(cu_seqlens)
    d = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    names = (ctypes.c_char_p * 32)()
    cnt = lib().kda_chunk_fwd_kernels(B, T, H, dk, dv, C, d, cu, n, ALGOS[algo], names, 32)
    if cnt < 0:
        raise KdaError(cnt, "kda_chunk_fwd_kernels")
    return [names[i].decode() for i in range(cnt)]


def set_test_wait_limit(kernels: int, limit_ns: int):
    """Failure-path test hook (``kda_set_test_wait_limit``): the next
    tensor-core prefill from this thread makes a bounded wait expire in the
    first CTA of the chosen kernels (bit 0 tc_intra, bit 1 tc_recur) and records
    KDA_ERR_TIMEOUT; 0 disarms."""
    st = lib().kda_set_test_wait_limit(int(kernels), int(limit_ns))
    if st != 0:
        raise KdaError(st, "kda_set_test_wait_limit")


def set_timing_events(events):
    """Per-kernel timing hook for the next chunk_fwd on this thread: a list of
    torch.cuda.Event (recorded before the first kernel and after each kernel).
    Each event must already exist (torch creates it on its first record)."""
    if any(e.cuda_event == 0 for e in events):
        raise ValueError("record every event once before handing it to the timing hook")
    arr = (ctypes.c_void_p * max(1, len(events)))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    st = lib().kda_set_timing_events(arr, len(events))
    if st != 0:
        raise KdaError(st, "kda_set_timing_events")


def chunk_fwd(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, C: int = 64,
              output_final_state: bool = True, o=None, final_state=None, workspace=None,
              algo: str = "auto", stream=None, prep: int = 0):
    """Chunkwise KDA prefill.

    q, k, log_alpha ``[B, T, H, dk]``; v ``[B, T, H, dv]``; beta ``[B, T, H]``;
    all one dtype (bf16 or fp32), contiguous, on one CUDA device.  ``cu_seqlens``
    (host sequence, N + 1 offsets) selects packed varlen mode with B = 1.
    ``init_state`` ``[N, H, dk, dv]`` fp32 or None.  Returns ``(o, final_state)``
    (final_state is None when ``output_final_state`` is False).  ``prep`` != 0
    calls ``kda_chunk_fwd_prep`` (tensor-core shapes only; ``algo`` must be
    "auto" or "tc"): log_alpha then holds gate logits and beta beta logits when
    the matching flag is set.
    """
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        _check_cuda(name, t, dt)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu, n_seqs, _keep = _cu_arg(cu_seqlens)
    N = n_seqs if cu_seqlens is not None else B
    _check_cuda("init_state", init_state, torch.float32)
    if prep and algo not in ("auto", "tc"):
        raise ValueError("prep is fused into the tensor-core path only")
    dev = q.device
    with _launch_on(dev, stream, (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta),
                                  ("init_state", init_state), ("o", o), ("final_state", final_state),
                                  ("workspace", workspace))) as (s, allocated):
        if o is None:
            o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
            allocated.append(o)
        if final_state is None and output_final_state:
            final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
            allocated.append(final_state)
        _check_cuda("o", o, dt)
        _check_cuda("final_state", final_state, torch.float32)
        need = lib().kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv, C, _DTYPES[dt], cu, n_seqs, ALGOS[algo])
        if workspace is None:
            workspace = torch.empty(max(int(need), 256), dtype=torch.uint8, device=dev)
            allocated.append(workspace)
        _check_cuda("workspace", workspace)
        wsb = workspace.numel() * workspace.element_size()
        if prep:
            st = lib().kda_chunk_fwd_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                          prep, _ptr(init_state), cu, n_seqs, B, T, H, dk, dv, C, _ptr(o),
                                          _ptr(final_state), _ptr(workspace), wsb, _stream_handle(s))
            what = "kda_chunk_fwd_prep"
        else:
            st = lib().kda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                        _ptr(init_state), cu, n_seqs, B, T, H, dk, dv, C, _ptr(o),
                                        _ptr(final_state), _ptr(workspace), wsb, _stream_handle(s), ALGOS[algo])
            what = "kda_chunk_fwd"
    if st != 0:
        raise KdaError(st, what)
    return o, final_state


def host_buffer_size(cu_seqlens, H, dk, dv, C: int = 64, dtype=torch.bfloat16, n_groups: int = 8) -> int:
    """Device bytes chunk_fwd_host needs for this batch (kda_chunk_fwd_host_buffer_size)."""
    cu, n, _keep = _cu_arg(cu_seqlens)
    return int(lib().kda_chunk_fwd_host_buffer_size(_DTYPES[dtype], cu, n, H, dk, dv, C, n_groups))


def _check_host(name, t, dtype=None):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def chunk_fwd_host(q, k, v, log_alpha, beta, cu_seqlens, init_state=None, C: int = 64, o=None,
                   final_state=None, output_final_state: bool = True, n_groups: int = 8, device_buffer=None,
                   device=None, stream=None, synchronize: bool = True):
    """Prefill of a packed batch held in host memory (``kda_chunk_fwd_host``):
    the library copies group after group of sequences to the device, computes
    them and copies the results back, with the copies of neighbouring groups
    overlapping the computation.

    q, k, log_alpha ``[1, T, H, dk]``, v ``[1, T, H, dv]``, beta ``[1, T, H]``:
    CPU tensors of one dtype (page-locked for the copies to overlap);
    ``cu_seqlens`` host offsets (N + 1); ``init_state`` CPU ``[N, H, dk, dv]``
    fp32 or None.  Returns CPU ``(o, final_state)``.  With ``synchronize`` the
    call waits for the stream, so the results are ready; without it the caller
    must keep every tensor alive and wait for ``stream`` before reading them.
    """
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        _check_host(name, t, dt)
    if cu_seqlens is None:
        raise ValueError("chunk_fwd_host takes a packed batch: cu_seqlens is required")
    _, T, H, dk = q.shape
    dv = v.shape[-1]
    cu, n_seqs, _keep = _cu_arg(cu_seqlens)
    _check_host("init_state", init_state, torch.float32)
    if o is None:
        o = torch.empty((1, T, H, dv), dtype=dt).pin_memory()
    if final_state is None and output_final_state:
        final_state = torch.empty((n_seqs, H, dk, dv), dtype=torch.float32).pin_memory()
    _check_host("o", o, dt)
    _check_host("final_state", final_state, torch.float32)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _launch_on(dev, stream, (("device_buffer", device_buffer),)) as (s, allocated):
        need = lib().kda_chunk_fwd_host_buffer_size(_DTYPES[dt], cu, n_seqs, H, dk, dv, C, n_groups)
        if device_buffer is None:
            device_buffer = torch.empty(max(int(need), 256), dtype=torch.uint8, device=dev)
            allocated.append(device_buffer)
        _check_cuda("device_buffer", device_buffer)
        st = lib().kda_chunk_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), log_alpha.data_ptr(),
                                      beta.data_ptr(), _DTYPES[dt],
                                      init_state.data_ptr() if init_state is not None else None, cu, n_seqs, H,
                                      dk, dv, C, o.data_ptr(), final_state.data_ptr() if final_state is not None
                                      else None, int(n_groups), _ptr(device_buffer),
                                      device_buffer.numel() * device_buffer.element_size(), _stream_handle(s))
        if st == 0 and synchronize:
            s.synchronize()
    if st != 0:
        raise KdaError(st, "kda_chunk_fwd_host")
    return o, final_state


def host_device_status(device_buffer, stream=None) -> int:
    """kda_chunk_fwd_host_device_status: 0, or the error a bounded device wait
    recorded during the last chunk_fwd_host call that used ``device_buffer``."""
    with _launch_on(device_buffer.device, stream, ()) as (s, _allocated):
        return int(lib().kda_chunk_fwd_host_device_status(_ptr(device_buffer), _stream_handle(s)))


# kernels of one kda_chunk_bwd call: the recompute (bf16 with d = 128: k1 and the tensor-core
# forward with its states, T and the key products stored; otherwise the CUDA-core k1-k3),
# then the gradient kernels (bf16 with d = 128: all four on the tensor cores)
BWD_KERNELS_TC = ["k1_cumsum", "tc_intra", "tc_recur", "kb_chain_tc", "kb_a_tc", "kb_b_tc", "kb_c_tc"]
BWD_KERNELS = ["k1_cumsum", "k2_wy", "k3_state", "kb_p", "kb_chain", "kb_a", "kb_b", "kb_c"]
# the timing hook's marks of kda_chunk_bwd: start, recompute, kb_p, kb_chain, kb_a, kb_b, kb_c
BWD_TIMED = ["recompute", "kb_p", "kb_chain", "kb_a", "kb_b", "kb_c"]
# the same marks on the tensor-core path, where nothing runs between the second and third
# (None): the recompute already stored the key products and the chain reads P from its images
BWD_TIMED_TC = ["recompute", None, "kb_chain_tc", "kb_a_tc", "kb_b_tc", "kb_c_tc"]


def _bwd_tc(dtype, dk, dv) -> bool:
    return dtype == torch.bfloat16 and dk == 128 and dv == 128


def bwd_kernels(dtype, dk, dv):
    """The kernels one kda_chunk_bwd call launches for this problem."""
    return BWD_KERNELS_TC if _bwd_tc(dtype, dk, dv) else BWD_KERNELS


def bwd_timed(dtype, dk, dv):
    """Labels of the intervals between kda_chunk_bwd's timing marks for this problem
    (None where no kernel runs in the interval)."""
    return BWD_TIMED_TC if _bwd_tc(dtype, dk, dv) else BWD_TIMED


def bwd_workspace_size(B, T, H, dk, dv, C=64, cu_seqlens=None) -> int:
    cu, n, _keep = _cu_arg(cu_seqlens)
    return int(lib().kda_chunk_bwd_workspace_size(B, T, H, dk, dv, C, cu, n))


def chunk_bwd(q, k, v, log_alpha, beta, d_o, init_state=None, d_final_state=None, cu_seqlens=None, C: int = 64,
              need_d_init_state: bool = True, grads=None, workspace=None, stream=None):
    """Gradients of ``sum(d_o * o) + sum(d_final_state * final_state)`` for the
    prefill :func:`chunk_fwd` computes from the same inputs.  Returns
    ``(dq, dk, dv, dlog_alpha, dbeta, d_init_state)`` (the first five in the
    input dtype, ``d_init_state`` fp32 ``[N, H, dk, dv]`` or None).  ``grads``
    may pass preallocated output tensors in that order."""
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta), ("d_o", d_o)):
        _check_cuda(name, t, dt)
    _check_cuda("init_state", init_state, torch.float32)
    _check_cuda("d_final_state", d_final_state, torch.float32)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu, n_seqs, _keep = _cu_arg(cu_seqlens)
    N = n_seqs if cu_seqlens is not None else B
    dev = q.device
    given = () if grads is None else tuple((f"grads[{i}]", t) for i, t in enumerate(grads))
    with _launch_on(dev, stream, (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta), ("d_o", d_o),
                                  ("init_state", init_state), ("d_final_state", d_final_state),
                                  ("workspace", workspace)) + given) as (s, allocated):
        if grads is None:
            grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(log_alpha),
                     torch.empty_like(beta),
                     torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) if need_d_init_state else None)
            allocated.extend(grads)
        dq, dk_, dv_, dla, dbeta, dinit = grads
        for name, t in (("dq", dq), ("dk", dk_), ("dv", dv_), ("dlog_alpha", dla), ("dbeta", dbeta)):
            _check_cuda(name, t, dt)
        _check_cuda("d_init_state", dinit, torch.float32)
        need = lib().kda_chunk_bwd_workspace_size(B, T, H, dk, dv, C, cu, n_seqs)
        if workspace is None:
            workspace = torch.empty(max(int(need), 256), dtype=torch.uint8, device=dev)
            allocated.append(workspace)
        _check_cuda("workspace", workspace)
        st = lib().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                 _ptr(init_state), cu, n_seqs, B, T, H, dk, dv, C, _ptr(d_o), _ptr(d_final_state),
                                 _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dla), _ptr(dbeta), _ptr(dinit),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(s))
    if st != 0:
        raise KdaError(st, "kda_chunk_bwd")
    return dq, dk_, dv_, dla, dbeta, dinit


def device_status(kind, workspace, dtype, B, T, H, dk, dv, C=64, cu_seqlens=None, algo="auto", stream=None,
                  device=None):
    """Synchronise ``stream`` and return the device-side status (0 or
    KDA_ERR_TIMEOUT) of the last call of ``kind`` ("fwd", "bwd" or "noalloc")
    that used ``workspace`` (ignored for "noalloc") with these sizes.  The
    query runs on the workspace's device (for "noalloc": ``device``, default the
    current device).  Raises KdaError for invalid arguments or a failed copy."""
    cu, n, _keep = _cu_arg(cu_seqlens)
    d = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    if kind not in ("fwd", "bwd", "noalloc"):
        raise ValueError(f"unknown kind {kind!r}")
    if workspace is not None:
        dev = workspace.device
    else:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with _launch_on(dev, stream) as (s, _):
        h = _stream_handle(s)
        if kind == "fwd":
            st = lib().kda_chunk_fwd_device_status(_ptr(workspace), d, cu, n, B, T, H, dk, dv, C, ALGOS[algo], h)
        elif kind == "bwd":
            st = lib().kda_chunk_bwd_device_status(_ptr(workspace), d, cu, n, B, T, H, dk, dv, C, h)
        else:
            st = lib().kda_chunk_fwd_noalloc_device_status(d, cu, n, B, T, H, dk, dv, C, h)
    if st not in (0, KDA_ERR_TIMEOUT):
        raise KdaError(st, f"device status ({kind})")
    return int(st)


def segment_map(q, k, v, log_alpha, beta, cu_seqlens=None, C: int = 64, M=None, F=None, workspace=None,
                stream=None):
    """Affine map of a segment (``kda_chunk_segment_map``): for every sequence
    and head, the segment takes a start state S to ``M S + F``.  Inputs as
    :func:`chunk_fwd`.  Returns ``(M [N, H, dk, dk], F [N, H, dk, dv])`` fp32."""
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        _check_cuda(name, t, dt)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu, n_seqs, _keep = _cu_arg(cu_seqlens)
    N = n_seqs if cu_seqlens is not None else B
    dev = q.device
    with _launch_on(dev, stream, (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta), ("M", M),
                                  ("F", F), ("workspace", workspace))) as (s, allocated):
        if M is None:
            M = torch.empty((N, H, dk, dk), dtype=torch.float32, device=dev)
            allocated.append(M)
        if F is None:
            F = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
            allocated.append(F)
        _check_cuda("M", M, torch.float32)
        _check_cuda("F", F, torch.float32)
        need = lib().kda_chunk_fwd_workspace_size(B, T, H, dk, dv, C, _DTYPES[dt], cu, n_seqs)
        if workspace is None:
            workspace = torch.empty(max(int(need), 256), dtype=torch.uint8, device=dev)
            allocated.append(workspace)
        _check_cuda("workspace", workspace)
        st = lib().kda_chunk_segment_map(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt], cu,
                                         n_seqs, B, T, H, dk, dv, C, _ptr(M), _ptr(F), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream_handle(s))
    if st != 0:
        raise KdaError(st, "kda_chunk_segment_map")
    return M, F


def compose_states(M, F, init_state=None, out=None, stream=None):
    """Start states of consecutive segments (``kda_compose_states``): ``M``
    ``[R, N, H, dk, dk]`` and ``F`` ``[R, N, H, dk, dv]`` (the segments' maps, in
    order), ``init_state`` ``[N, H, dk, dv]`` or None.  Returns ``[R + 1, N, H,
    dk, dv]``: entry r is the state segment r starts from, the last one the
    state after all R segments."""
    R, N, H, dk, _ = M.shape
    dv = F.shape[-1]
    for name, t in (("M", M), ("F", F), ("init_state", init_state)):
        _check_cuda(name, t, torch.float32)
    dev = M.device
    with _launch_on(dev, stream, (("F", F), ("init_state", init_state), ("out", out))) as (s, allocated):
        if out is None:
            out = torch.empty((R + 1, N, H, dk, dv), dtype=torch.float32, device=dev)
            allocated.append(out)
        _check_cuda("out", out, torch.float32)
        st = lib().kda_compose_states(_ptr(M), _ptr(F), _ptr(init_state), R, N, H, dk, dv, _ptr(out),
                                      _stream_handle(s))
    if st != 0:
        raise KdaError(st, "kda_compose_states")
    return out


NOALLOC_SCRATCH_BYTES = 64 << 20   # KDA_NOALLOC_SCRATCH_BYTES in include/kda.h


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, C: int = 64,
                      o=None, final_state=None, stream=None):
    """Prefill through ``kda_chunk_fwd_noalloc``: no workspace argument, the
    library's own fixed device scratch is used (for callers that cannot
    allocate).  Problems needing more than NOALLOC_SCRATCH_BYTES of scratch
    raise KdaError (KDA_ERR_SCRATCH).  Calls that overlap on the GPU share the
    scratch and must be serialised."""
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        _check_cuda(name, t, dt)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cu, n_seqs, _keep = _cu_arg(cu_seqlens)
    N = n_seqs if cu_seqlens is not None else B
    _check_cuda("init_state", init_state, torch.float32)
    dev = q.device
    with _launch_on(dev, stream, (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta),
                                  ("init_state", init_state), ("o", o), ("final_state", final_state))) \
            as (s, allocated):
        if o is None:
            o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
            allocated.append(o)
        if final_state is None:
            final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
            allocated.append(final_state)
        _check_cuda("o", o, dt)
        _check_cuda("final_state", final_state, torch.float32)
        st = lib().kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                         _ptr(init_state), cu, n_seqs, B, T, H, dk, dv, C, _ptr(o),
                                         _ptr(final_state), _stream_handle(s))
    if st != 0:
        raise KdaError(st, "kda_chunk_fwd_noalloc")
    return o, final_state


def decode_step(q, k, v, log_alpha, beta, state, o=None, stream=None, prep: int = 0):
    """One KDA decode step for N sequences; ``state`` ``[N, H, dk, dv]`` fp32 is
    updated in place.  q, k, log_alpha ``[N, H, dk]``, v ``[N, H, dv]``, beta
    ``[N, H]``.  Returns o ``[N, H, dv]``.  ``prep`` != 0 calls
    ``kda_decode_step_prep`` (raw inputs normalised / activated in the kernel)."""
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        _check_cuda(name, t, dt)
    _check_cuda("state", state, torch.float32)
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    with _launch_on(dev, stream, (("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta),
                                  ("state", state), ("o", o))) as (s, allocated):
        if o is None:
            o = torch.empty((N, H, dv), dtype=dt, device=dev)
            allocated.append(o)
        _check_cuda("o", o, dt)
        if prep:
            st = lib().kda_decode_step_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                            prep, _ptr(state), N, H, dk, dv, _ptr(o), _stream_handle(s))
            what = "kda_decode_step_prep"
        else:
            st = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _DTYPES[dt],
                                       _ptr(state), N, H, dk, dv, _ptr(o), _stream_handle(s))
            what = "kda_decode_step"
    if st != 0:
        raise KdaError(st, what)
    return o
