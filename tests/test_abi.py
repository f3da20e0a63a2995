"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects invalid arguments on the host before launching."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_30_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, E_NULL, E_SHAPE, E_DTYPE, E_ALIGN, E_CHUNK, E_SEQ, E_WS = 0, -1, -2, -3, -4, -5, -6, -7


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]*?\b(kda_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = header_functions()
    assert "kda_chunk_fwd" in names and "kda_decode_step" in names
    assert set(names) == set(kda.exported_symbols())


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(kda.lib()._name)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    lib = kda.lib()
    for code in range(-11, 1):
        s = lib.kda_status_string(code).decode()
        assert s.startswith("KDA")
    assert "unknown" in lib.kda_status_string(-99).decode()
    assert lib.kda_version() >= 100


def _ws(B=1, T=256, H=2, dk=64, dv=64, C=64, dtype=1, cu=None, algo="auto"):
    return kda.workspace_size(B, T, H, dk, dv, C, dtype, cu_seqlens=cu, algo=algo)


def test_workspace_size_queries():
    assert _ws() > 0
    assert _ws(C=32) == 0
    assert _ws(dk=96) == 0
    assert _ws(dtype=7) == 0
    assert _ws(B=1, T=10, cu=[0, 4, 10]) > 0
    assert _ws(B=2, T=10, cu=[0, 4, 10]) == 0          # varlen needs B = 1
    assert _ws(B=1, T=10, cu=[0, 6, 4, 10]) == 0       # decreasing
    assert _ws(B=1, T=10, cu=[1, 4, 10]) == 0          # does not start at 0
    assert _ws(B=1, T=10, cu=[0, 4, 9]) == 0           # does not end at T
    assert _ws(T=0) > 0                                # empty problem is valid
    # SIMT workspace holds g, U, Wk, W and the chunk start states
    B, T, H, d, C = 2, 200, 3, 64, 64
    n_chunks = B * ((T + C - 1) // C)
    need = B * T * H * d * 4 * 4 + n_chunks * H * d * d * 4
    assert _ws(B=B, T=T, H=H, dk=d, dv=d, C=C, dtype=1, algo="simt") >= need


def test_tensor_core_path_serves_both_chunk_sizes_with_64_token_chunks():
    # bf16, d = 128: the tensor-core workspace for C = 128 is the one for C = 64
    for cu in (None, [0, 100, 300, 301]):
        B, T = (2, 300) if cu is None else (1, 301)
        w64 = _ws(B=B, T=T, H=3, dk=128, dv=128, C=64, dtype=0, cu=cu, algo="tc")
        w128 = _ws(B=B, T=T, H=3, dk=128, dv=128, C=128, dtype=0, cu=cu, algo="tc")
        assert w64 > 0 and w64 == w128
    # the CUDA-core path keeps the chunk size it is given
    assert _ws(B=2, T=300, H=3, dk=128, dv=128, C=64, dtype=0, algo="simt") != \
        _ws(B=2, T=300, H=3, dk=128, dv=128, C=128, dtype=0, algo="simt")


def test_packed_batches_launch_the_table_writes_first():
    """A packed batch starts with the sequence-table write and the per-chunk table
    (one 16-byte entry per chunk in the workspace); an equal-length batch has
    neither."""
    import torch
    H, d = 3, 128
    cu = [0, 100, 300, 301, 301, 365]          # an empty sequence included
    for algo, first in (("tc", "tc_intra"), ("simt", "k1_cumsum")):
        names = kda.chunk_kernels(1, 365, H, d, d, 64, torch.bfloat16, cu_seqlens=cu, algo=algo)
        assert names[:3] == ["seq_table_write", "chunk_table_fill", first], names
        names = kda.chunk_kernels(2, 365, H, d, d, 64, torch.bfloat16, algo=algo)
        assert names[0] == first and "chunk_table_fill" not in names, names
    # the two sequence tables (16 bytes per sequence each) and the chunk table sit
    # ahead of the scratch: one more 64-token chunk adds its 16-byte entry besides
    # the scratch it needs
    w = _ws(B=1, T=365, H=H, dk=d, dv=d, C=64, dtype=0, cu=cu, algo="tc")
    w_more = _ws(B=1, T=429, H=H, dk=d, dv=d, C=64, dtype=0, cu=cu[:-1] + [365, 429], algo="tc")
    w_eq = _ws(B=1, T=365, H=H, dk=d, dv=d, C=64, dtype=0, algo="tc")
    assert w > w_eq and w_more > w


def test_simt_offsets_are_disjoint_and_ordered():
    off = kda.simt_offsets(2, 200, 3, 64, 64, 64)
    assert off == sorted(off) and len(set(off)) == 5
    assert all(o % 256 == 0 for o in off)


def _call(**kw):
    """kda_chunk_fwd_ex with fake (never dereferenced) device pointers."""
    lib = kda.lib()
    a = dict(q=0x10000, k=0x20000, v=0x30000, la=0x40000, beta=0x50000, dtype=1, s0=None, cu=None, n=0,
             B=1, T=256, H=2, dk=64, dv=64, C=64, o=0x60000, fs=None, ws=0x100000, wsb=1 << 40, algo=0)
    a.update(kw)
    cu = None
    keep = None
    if a["cu"] is not None:
        keep = (ctypes.c_int32 * len(a["cu"]))(*a["cu"])
        cu = ctypes.cast(keep, ctypes.POINTER(ctypes.c_int32))
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.kda_chunk_fwd_ex(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]), vp(a["beta"]), a["dtype"],
                                vp(a["s0"]), cu, a["n"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["C"],
                                vp(a["o"]), vp(a["fs"]), vp(a["ws"]), a["wsb"], None, a["algo"])


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=5), E_DTYPE),
    (dict(C=32), E_CHUNK),
    (dict(dk=96), E_SHAPE),
    (dict(H=0), E_SHAPE),
    (dict(q=None), E_NULL),
    (dict(o=None), E_NULL),
    (dict(ws=None), E_WS),
    (dict(wsb=16), E_WS),
    (dict(k=0x20004), E_ALIGN),
    (dict(ws=0x100010), E_ALIGN),
    (dict(cu=[0, 100, 50, 256], n=3), E_SEQ),
    (dict(cu=[0, 100, 200], n=2), E_SEQ),
    (dict(cu=[0, 256], n=1, B=2), E_SEQ),
    (dict(algo=2, dtype=1), E_SHAPE),          # tensor-core path is bf16 only
    (dict(algo=9), E_SHAPE),
])
def test_chunk_fwd_rejects_before_launch(kw, code):
    assert _call(**kw) == code


def test_decode_rejects_before_launch():
    lib = kda.lib()
    vp = ctypes.c_void_p
    args = [vp(0x10000)] * 5
    assert lib.kda_decode_step(*args, 3, vp(0x70000), 4, 2, 64, 64, vp(0x80000), None) == E_DTYPE
    assert lib.kda_decode_step(*args, 0, vp(0x70000), 4, 2, 96, 64, vp(0x80000), None) == E_SHAPE
    assert lib.kda_decode_step(*args, 0, None, 4, 2, 64, 64, vp(0x80000), None) == E_NULL
    assert lib.kda_decode_step(*args, 0, vp(0x70004), 4, 2, 64, 64, vp(0x80000), None) == E_ALIGN
    assert lib.kda_decode_step(*args, 0, vp(0x70000), 0, 2, 64, 64, vp(0x80000), None) == OK   # N = 0: no work


def _call_prep(prep, dtype=0, dk=128, dv=128, C=64, ws=0x100000):
    lib = kda.lib()
    vp = ctypes.c_void_p
    return lib.kda_chunk_fwd_prep(vp(0x10000), vp(0x20000), vp(0x30000), vp(0x40000), vp(0x50000), dtype, prep,
                                  None, None, 0, 1, 256, 2, dk, dv, C, vp(0x60000), None, vp(ws), 1 << 40, None)


def test_prep_entry_points_reject_before_launch():
    assert _call_prep(8) == E_SHAPE                       # unknown flag
    assert _call_prep(1 << 31) == E_SHAPE
    assert _call_prep(7, dtype=1) == E_SHAPE              # fp32: not the tensor-core path
    assert _call_prep(1, dk=64, dv=64) == E_SHAPE         # d = 64: not the tensor-core path
    assert _call_prep(7, dtype=5) == E_DTYPE
    assert _call_prep(7, C=32) == E_CHUNK
    assert _call_prep(7, ws=0) == E_WS
    assert _call_prep(7, ws=0x100010) == E_ALIGN
    lib = kda.lib()
    vp = ctypes.c_void_p
    args = [vp(0x10000)] * 5
    assert lib.kda_decode_step_prep(*args, 0, 8, vp(0x70000), 4, 2, 64, 64, vp(0x80000), None) == E_SHAPE
    assert lib.kda_decode_step_prep(*args, 3, 7, vp(0x70000), 4, 2, 64, 64, vp(0x80000), None) == E_DTYPE
    assert lib.kda_decode_step_prep(*args, 0, 7, None, 4, 2, 64, 64, vp(0x80000), None) == E_NULL
    assert lib.kda_decode_step_prep(*args, 1, 7, vp(0x70000), 0, 2, 64, 64, vp(0x80000), None) == OK   # N = 0


def test_prep_flags_match_the_header():
    text = open(HEADER).read()
    for name, val in (("KDA_PREP_NONE", kda.PREP_NONE), ("KDA_PREP_QK_L2NORM", kda.PREP_QK_L2NORM),
                      ("KDA_PREP_GATE_SOFTPLUS", kda.PREP_GATE_SOFTPLUS),
                      ("KDA_PREP_BETA_SIGMOID", kda.PREP_BETA_SIGMOID)):
        assert re.search(rf"{name}\s*=\s*{val}\b", text), name
    import oracle.prep as op
    assert (op.QK_L2NORM, op.GATE_SOFTPLUS, op.BETA_SIGMOID) == (kda.PREP_QK_L2NORM, kda.PREP_GATE_SOFTPLUS,
                                                                 kda.PREP_BETA_SIGMOID)


def _call_bwd(**kw):
    """kda_chunk_bwd with fake (never dereferenced) device pointers."""
    lib = kda.lib()
    a = dict(q=0x10000, k=0x20000, v=0x30000, la=0x40000, beta=0x50000, dtype=1, s0=None, cu=None, n=0,
             B=1, T=256, H=2, dk=64, dv=64, C=64, do=0x60000, dfs=None, dq=0x70000, dk_=0x80000, dv_=0x90000,
             dla=0xa0000, db=0xb0000, ds0=None, ws=0x100000, wsb=1 << 40)
    a.update(kw)
    cu = None
    keep = None
    if a["cu"] is not None:
        keep = (ctypes.c_int32 * len(a["cu"]))(*a["cu"])
        cu = ctypes.cast(keep, ctypes.POINTER(ctypes.c_int32))
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.kda_chunk_bwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["la"]), vp(a["beta"]), a["dtype"],
                             vp(a["s0"]), cu, a["n"], a["B"], a["T"], a["H"], a["dk"], a["dv"], a["C"], vp(a["do"]),
                             vp(a["dfs"]), vp(a["dq"]), vp(a["dk_"]), vp(a["dv_"]), vp(a["dla"]), vp(a["db"]),
                             vp(a["ds0"]), vp(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=5), E_DTYPE),
    (dict(C=32), E_CHUNK),
    (dict(dk=96), E_SHAPE),
    (dict(H=0), E_SHAPE),
    (dict(do=None), E_NULL),
    (dict(dla=None), E_NULL),
    (dict(db=None), E_NULL),
    (dict(ws=None), E_WS),
    (dict(wsb=16), E_WS),
    (dict(dq=0x70004), E_ALIGN),
    (dict(ds0=0x110008), E_ALIGN),
    (dict(ws=0x100010), E_ALIGN),
    (dict(cu=[0, 100, 50, 256], n=3), E_SEQ),
])
def test_chunk_bwd_rejects_before_launch(kw, code):
    assert _call_bwd(**kw) == code


def test_bwd_workspace_size():
    B, T, H, d = 2, 200, 3, 64
    w = kda.bwd_workspace_size(B, T, H, d, d, 64)
    assert w > kda.workspace_size(B, T, H, d, d, 64, 1, algo="simt")   # holds the CUDA-core forward's scratch
    assert w == kda.bwd_workspace_size(B, T, H, d, d, 128)           # 64-token chunks either way
    assert kda.bwd_workspace_size(B, T, H, d, d, 32) == 0
    assert kda.bwd_workspace_size(1, 10, H, d, d, 64, cu_seqlens=[0, 4, 10]) > 0
    assert kda.bwd_workspace_size(1, 10, H, d, d, 64, cu_seqlens=[0, 6, 4, 10]) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        kda.chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))


def _status_fwd(ws=0x100000, dtype=1, cu=None, B=1, T=256, H=2, dk=64, dv=64, C=64, algo=0):
    lib = kda.lib()
    cu_p, n, _keep = kda._cu_arg(cu)
    return lib.kda_chunk_fwd_device_status(None if ws is None else ctypes.c_void_p(ws), dtype, cu_p, n, B, T, H,
                                           dk, dv, C, algo, None)


def _status_bwd(ws=0x100000, dtype=1, cu=None, B=1, T=256, H=2, dk=64, dv=64, C=64):
    lib = kda.lib()
    cu_p, n, _keep = kda._cu_arg(cu)
    return lib.kda_chunk_bwd_device_status(None if ws is None else ctypes.c_void_p(ws), dtype, cu_p, n, B, T, H,
                                           dk, dv, C, None)


def test_device_status_validates_on_the_host():
    # invalid arguments are rejected before anything touches the device
    assert _status_fwd(ws=None) == E_NULL
    assert _status_fwd(dtype=5) == E_DTYPE
    assert _status_fwd(algo=9) == E_SHAPE
    assert _status_fwd(dk=96) == E_SHAPE
    assert _status_fwd(cu=[0, 100, 50, 256]) == E_SEQ
    assert _status_bwd(ws=None) == E_NULL
    assert _status_bwd(C=32) == E_CHUNK
    assert _status_bwd(dtype=5) == E_DTYPE
    # the CUDA-core path never waits on the device: OK without reading the (fake) workspace
    assert _status_fwd(dk=64, dv=64) == OK
    assert _status_fwd(dk=128, dv=128, algo=kda.ALGOS["simt"]) == OK
    assert _status_bwd(dk=64, dv=64, dtype=1) == OK
    # zero sequences launch nothing, on either path
    assert _status_bwd(dtype=0, dk=128, dv=128, B=0) == OK
    assert _status_fwd(dtype=0, dk=128, dv=128, B=0) == OK


def test_test_wait_limit_arguments():
    """kda_set_test_wait_limit checks its arguments on the host and disarms with 0."""
    lib = kda.lib()
    assert lib.kda_set_test_wait_limit(4, 1000) == E_SHAPE          # unknown kernel bit
    assert lib.kda_set_test_wait_limit(1, 0) == E_SHAPE             # zero limit
    assert lib.kda_set_test_wait_limit(2, 2_000_000_000) == E_SHAPE  # above one second
    assert lib.kda_set_test_wait_limit(3, 1000) == OK
    assert lib.kda_set_test_wait_limit(0, 0) == OK                  # disarm


def _host_call(cu=(0, 100, 300, 700), n_groups=3, buf=0x100000, bufb=1 << 40, dtype=0, H=2, dk=128, dv=128):
    lib = kda.lib()
    vp = ctypes.c_void_p
    cua = None if cu is None else (ctypes.c_int32 * len(cu))(*cu)
    n = 0 if cu is None else len(cu) - 1
    args = [vp(0x10000)] * 5
    return lib.kda_chunk_fwd_host(*args, dtype, None, cua, n, H, dk, dv, 64, vp(0x20000), None, n_groups,
                                  None if buf is None else vp(buf), bufb, None)


def test_host_pipeline_buffer_size_and_rejections():
    """kda_chunk_fwd_host_buffer_size / kda_chunk_fwd_host check their arguments on
    the host: the buffer holds at least one workspace for the largest group and two
    staging slots, and shrinks as the batch is cut into more groups."""
    lib = kda.lib()
    cu = [0, 1000, 2000, 3000, 4000, 5000, 6000, 7000, 8000]
    cua = (ctypes.c_int32 * len(cu))(*cu)
    H, d = 4, 128
    one = lib.kda_chunk_fwd_host_buffer_size(0, cua, 8, H, d, d, 64, 1)
    four = lib.kda_chunk_fwd_host_buffer_size(0, cua, 8, H, d, d, 64, 4)
    eight = lib.kda_chunk_fwd_host_buffer_size(0, cua, 8, H, d, d, 64, 8)
    whole = lib.kda_chunk_fwd_workspace_size(1, 8000, H, d, d, 64, 0, cua, 8)
    io = 8000 * H * d * 2 * 5 + 8000 * H * 2 + 2 * 8 * H * d * d * 4   # q k log_alpha v o, beta, states
    assert one >= whole + 2 * io
    assert one > four > eight > 0
    assert lib.kda_chunk_fwd_host_buffer_size(0, None, 8, H, d, d, 64, 4) == 0
    assert lib.kda_chunk_fwd_host_buffer_size(0, cua, 8, H, d, d, 64, 0) == 0
    assert lib.kda_chunk_fwd_host_buffer_size(5, cua, 8, H, d, d, 64, 4) == 0
    # rejections before anything touches a device
    assert _host_call(cu=None) == E_SEQ
    assert _host_call(cu=(0, 100, 50)) == E_SEQ
    assert _host_call(n_groups=0) == E_SHAPE
    assert _host_call(dtype=5) == E_DTYPE
    assert _host_call(buf=None) == E_WS
    assert _host_call(bufb=1024) == E_WS
    assert _host_call(buf=0x100010) == E_ALIGN
    assert lib.kda_chunk_fwd_host_device_status(None, None) == E_NULL
