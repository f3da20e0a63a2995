"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bar: max |got - ref| / rms(ref) <= 2e-2 for bf16 inputs and <= 1e-4 for fp32
inputs, on o and on the final state (the tolerances the operator is specified
to, with fp32 state and fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_30_b200 as kda
import oracle
from kda_inputs import WORKLOADS, make_decode_state, make_decode_token, make_prefill, to_f64
from kda_testlib import TOL, gpu_slices, oracle_prefill, parity, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _to(inp, dev):
    for name in ("q", "k", "v", "log_alpha", "beta"):
        setattr(inp, name, getattr(inp, name).to(dev))
    if inp.init_state is not None:
        inp.init_state = inp.init_state.to(dev)
    return inp


def _run(inp, algo="auto", C=None):
    o, fs = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state,
                          cu_seqlens=inp.cu_seqlens, C=C or inp.C, algo=algo)
    torch.cuda.synchronize()
    return o, fs


def _check_all(inp, o, fs, tol, label="prefill"):
    o_ref, fs_ref, ti, seqs, heads = oracle_prefill(inp)
    og, fg = gpu_slices(o, fs, ti, seqs, heads)
    eo = parity(f"{label} o", og, o_ref, tol, stored_as=inp.dtype)
    es = parity(f"{label} state", fg, fs_ref, tol)
    assert np.isfinite(og).all() and np.isfinite(fg).all()
    assert eo <= tol, f"o rel err {eo:.3e} > {tol}"
    assert es <= tol, f"state rel err {es:.3e} > {tol}"
    return eo, es


# --------------------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_decode_steps_small(cuda_ok, dtype, dk, dv):
    from dataclasses import replace
    wl = replace(WORKLOADS["decode"], dtype=dtype, dk=dk, dv=dv)
    N, H = 5, 3
    state = make_decode_state(wl, N=N, H=H, seed=3)
    s_gpu = state.to(DEV).clone()
    s_ref = to_f64(state)
    for step in range(4):
        tok = make_decode_token(wl, step=step, N=N, H=H, seed=3)
        o = kda.decode_step(tok.q.to(DEV), tok.k.to(DEV), tok.v.to(DEV), tok.log_alpha.to(DEV),
                            tok.beta.to(DEV), s_gpu)
        o_ref, s_ref = oracle.decode_step(to_f64(tok.q), to_f64(tok.k), to_f64(tok.v), to_f64(tok.log_alpha),
                                          to_f64(tok.beta), s_ref)
        torch.cuda.synchronize()
        assert rel_err(to_f64(o), o_ref, stored_as=dtype) <= TOL[dtype]
        assert rel_err(to_f64(s_gpu), s_ref) <= TOL[dtype]


def test_decode_alpha_zero_and_beta_edges(cuda_ok):
    """log alpha = -inf (memory cleared), beta = 0 and beta = 1."""
    N, H, d = 4, 2, 128
    state = make_decode_state("decode", N=N, H=H, seed=5)
    tok = make_decode_token("decode", step=0, N=N, H=H, seed=5)
    tok.log_alpha[0] = float("-inf")
    tok.beta[1] = 0.0
    tok.beta[2] = 1.0
    s_gpu = state.to(DEV).clone()
    o = kda.decode_step(tok.q.to(DEV), tok.k.to(DEV), tok.v.to(DEV), tok.log_alpha.to(DEV), tok.beta.to(DEV), s_gpu)
    o_ref, s_ref = oracle.decode_step(to_f64(tok.q), to_f64(tok.k), to_f64(tok.v), to_f64(tok.log_alpha),
                                      to_f64(tok.beta), to_f64(state))
    torch.cuda.synchronize()
    assert rel_err(to_f64(o), o_ref, stored_as="bf16") <= 2e-2
    assert rel_err(to_f64(s_gpu), s_ref) <= 2e-2


def test_decode_full_size_sampled(cuda_ok):
    """256 sequences x 32 heads x 128 x 128 (the decode benchmark's launch),
    all 64 consecutive steps of the workload: the sampled sequences' outputs at
    every step and their states after the last step vs the oracle."""
    wl = WORKLOADS["decode"]
    state = make_decode_state(wl, device=DEV)
    idx = [0, 17, 128, 255]
    s_ref = to_f64(state[idx])
    worst = 0.0
    for step in range(wl.steps):
        tok = make_decode_token(wl, step=step, device=DEV)
        o = kda.decode_step(tok.q, tok.k, tok.v, tok.log_alpha, tok.beta, state)
        o_ref, s_ref = oracle.decode_step(to_f64(tok.q[idx]), to_f64(tok.k[idx]), to_f64(tok.v[idx]),
                                          to_f64(tok.log_alpha[idx]), to_f64(tok.beta[idx]), s_ref)
        torch.cuda.synchronize()
        e = parity(f"decode N=256 H=32 step {step} o", to_f64(o[idx]), o_ref, 2e-2, stored_as="bf16")
        worst = max(worst, e)
        assert e <= 2e-2, step
    assert parity("decode N=256 H=32 state after 64 steps", to_f64(state[idx]), s_ref, 2e-2) <= 2e-2
    assert torch.isfinite(state).all()


# --------------------------------------------------------------------------- prefill, small

def test_prefill_tiny_f32(cuda_ok):
    """fp32 prefill B=1, H=2, T=256, d=64, C=64 (zero initial state), tol 1e-4."""
    inp = _to(make_prefill("tiny_f32"), DEV)
    o, fs = _run(inp)
    _check_all(inp, o, fs, TOL["f32"])


@pytest.mark.parametrize("algo,C", [("auto", 64), ("auto", 128), ("simt", 64), ("simt", 128), ("tc", 64),
                                    ("tc", 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 200, 300])
def test_prefill_bf16_ragged(cuda_ok, algo, C, T):
    """bf16, d=128, several chunks and a ragged tail, random initial state;
    the tensor-core path (64-token chunks, asked for 64 or 128) and the CUDA-core
    split (the chunk size as given)."""
    inp = _to(make_prefill("prefill", B=2, T=T, H=3, seed=T), DEV)
    o, fs = _run(inp, algo=algo, C=C)
    _check_all(inp, o, fs, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_prefill_small_heads(cuda_ok, dk, dv):
    from dataclasses import replace
    wl = replace(WORKLOADS["prefill"], dk=dk, dv=dv)
    for dt in ("bf16", "f32"):
        inp = _to(make_prefill(replace(wl, dtype=dt), B=2, T=150, H=2, seed=9), DEV)
        o, fs = _run(inp)
        _check_all(inp, o, fs, TOL[dt])


@pytest.mark.parametrize("algo,C", [("auto", 64), ("auto", 128), ("simt", 64)])
def test_prefill_varlen_with_empty_and_tiny_sequences(cuda_ok, algo, C):
    lengths = [5, 0, 64, 129, 1, 300, 0, 77]
    inp = _to(make_prefill("varlen", H=4, lengths=lengths, seed=11, C=C), DEV)
    o, fs = _run(inp, algo=algo, C=C)
    _check_all(inp, o, fs, TOL["bf16"])


@pytest.mark.parametrize("algo", ["auto", "simt"])
def test_prefill_gate_regimes_and_special_heads(cuda_ok, algo):
    """Near-0 gates (log alpha down to -16 per token: the tensor-core path's
    pairwise fallback for diagonal blocks), near-1 gates, mixed; and the
    alpha = 1 / scalar-alpha heads."""
    inp = _to(make_prefill("varlen", H=6, lengths=[700, 333], seed=12), DEV)
    o, fs = _run(inp, algo=algo)
    _check_all(inp, o, fs, TOL["bf16"])
    inp = _to(make_prefill("long", T=500, H=4, seed=13), DEV)
    o, fs = _run(inp, algo=algo)
    _check_all(inp, o, fs, TOL["bf16"])


@pytest.mark.parametrize("algo", ["auto", "simt"])
def test_prefill_alpha_zero_beta_edges(cuda_ok, algo):
    inp = make_prefill("prefill", B=1, T=200, H=2, seed=14)
    inp.log_alpha[0, 50:60, 0] = float("-inf")
    inp.log_alpha[0, 100, 1, :7] = float("-inf")
    inp.beta[0, 10:20, 0] = 0.0
    inp.beta[0, 30:40, 1] = 1.0
    inp = _to(inp, DEV)
    o, fs = _run(inp, algo=algo)
    _check_all(inp, o, fs, TOL["bf16"])


def test_prefill_empty_and_no_final_state(cuda_ok):
    inp = _to(make_prefill("prefill", B=2, T=0, H=2, seed=15), DEV)
    o, fs = _run(inp)
    assert o.numel() == 0
    torch.testing.assert_close(fs, inp.init_state)
    inp = _to(make_prefill("prefill", B=1, T=70, H=2, seed=16), DEV)
    o1, _ = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state,
                          output_final_state=False)
    o2, _ = _run(inp)
    torch.testing.assert_close(o1, o2, rtol=0, atol=0)


@pytest.mark.parametrize("algo", ["tc", "simt"])
def test_prefill_final_state_may_alias_init_state(cuda_ok, algo):
    """final_state may be the init_state buffer (updated in place): same o and
    state, bit for bit, as with separate buffers; also through the no-alloc call."""
    inp = _to(make_prefill("prefill", lengths=[130, 0, 64, 200], H=3, seed=77), DEV)
    o1, f1 = _run(inp, algo=algo)
    st = inp.init_state.clone()
    o2, f2 = kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=st, final_state=st,
                           cu_seqlens=inp.cu_seqlens, C=64, algo=algo)
    torch.cuda.synchronize()
    assert f2 is st
    assert torch.equal(o2, o1) and torch.equal(st, f1)
    if algo == "tc":
        st = inp.init_state.clone()
        o3, _ = kda.chunk_fwd_noalloc(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=st, final_state=st,
                                      cu_seqlens=inp.cu_seqlens, C=64)
        torch.cuda.synchronize()
        assert torch.equal(o3, o1) and torch.equal(st, f1)


def test_device_status_after_tensor_core_calls(cuda_ok):
    """The error word of the bounded device-side waits reads 0 after calls that
    finished normally (forward, fused-prep forward and backward)."""
    inp = _to(make_prefill("prefill", B=2, T=200, H=4, seed=77), DEV)
    B, T, H, dk = inp.q.shape
    ws = torch.empty(kda.workspace_size(B, T, H, dk, dk, 64, torch.bfloat16), dtype=torch.uint8, device=DEV)
    kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, C=64, workspace=ws)
    assert kda.device_status("fwd", ws, torch.bfloat16, B, T, H, dk, dk, 64) == 0
    kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, C=64, workspace=ws, prep=kda.PREP_QK_L2NORM)
    assert kda.device_status("fwd", ws, torch.bfloat16, B, T, H, dk, dk, 64) == 0
    wsb = torch.empty(kda.bwd_workspace_size(B, T, H, dk, dk, 64), dtype=torch.uint8, device=DEV)
    kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, torch.randn_like(inp.v), C=64, workspace=wsb)
    assert kda.device_status("bwd", wsb, torch.bfloat16, B, T, H, dk, dk, 64) == 0


def test_prefill_resume_and_handoff(cuda_ok):
    """Prefill of x[:t1] then x[t1:] from the carried state equals one prefill;
    prefill of T tokens then decode steps equals prefill of T + m tokens."""
    inp = _to(make_prefill("prefill", B=2, T=260, H=2, seed=17), DEV)
    o_all, fs_all = _run(inp)
    t1 = 130
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = kda.chunk_fwd(sl(inp.q, 0, t1), sl(inp.k, 0, t1), sl(inp.v, 0, t1), sl(inp.log_alpha, 0, t1),
                           sl(inp.beta, 0, t1), init_state=inp.init_state)
    o2, s2 = kda.chunk_fwd(sl(inp.q, t1, 260), sl(inp.k, t1, 260), sl(inp.v, t1, 260),
                           sl(inp.log_alpha, t1, 260), sl(inp.beta, t1, 260), init_state=s1)
    torch.cuda.synchronize()
    # two stored bf16 outputs: the storage half-ulp of each side is allowed
    assert rel_err(to_f64(torch.cat([o1, o2], 1)), to_f64(o_all), stored_as="bf16", both_stored=True) <= 2e-2
    assert rel_err(to_f64(s2), to_f64(fs_all)) <= 2e-2
    # prefill 250 tokens, then 10 decode steps
    o_p, st = kda.chunk_fwd(sl(inp.q, 0, 250), sl(inp.k, 0, 250), sl(inp.v, 0, 250), sl(inp.log_alpha, 0, 250),
                            sl(inp.beta, 0, 250), init_state=inp.init_state)
    outs = []
    for t in range(250, 260):
        outs.append(kda.decode_step(inp.q[:, t].contiguous(), inp.k[:, t].contiguous(), inp.v[:, t].contiguous(),
                                    inp.log_alpha[:, t].contiguous(), inp.beta[:, t].contiguous(), st))
    torch.cuda.synchronize()
    assert rel_err(to_f64(torch.stack(outs, 1)), to_f64(o_all[:, 250:]), stored_as="bf16", both_stored=True) <= 2e-2
    assert rel_err(to_f64(st), to_f64(fs_all)) <= 2e-2


def test_simt_intermediates_match_oracle(cuda_ok):
    """Rows of the four-kernel split against the oracle's chunk-form
    intermediates: cumulative log decay g, U, Wk, W and the chunk start states."""
    for dt, tol in (("f32", 1e-4), ("bf16", 2e-2)):
        from dataclasses import replace
        wl = replace(WORKLOADS["prefill"], dtype=dt, dk=64, dv=64)
        lengths = [130, 64, 7]
        inp = _to(make_prefill(wl, H=2, lengths=lengths, seed=21), DEV)
        C = 64
        B, T, H = 1, int(inp.seq_start[-1]), 2
        ws_bytes = kda.workspace_size(B, T, H, 64, 64, C, inp.q.dtype, cu_seqlens=inp.cu_seqlens, algo="simt")
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
        kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state,
                      cu_seqlens=inp.cu_seqlens, C=C, workspace=ws, algo="simt")
        torch.cuda.synchronize()
        off = kda.simt_offsets(B, T, H, 64, 64, C, cu_seqlens=inp.cu_seqlens)
        n_chunks = sum((L + C - 1) // C for L in lengths)

        def view(i, shape):
            n = int(np.prod(shape))
            return ws[off[i]:off[i] + 4 * n].view(torch.float32).reshape(shape).double().cpu().numpy()

        ref = oracle.chunkform(*(to_f64(x).reshape(T, H, -1) if x.dim() == 4 else to_f64(x).reshape(T, H)
                                 for x in (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)),
                               inp.seq_start, C, init_state=to_f64(inp.init_state), intermediates=True)
        assert rel_err(view(0, (T, H, 64)), ref["g"]) <= tol
        assert rel_err(view(1, (T, H, 64)), ref["u"]) <= tol
        assert rel_err(view(2, (T, H, 64)), ref["wk"]) <= tol
        assert rel_err(view(3, (T, H, 64)), ref["w"]) <= tol
        assert rel_err(view(4, (n_chunks, H, 64, 64)), ref["s_chunk"]) <= tol


# --------------------------------------------------------------------------- prefill, full size

def test_full_prefill_b4_h16_t4096(cuda_ok):
    """B=4, H=16, T=4096, d=128, C=64 bf16 (the prefill benchmark's launch);
    sampled (sequence, head) pairs over all 4096 tokens."""
    inp = make_prefill("prefill", device=DEV)
    o, fs = _run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    for seqs, heads in (([0], [0, 5]), ([1], [15]), ([3], [8])):
        o_ref, fs_ref, ti, s_, h_ = oracle_prefill(inp, heads=heads, seqs=seqs)
        og, fg = gpu_slices(o, fs, ti, s_, h_)
        assert parity(f"prefill B=4 H=16 T=4096 seqs {seqs} heads {heads} o", og, o_ref, 2e-2,
                      stored_as="bf16") <= 2e-2
        assert parity(f"prefill B=4 H=16 T=4096 seqs {seqs} heads {heads} state", fg, fs_ref, 2e-2) <= 2e-2


def test_full_prefill_long_t65536(cuda_ok):
    """B=1, H=32, T=65536, bf16; head 0 alpha = 1, head 1 scalar alpha; sampled
    heads.  Chunk independence on the GPU: the tensor-core path (64-token
    chunks) and the CUDA-core split with 128-token chunks agree with the oracle
    and with each other."""
    inp = make_prefill("long", device=DEV)
    o_ref, fs_ref, ti, s_, h_ = oracle_prefill(inp, heads=[0, 1, 20])
    got = {}
    for algo, C in (("tc", 64), ("tc", 128), ("simt", 128)):
        o, fs = _run(inp, C=C, algo=algo)
        assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
        og, fg = gpu_slices(o, fs, ti, s_, h_)
        for j in range(3):
            lab = f"long T=65536 {algo} C={C} head {h_[j]}"
            assert parity(lab + " o", og[:, j], o_ref[:, j], 2e-2, stored_as="bf16") <= 2e-2, (algo, C, j)
            assert parity(lab + " state", fg[:, j], fs_ref[:, j], 2e-2) <= 2e-2, (algo, C, j)
        got[(algo, C)] = (og, fg)
        del o, fs
    og64, fg64 = got[("tc", 64)]
    og128, fg128 = got[("simt", 128)]
    assert rel_err(og64, og128, stored_as="bf16", both_stored=True) <= 2e-2
    assert rel_err(fg64, fg128) <= 2e-2
    assert np.array_equal(got[("tc", 128)][0], og64)      # the same 64-token computation


def test_full_prefill_varlen_64_seqs(cuda_ok):
    """64 packed sequences, lengths U[512, 32768] (~1.07M tokens), H=32, C=64;
    sampled (sequence, head) pairs covering the three gate regimes."""
    inp = make_prefill("varlen", device=DEV)
    o, fs = _run(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    lens = np.diff(inp.seq_start)
    longest = int(np.argmax(lens))
    for seqs, heads in (([0, 1], [0, 1, 2]), ([longest], [3, 31])):
        o_ref, fs_ref, ti, s_, h_ = oracle_prefill(inp, heads=heads, seqs=seqs)
        og, fg = gpu_slices(o, fs, ti, s_, h_)
        for j in range(len(heads)):
            lab = f"varlen 64 seqs, seqs {seqs} head {heads[j]}"
            assert parity(lab + " o", og[:, j], o_ref[:, j], 2e-2, stored_as="bf16") <= 2e-2
            assert parity(lab + " state", fg[:, j], fs_ref[:, j], 2e-2) <= 2e-2


@pytest.mark.parametrize("call", ["fwd", "bwd"])
def test_varlen_call_returns_before_earlier_work_finishes(cuda_ok, call):
    """A packed-batch call is asynchronous: its sequence tables reach the device
    as launch parameters, so the host returns while work queued before it on
    the stream is still running (a copy from pageable host memory would first
    wait for that work).  The results still match the oracle."""
    inp = _to(make_prefill("varlen", H=4, lengths=[300, 70, 0, 129], seed=51), DEV)
    args = (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)
    d_o = torch.randn_like(inp.v)
    run = (lambda: kda.chunk_fwd(*args, init_state=inp.init_state, cu_seqlens=inp.cu_seqlens)) if call == "fwd" \
        else (lambda: kda.chunk_bwd(*args, d_o, init_state=inp.init_state, cu_seqlens=inp.cu_seqlens))
    run()                                  # library loaded, kernels resident
    torch.cuda.synchronize()
    torch.cuda._sleep(1_000_000_000)       # ~0.5 s of spinning on the current stream
    before = torch.cuda.Event()
    before.record()
    out = run()
    pending = not before.query()
    torch.cuda.synchronize()
    assert pending, "the call waited for earlier work on its stream"
    if call == "fwd":
        _check_all(inp, out[0], out[1], TOL["bf16"], label="varlen async call")


@pytest.mark.parametrize("kernels", [1, 2, 3])
def test_device_wait_timeout_is_reported_and_recoverable(cuda_ok, kernels):
    """The failure path of the bounded device-side waits, without breaking the
    GPU: kda_set_test_wait_limit makes one wait in the first CTA of tc_intra
    (1), tc_recur (2) or both (3) wait 1 ms on a barrier that nothing completes.
    The call then reports KDA_ERR_TIMEOUT through the device status, and the
    next call on the same stream and workspace is normal and matches the
    oracle."""
    inp = _to(make_prefill("prefill", B=2, T=300, H=4, seed=61), DEV)
    B, T, H, dk = inp.q.shape
    ws = torch.empty(kda.workspace_size(B, T, H, dk, dk, 64, torch.bfloat16), dtype=torch.uint8, device=DEV)
    args = (inp.q, inp.k, inp.v, inp.log_alpha, inp.beta)
    kda.set_test_wait_limit(kernels, 1_000_000)
    kda.chunk_fwd(*args, init_state=inp.init_state, C=64, workspace=ws)
    assert kda.device_status("fwd", ws, torch.bfloat16, B, T, H, dk, dk, 64) == kda.KDA_ERR_TIMEOUT
    o, fs = kda.chunk_fwd(*args, init_state=inp.init_state, C=64, workspace=ws)
    assert kda.device_status("fwd", ws, torch.bfloat16, B, T, H, dk, dk, 64) == 0
    _check_all(inp, o, fs, TOL["bf16"], label=f"after a timeout in kernels {kernels}")
