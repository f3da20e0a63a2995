#!/usr/bin/env python
"""KDA benchmark: prefill tokens/s + tensor-pipe %, decode tokens/s + HBM GB/s, one B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one ``kda_chunk_fwd`` over the headline workload, inputs resident in
HBM: the packed variable-length batch of 64 sequences (lengths uniform in
[512, 32768], about 1.07 M tokens), H = 32, d_k = d_v = 128, chunk 64, bf16
inputs, fp32 states, three gate regimes.  Its inputs (about 35 GB) are far
larger than L2, so no flush is needed between steps; each step is timed with
CUDA events on the launching stream.  In the same run, each with its own JSON
object:

* ``prefill_b4``: B = 4, H = 16, T = 4096 (L2 flushed before every step);
* ``long``: one 65,536-token sequence, H = 32, at C = 64 and C = 128 on the
  tensor-core path (64-token chunks either way) and at C = 128 on the
  CUDA-core split, with the state carry's time per chunk step;
* ``decode``: 256 sequences x 32 heads, 64 consecutive steps, timed per launch;
* ``prep``: the prefill_b4 and decode launches on raw inputs, preprocessing
  fused (``kda_chunk_fwd_prep`` / ``kda_decode_step_prep``);
* ``backward``: ``kda_chunk_bwd`` on the prefill_b4 workload;
* ``seqpar``: one long sequence split into segments (projection on one GPU);
* ``e2e``: the headline through the public API with pinned host buffers (H2D
  of the inputs and D2H of the outputs inside the timed region);
* ``cpu_baseline``: the fp64 oracle on a bounded sample of the headline
  workload on the host cores (rank 0, N = 1).

Roofline: ``achieved`` divides the method's algorithmic bytes (q, k, v,
log alpha, beta in, o out: 1,282 B per token-head at d = 128 in bf16, plus the
initial and final states) by the dominant kernel's average launch time; the
bytes each kernel moves by its own design are reported beside it as
``design_bytes``.  Tensor figures use the algorithmic FLOPs of the chunk
algorithm (6 dk dv + C (3 dk + 2 dv) + C^2 / 3 per token-head).

With N > 1 (torchrun) every rank runs its own independent batch (weak scaling,
no collective on the data path); times are the max over ranks.
Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s + tensor-pipe %; decode tokens/s + HBM GB/s (1xB200)"
D = 128
PREFILL_B4 = dict(B=4, T=4096, H=16)
LONG = dict(B=1, T=65536, H=32)
DECODE = dict(N=256, H=32, dk=128, dv=128, steps=64)
SM_COUNT = 148
TC_FLOP_PER_CLK_SM = 8192      # dense bf16 tcgen05 FLOPs per SM per clock (2.25 PFLOP/s at ~1.86 GHz)


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--workload", default="varlen", choices=["varlen", "prefill_b4", "long"],
                    help="headline prefill workload (profiling aid; the default is the packed 64-sequence batch)")
    ap.add_argument("--varlen-seqs", type=int, default=64,
                    help="profiling aid: only the first n sequences of the packed batch")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prep", action="store_true", help="skip the fused-preprocessing timings")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward-pass timings")
    ap.add_argument("--no-seqpar", action="store_true", help="skip the sequence-parallel timings")
    ap.add_argument("--no-b4", action="store_true", help="skip the B=4 H=16 T=4096 prefill line")
    ap.add_argument("--no-long", action="store_true", help="skip the T=65536 prefill lines")
    ap.add_argument("--seqpar", action="store_true",
                    help="with N > 1 ranks, also time one long sequence split over the ranks (NCCL all-gather)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle sample length")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode"],
                    help="profiling aid: run only the headline prefill or only decode")
    ap.add_argument("--decode-n", type=int, default=DECODE["N"], help="profiling aid: decode sequences")
    a = ap.parse_args()
    a.warmup = max(3, a.warmup)
    return a


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_helpers(world, device=None):
    """barrier() and max_over_ranks(x) for a step timed on every rank: with one
    rank both are no-ops; otherwise they use the initialised process group
    (NCCL on GPUs, gloo in the CPU tests)."""
    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(x):
        if world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def job_throughput(world, units_per_rank_step, steps, max_total_ms):
    """Whole-job units/s: every rank processes its own batch (weak scaling), the
    job takes as long as its slowest rank."""
    return world * units_per_rank_step * steps / (max_total_ms / 1e3)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if gpu_id:
                cmd += ["-i", gpu_id]
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:  # noqa: BLE001 - clocks are best-effort metadata
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * (max(smax) if smax else 1)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- work and bytes

class Geometry:
    """Sizes of one prefill problem: token-heads, chunk-heads (64-token chunks,
    the tensor-core kernels' tile, restarting at every sequence), states."""

    def __init__(self, lengths, H, dk=D, dv=D, C=64):
        self.lengths = [int(x) for x in lengths]
        self.H, self.dk, self.dv, self.C = H, dk, dv, C
        self.tokens = sum(self.lengths)
        self.token_heads = self.tokens * H
        self.n_seqs = len(self.lengths)
        self.chunk_heads = sum((L + 63) // 64 for L in self.lengths) * H
        self.state_bytes = self.n_seqs * H * dk * dv * 4


def algorithmic_flops(g: Geometry, C: int) -> float:
    """FLOPs of the chunk algorithm, masked work counted once:
    6 dk dv + C (3 dk + 2 dv) + C^2 / 3 per token-head (140,629 at d = 128, C = 64)."""
    return g.token_heads * (6 * g.dk * g.dv + C * (3 * g.dk + 2 * g.dv) + C * C / 3)


def minimal_bytes(g: Geometry, in_bytes=2) -> int:
    """The method's algorithmic bytes: q, k, v, log alpha, beta in and o out once
    (1,282 B per token-head at d = 128, bf16), plus the initial and final states."""
    per_th = (2 * g.dk + g.dv + g.dk + 1) * in_bytes + g.dv * in_bytes
    return g.token_heads * per_th + 2 * g.state_bytes


# tensor-core path: bytes of one (chunk, head) workspace image (kda_chunk_tc.cu) and
# the dense tcgen05 work each kernel issues per (chunk, head), counted as M = 128 tiles
TC_CHUNK_BYTES = 147968
TC_ISSUED_FLOPS = {
    # [K e ; Q e] x decayed keys: M 128, N 160, K 128, three terms; T [bV | bK e^g]: M 64 (a
    # 128-row tile's time), N 256, K 64, three terms
    "tc_intra": 2 * 128 * 160 * 128 * 3 + 2 * 128 * 256 * 64 * 3,
    # per chunk over all 128 state columns: [Wk ; Q e^g] S (K 128), Kd^T W and [0 ; P] W (K 64), three terms
    "tc_recur": 2 * 128 * 128 * (128 + 64 + 64) * 3,
}


def design_bytes(kernel: str, g: Geometry, in_bytes=2):
    """Bytes a kernel moves by its own design (inputs read once, outputs and
    workspace written once, workspace read back once)."""
    th = g.token_heads
    ws = g.chunk_heads * TC_CHUNK_BYTES
    simt_ws = th * 4 * (3 * g.dk + 2 * g.dv)
    schunk = g.chunk_heads * g.dk * g.dv * 4
    table = {
        "tc_intra": th * ((3 * g.dk + g.dv + 1) * in_bytes) + ws,
        "tc_recur": ws + th * g.dv * in_bytes + 2 * g.state_bytes,
        "k1_cumsum": th * g.dk * (in_bytes + 8),
        "k2_wy": th * (2 * g.dk * in_bytes + g.dv * in_bytes + in_bytes + 8 * g.dk) + th * 4 * (g.dv + g.dk),
        "k3_state": th * (4 * g.dk + 4 * g.dv + in_bytes * g.dk + 8 * g.dk) + th * 4 * g.dv + schunk
        + 2 * g.state_bytes,
        "k4_output": th * (2 * g.dk * in_bytes + 8 * g.dk + 4 * g.dv + g.dv * in_bytes) + schunk,
        "seq_table_write": 0,
        "chunk_table_fill": 0,
    }
    return table.get(kernel, None) if kernel != "simt" else simt_ws


def _tc_digest():
    csrc = os.path.join(ROOT, "kimi_delta_attention_30_b200", "csrc")
    h = hashlib.sha256()
    for f in ("kda_chunk_tc.cu", "kda_tc.cuh", "kda_tc_image.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profile_rows(name):
    """Rows of a committed ncu table under profiles/ whose source digest matches
    the kernels as built now (columns: kernel workload units value... digest)."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return []
    digest = _tc_digest()
    rows = []
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        f = line.split()
        if f[-1] == digest:
            rows.append(f)
    return rows


def measured_traffic(kernel, g: Geometry):
    """DRAM bytes per launch of `kernel` for this problem: the committed ncu
    capture's bytes per (chunk, head), times this problem's chunk-heads; None
    when there is none or the kernel sources changed since it was taken."""
    for f in _profile_rows("dram_traffic.txt"):
        if len(f) == 6 and f[0] == kernel:
            units, rd, wr = int(f[2]), int(f[3]), int(f[4])
            return int(round((rd + wr) / units * g.chunk_heads))
    return None


def measured_tensor_pct(kernel):
    """sm__pipe_tensor_cycles_active (% of peak, elapsed) from the committed ncu
    capture, or None when none matches the kernels as built now."""
    for f in _profile_rows("tensor_pipe.txt"):
        if len(f) == 5 and f[0] == kernel:
            return float(f[3])
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def prefill_report(g: Geometry, C_req: int, C_run: int, kernels, k_avg_ms, ms_per_step, pk, sm_mhz):
    """Roofline and tensor figures of one timed prefill."""
    t = ms_per_step / 1e3
    algo_b = minimal_bytes(g)
    flops = algorithmic_flops(g, C_run)
    timed = [j for j, n in enumerate(kernels) if n not in ("seq_table_write", "chunk_table_fill")]
    dom = max(timed, key=lambda j: k_avg_ms[j])
    dom_s = k_avg_ms[dom] / 1e3
    ach = algo_b / dom_s / 1e9
    roof = {"kernel": kernels[dom], "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": measured_traffic(kernels[dom], g),
            "algorithmic_bytes": algo_b, "design_bytes": design_bytes(kernels[dom], g),
            "peak_source": pk["source"],
            "note": "achieved = the method's algorithmic bytes (1,282 B per token-head + 2 states) / the dominant "
                    "kernel's average launch time; peak = measured HBM copy bandwidth"}
    clk = (sm_mhz or 1965.0) * 1e6
    ktab = {}
    for j in timed:
        n = kernels[j]
        s = k_avg_ms[j] / 1e3
        db = design_bytes(n, g)
        e = {"avg_us": k_avg_ms[j] * 1e3, "share": k_avg_ms[j] / max(sum(k_avg_ms[i] for i in timed), 1e-12),
             "design_bytes": db, "design_gbs": (db / s / 1e9) if db else None,
             "traffic": measured_traffic(n, g)}
        if n in TC_ISSUED_FLOPS:
            issued = TC_ISSUED_FLOPS[n] * g.chunk_heads
            e["issued_tensor_flops"] = issued
            e["tensor_pipe_pct_est"] = 100.0 * issued / (s * SM_COUNT * TC_FLOP_PER_CLK_SM * clk)
            e["tensor_pipe_pct_ncu"] = measured_tensor_pct(n)
        ktab[n] = e
    t_hbm = algo_b / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk["bf16_tflops"] * 1e12)
    tensor = {"algorithmic_flops": flops, "tflops": flops / t / 1e12,
              "frac_of_burst_peak": flops / t / (pk["bf16_tflops"] * 1e12),
              "frac_of_sustained_peak": flops / t / (pk["bf16_tflops_sustained"] * 1e12)
              if pk.get("bf16_tflops_sustained") else None,
              "flops_per_token_head": 6 * D * D + C_run * 5 * D + C_run * C_run / 3,
              "chunk_computed": C_run, "chunk_requested": C_req}
    path = {"algorithmic_bytes": algo_b, "time_min_us": max(t_hbm, t_tc) * 1e6,
            "frac_of_hbm_bound": t_hbm / t, "time_min_over_time": max(t_hbm, t_tc) / t}
    return roof, tensor, path, ktab


# ----------------------------------------------------------------------------- oracle timing

class OracleSample:
    """The fp64 oracle timed on a bounded sample of the headline workload: the
    first `n_seqs` sequences of the packed batch (their lengths drawn as the
    workload draws them) over `heads` heads (gate regimes by head index mod 3),
    one (sequence, head) pair per host thread; the pass is repeated to fill about
    `seconds` of wall time.  Throughput is in full 32-head tokens per second."""

    def __init__(self, seconds: float, seed: int = 0, n_seqs: int = 6, heads: int = 12):
        import oracle
        from kda_inputs import WORKLOADS, make_prefill, to_f64, varlen_lengths
        wl = WORKLOADS["varlen"]
        self.oracle = oracle
        self.threads = oracle.max_threads()
        self.H_full = wl.H
        lens = varlen_lengths(wl.n_seqs, *wl.len_range, seed=seed)[:n_seqs]
        inp = make_prefill("varlen", lengths=lens, H=heads, seed=seed)
        n = int(inp.seq_start[-1])
        f = lambda t: to_f64(t).reshape(n, heads, -1)
        self.args = (f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha), to_f64(inp.beta).reshape(n, heads))
        self.s0 = to_f64(inp.init_state)
        self.seq = inp.seq_start
        self.lens = [int(x) for x in lens]
        self.heads = heads
        self.reps = 1
        t1 = self.time()
        self.reps = max(1, int(round(seconds / max(t1, 1e-3))))

    def time(self) -> float:
        t0 = time.perf_counter()
        for _ in range(self.reps):
            self.oracle.forward(*self.args, self.seq, init_state=self.s0, n_threads=self.threads)
        return time.perf_counter() - t0

    def tokens(self) -> float:
        return self.reps * sum(self.lens) * self.heads / self.H_full   # a token carries all 32 heads

    def single_core(self) -> dict:
        """The shortest sampled sequence, one head, on one thread."""
        j = min(range(len(self.lens)), key=lambda i: self.lens[i])
        a, b = int(self.seq[j]), int(self.seq[j + 1])
        sl = [x[a:b, :1] for x in self.args]
        t0 = time.perf_counter()
        self.oracle.forward(*sl, [0, b - a], init_state=self.s0[j:j + 1, :1], n_threads=1)
        dt = time.perf_counter() - t0
        return {"value": (b - a) / self.H_full / dt, "unit": "tokens/s", "cores": 1,
                "sample": f"1 (sequence, head) pair x {b - a} tokens, {dt:.2f} s"}

    def describe(self, dt: float) -> str:
        return (f"{len(self.lens)} sequences of the packed batch ({sum(self.lens)} tokens, lengths "
                f"{min(self.lens)}-{max(self.lens)}) x {self.heads} of its 32 heads"
                f"{f', {self.reps} passes' if self.reps > 1 else ''} (= {self.tokens():.0f} full 32-head tokens), "
                f"fp64 token recurrence, {self.threads} threads, {dt:.1f} s")


def headline_config(lengths, C, extra=None):
    c = {"workload": f"packed varlen prefill: {len(lengths)} sequences, lengths U[512, 32768] "
                     f"({sum(lengths)} tokens), H=32, d_k=d_v=128, C={C}, bf16 inputs, fp32 states, "
                     "gate regimes by head mod 3 (near-1, near-0, mixed), beta ~ U(0,1)",
         "n_seqs": len(lengths), "tokens": int(sum(lengths)), "H": 32, "dk": D, "dv": D, "C": C}
    if extra:
        c.update(extra)
    return c


def run_reference(a, world, rank):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from kda_inputs import WORKLOADS, varlen_lengths
    wl = WORKLOADS["varlen"]
    lengths = list(varlen_lengths(wl.n_seqs, *wl.len_range, seed=0))
    steps = a.warmup + a.steps
    smp = OracleSample(max(0.5, min(8.0, 120.0 / steps)))
    vals, dts = [], []
    for i in range(steps):
        dt = smp.time()
        if i >= a.warmup:
            vals.append(smp.tokens() / dt)
            dts.append(dt)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": statistics.mean(dts) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(lengths, 64, {"sample": "each step: the oracle on a bounded sample of the "
                                                               "workload"}),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.threads, "kind": "oracle",
                             "sample": smp.describe(statistics.mean(dts))},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def main():
    a = _args()
    world, rank, local = _dist()
    if a.impl == "reference":
        return run_reference(a, world, rank)

    import torch
    import torch.distributed as dist

    import kimi_delta_attention_30_b200 as kda
    from kda_inputs import (RAW_PREP, WORKLOADS, make_decode_state, make_decode_token, make_grad_outputs,
                            make_prefill, varlen_lengths)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    barrier, max_over_ranks = rank_helpers(world, dev)

    props = torch.cuda.get_device_properties(dev)
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(props.uuid)
    except Exception:  # noqa: BLE001
        gpu_id = None
    pk = peaks()
    DECODE["N"] = a.decode_n
    run_prefill = a.only in ("all", "prefill")
    run_decode = a.only in ("all", "decode") and not a.no_decode
    extras = a.only == "all"
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(gpu_id if rank == 0 else None)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2

    def time_prefill(inp, C, algo="auto", steps=None, do_flush=False, prep=0, geom=None):
        """Time `steps` calls after `warmup`; per-kernel times through the library's
        timing hook.  Returns (ms_per_step max over ranks, kernel names, per-kernel avg ms)."""
        steps = a.steps if steps is None else steps
        B, T, H, dk = inp.q.shape
        cu = inp.cu_seqlens
        names = kda.chunk_kernels(B, T, H, dk, dk, C, inp.q.dtype, cu_seqlens=cu, algo=algo)
        nk = len(names)
        ws = torch.empty(kda.workspace_size(B, T, H, dk, dk, C, inp.q.dtype, cu_seqlens=cu, algo=algo),
                         dtype=torch.uint8, device=dev)
        o = torch.empty(inp.v.shape, dtype=inp.v.dtype, device=dev)
        fs = torch.empty(inp.init_state.shape, dtype=torch.float32, device=dev)

        def step(evs=None):
            if evs is not None:
                kda.set_timing_events(evs)
            kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state, cu_seqlens=cu,
                          C=C, o=o, final_state=fs, workspace=ws, algo=algo, prep=prep)

        for _ in range(a.warmup):
            if do_flush:
                flush.zero_()
            step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(steps)]
        for row in ev:            # torch creates the CUDA event on its first record
            for e in row:
                e.record(stream)
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            if do_flush:
                flush.zero_()
            step(ev[i])
        torch.cuda.synchronize()
        barrier()
        total = max_over_ranks(sum(ev[i][0].elapsed_time(ev[i][nk]) for i in range(steps)))
        k_avg = [statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps)) for j in range(nk)]
        del ws, o, fs
        return total / steps, names, k_avg

    value = ms_per_step = roofline = tensor = path_roofline = kernel_table = headline = None
    kernels, lengths = [], []
    hl_inp = None
    gpu_launches = None
    sm_guess = 1965.0
    if run_prefill:
        wlname = a.workload
        if wlname == "varlen":
            wl = WORKLOADS["varlen"]
            lengths = [int(x) for x in varlen_lengths(wl.n_seqs, *wl.len_range, seed=rank)][:a.varlen_seqs]
            hl_inp = make_prefill("varlen", device=dev, seed=rank, lengths=lengths)
            C = 64
            geom = Geometry(lengths, 32)
            cfg = headline_config(lengths, C)
            do_flush = False
            cfg["l2"] = "inputs (35 GB) far larger than L2: no flush between steps" if a.varlen_seqs == 64 \
                else "no flush between steps"
        elif wlname == "prefill_b4":
            p = PREFILL_B4
            hl_inp = make_prefill("prefill", device=dev, seed=rank, B=p["B"])
            C = 64
            lengths = [p["T"]] * p["B"]
            geom = Geometry(lengths, p["H"])
            cfg = {"workload": f"prefill B={p['B']} H={p['H']} T={p['T']} d_k=d_v=128 C=64 bf16 inputs, fp32 state",
                   "l2": "flushed before every timed step (256 MiB write)"}
            do_flush = True
        else:
            p = LONG
            hl_inp = make_prefill("long", device=dev, seed=rank)
            C = 64
            lengths = [p["T"]]
            geom = Geometry(lengths, p["H"])
            cfg = {"workload": "long prefill B=1 H=32 T=65536 d_k=d_v=128 C=64 bf16, head 0 alpha=1, head 1 scalar "
                               "alpha", "l2": "inputs larger than L2: no flush"}
            do_flush = False
        ms_per_step, kernels, k_avg = time_prefill(hl_inp, C, a.algo, do_flush=do_flush)
        value = job_throughput(world, geom.tokens, 1, ms_per_step)
        roofline, tensor, path_roofline, kernel_table = prefill_report(geom, C, 64 if a.algo != "simt" else C,
                                                                       kernels, k_avg, ms_per_step, pk, sm_guess)
        gpu_launches = len(kernels) * a.steps
        cfg.update({"algo": a.algo, "kernels": kernels,
                    "parallelism": f"replicas x{world} (independent batches per GPU)"})
        headline = cfg

    # ---------------------------------------------------------------- e2e (headline, host buffers)
    e2e = None
    if run_prefill and not a.no_e2e:
        names = ("q", "k", "v", "log_alpha", "beta")
        need = sum(getattr(hl_inp, n).numel() * getattr(hl_inp, n).element_size() for n in names) \
            + hl_inp.init_state.numel() * 4 + hl_inp.v.numel() * 2 + hl_inp.init_state.numel() * 4
        avail = None
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except Exception:  # noqa: BLE001
            pass
        if avail is not None and avail < 2 * need:
            e2e = {"value": None, "unit": "tokens/s", "skipped": f"host memory: {avail / 2**30:.0f} GiB available, "
                   f"{need / 2**30:.0f} GiB of pinned buffers needed"}
        else:
            host = {n: getattr(hl_inp, n).to("cpu").pin_memory() for n in names}
            host["init_state"] = hl_inp.init_state.to("cpu").pin_memory()
            B, T, H, dk = hl_inp.q.shape
            o_h = torch.empty(hl_inp.v.shape, dtype=hl_inp.v.dtype).pin_memory()
            fs_h = torch.empty(hl_inp.init_state.shape, dtype=torch.float32).pin_memory()
            # the device copies of the inputs are not needed for this part
            for n in names:
                setattr(hl_inp, n, None)
            hl_inp.init_state = None
            torch.cuda.empty_cache()
            e2e_groups = 16
            buf = torch.empty(kda.host_buffer_size(hl_inp.cu_seqlens, H, dk, dk, 64, torch.bfloat16, e2e_groups),
                              dtype=torch.uint8, device=dev)
            h2d = sum(t.numel() * t.element_size() for t in host.values())
            d2h = o_h.numel() * o_h.element_size() + fs_h.numel() * fs_h.element_size()
            e2e_steps = max(3, min(a.steps, 10))

            def e2e_step():
                kda.chunk_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"],
                                   hl_inp.cu_seqlens, init_state=host["init_state"], C=64, o=o_h, final_state=fs_h,
                                   n_groups=e2e_groups, device_buffer=buf, stream=stream, synchronize=False)

            for _ in range(a.warmup):
                e2e_step()
            barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(e2e_steps):
                e2e_step()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            et = max_over_ranks(e0.elapsed_time(e1))
            e2e = {"value": job_throughput(world, sum(lengths), e2e_steps, et), "unit": "tokens/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": et / e2e_steps,
                   "steps": e2e_steps, "n_groups": e2e_groups,
                   "path": "kda_chunk_fwd_host (public API): pinned host buffers in, the packed batch in "
                           f"{e2e_groups} groups of sequences whose copies both ways overlap the kernels, "
                           "pinned host buffers out"}
            del host, o_h, fs_h, buf
    if hl_inp is not None:
        del hl_inp
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- B=4 H=16 T=4096 prefill
    b4 = None
    prep = {} if (run_prefill and extras and not a.no_prep and a.algo in ("auto", "tc")) else None
    b4_inp = None
    if run_prefill and extras and not a.no_b4:
        p = PREFILL_B4
        b4_inp = make_prefill("prefill", device=dev, seed=rank, B=p["B"])
        g4 = Geometry([p["T"]] * p["B"], p["H"])
        ms4, names4, k4 = time_prefill(b4_inp, 64, a.algo, do_flush=True)
        r4, t4, p4, kt4 = prefill_report(g4, 64, 64, names4, k4, ms4, pk, sm_guess)
        b4 = {"value": job_throughput(world, g4.tokens, 1, ms4), "unit": "tokens/s", "ms_per_step": ms4,
              "roofline": r4, "tensor": t4, "path_roofline": p4, "kernel_times": kt4,
              "config": {"workload": f"prefill B={p['B']} H={p['H']} T={p['T']} d_k=d_v=128 C=64 bf16, fp32 state",
                         "l2": "flushed before every timed step (256 MiB write)"}}
        if prep is not None:
            raw = make_prefill("prefill_raw", device=dev, seed=rank, B=p["B"])
            msp, namesp, kp = time_prefill(raw, 64, a.algo, do_flush=True, prep=RAW_PREP)
            F = torch.nn.functional
            qn, kn, lan, bn = (torch.empty_like(t) for t in (raw.q, raw.k, raw.log_alpha, raw.beta))
            ws = torch.empty(kda.workspace_size(p["B"], p["T"], p["H"], D, D, 64, torch.bfloat16),
                             dtype=torch.uint8, device=dev)

            def unfused_step():
                qn.copy_(F.normalize(raw.q.float(), dim=-1))
                kn.copy_(F.normalize(raw.k.float(), dim=-1))
                lan.copy_(-F.softplus(raw.log_alpha.float()))
                bn.copy_(torch.sigmoid(raw.beta.float()))
                kda.chunk_fwd(qn, kn, raw.v, lan, bn, init_state=raw.init_state, C=64, workspace=ws, algo=a.algo)

            for _ in range(a.warmup):
                flush.zero_()
                unfused_step()
            uev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(a.steps)]
            barrier()
            torch.cuda.synchronize()
            for i in range(a.steps):
                flush.zero_()
                uev[i][0].record(stream)
                unfused_step()
                uev[i][1].record(stream)
            torch.cuda.synchronize()
            barrier()
            u_total = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in uev))
            del qn, kn, lan, bn, ws, raw
            sep = 2 * g4.token_heads * (3 * D + 1) * 2
            prep["prefill"] = {
                "value": job_throughput(world, g4.tokens, 1, msp), "unit": "tokens/s", "ms_per_step": msp,
                "added_ms_vs_plain": msp - ms4,
                "kernel_times": {namesp[j]: {"avg_us": kp[j] * 1e3} for j in range(len(namesp))},
                "separate_pass_bytes": sep, "separate_pass_min_ms": sep / (pk["hbm_gbs"] * 1e9) * 1e3,
                "unfused_torch_ms_per_step": u_total / a.steps,
                "config": {"workload": f"prefill B={p['B']} H={p['H']} T={p['T']} d=128 C=64 bf16, raw q/k "
                           "(unnormalised), gate logits, beta logits; flags QK_L2NORM|GATE_SOFTPLUS|BETA_SIGMOID",
                           "l2": "flushed before every timed step (256 MiB write)"}}

    # ---------------------------------------------------------------- backward (B=4 workload)
    bwd = None
    if b4_inp is not None and not a.no_bwd:
        p = PREFILL_B4
        B, T, H = p["B"], p["T"], p["H"]
        d_o, dfs = make_grad_outputs(b4_inp, seed=rank)
        grads = (torch.empty_like(b4_inp.q), torch.empty_like(b4_inp.k), torch.empty_like(b4_inp.v),
                 torch.empty_like(b4_inp.log_alpha), torch.empty_like(b4_inp.beta),
                 torch.empty_like(b4_inp.init_state))
        bws = torch.empty(kda.bwd_workspace_size(B, T, H, D, D, 64), dtype=torch.uint8, device=dev)
        nb = len(kda.BWD_TIMED)

        def bwd_step(evs=None):
            if evs is not None:
                kda.set_timing_events(evs)
            kda.chunk_bwd(b4_inp.q, b4_inp.k, b4_inp.v, b4_inp.log_alpha, b4_inp.beta, d_o,
                          init_state=b4_inp.init_state, d_final_state=dfs, C=64, grads=grads, workspace=bws)

        for _ in range(a.warmup):
            flush.zero_()
            bwd_step()
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(nb + 1)] for _ in range(a.steps)]
        for row in bev:
            for e in row:
                e.record(stream)
        barrier()
        torch.cuda.synchronize()
        for i in range(a.steps):
            flush.zero_()
            bwd_step(bev[i])
        torch.cuda.synchronize()
        barrier()
        b_total = max_over_ranks(sum(bev[i][0].elapsed_time(bev[i][nb]) for i in range(a.steps)))
        b_avg = [statistics.mean(bev[i][j].elapsed_time(bev[i][j + 1]) for i in range(a.steps)) for j in range(nb)]
        # an interval with no kernel (the events' own gap) is added to the one before it
        b_times = {}
        last = None
        for lab, t in zip(kda.bwd_timed(torch.bfloat16, D, D), b_avg):
            if lab is None:
                b_times[last]["avg_us"] += t * 1e3
                continue
            b_times[lab] = {"avg_us": t * 1e3}
            last = lab
        for v in b_times.values():
            v["share"] = v["avg_us"] / max(sum(w["avg_us"] for w in b_times.values()), 1e-12)
        tok_h = B * T * H
        min_bwd = tok_h * ((3 * D + D + 1) * 2 + D * 2 + (3 * D + D + 1) * 2) + 3 * B * H * D * D * 4
        b_ms = b_total / a.steps
        bwd = {"value": job_throughput(world, B * T, a.steps, b_total), "unit": "tokens/s", "ms_per_step": b_ms,
               "kernel_times": b_times,
               "path_roofline": {"minimal_bytes": min_bwd,
                                 "time_min_us": min_bwd / (pk["hbm_gbs"] * 1e9) * 1e6,
                                 "frac_of_hbm_bound": min_bwd / (pk["hbm_gbs"] * 1e9) / (b_ms / 1e3)},
               "gpu_launches": len(kda.bwd_kernels(torch.bfloat16, D, D)) * a.steps,
               "config": {"workload": f"backward of the prefill B={B} H={H} T={T} d=128 (d_o ~ N(0,1) bf16, "
                                      "d_final_state ~ N(0, 0.1^2))",
                          "l2": "flushed before every timed step (256 MiB write)"}}
        del grads, bws, d_o, dfs
    if b4_inp is not None:
        del b4_inp

    # ---------------------------------------------------------------- T = 65536, C = 64 and C = 128
    long = None
    if run_prefill and extras and not a.no_long:
        p = LONG
        linp = make_prefill("long", device=dev, seed=rank)
        gl = Geometry([p["T"]], p["H"])
        long = {"config": {"workload": "one sequence B=1 H=32 T=65536 d_k=d_v=128 bf16, head 0 alpha=1, head 1 "
                                       "scalar alpha; inputs larger than L2, no flush"}}
        runs = [("tc", 64, a.steps), ("tc", 128, a.steps), ("simt", 128, max(3, min(a.steps, 5)))]
        for algo, C, n in runs:
            msl, nl, kl = time_prefill(linp, C, algo, steps=n)
            C_run = 64 if algo == "tc" else C
            rl, tl, pl, ktl = prefill_report(gl, C, C_run, nl, kl, msl, pk, sm_guess)
            chain = {"tc": "tc_recur", "simt": "k3_state"}[algo]
            n_chunks = (p["T"] + C_run - 1) // C_run
            long[f"{algo}_C{C}"] = {"value": job_throughput(world, gl.tokens, 1, msl), "unit": "tokens/s",
                                    "ms_per_step": msl, "chunk_computed": C_run, "roofline": rl, "tensor": tl,
                                    "path_roofline": pl, "kernel_times": ktl,
                                    "state_carry_us_per_chunk_step": ktl[chain]["avg_us"] / n_chunks,
                                    "steps": n}
        del linp

    # ---------------------------------------------------------------- sequence parallelism
    seqp = None
    if run_prefill and extras and not a.no_seqpar and (world == 1 or a.seqpar):
        from kimi_delta_attention_30_b200 import seqpar
        Tl, Hl = 65536, 32
        nseg = world if world > 1 else 8
        seg = Tl // nseg
        sin = make_prefill("prefill", device=dev, seed=rank, B=1, T=seg, H=Hl)
        args5 = (sin.q, sin.k, sin.v, sin.log_alpha, sin.beta)

        def timed(fn, n):
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            for _ in range(a.warmup):
                flush.zero_()
                fn()
            barrier()
            torch.cuda.synchronize()
            for e0, e1 in evs:
                flush.zero_()
                e0.record(stream)
                fn()
                e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            return max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs)) / n

        if world > 1:
            ms = timed(lambda: seqpar.seqpar_forward(*args5, init_state=sin.init_state[:1]), a.steps)
            seqp = {"value": Tl / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "measured": True}
        else:
            s0 = sin.init_state[:1].contiguous()
            ms_maps = timed(lambda: seqpar.segment_maps(*args5), a.steps)
            ms_pass = timed(lambda: kda.chunk_fwd(*args5, init_state=s0), a.steps)
            full = make_prefill("prefill", device=dev, seed=rank, B=1, T=Tl, H=Hl)
            ms_full = timed(lambda: kda.chunk_fwd(full.q, full.k, full.v, full.log_alpha, full.beta,
                                                  init_state=full.init_state[:1]), a.steps)
            del full
            seqp = {"measured": False, "projected_ranks": nseg, "ms_maps_one_segment": ms_maps,
                    "ms_prefill_one_segment": ms_pass, "projected_ms_per_rank": ms_maps + ms_pass,
                    "single_gpu_ms": ms_full, "projected_speedup": ms_full / (ms_maps + ms_pass),
                    "note": "per-rank critical path without the all-gather (2 MiB per rank)"}
        seqp["config"] = {"workload": f"one sequence T={Tl} H={Hl} d=128 bf16 split into {nseg} segments"}
        del sin

    # ---------------------------------------------------------------- decode
    decode = None
    if run_decode:
        d = DECODE
        state = make_decode_state("decode", device=dev, seed=rank, N=d["N"])
        toks = [make_decode_token("decode", step=s, device=dev, seed=rank, N=d["N"]) for s in range(d["steps"])]
        od = torch.empty((d["N"], d["H"], d["dv"]), dtype=torch.bfloat16, device=dev)

        def decode_round(evs=None, tk=toks, flags=0):
            for s in range(d["steps"]):
                t = tk[s]
                if evs is not None:
                    evs[s][0].record(stream)
                kda.decode_step(t.q, t.k, t.v, t.log_alpha, t.beta, state, o=od, prep=flags)
                if evs is not None:
                    evs[s][1].record(stream)

        def timed_rounds(**kw):
            for _ in range(a.warmup):
                decode_round(**kw)
            dev_ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(d["steps"])]
                      for _ in range(a.steps)]
            barrier()
            torch.cuda.synchronize()
            for i in range(a.steps):
                decode_round(dev_ev[i], **kw)
            torch.cuda.synchronize()
            barrier()
            return max_over_ranks(sum(e[0].elapsed_time(e[1]) for r in dev_ev for e in r))

        dtot = timed_rounds()
        n_launch = a.steps * d["steps"]
        us = dtot / n_launch * 1e3
        st_bytes = d["N"] * d["H"] * d["dk"] * d["dv"] * 4
        tok_bytes = d["N"] * d["H"] * ((3 * d["dk"] + 2 * d["dv"]) * 2 + 2)
        alg = 2 * st_bytes + tok_bytes
        gbs = alg / (us * 1e-6) / 1e9
        decode = {"value": job_throughput(world, d["N"], n_launch, dtot), "unit": "tokens/s",
                  "us_per_step": us, "hbm_gbs": gbs,
                  "roofline": {"kernel": "decode_kernel", "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": gbs / pk["hbm_gbs"], "traffic": None,
                               "algorithmic_bytes": alg, "frac_of_8TBs_spec": gbs / 8000.0},
                  "config": {"workload": f"decode N={d['N']} H={d['H']} d={d['dk']} fp32 state, bf16 tokens, "
                             f"{d['steps']} consecutive steps", "l2": "state 512 MiB > L2"},
                  "gpu_launches": n_launch}
        if prep is not None:
            del toks
            raw_toks = [make_decode_token("decode_raw", step=s, device=dev, seed=rank, N=d["N"])
                        for s in range(d["steps"])]
            ptot = timed_rounds(tk=raw_toks, flags=RAW_PREP)
            pus = ptot / n_launch * 1e3
            prep["decode"] = {"value": job_throughput(world, d["N"], n_launch, ptot), "unit": "tokens/s",
                              "us_per_step": pus, "hbm_gbs": alg / (pus * 1e-6) / 1e9,
                              "added_us_vs_plain": pus - us,
                              "config": {"workload": f"decode N={d['N']} H={d['H']} d={d['dk']} raw bf16 tokens, "
                                         "flags QK_L2NORM|GATE_SOFTPLUS|BETA_SIGMOID"}}
            del raw_toks
        del state

    clk = clocks.stop() if rank == 0 else None
    if clk and clk.get("sm_mhz") and kernel_table:
        # tensor-pipe estimates at the clock seen during the run
        for tab in [kernel_table] + ([b4["kernel_times"]] if b4 else []) + \
                   ([v["kernel_times"] for kk, v in long.items() if kk != "config"] if long else []):
            for e in tab.values():
                if "tensor_pipe_pct_est" in e:
                    e["tensor_pipe_pct_est"] *= sm_guess / clk["sm_mhz"]

    # ---------------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and run_prefill and not a.no_cpu:
        smp = OracleSample(a.cpu_seconds)
        dt = smp.time()
        cpu = {"value": smp.tokens() / dt, "unit": "tokens/s", "cores": smp.threads, "kind": "oracle",
               "sample": smp.describe(dt), "single_core": smp.single_core()}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
                "warmup": a.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": headline,
                "roofline": roofline, "tensor": tensor, "path_roofline": path_roofline,
                "kernel_times": kernel_table, "gpu_launches": gpu_launches,
                "prefill_b4": b4, "long": long, "decode": decode, "prep": prep, "backward": bwd, "seqpar": seqp,
                "e2e": e2e, "cpu_baseline": cpu,
                "clocks": clk, "gpu": props.name}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
