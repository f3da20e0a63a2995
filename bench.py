#!/usr/bin/env python
"""KDA benchmark: prefill tokens/s (headline) and decode tokens/s on one B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one ``kda_chunk_fwd`` over the prefill workload (B=4, H=16, T=4096,
d_k=d_v=128, chunk 64, bf16 inputs, fp32 state), inputs resident in HBM; L2 is
flushed (256 MiB write) before every timed step and each step is timed with
CUDA events on the launching stream.  In the same run: the decode workload
(256 sequences x 32 heads, d=128, fp32 state, 64 consecutive steps per bench
step, timed per launch), the end-to-end prefill through the public API with
pinned host buffers (H2D inputs + D2H outputs inside the timed region), and the
fp64 oracle on a bounded sample on the host cores (rank 0, N = 1).  The
"prep" object times the same prefill and decode launches on raw inputs with the
input preprocessing fused in (``kda_chunk_fwd_prep`` / ``kda_decode_step_prep``:
q/k L2 norm, -softplus gate, sigmoid beta).

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

PREFILL = dict(B=4, T=4096, H=16, dk=128, dv=128, C=64)
DECODE = dict(N=256, H=32, dk=128, dv=128, steps=64)
METRIC = "KDA prefill tokens/s (B=4 H=16 T=4096 d=128 C=64 bf16); decode tokens/s + HBM GB/s"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prep", action="store_true", help="skip the fused-preprocessing timings")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward-pass timings")
    ap.add_argument("--no-seqpar", action="store_true", help="skip the sequence-parallel timings")
    ap.add_argument("--seqpar", action="store_true",
                    help="with N > 1 ranks, also time one long sequence split over the ranks (NCCL all-gather)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle sample length")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode"],
                    help="profiling aid: run only one part (the JSON line then lacks the other)")
    ap.add_argument("--decode-n", type=int, default=DECODE["N"], help="profiling aid: decode sequences")
    ap.add_argument("--prefill-b", type=int, default=PREFILL["B"], help="profiling aid: prefill batch")
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


# ----------------------------------------------------------------------------- algorithmic bytes

def kernel_bytes(name, B, T, H, dk, dv, C, in_bytes=2):
    """Bytes each kernel must move by design (inputs read once, outputs written once)."""
    tok = B * T * H
    n_chunks = B * ((T + C - 1) // C)
    st = B * H * dk * dv * 4
    schunk = n_chunks * H * dk * dv * 4
    # workspace per token-head of the tensor-core path: Wk, Q exp(g), Kd (hi+lo bf16, 4 B per
    # channel each), U (fp32), one row of P (hi+lo bf16, C entries)
    ws_tok = 3 * 4 * dk + 4 * dv + 4 * C
    table = {
        "tc_intra": tok * ((3 * dk + dv) * in_bytes + in_bytes) + tok * ws_tok + n_chunks * H * dk * 4,
        "tc_recur": tok * ws_tok + n_chunks * H * dk * 4 + tok * dv * in_bytes + 2 * st,
        "k1_cumsum": tok * dk * (in_bytes + 4),
        "k2_wy": tok * (2 * dk * in_bytes + dv * in_bytes + in_bytes + 4 * dk) + tok * 4 * (dv + dk),
        "k3_state": tok * (4 * dk + 4 * dv + in_bytes * dk + 4 * dk) + tok * 4 * dv + schunk + 2 * st,
        "k4_output": tok * (2 * dk * in_bytes + 4 * dk + 4 * dv + dv * in_bytes) + schunk,
    }
    return table.get(name)


def algorithmic_flops(B, T, H, dk, dv, C):
    """FLOPs of the chunk algorithm per call, masked work counted once:
    6 dk dv + C (3 dk + 2 dv) + C^2 / 3 per token-head."""
    return B * T * H * (6 * dk * dv + C * (3 * dk + 2 * dv) + C * C / 3)


def minimal_bytes(B, T, H, dk, dv, in_bytes=2, with_state=True):
    """q, k, v, log alpha, beta in; o out; initial and final state."""
    tok = B * T * H
    b = tok * ((2 * dk + dv + dk + 1) * in_bytes + dv * in_bytes)
    if with_state:
        b += 2 * B * H * dk * dv * 4
    return b


def separate_prep_bytes(n_tok_heads, dk, in_bytes=2):
    """A stand-alone preprocessing pass: read raw q, k, gate (dk each) and beta,
    write them back processed."""
    return 2 * n_tok_heads * (3 * dk + 1) * in_bytes


def measured_traffic(kernel, B, T, H, C, workload="prefill"):
    """DRAM bytes per launch of `kernel` on this workload from the committed ncu
    table, or None when there is none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    csrc = os.path.join(ROOT, "kimi_delta_attention_30_b200", "csrc")
    h = hashlib.sha256()
    for f in ("kda_chunk_tc.cu", "kda_tc.cuh", "kda_internal.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    want = f"{workload}_b{B}_h{H}_t{T}_c{C}"
    for line in open(path):
        f = line.split()
        if len(f) == 5 and not line.startswith("#") and f[0] == kernel and f[1] == want and f[4] == digest:
            return int(f[2]) + int(f[3])
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- oracle timing

class OracleSample:
    """The fp64 oracle timed on whole prefill sequences (T = 4096) of the prefill
    workload: one (sequence, head) pair per host thread, as many pairs as fit
    about `seconds` of wall time (at most the workload's 64 pairs); when all 64
    take less than that, the whole workload is repeated to fill it.  Inputs are
    drawn once; each call of :meth:`time` reruns the oracle on them."""

    def __init__(self, seconds: float, seed: int = 0):
        import oracle
        from kda_inputs import make_prefill, to_f64
        self.oracle = oracle
        self.threads = oracle.max_threads()
        T, H = PREFILL["T"], PREFILL["H"]
        self.T, self.H = T, H
        inp = make_prefill("prefill", B=1, T=T, H=64, seed=seed)
        f = lambda t: to_f64(t).reshape(T, 64, -1)
        self.full = (f(inp.q), f(inp.k), f(inp.v), f(inp.log_alpha), to_f64(inp.beta).reshape(T, 64),
                     to_f64(inp.init_state))
        self.seq = inp.seq_start
        self.n_pairs, self.reps = 1, 1
        t1 = self.time()
        n = max(1, min(64, int(self.threads * max(1.0, seconds / max(t1, 1e-3)))))
        if n > self.threads:
            n -= n % self.threads              # whole waves of threads
        self.n_pairs = n
        if n == 64:
            self.reps = max(1, int(round(seconds / max(self.time(), 1e-3))))

    def time(self) -> float:
        n = self.n_pairs
        q, k, v, la, beta, s0 = self.full
        args = (q[:, :n], k[:, :n], v[:, :n], la[:, :n], beta[:, :n])
        t0 = time.perf_counter()
        for _ in range(self.reps):
            self.oracle.forward(*args, self.seq, init_state=s0[:, :n], n_threads=self.threads)
        return time.perf_counter() - t0

    def tokens(self) -> float:
        return self.reps * self.n_pairs * self.T / self.H      # a token carries all H heads

    def single_core(self) -> dict:
        """One (sequence, head) pair on one thread (tokens/s in full H-head tokens)."""
        q, k, v, la, beta, s0 = self.full
        t0 = time.perf_counter()
        self.oracle.forward(q[:, :1], k[:, :1], v[:, :1], la[:, :1], beta[:, :1], self.seq, init_state=s0[:, :1],
                            n_threads=1)
        dt = time.perf_counter() - t0
        return {"value": self.T / self.H / dt, "unit": "tokens/s", "cores": 1,
                "sample": f"1 (sequence, head) pair x {self.T} tokens, {dt:.2f} s"}

    def describe(self, dt: float) -> str:
        return (f"{self.n_pairs} (sequence, head) pairs x {self.T} tokens of the prefill workload"
                f"{f', {self.reps} passes' if self.reps > 1 else ''} "
                f"(= {self.tokens():.0f} full {self.H}-head tokens), fp64 token recurrence, "
                f"{self.threads} threads, {dt:.1f} s")


def run_reference(a, world, rank):
    """Reference arm: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return
    steps = a.warmup + a.steps
    smp = OracleSample(max(0.5, min(8.0, 120.0 / steps)))
    vals, dts = [], []
    for i in range(steps):
        dt = smp.time()
        if i >= a.warmup:
            vals.append(smp.tokens() / dt)
            dts.append(dt)
    value = statistics.mean(vals)
    p = PREFILL
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": statistics.mean(dts) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"prefill B={p['B']} H={p['H']} T={p['T']} d_k=d_v={p['dk']} C={p['C']} bf16 inputs, fp32 state",
                       "sample": "each step: the oracle on a bounded sample of the workload"},
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
    from kda_inputs import RAW_PREP, make_decode_state, make_decode_token, make_grad_outputs, make_prefill

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
    p = PREFILL
    B, T, H, dk, dv, C = a.prefill_b, p["T"], p["H"], p["dk"], p["dv"], p["C"]
    DECODE["N"] = a.decode_n

    run_prefill = a.only in ("all", "prefill")
    run_decode = a.only in ("all", "decode") and not a.no_decode
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(gpu_id if rank == 0 else None)
    value = ms_per_step = roofline = path_roofline = kernel_table = t_wall = None
    kernels, nk = [], 0
    run_prep = not a.no_prep and a.algo in ("auto", "tc")
    prep = {} if run_prep else None
    if run_prefill:
        inp = make_prefill("prefill", device=dev, seed=rank, B=B)
        kernels = kda.chunk_kernels(B, T, H, dk, dv, C, torch.bfloat16, algo=a.algo)
        nk = len(kernels)
        ws = torch.empty(kda.workspace_size(B, T, H, dk, dv, C, torch.bfloat16, algo=a.algo), dtype=torch.uint8,
                         device=dev)
        o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
        fs = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
        flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB > L2

        def prefill_step(evs=None):
            if evs is not None:
                kda.set_timing_events(evs)
            kda.chunk_fwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, init_state=inp.init_state, C=C, o=o,
                          final_state=fs, workspace=ws, algo=a.algo)

        for _ in range(a.warmup):
            flush.zero_()
            prefill_step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(a.steps)]
        for row in ev:            # torch creates the CUDA event on its first record
            for e in row:
                e.record(stream)
        barrier()
        torch.cuda.synchronize()
        t_wall = time.perf_counter()
        for i in range(a.steps):
            flush.zero_()
            prefill_step(ev[i])
        torch.cuda.synchronize()
        barrier()
        t_wall = time.perf_counter() - t_wall
        step_ms = [ev[i][0].elapsed_time(ev[i][nk]) for i in range(a.steps)]
        k_ms = [[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(a.steps)] for j in range(nk)]
        total_ms = max_over_ranks(sum(step_ms))
        ms_per_step = total_ms / a.steps
        tokens = B * T
        value = job_throughput(world, tokens, a.steps, total_ms)
        k_avg = [statistics.mean(x) for x in k_ms]
        dom = max(range(nk), key=lambda j: k_avg[j])
        dom_bytes = kernel_bytes(kernels[dom], B, T, H, dk, dv, C)
        kernel_table = {kernels[j]: {"avg_us": k_avg[j] * 1e3, "share": k_avg[j] / max(sum(k_avg), 1e-12)}
                        for j in range(nk)}
        roofline = None
        if dom_bytes is not None:
            ach = dom_bytes / (k_avg[dom] / 1e3) / 1e9
            roofline = {"kernel": kernels[dom], "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / pk["hbm_gbs"], "traffic": measured_traffic(kernels[dom], B, T, H, C),
                        "algorithmic_bytes": dom_bytes,
                        "peak_source": pk["source"]}
        min_b = minimal_bytes(B, T, H, dk, dv)
        flops = algorithmic_flops(B, T, H, dk, dv, C)
        t_hbm = min_b / (pk["hbm_gbs"] * 1e9)
        t_tc = flops / (pk["bf16_tflops"] * 1e12)
        path_roofline = {"minimal_bytes": min_b, "time_min_us": max(t_hbm, t_tc) * 1e6,
                         "frac_of_hbm_bound": t_hbm / (ms_per_step / 1e3),
                         "algorithmic_flops": flops, "tflops": flops / (ms_per_step / 1e3) / 1e12,
                         "frac_of_tensor_peak": flops / (ms_per_step / 1e3) / (pk["bf16_tflops"] * 1e12),
                         "time_min_over_time": max(t_hbm, t_tc) / (ms_per_step / 1e3)}

        # ------------------------------------------------ prefill, preprocessing fused
        if run_prep:
            raw = make_prefill("prefill_raw", device=dev, seed=rank, B=B)

            def prep_step(evs=None):
                if evs is not None:
                    kda.set_timing_events(evs)
                kda.chunk_fwd(raw.q, raw.k, raw.v, raw.log_alpha, raw.beta, init_state=raw.init_state, C=C, o=o,
                              final_state=fs, workspace=ws, algo=a.algo, prep=RAW_PREP)

            for _ in range(a.warmup):
                flush.zero_()
                prep_step()
            pev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(a.steps)]
            for row in pev:
                for e in row:
                    e.record(stream)
            barrier()
            torch.cuda.synchronize()
            for i in range(a.steps):
                flush.zero_()
                prep_step(pev[i])
            torch.cuda.synchronize()
            barrier()
            p_total = max_over_ranks(sum(pev[i][0].elapsed_time(pev[i][nk]) for i in range(a.steps)))
            pk_avg = [statistics.mean(pev[i][j].elapsed_time(pev[i][j + 1]) for i in range(a.steps))
                      for j in range(nk)]
            # the unfused alternative: torch kernels preprocess into bf16 buffers, then the plain operator
            F = torch.nn.functional
            qn, kn, lan, bn = (torch.empty_like(t) for t in (raw.q, raw.k, raw.log_alpha, raw.beta))

            def unfused_step():
                qn.copy_(F.normalize(raw.q.float(), dim=-1))
                kn.copy_(F.normalize(raw.k.float(), dim=-1))
                lan.copy_(-F.softplus(raw.log_alpha.float()))
                bn.copy_(torch.sigmoid(raw.beta.float()))
                kda.chunk_fwd(qn, kn, raw.v, lan, bn, init_state=raw.init_state, C=C, o=o, final_state=fs,
                              workspace=ws, algo=a.algo)

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
            del qn, kn, lan, bn
            sep = separate_prep_bytes(tokens * H, dk)
            prep["prefill"] = {
                "value": job_throughput(world, tokens, a.steps, p_total), "unit": "tokens/s",
                "ms_per_step": p_total / a.steps, "added_ms_vs_plain": p_total / a.steps - ms_per_step,
                "kernel_times": {kernels[j]: {"avg_us": pk_avg[j] * 1e3,
                                              "traffic": measured_traffic(kernels[j], B, T, H, C, "prefill_raw")}
                                 for j in range(nk)},
                "separate_pass_bytes": sep, "separate_pass_min_ms": sep / (pk["hbm_gbs"] * 1e9) * 1e3,
                "unfused_torch_ms_per_step": u_total / a.steps,
                "config": {"workload": f"prefill B={B} H={H} T={T} d={dk} C={C} bf16, raw q/k (unnormalised), "
                           "gate logits, beta logits; flags QK_L2NORM|GATE_SOFTPLUS|BETA_SIGMOID",
                           "l2": "flushed before every timed step (256 MiB write)"}}
            del raw

    # ---------------------------------------------------------------- backward
    bwd = None
    if run_prefill and not a.no_bwd:
        d_o, dfs = make_grad_outputs(inp, seed=rank)
        grads = (torch.empty_like(inp.q), torch.empty_like(inp.k), torch.empty_like(inp.v),
                 torch.empty_like(inp.log_alpha), torch.empty_like(inp.beta), torch.empty_like(inp.init_state))
        bws = torch.empty(kda.bwd_workspace_size(B, T, H, dk, dv, C), dtype=torch.uint8, device=dev)
        nb = len(kda.BWD_TIMED)

        def bwd_step(evs=None):
            if evs is not None:
                kda.set_timing_events(evs)
            kda.chunk_bwd(inp.q, inp.k, inp.v, inp.log_alpha, inp.beta, d_o, init_state=inp.init_state,
                          d_final_state=dfs, C=C, grads=grads, workspace=bws)

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
        # minimal traffic of a backward pass: the forward's inputs and d_o in, five gradients out, plus the
        # initial state, the final-state gradient and the initial-state gradient
        tok_h = tokens * H
        min_bwd = tok_h * ((3 * dk + dv + 1) * 2 + dv * 2 + (3 * dk + dv + 1) * 2) + 3 * B * H * dk * dv * 4
        b_ms = b_total / a.steps
        bwd = {"value": job_throughput(world, tokens, a.steps, b_total), "unit": "tokens/s", "ms_per_step": b_ms,
               "kernel_times": {kda.BWD_TIMED[j]: {"avg_us": b_avg[j] * 1e3, "share": b_avg[j] / max(sum(b_avg), 1e-12)}
                                for j in range(nb)},
               "path_roofline": {"minimal_bytes": min_bwd,
                                 "time_min_us": min_bwd / (pk["hbm_gbs"] * 1e9) * 1e6,
                                 "frac_of_hbm_bound": min_bwd / (pk["hbm_gbs"] * 1e9) / (b_ms / 1e3)},
               "gpu_launches": len(kda.bwd_kernels(torch.bfloat16, dk, dv)) * a.steps,
               "config": {"workload": f"backward of the prefill workload (B={B} H={H} T={T} d={dk}), d_o ~ N(0,1) "
                                      "bf16, d_final_state ~ N(0, 0.1^2); recompute on the tensor-core forward, "
                                      "gradient kernels fp32 on CUDA cores, 64-token chunks",
                          "l2": "flushed before every timed step (256 MiB write)"}}
        del grads, bws, d_o, dfs

    # ---------------------------------------------------------------- sequence parallelism
    # one 65,536-token sequence (H = 32, d = 128, bf16) split into contiguous segments, one per
    # rank, start states exchanged by one all-gather of per-segment affine maps (seqpar.py).
    # With N > 1 ranks this is measured when --seqpar is given (the replicas' scaling line does not
    # depend on it); on one GPU the per-rank critical path of an 8-way split
    # (maps of one segment, then its prefill from the start state) is timed and reported as a
    # projection beside the single-GPU prefill of the whole sequence.
    seqp = None
    if run_prefill and not a.no_seqpar and (world == 1 or a.seqpar):
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
        if run_prep:
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

    # ---------------------------------------------------------------- end to end
    e2e = None
    if run_prefill and not a.no_e2e:
        host = {n: getattr(inp, n).to("cpu").pin_memory() for n in ("q", "k", "v", "log_alpha", "beta")}
        host["init_state"] = inp.init_state.to("cpu").pin_memory()
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        fs_h = torch.empty(fs.shape, dtype=fs.dtype).pin_memory()
        dbuf = {n: torch.empty_like(getattr(inp, n)) for n in ("q", "k", "v", "log_alpha", "beta", "init_state")}
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_h.numel() * o_h.element_size() + fs_h.numel() * fs_h.element_size()

        def e2e_step():
            for n, t in host.items():
                dbuf[n].copy_(t, non_blocking=True)
            kda.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"],
                          init_state=dbuf["init_state"], C=C, o=o, final_state=fs, workspace=ws, algo=a.algo)
            o_h.copy_(o, non_blocking=True)
            fs_h.copy_(fs, non_blocking=True)

        for _ in range(a.warmup):
            e2e_step()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(a.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        et = max_over_ranks(e0.elapsed_time(e1))
        e2e = {"value": job_throughput(world, tokens, a.steps, et), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": et / a.steps}

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
                "config": {"workload": f"prefill B={B} H={H} T={T} d_k=d_v={dk} C={C} bf16 inputs, fp32 state",
                           "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "C": C, "algo": a.algo,
                           "kernels": kernels, "l2": "flushed before every timed step (256 MiB write)",
                           "parallelism": f"replicas x{world} (independent sequences per GPU)"},
                "roofline": roofline, "path_roofline": path_roofline, "kernel_times": kernel_table,
                "gpu_launches": nk * a.steps if run_prefill else None, "decode": decode, "prep": prep, "backward": bwd, "seqpar": seqp,
                "e2e": e2e, "cpu_baseline": cpu,
                "clocks": clk, "wall_s_timed": t_wall, "gpu": props.name}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
