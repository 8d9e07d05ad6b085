#!/usr/bin/env python
"""Benchmark of the retention hot path on B200, one JSON line on stdout.

Step: one chunkwise retention forward (xPos, QK^T/sqrt(d), D~) over one batch of the
workload "chunkwise forward bf16: batch 8, d_model 1024, h 8, d_k = d_v = 128, seq 2048,
chunk 64", raw output in bf16, through the C interface.  value = tokens/s of the whole job.
Inputs rotate over 4 resident sets (4 x 134 MB > the 126 MB L2), so no step re-reads the
previous step's operands from L2.

Alongside the step (1 GPU only), the same line carries: the decode step on the workload
"batch 64, h 16, d_k 256, d_v 512, fp32 state" (state GB/s), and, where enabled, the
long-sequence and MSR workloads.  --impl reference times the fp64 CPU oracle instead.

Multi-GPU (one process per GPU): every rank runs its own batch (weak scaling); the path has no
exchange step, so the only collectives of the timed step are the barrier and the max of the
timed durations.  `--gpus N` without a torchrun environment relaunches this script under
torch.distributed.run with N processes; a run whose world size differs from --gpus fails.  The
sequence-sharded leg (`seqshard`) runs one long sequence cut into one shard per rank, whose
states cross ranks in one all-gather (the path's only real exchange).
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

MAIN = dict(workload="chunkwise_fwd_bf16_b8_L2048_h8_dk128_dv128_B64", batch=8, seqlen=2048, heads=8, d_k=128,
            d_v=128, chunk=64)
DECODE = dict(workload="decode_step_b64_h16_dk256_dv512_fp32state", batch=64, heads=16, d_k=256, d_v=512)
LONG = dict(workload="chunkwise_fwd_bf16_b2_L8192_h16_dk256_dv512", batch=2, seqlen=8192, heads=16, d_k=256, d_v=512)
MSR = dict(workload="msr_fwd_bf16_b4_L4096_h8_dk256_dv256_B256", batch=4, seqlen=4096, heads=8, d_k=256, d_v=256,
           chunk=256)
FLAGS = 1 | 2 | 4  # XPOS | SCALE_SQRT_D | NORM_D
N_SETS = 4


def flops_per_token_head(dk, dv, B):
    """Algorithmic FLOPs: causal inner-chunk QK^T and PV, cross-chunk Q R, state update K^T V."""
    return (dk + dv) * (B + 1) + 4 * dk * dv


def bytes_per_token_head(dk, dv, elt=2):
    """Algorithmic HBM bytes: read q, k, v, write o, each once."""
    return elt * (2 * dk + 2 * dv)


def ncu_traffic(name):
    """DRAM bytes per launch from the committed ncu record, if the kernel's sources still hash
    to the profiled version (else None: the counters no longer describe the compiled kernels)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[name]
        h = hashlib.sha256()
        for f in rec["sources"]:
            h.update(open(os.path.join(ROOT, f), "rb").read())
        return rec["dram_bytes_per_launch"] if h.hexdigest()[:16] == rec["hash"] else None
    except (OSError, KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


# ---- clocks during the timed region ----------------------------------------------------------

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML every 10 ms (read-only)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        self.samples = []
        self.ok = False
        self.marks = []
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self):
        self.marks.append(time.perf_counter())

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(win) < 3:  # the timed region is shorter than a few samples: use the whole run
            win = self.samples
            window = "whole benchmark run (timed region shorter than the sampling interval)"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = sorted({name for _, _, r in win for name, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(m for _, m, _ in win), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(win), "window": window}


# ---- distributed plumbing --------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---- our arm -------------------------------------------------------------------------------

def make_main_inputs(cfg, device, rank):
    import torch

    import synth_inputs as si
    sets = []
    for i in range(N_SETS):
        q, k, v = si.qkv(cfg["batch"], cfg["seqlen"], cfg["heads"], cfg["d_k"], cfg["d_v"], 2 + 100 * rank + i,
                         "bf16")
        o = torch.empty(cfg["batch"], cfg["seqlen"], cfg["heads"], cfg["d_v"], dtype=torch.bfloat16, device=device)
        sets.append((q.to(device), k.to(device), v.to(device), o))
    return sets


def run_chunkwise(rn, s, cfg, gamma, theta, stream, ws):
    """One step: the chunkwise call with its workspace (allocated once by the caller)."""
    q, k, v, o = s
    rn.retnet_retention_chunkwise_ws(q, k, v, o, gamma, theta, 0, FLAGS, cfg["chunk"], workspace=ws, stream=stream)


def time_steps(fn, steps, stream):
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        fn(i)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3  # seconds


def bench_decode(rn, device, stream, steps, warmup, peaks):
    import torch

    import synth_inputs as si
    c = DECODE
    b, h, dk, dv = c["batch"], c["heads"], c["d_k"], c["d_v"]
    S = si.decode_state(b, h, dk, dv, 4).to(device)
    toks = []  # new q, k, v for every step, as the workload states (the same draws as the parity test)
    for t in range(steps + warmup):
        q, k, v = si.decode_token(b, h, dk, dv, 4, t)
        toks.append((q.to(device), k.to(device), v.to(device)))
    o = torch.empty(b, h, dv, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)

    def step(i):
        q, k, v = toks[i]
        rn.retnet_retention_step(q, k, v, o, S, g, th, i, FLAGS, None, stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    secs = time_steps(lambda i: step(warmup + i), steps, stream)
    per = secs / steps
    state_bytes = 2 * b * h * dk * dv * 4
    io_bytes = b * h * (2 * dk + dv) * 2 + b * h * dv * 4
    gbs = (state_bytes + io_bytes) / per / 1e9
    return {"workload": c["workload"], "steps": steps, "positions": f"{warmup}..{warmup + steps - 1}",
            "us_per_step": per * 1e6,
            "bytes_per_step": state_bytes + io_bytes, "gbs": gbs, "frac_of_measured_hbm": gbs / peaks["hbm"],
            "frac_of_8tbs": gbs / 8000.0, "gpu_launches": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm"], "traffic": ncu_traffic("decode_step"),
                         "peak_source": peaks["source"]}}


def bench_long(rn, device, stream, steps, peaks):
    """Long-sequence chunkwise forward (chunks 128 and 512): TFLOP/s against the bf16 peak."""
    import torch

    import synth_inputs as si
    c = LONG
    b, L, h, dk, dv = c["batch"], c["seqlen"], c["heads"], c["d_k"], c["d_v"]
    q, k, v = si.qkv(b, L, h, dk, dv, 3, "bf16")
    q, k, v = q.to(device), k.to(device), v.to(device)
    o = torch.empty(b, L, h, dv, dtype=torch.bfloat16, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device=device)
    out = {"workload": c["workload"], "workspace_bytes": ws.numel()}
    for B in (128, 512):
        path = rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, g)
        launches = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g, ws.numel())

        def step(i):
            rn.retnet_retention_chunkwise_ws(q, k, v, o, g, th, 0, FLAGS, B, workspace=ws, stream=stream)

        for i in range(2):
            step(i)
        torch.cuda.synchronize()
        secs = time_steps(step, steps, stream) / steps
        flops = b * L * h * flops_per_token_head(dk, dv, B)
        byt = b * L * h * bytes_per_token_head(dk, dv)
        out[f"chunk{B}"] = {"us_per_step": secs * 1e6, "tokens_per_s": b * L / secs, "tflops": flops / secs / 1e12,
                            "frac_bf16_peak": flops / secs / 1e12 / peaks["bf16"], "gbs": byt / secs / 1e9,
                            "frac_hbm": byt / secs / 1e9 / peaks["hbm"],
                            "kernel": "tcgen05" if path == 1 else "fp32 CUDA cores",
                            "launches_per_step": launches, "gpu_launches": launches * steps}
    return out


def bench_msr(rn, device, stream, steps, peaks):
    """MSR forward (chunk 256, bf16 out): the fused kernel (retention, GroupNorm and swish gate
    in one tensor-core kernel per cluster of d_v slices), and beside it the two-kernel form
    (chunkwise retention to HBM, then the GroupNorm + gate kernel).  Both with split fp16
    operands, which the post-epilogue accuracy needs."""
    import torch

    import synth_inputs as si
    c = MSR
    b, L, h, dk, dv, B = c["batch"], c["seqlen"], c["heads"], c["d_k"], c["d_v"], c["chunk"]
    q, k, v = si.qkv(b, L, h, dk, dv, 5, "bf16")
    q, k, v = q.to(device), k.to(device), v.to(device)
    gt = si.gate(b, L, h, dv, 5, "bf16").to(device)
    y = torch.empty(b, L, h, dv, dtype=torch.bfloat16, device=device)
    out = torch.empty(b, L, h * dv, dtype=torch.bfloat16, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    path = rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS | rn.F_PRECISE, B, g)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device=device)
    two_launches = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS | rn.F_PRECISE, B, g,
                                                ws.numel()) + 1
    fused_launches = rn.retnet_msr_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, g, ws.numel())

    def two_kernel(i):
        rn.retnet_retention_chunkwise_ws(q, k, v, y, g, th, 0, FLAGS | rn.F_PRECISE, B, workspace=ws, stream=stream)
        rn.retnet_msr_epilogue(y.view(b, L, h * dv), gt, out, h, 1e-5, stream)

    def fused(i):
        rn.retnet_msr_chunkwise(q, k, v, gt.view(b, L, h, dv), out.view(b, L, h, dv), g, th, 0, FLAGS, B, 1e-5,
                                workspace=ws, stream=stream)

    flops = b * L * h * flops_per_token_head(dk, dv, B)
    res = {"workload": c["workload"], "workspace_bytes": ws.numel()}
    legs = [("two_kernel", two_kernel, two_launches, 4 * dv, "tcgen05 split operands + epilogue" if path == 1 else
             "fp32 CUDA cores + epilogue")]
    if fused_launches > 0:
        legs.insert(0, ("fused", fused, fused_launches, 2 * dv, "tcgen05 split operands, fused GroupNorm + gate"))
    for name, fn, launches, extra, kernel in legs:
        for i in range(2):
            fn(i)
        torch.cuda.synchronize()
        secs = time_steps(fn, steps, stream) / steps
        # algorithmic bytes: q, k, v, out (+ the gate; the two-kernel form also re-reads y and writes out)
        byt = b * L * h * (bytes_per_token_head(dk, dv) + extra)
        res[name] = {"us_per_step": secs * 1e6, "tokens_per_s": b * L / secs, "tflops": flops / secs / 1e12,
                     "frac_bf16_peak": flops / secs / 1e12 / peaks["bf16"], "gbs": byt / secs / 1e9,
                     "frac_hbm": byt / secs / 1e9 / peaks["hbm"], "kernel": kernel, "launches_per_step": launches,
                     "gpu_launches": launches * steps}
    return res


def bench_backward(rn, device, stream, steps, peaks):
    """Gradient of the forward (dq, dk, dv) on the headline workload, bf16 inputs, fp32 out, on
    the path the library takes (tensor cores: three runs of the chunkwise kernel), against the
    bf16 tensor peak with 2x the forward's algorithmic FLOPs (the usual backward/forward ratio)."""
    import torch

    import synth_inputs as si
    c = MAIN
    b, L, h, dk, dv, B = c["batch"], c["seqlen"], c["heads"], c["d_k"], c["d_v"], c["chunk"]
    q, k, v = si.qkv(b, L, h, dk, dv, 11, "bf16")
    q, k, v = q.to(device), k.to(device), v.to(device)
    do = si.randn((b, L, h, dv), 12, "bf16").to(device)
    dq, dk_ = torch.empty(b, L, h, dk, device=device), torch.empty(b, L, h, dk, device=device)
    dv_ = torch.empty(b, L, h, dv, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    ws = torch.empty(rn.retnet_backward_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device=device)
    path = rn.retnet_backward_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, g, ws.numel())
    launches = rn.retnet_backward_launches((b, L, h, dk), dv, rn.BF16, FLAGS, g, ws.numel())

    def step(i):
        rn.retnet_retention_backward(q, k, v, do, dq, dk_, dv_, g, th, 0, FLAGS, workspace=ws, stream=stream)

    step(0)
    torch.cuda.synchronize()
    secs = time_steps(step, steps, stream) / steps
    flops = 2 * b * L * h * flops_per_token_head(dk, dv, B)
    tf = flops / secs / 1e12
    return {"workload": "backward_" + c["workload"], "us_per_step": secs * 1e6, "tokens_per_s": b * L / secs,
            "tflops": tf, "frac_bf16_peak": tf / peaks["bf16"],
            "kernel": "tcgen05 (three chunkwise runs, fp16 value rows)" if path == 1 else "fp32 CUDA cores",
            "workspace_bytes": ws.numel(), "launches_per_step": launches, "gpu_launches": launches * steps}


def bench_flag_variants(rn, device, stream, steps, peaks, ws):
    """The headline workload with R~ (key-sum pass + split operands) and with split operands
    alone (RETNET_F_PRECISE), beside the timed step's single-copy operands."""
    import torch

    import synth_inputs as si
    c = MAIN
    b, L, h, dk, dv, B = c["batch"], c["seqlen"], c["heads"], c["d_k"], c["d_v"], c["chunk"]
    q, k, v = si.qkv(b, L, h, dk, dv, 2, "bf16")
    q, k, v = q.to(device), k.to(device), v.to(device)
    o = torch.empty(b, L, h, dv, dtype=torch.bfloat16, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    out = {"workload": c["workload"]}
    byt = b * L * h * bytes_per_token_head(dk, dv)
    for name, fl in (("norm_r", FLAGS | rn.F_NORM_R), ("precise", FLAGS | rn.F_PRECISE)):
        launches = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, fl, B, g, ws.numel())

        def step(i):
            rn.retnet_retention_chunkwise_ws(q, k, v, o, g, th, 0, fl, B, workspace=ws, stream=stream)

        for i in range(3):
            step(i)
        torch.cuda.synchronize()
        secs = time_steps(step, steps, stream) / steps
        out[name] = {"us_per_step": secs * 1e6, "tokens_per_s": b * L / secs, "gbs": byt / secs / 1e9,
                     "frac_hbm": byt / secs / 1e9 / peaks["hbm"], "launches_per_step": launches,
                     "gpu_launches": launches * steps}
    return out


def bench_seqshard(rn, device, stream, steps, world, rank):
    """One long sequence (b2 / L8192 / h16 / d_k 256 / d_v 512, chunk 128) cut into one shard
    per rank: each rank computes its shard's state, the states are all-gathered (NCCL), each
    rank folds the earlier ones into its start state and runs its shard (strong scaling: the
    sequence is fixed).  Timed on the device, max over ranks."""
    import torch

    import synth_inputs as si
    from linear_attention_sequence_chunkwise_b200 import seqshard
    c = LONG
    b, L, h, dk, dv, B = c["batch"], c["seqlen"], c["heads"], c["d_k"], c["d_v"], 128
    Ls = L // world
    q, k, v = si.qkv(b, Ls, h, dk, dv, 3 + 100 * rank, "bf16")
    q, k, v = q.to(device), k.to(device), v.to(device)
    o = torch.empty(b, Ls, h, dv, dtype=torch.bfloat16, device=device)
    so = torch.empty(b, h, dk, dv, dtype=torch.float32, device=device)
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)

    def step(i):
        seqshard.retention_chunkwise_sharded(q, k, v, o, g, th, 0, FLAGS, B, state_out=so)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    secs = max_over_ranks(time_steps(step, steps, stream), world, device) / steps
    return {"workload": f"seqshard_{c['workload']}_B{B}", "shards": world, "tokens_per_shard": Ls,
            "us_per_step": secs * 1e6, "tokens_per_s": b * L / secs, "scaling": "strong",
            "exchange": "one all-gather of b*h*d_k*d_v fp32 per rank (NCCL)",
            # segment-state pass, one state advance per earlier shard, the shard's chunkwise call
            "gpu_launches_per_rank_step": 1 + rank + rn.retnet_chunkwise_launches((b, Ls, h, dk), dv, rn.BF16, FLAGS,
                                                                                 B, g, 0)}


def oracle_sample(cfg, budget_s):
    """Size a bounded sample of the workload for the fp64 oracle: whole batch rows (all heads)."""
    import oracle
    import synth_inputs as si
    threads = oracle.num_threads(0)
    b, L, h, dk, dv = cfg["batch"], cfg["seqlen"], cfg["heads"], cfg["d_k"], cfg["d_v"]
    q, k, v = si.qkv(1, L, h, dk, dv, 2, "bf16")
    g, th = si.gamma_schedule(h), si.theta_schedule(dk)
    t0 = time.perf_counter()
    oracle.recurrent(q[:, :, :1], k[:, :, :1], v[:, :, :1], g[:1], th, 0, FLAGS)  # one (row, head) pair
    one = time.perf_counter() - t0
    rows = int(min(b, max(1, round(budget_s * threads / (one * h)))))
    q, k, v = si.qkv(rows, L, h, dk, dv, 2, "bf16")
    desc = (f"{rows} of {b} batch rows (all {h} heads, L={L}, d_k={dk}, d_v={dv}) through the fp64 "
            f"recurrent-form oracle, OpenMP over (row, head) pairs")
    return dict(q=q, k=k, v=v, g=g, th=th, rows=rows, L=L, threads=threads, desc=desc)


def run_oracle(smp):
    import oracle
    t0 = time.perf_counter()
    oracle.recurrent(smp["q"], smp["k"], smp["v"], smp["g"], smp["th"], 0, FLAGS)
    return time.perf_counter() - t0


def cpu_baseline(cfg, budget_s=15.0):
    """The oracle as it stands, timed on this host's cores on a bounded sample of the workload."""
    smp = oracle_sample(cfg, budget_s)
    secs = run_oracle(smp)
    return {"value": smp["rows"] * smp["L"] / secs, "unit": "tokens/s", "cores": smp["threads"], "kind": "oracle",
            "sample": smp["desc"], "seconds": secs}


def main_ours(args):
    import torch

    import linear_attention_sequence_chunkwise_b200 as rn
    import synth_inputs as si
    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    rn.load()
    peaks = load_peaks()
    cfg = MAIN
    b, L, h, dk, dv, B = cfg["batch"], cfg["seqlen"], cfg["heads"], cfg["d_k"], cfg["d_v"], cfg["chunk"]
    gamma, theta = si.gamma_schedule(h), si.theta_schedule(dk)
    path = rn.retnet_chunkwise_kernel((b, L, h, dk), dv, rn.BF16, FLAGS, B, gamma)
    dtype_label = "f16" if path == 1 else "f32"  # arithmetic type of the kernel that runs
    sets = make_main_inputs(cfg, device, rank)
    ws = torch.empty(rn.retnet_chunkwise_workspace_size((b, L, h, dk, dv)), dtype=torch.uint8, device=device)
    launches = rn.retnet_chunkwise_launches((b, L, h, dk), dv, rn.BF16, FLAGS, B, gamma, ws.numel())
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()

    def step(i):
        run_chunkwise(rn, sets[i % N_SETS], cfg, gamma, theta, stream, ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    secs = time_steps(step, args.steps, stream)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    barrier(world)
    secs_max = max_over_ranks(secs, world, device)
    clk = clocks.summary(t_wall0, t_wall1)

    tokens = b * L * world * args.steps
    value = tokens / secs_max
    per_launch = secs / args.steps
    alg_bytes = b * L * h * bytes_per_token_head(dk, dv)
    alg_flops = b * L * h * flops_per_token_head(dk, dv, B)
    achieved_gbs = alg_bytes / per_launch / 1e9
    tflops = alg_flops / per_launch / 1e12
    line = {
        "metric": "retention fwd tokens/s + TFLOP/s (% bf16 peak); decode-step state GB/s",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs_max / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_label, "input_dtype": "bf16",
        "kernel": "tcgen05 tensor-core chunkwise" if path == 1 else "fp32 CUDA-core chunkwise",
        "data": "synthetic",
        "config": {"workload": cfg["workload"], "batch_per_gpu": b, "global_batch": b * world, "seq_len": L,
                   "heads": h, "d_k": dk, "d_v": dv, "chunk": B, "flags": "xpos|sqrt_d|norm_d",
                   "out_dtype": "bf16", "l2": f"inputs rotate over {N_SETS} resident sets "
                                             f"({N_SETS * alg_bytes / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"dp{world}"},
        "tflops": tflops, "frac_bf16_peak": tflops * 1e12 / (peaks["bf16"] * 1e12),
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm"], "traffic": ncu_traffic("chunkwise_tc") if path == 1 else None,
                     "peak_source": peaks["source"], "algorithmic_bytes_per_step": alg_bytes,
                     "step_us": per_launch * 1e6,
                     "scope": "one step = the chunkwise call: " + (
                         "segment-state pre-pass + output pass (two launches)" if launches == 2 else "one launch")},
        "gpu_launches": args.steps * launches,
        "launches_per_step": launches,
        "workspace_bytes": ws.numel(),
        "clocks": clk,
    }
    # e2e: host buffers in pinned memory, copies inside the timed region, through the same C call.
    # Steps are pipelined as a serving loop would run them: step i's inputs go up on a copy
    # stream while step i-1 computes and step i-2's output comes down on a third stream (two
    # device buffer sets, each reused only after its previous step's output has been read back).
    if "e2e" not in args.sections:
        line["e2e"] = None
    e2e_steps = max(3, min(args.steps, 50)) if "e2e" in args.sections else 0
    hq = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in sets[0][:3]]
    for hx, dx in zip(hq, sets[0][:3]):
        hx.copy_(dx.cpu())
    ho = [torch.empty(sets[0][3].shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_back = [torch.cuda.Event() for _ in range(2)]
    for e in ev_out + ev_back:
        e.record(stream)

    def e2e_step(i):
        j = i % 2
        dq, dk_, dv_, do = sets[j]
        up.wait_event(ev_out[j])  # the compute that last read these inputs is done
        with torch.cuda.stream(up):
            dq.copy_(hq[0], non_blocking=True)
            dk_.copy_(hq[1], non_blocking=True)
            dv_.copy_(hq[2], non_blocking=True)
        ev_in[j].record(up)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_back[j])  # this buffer's previous output has been read back
        run_chunkwise(rn, (dq, dk_, dv_, do), cfg, gamma, theta, stream, ws)
        ev_out[j].record(stream)
        down.wait_event(ev_out[j])
        with torch.cuda.stream(down):
            ho[j].copy_(do, non_blocking=True)
        ev_back[j].record(down)

    def e2e_run(i):
        if i == 0:  # the first copy starts after the timed region's start event
            up.wait_stream(stream)
        e2e_step(i)
        if i == e2e_steps - 1:  # the timed region ends when the last output is on the host
            stream.wait_stream(down)

    if e2e_steps:
        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        barrier(world)
        e_secs = time_steps(e2e_run, e2e_steps, stream)
        barrier(world)
        e_secs = max_over_ranks(e_secs, world, device)
        line["e2e"] = {"value": b * L * world * e2e_steps / e_secs, "unit": "tokens/s",
                       "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in hq),
                       "d2h_bytes_per_step": ho[0].numel() * ho[0].element_size(), "steps": e2e_steps,
                       "pipelining": "copy-in, compute and copy-out of successive steps on three streams"}
    if world == 1 and "decode" in args.sections:
        line["decode"] = bench_decode(rn, device, stream, args.decode_steps, 3, peaks)
    if world == 1 and "long" in args.sections:
        line["long"] = bench_long(rn, device, stream, 10, peaks)
    if world == 1 and "msr" in args.sections:
        line["msr"] = bench_msr(rn, device, stream, 10, peaks)
    if world == 1 and "backward" in args.sections:
        line["backward"] = bench_backward(rn, device, stream, 3, peaks)
    if world == 1 and "variants" in args.sections:
        line["variants"] = bench_flag_variants(rn, device, stream, 20, peaks, ws)
    if "seqshard" in args.sections:
        import datetime

        import torch.distributed as dist
        own_group = not dist.is_initialized()
        if own_group:  # one rank: a one-member NCCL group carries the (trivial) all-gather
            dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=120), device_id=device)
        line["seqshard"] = bench_seqshard(rn, device, stream, 5, world, rank)
        if own_group:
            dist.destroy_process_group()
    clocks.stop()
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main_reference(args):
    """The oracle on the host cores, on the same workload, metric and unit as our arm."""
    world, rank, _ = dist_env()
    if rank != 0:
        return  # rank 0 alone runs and prints
    cfg = MAIN
    smp = oracle_sample(cfg, max(0.5, args.cpu_seconds / max(1, args.steps)))
    for _ in range(args.warmup):
        run_oracle(smp)
    secs = sum(run_oracle(smp) for _ in range(args.steps))
    value = smp["rows"] * smp["L"] * args.steps / secs
    line = {"metric": "retention fwd tokens/s + TFLOP/s (% bf16 peak); decode-step state GB/s", "impl": "reference",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg["workload"], "batch": cfg["batch"], "seq_len": cfg["seqlen"],
                       "heads": cfg["heads"], "d_k": cfg["d_k"], "d_v": cfg["d_v"], "chunk": cfg["chunk"],
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp["threads"], "kind": "oracle",
                             "sample": "each step: " + smp["desc"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch(n):
    """Run this script under torch.distributed.run with n processes (one per GPU); returns its
    exit status.  Rank 0's JSON line reaches stdout through the launcher."""
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main_stub(args):
    """Launch plumbing only (no GPU, no kernels, nothing timed): every rank joins a gloo group,
    the ranks are counted with an all-reduce, and rank 0 prints the count.  Used by the CPU
    tests of the multi-process launch."""
    world, rank, _ = dist_env()
    seen = 1
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        t = torch.ones(1)
        dist.all_reduce(t)
        seen = int(t.item())
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"stub": True, "n_gpus": world, "ranks_seen": seen, "value": None}), flush=True)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sections", default="e2e,decode,long,msr,backward,variants,seqshard",
                    help="comma list of extra legs to run beside the timed step: e2e, decode, long, msr, backward, "
                         "variants, seqshard")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--stub", action="store_true",
                    help="check the multi-process launch only (CPU, gloo): print the rank count, run no kernels")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args(argv)
    if a.warmup < 3 and a.impl == "ours":
        a.warmup = 3
    return a


if __name__ == "__main__":
    args = parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus))
    if int(os.environ.get("WORLD_SIZE", "1")) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started {os.environ.get('WORLD_SIZE', '1')} ranks",
              file=sys.stderr)
        sys.exit(2)
    if args.stub:
        main_stub(args)
    elif args.impl == "reference":
        main_reference(args)
    else:
        main_ours(args)
