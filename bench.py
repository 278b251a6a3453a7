#!/usr/bin/env python
"""Throughput of the MoE layer with zero-computation experts on B200, one JSON line.

A step is one pass of the whole hot path over one batch: moe_forward (router GEMM, softmax
and biased top-K, dispatch, SwiGLU expert GEMMs, combine) followed by the PID bias update,
inputs resident in HBM.  Default workload: prefill (T=16384 tokens, d=6144, 512 SwiGLU experts
of width 2048 plus 256 zero experts, K=12).  Weights (38.7 GB) and x (201 MB) are far larger
than the 126 MB L2, so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skewed|mid|tiny]
  python bench.py --impl reference ...     # the CPU oracle on a bounded sample, host cores

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica on its own
tokens: the layer has no exchange step, so there is no data-path collective; the elapsed time
is the maximum over ranks.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_38_b200 import binding as mb  # noqa: E402
from mixture_experts_layer_38_b200.workloads import WORKLOADS, make_tokens, make_weights  # noqa

METRIC = "MoE-layer tokens/s"
UNIT = "tokens/s"
PID_GAINS = (0.005, 0.002, 0.0)  # kp, ki, kd
LAUNCHES_PER_STEP = 10  # router GEMM, top-K, histogram, scan, permute, gather, 2 GEMMs,
                        # combine, PID
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel from an ncu capture (profiles/), valid only
# while the kernel source is unchanged (sha1 of the GEMM source at capture time).
NCU_TRAFFIC = {}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def gemm_source_hash():
    h = hashlib.sha1()
    for name in ("gemm.cu", "device.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_layer_38_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


# ------------------------------------------------------------------------------ replicas
def max_over_ranks(value: float, world: int, device=None) -> float:
    """Elapsed time of the job: the maximum over ranks (a timing collective, not data)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms: float) -> float:
    """Tokens per second of the whole job: every rank processes its own batch each step."""
    return world * tokens_per_rank * steps / (ms / 1e3)


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            uuid = str(device)
        self.gpu = uuid

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception as e:  # nvidia-smi missing: report no clocks
            log("clock sampling unavailable:", e)
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------------------ work model
def work_model(w, counts):
    """Algorithmic FLOPs and bytes of one step from the routing actually taken."""
    counts = np.asarray(counts, np.int64)
    A = int(counts[:w.N].sum())
    U = int((counts[:w.N] > 0).sum())
    d, I, T, E = w.d, w.I, w.T, w.E
    flops = {
        "router_gemm": 2 * T * d * E,
        "ffn_up_gemm": 2 * A * d * 2 * I,
        "ffn_down_gemm": 2 * A * I * d,
    }
    bytes_ = {
        "router_gemm": E * d * 2 + T * d * 2 + T * E * 4,
        "ffn_up_gemm": U * 2 * I * d * 2 + A * d * 2 + A * I * 2,
        "ffn_down_gemm": U * d * I * 2 + A * I * 2 + A * d * 2,
        "dispatch": 2 * A * d * 2,
        "combine": (A + 2 * T) * d * 2,
    }
    return A, U, flops, bytes_


# ------------------------------------------------------------------------------ CPU oracle
def oracle_tokens_per_s(w, x_dev, wt, b, n_tokens, seed, cache=None):
    """The oracle, as it stands, on a seeded sample of tokens; weight fetches not timed."""
    import oracle  # test infrastructure: only this leg of the benchmark may use it
    rng = np.random.default_rng(seed)
    tokens = np.sort(rng.choice(w.T, n_tokens, replace=False))
    xs = x_dev[torch.from_numpy(tokens).to(x_dev.device)].cpu()
    W_r = wt["W_r"].cpu()
    b_cpu = b.cpu()
    fetch_s = [0.0]

    def fetch(e):
        t0 = time.perf_counter()
        if cache is not None and e in cache:
            out = cache[e]
        else:
            out = (wt["W_g"][e].cpu(), wt["W_u"][e].cpu(), wt["W_d"][e].cpu())
            if cache is not None:
                cache[e] = out
        fetch_s[0] += time.perf_counter() - t0
        return out
    t0 = time.perf_counter()
    oracle.forward_sampled(np.arange(n_tokens), xs, W_r, b_cpu, w.N, w.Z, w.K, fetch)
    elapsed = time.perf_counter() - t0 - fetch_s[0]
    threads = int(os.environ.get("OMP_NUM_THREADS", 0)) or len(os.sched_getaffinity(0))
    return n_tokens / elapsed, elapsed, threads


def default_sample(w):
    # ~10-30 s of fp64 work on a few dozen host cores: scale by the per-token FFN work.
    per_token = 6.0 * w.d * w.I * min(w.K, 9)
    return int(max(4, min(w.T, 64, round(1.5e11 / per_token))))


# ------------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    w = WORKLOADS[args.workload]
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    log(f"[rank {rank}] generating {w.name} weights ({w.weight_bytes / 1e9:.1f} GB)")
    wt = make_weights(w, device, seed=args.seed)
    x = make_tokens(w, device, seed=args.seed + rank)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = mb.alloc_workspace(dm, device)
    y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=device)
    b = wt["b"].clone()
    pid_state = torch.zeros(2, dtype=torch.float32, device=device)
    params = mb.PidParams(w.pid_target, *PID_GAINS)
    n_steps = args.warmup + args.steps
    counts = torch.zeros((n_steps + args.steps, w.E), dtype=torch.int32, device=device)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(mb.NUM_STAGE_EVENTS)]
              for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    for ev in events:  # torch creates the CUDA event handle on first record
        for e in ev:
            e.record(stream)

    def step(i, ev=None):
        if ev is None:
            mb.moe_forward(dm, x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y, counts[i], ws)
        else:
            mb.moe_forward_timed(dm, x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y,
                                 counts[i], ws, ev)
        mb.moe_bias_update(dm, counts[i], b, pid_state, params)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(device)
    clocks.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, events[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, world, device)
    status = mb.moe_last_device_error(ws)
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the timed steps")

    # per-stage durations and algorithmic work of the timed steps
    stage_ms = {n: 0.0 for n in mb.STAGE_NAMES}
    for ev in events:
        for si, n in enumerate(mb.STAGE_NAMES):
            stage_ms[n] += ev[si].elapsed_time(ev[si + 1])
    hist = counts[args.warmup:n_steps].cpu().numpy()
    tot_flops = {k: 0 for k in ("router_gemm", "ffn_up_gemm", "ffn_down_gemm")}
    tot_bytes = {k: 0 for k in ("router_gemm", "ffn_up_gemm", "ffn_down_gemm", "dispatch",
                                "combine")}
    A_steps, U_steps = [], []
    for c in hist:
        A, U, fl, by = work_model(w, c)
        A_steps.append(A)
        U_steps.append(U)
        for k in fl:
            tot_flops[k] += fl[k]
        for k in by:
            tot_bytes[k] += by[k]
    pk, pk_src = peaks()
    dominant = max(stage_ms, key=stage_ms.get)
    hbm_bound = w.name == "decode"
    kernel = dominant
    if hbm_bound or kernel not in tot_flops:
        achieved = tot_bytes[kernel] / (stage_ms[kernel] / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s"}
        peak_name = "hbm_gbs"
    else:
        achieved = tot_flops[kernel] / (stage_ms[kernel] / 1e3) / 1e12
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s"}
        peak_name = "bf16_tflops_sustained"
    roof["frac"] = round(achieved / peak, 4)
    tr = NCU_TRAFFIC.get((w.name, kernel))
    roof["traffic"] = tr["bytes_per_launch"] if tr and tr["src"] == gemm_source_hash() else None
    roof["kernel"] = kernel
    roof["peak_source"] = f"{pk_src} {peak_name}"
    layer_flops = sum(tot_flops.values())
    layer = {"tflops": round(layer_flops / (ms / 1e3) / 1e12, 1),
             "frac_of_bf16_peak": round(layer_flops / (ms / 1e3) / 1e12 / pk["bf16_tflops"], 4)}

    # ---------------------------------------------------------------- end to end, host buffers
    if args.no_e2e:
        return finish(args, w, world, rank, ms_max, A_steps, U_steps, roof, layer, stage_ms,
                      clk, None, x, wt, b)
    x_host = torch.empty((w.T, w.d), dtype=torch.bfloat16).pin_memory()
    x_host.copy_(x.cpu())
    y_host = torch.empty((w.T, w.d), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_steps = args.steps
    for i in range(2):  # warm the copy path
        x_dev.copy_(x_host, non_blocking=True)
        step(n_steps + i)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        mb.moe_forward(dm, x_dev, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y,
                       counts[n_steps + (i % args.steps)], ws)
        mb.moe_bias_update(dm, counts[n_steps + (i % args.steps)], b, pid_state, params)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e = {"value": round(job_throughput(world, w.T, e2e_steps, e2e_ms), 1), "unit": UNIT,
           "h2d_bytes_per_step": int(x_host.numel() * 2),
           "d2h_bytes_per_step": int(y_host.numel() * 2)}
    return finish(args, w, world, rank, ms_max, A_steps, U_steps, roof, layer, stage_ms, clk,
                  e2e, x, wt, b)


def finish(args, w, world, rank, ms_max, A_steps, U_steps, roof, layer, stage_ms, clk, e2e,
           x, wt, b):
    result = {
        "metric": METRIC, "value": round(job_throughput(world, w.T, args.steps, ms_max), 1),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; x~N(0,1), weights~N(0,0.02^2) bf16, biases~U(-0.05,0.05))",
        "config": {
            "workload": w.name, "T": w.T, "d": w.d, "N": w.N, "Z": w.Z, "K": w.K, "I": w.I,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (weights %.1f GB, x %.0f MB); no flush"
                  % (w.weight_bytes / 1e9, w.T * w.d * 2 / 1e6),
            "step": "moe_forward + moe_bias_update (PID target %.1f, kp=%g ki=%g kd=%g)"
                    % ((w.pid_target,) + PID_GAINS),
            "mean_ffn_experts_per_token": round(float(np.mean(A_steps)) / w.T, 4),
            "distinct_ffn_experts": int(np.mean(U_steps)),
        },
        "roofline": roof,
        "layer": layer,
        "stages_ms": {k: round(v / args.steps, 4) for k, v in stage_ms.items()},
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        n = args.cpu_sample or default_sample(w)
        log(f"oracle CPU baseline on {n} sampled tokens ...")
        tps, secs, threads = oracle_tokens_per_s(w, x, wt, b, n, args.seed)
        result["cpu_baseline"] = {
            "value": round(tps, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} seeded tokens of {w.name} (router + SwiGLU experts + combine, "
                      f"fp64, weight fetches excluded), {secs:.1f} s"}
    return result


# ------------------------------------------------------------------------------ reference arm
def run_reference(args, rank, world, local_rank):
    """The oracle as it stands, on the host cores: each step a bounded token sample."""
    w = WORKLOADS[args.workload]
    use_cuda = torch.cuda.is_available()
    device = torch.device("cuda", local_rank) if use_cuda else torch.device("cpu")
    if use_cuda:
        torch.cuda.set_device(device)
    log(f"reference arm: generating {w.name} inputs on {device}")
    wt = make_weights(w, device, seed=args.seed)
    x = make_tokens(w, device, seed=args.seed)
    n = args.cpu_sample or max(2, default_sample(w) // 4)
    per_step = []
    total_tokens = 0
    total_s = 0.0
    threads = 0
    cache = {}
    for i in range(args.warmup + args.steps):
        tps, secs, threads = oracle_tokens_per_s(w, x, wt, wt["b"], n, args.seed + 1 + i, cache)
        if len(cache) > 64:
            cache.clear()
        if i >= args.warmup:
            per_step.append(secs)
            total_tokens += n
            total_s += secs
    value = total_tokens / total_s
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_s / args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same generator as the GPU arm)",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "N": w.N, "Z": w.Z, "K": w.K,
                   "I": w.I, "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": threads,
                         "kind": "oracle",
                         "sample": f"{n} seeded tokens per step of {w.name}, fp64"},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default="prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-sample", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world, local_rank)), flush=True)
        return 0
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=300),
            device_id=torch.device("cuda", local_rank))
    try:
        result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
