#!/usr/bin/env python
"""Throughput of the MoE layer with zero-computation experts on B200, one JSON line.

A step is one pass of the whole hot path over one batch: moe_forward (router GEMM, softmax
and biased top-K, dispatch, SwiGLU expert GEMMs, combine) followed by the PID bias update,
inputs resident in HBM.  Default workload: prefill (T=16384 tokens, d=6144, 512 SwiGLU experts
of width 2048 plus 256 zero experts, K=12).  Weights (38.7 GB) and x (201 MB) are far larger
than the 126 MB L2, so no L2 flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W]
      [--workload prefill|decode|skewed|mid|tiny|prefill_small]
  python bench.py --impl reference ...     # the CPU oracle on a bounded sample, host cores

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica on its own
tokens: the layer has no exchange step, so there is no data-path collective; the elapsed time
is the maximum over ranks.
"""
import argparse
import datetime
import hashlib
import re
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
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 datasheet figure
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e datasheet figure
PID_GAINS = (0.005, 0.002, 0.0)  # kp, ki, kd
LAUNCHES_PER_STEP = 10  # router GEMM, top-K, histogram, scan, permute, gather, 2 GEMMs,
                        # combine, PID
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of the dominant kernel from an ncu capture (profiles/), valid only
# while the kernel and its launch set-up are unchanged (sha1 of the code, comments removed, of
# the GEMM kernel and of the file that builds its tensor maps, at capture time).
NCU_TRAFFIC = {
    # DRAM bytes per launch of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum)
    # for the sources hashing to "src".  Decode streams each used expert's weights once, so the
    # figures come from a decode-shaped capture with 128 experts (102 used) scaled to the decode
    # workload's 145 used experts (the decode-shaped DRAM summary under profiles/); prefill's
    # traffic does not scale that way and was not captured at full size for this build (null).
    ("decode", "ffn_up_gemm"): {"bytes_per_launch": 7315470758, "src": "869fc7a06349"},
    ("decode+fp8+act", "ffn_up_gemm"): {"bytes_per_launch": 3779534105, "src": "869fc7a06349"},
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _code_only(text):
    """C/C++ source without comments and blank space, so comment edits keep the hash."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def gemm_source_hash(read=None):
    h = hashlib.sha1()
    for name in ("gemm.cu", "gemm_common.cuh", "gemm_f8.cu", "device.cuh", "kernels.cuh",
                 "moe_api.cu"):
        path = os.path.join("mixture_experts_layer_38_b200", "csrc", name)
        if read is None:
            with open(os.path.join(ROOT, path), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(path)
        h.update(_code_only(text).encode())
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
    """SM clock, power and clock-event reasons sampled DURING the timed region (read-only).

    NVML (the library nvidia-smi reads) polled every 10 ms from a thread, so even a timed region
    of a few hundred ms yields dozens of samples; nvidia-smi's loop mode is the fallback."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))
    SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.samples = []
        self.max_mhz = None
        self.power_limit_w = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._path = None
        self.source = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else \
                pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            try:
                self.power_limit_w = pynvml.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
            except Exception:
                pass
            bits = [(name, getattr(pynvml, const)) for name, const in self.REASONS]
            self._stop = threading.Event()

            def loop():
                while not self._stop.is_set():
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        watts = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((mhz, watts, [n for n, bit in bits if r & bit]))
                    except Exception:
                        pass
                    self._stop.wait(0.01)
            self._thread = threading.Thread(target=loop, daemon=True)
            self._thread.start()
            self.source = "nvml 10 ms"
            return
        except Exception as e:
            log("NVML clock sampling unavailable, falling back to nvidia-smi:", e)
        fd, self._path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid or "0", f"--query-gpu={self.SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self._path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi 100 ms"
        except Exception as e:
            log("clock sampling unavailable:", e)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        elif self._proc is not None:
            time.sleep(0.15)
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            with open(self._path) as f:
                for line in f:
                    r = [x.strip() for x in line.split(",")]
                    if len(r) < 9:
                        continue
                    try:
                        self.samples.append((float(r[1]), float(r[3]),
                                             [names[i] for i in range(4) if r[5 + i] == "Active"]))
                        self.max_mhz = float(r[2])
                    except ValueError:
                        pass
            os.unlink(self._path)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"],
                    "source": self.source}
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(s[0] for s in self.samples),
                "power_w_max": round(max(s[1] for s in self.samples), 1),
                "power_limit_w": self.power_limit_w,
                "samples": len(self.samples),
                "reasons": sorted({r for s in self.samples for r in s[2]}),
                "source": self.source}


# ------------------------------------------------------------------------------ work model
def work_model(w, counts, wb=2, ab=2):
    """Algorithmic FLOPs and bytes of one step from the routing actually taken; `wb` bytes per
    expert weight (2 for bf16, 1 for the FP8 codes; their block scales add 4 bytes per 16384
    weights, negligible), `ab` bytes per GEMM activation (2 for bf16, 1 for FP8 activations,
    whose up-projection stage also holds the quantisation of x_perm: 2 bytes read, 1 written
    per element; block scales again negligible)."""
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
        "ffn_up_gemm": U * 2 * I * d * wb + A * d * ab + A * I * ab +
                       (A * d * 3 if ab == 1 else 0),
        "ffn_down_gemm": U * d * I * wb + A * I * ab + A * d * 2,
        "dispatch": (T + A) * d * 2,  # each token row read once, each slot row written
        "combine": (A + 2 * T) * d * 2,
    }
    return A, U, flops, bytes_


def stage_durations(events):
    """Per-stage milliseconds summed over the timed steps (events recorded by moe_forward_timed)."""
    stage_ms = {n: 0.0 for n in mb.STAGE_NAMES}
    for ev in events:
        for si, n in enumerate(mb.STAGE_NAMES):
            stage_ms[n] += ev[si].elapsed_time(ev[si + 1])
    return stage_ms


def step_work(w, hist, wb=2, ab=2):
    """Algorithmic FLOPs and bytes summed over the steps whose per-expert counts are `hist`."""
    tot_flops = {k: 0 for k in ("router_gemm", "ffn_up_gemm", "ffn_down_gemm")}
    tot_bytes = {k: 0 for k in ("router_gemm", "ffn_up_gemm", "ffn_down_gemm", "dispatch",
                                "combine")}
    A_steps, U_steps, load_ratio = [], [], []
    for c in hist:
        A, U, fl, by = work_model(w, c, wb=wb, ab=ab)
        A_steps.append(A)
        U_steps.append(U)
        ffn = c[:w.N]
        load_ratio.append(float(ffn.max()) / max(float(ffn.mean()), 1e-30))
        for k in fl:
            tot_flops[k] += fl[k]
        for k in by:
            tot_bytes[k] += by[k]
    return tot_flops, tot_bytes, (A_steps, U_steps, load_ratio)


def roofline_of(w, stage_ms, tot_flops, tot_bytes, fp8=False, fp8_act=False):
    """Roofline record of the dominant (longest) stage: FLOP/s against the burst bf16 peak for
    a contraction at prefill-like sizes, bytes/s against the HBM copy peak at decode."""
    pk, pk_src = peaks()
    kernel = max(stage_ms, key=stage_ms.get)
    if w.name == "decode" or kernel not in tot_flops:
        achieved = tot_bytes[kernel] / (stage_ms[kernel] / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s"}
        peak_name = "hbm_gbs"
    else:
        # The kernel is event-timed over a sub-second run of steps: the burst peak applies.
        achieved = tot_flops[kernel] / (stage_ms[kernel] / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s"}
        peak_name = "bf16_tflops (burst)"
        if "bf16_tflops_sustained" in pk:
            roof["frac_of_sustained"] = round(achieved / pk["bf16_tflops_sustained"], 4)
    roof["frac"] = round(achieved / peak, 4)
    # the datasheet figures (dense bf16 2250 TFLOP/s, HBM3e 8000 GB/s), for context
    roof["frac_of_nominal"] = round(achieved / (NOMINAL_HBM_GBS if roof["bound"] == "hbm"
                                                else NOMINAL_BF16_TFLOPS), 4)
    tr = NCU_TRAFFIC.get((w.name + ("+fp8" if fp8 else "") + ("+act" if fp8_act else ""), kernel))
    roof["traffic"] = tr["bytes_per_launch"] if tr and tr["src"] == gemm_source_hash() else None
    roof["kernel"] = kernel
    roof["peak_source"] = f"{pk_src} {peak_name}"
    return roof


def layer_of(flops, bytes_, ms, decode=False):
    """The whole step against both rooflines, and the target the workload is held to: at
    prefill-like sizes >= 0.60 of the bf16 peak, at decode >= 0.70 of HBM bandwidth."""
    pk, _ = peaks()
    tflops = flops / (ms / 1e3) / 1e12
    gbs = bytes_ / (ms / 1e3) / 1e9
    layer = {"tflops": round(tflops, 1),
             "frac_of_bf16_peak": round(tflops / pk["bf16_tflops"], 4),
             "frac_of_nominal_bf16": round(tflops / NOMINAL_BF16_TFLOPS, 4),
             "gbs": round(gbs, 1),
             "frac_of_hbm_peak": round(gbs / pk["hbm_gbs"], 4),
             "frac_of_nominal_hbm": round(gbs / NOMINAL_HBM_GBS, 4)}
    if decode:
        layer["target"] = {"what": "whole step >= 0.70 of measured HBM bandwidth",
                           "frac": layer["frac_of_hbm_peak"],
                           "met": layer["frac_of_hbm_peak"] >= 0.70}
    else:
        layer["target"] = {"what": "whole step >= 0.60 of measured burst bf16 peak",
                           "frac": layer["frac_of_bf16_peak"],
                           "met": layer["frac_of_bf16_peak"] >= 0.60}
    return layer


def near_tie_tokens(dm, x, W_r, b, ws):
    """Tokens whose K-th vs (K+1)-th biased-score gap (the GPU's fp32 gap from moe_route) is at
    most 1e-4 on the bench's x with the current biases: where the routing rule allows any
    eps-valid set instead of one bit-exact set."""
    idx = torch.empty((dm.T, dm.K), dtype=torch.int32, device=x.device)
    gate = torch.empty((dm.T, dm.K), dtype=torch.float32, device=x.device)
    gap = torch.empty((dm.T,), dtype=torch.float32, device=x.device)
    mb.moe_route(dm, x, W_r, b, idx, gate, gap, ws)
    return int((gap <= 1e-4).sum().item())


def decode_record(args, wt, device, rank, world, fp8_act=False):
    """The decode workload (T = 128) timed on the given expert weights, as its own record:
    ms per step, tokens/s, the dominant kernel against the HBM peak, the whole step's
    fractions, per-stage times and clocks.  Every rank runs it (the max over ranks is taken).
    With fp8_act the weights are first quantised to block-wise FP8 (outside the timed region)
    and the layer runs with FP8 activations (E4M3 x E4M3 MMAs, moe_forward_fp8)."""
    w = WORKLOADS["decode"]
    x = make_tokens(w, device, seed=args.seed + rank)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=mb.FP8_ACTIVATIONS if fp8_act else 0)
    fw = None
    if fp8_act:
        log(f"[rank {rank}] quantising the expert weights to block-wise FP8 for the FP8 decode")
        fw = mb.quantize_expert_weights_fp8(dm, wt["W_g"], wt["W_u"], wt["W_d"])

    def forward(c, ev=None):
        if fw is not None:
            mb.moe_forward_fp8(dm, x, wt["W_r"], b, fw, y, c, ws, events=ev)
        elif ev is None:
            mb.moe_forward(dm, x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y, c, ws)
        else:
            mb.moe_forward_timed(dm, x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y, c, ws,
                                 ev)
    ws = mb.alloc_workspace(dm, device)
    y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=device)
    b = wt["b"].clone()
    pid_state = torch.zeros(2, dtype=torch.float32, device=device)
    params = mb.PidParams(w.pid_target, *PID_GAINS, 0.0)
    steps = max(args.steps, 60)  # ~0.1 s: enough clock samples
    counts = torch.zeros((args.warmup + steps, w.E), dtype=torch.int32, device=device)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(mb.NUM_STAGE_EVENTS)]
              for _ in range(steps)]
    stream = torch.cuda.current_stream()
    for ev in events:
        for e in ev:
            e.record(stream)
    for i in range(args.warmup):
        forward(counts[i])
        mb.moe_bias_update(dm, counts[i], b, pid_state, params)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(device)
    clocks.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        c = counts[args.warmup + i]
        forward(c, events[i])
        mb.moe_bias_update(dm, c, b, pid_state, params)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(start.elapsed_time(end), world, device)
    status = mb.moe_last_device_error(ws)
    if status != 0:
        raise RuntimeError(f"device status {status:#x} after the decode steps")
    stage_ms = stage_durations(events)
    tot_flops, tot_bytes, (A_steps, U_steps, _) = step_work(
        w, counts[args.warmup:].cpu().numpy(), wb=1 if fp8_act else 2, ab=1 if fp8_act else 2)
    layer = layer_of(sum(tot_flops.values()), sum(tot_bytes.values()), ms, decode=True)
    rec = {
        "workload": w.name, "T": w.T, "steps": steps,
        "ms_per_step": round(ms / steps, 4),
        "value": round(job_throughput(world, w.T, steps, ms), 1), "unit": UNIT,
        "roofline": roofline_of(w, stage_ms, tot_flops, tot_bytes, fp8=fp8_act,
                                fp8_act=fp8_act),
        "layer": layer,
        "stages_ms": {k: round(v / steps, 4) for k, v in stage_ms.items()},
        "mean_ffn_experts_per_token": round(float(np.mean(A_steps)) / w.T, 4),
        "distinct_ffn_experts": int(np.mean(U_steps)),
        "near_tie_tokens": near_tie_tokens(dm, x, wt["W_r"], b, ws),
        "clocks": clk,
        "gpu_launches": (LAUNCHES_PER_STEP + (1 if fp8_act else 0)) * steps,
    }
    if fp8_act:
        rec["variant"] = {"expert_weights": "fp8 e4m3, 128x128 blocks",
                          "activations": "fp8 e4m3, 1x128 blocks (E4M3 x E4M3 MMAs)",
                          "bytes_model": "1 byte per weight and per GEMM activation"}
        del fw
    return rec


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
    # ~10-30 s of fp64 work on a 16-core host (the full-size layer costs ~56 ms per token
    # there): scale by the per-token FFN work.
    per_token = 6.0 * w.d * w.I * min(w.K, 9)
    return int(max(4, min(w.T, 512, round(2.0e11 / per_token))))


# ------------------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    w = WORKLOADS[args.workload]
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    log(f"[rank {rank}] generating {w.name} weights ({w.weight_bytes / 1e9:.1f} GB)")
    wt = make_weights(w, device, seed=args.seed)
    x = make_tokens(w, device, seed=args.seed + rank)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I,
                 flags=(mb.RENORMALIZE_GATES if args.renormalize_gates else 0) |
                 (mb.FP8_ACTIVATIONS if args.fp8_activations else 0) |
                 (mb.FUSED_COMBINE if args.fused_combine else 0))
    ws = mb.alloc_workspace(dm, device)
    y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=device)
    b = wt["b"].clone()
    dense = None
    if args.scmoe > 0:
        # ScMoE shortcut branch: a dense SwiGLU FFN on its own input, on a second stream
        g = torch.Generator(device=device).manual_seed(args.seed + 77)
        Id = args.scmoe
        dense = {
            "dm": mb.dims(w.T, w.d, 1, 0, 1, Id),
            "x": torch.randn((w.T, w.d), generator=g, device=device).to(torch.bfloat16),
            "W_g": (torch.randn((Id, w.d), generator=g, device=device) * 0.02).to(torch.bfloat16),
            "W_u": (torch.randn((Id, w.d), generator=g, device=device) * 0.02).to(torch.bfloat16),
            "W_d": (torch.randn((w.d, Id), generator=g, device=device) * 0.02).to(torch.bfloat16),
            "h": torch.empty((w.T, Id), dtype=torch.bfloat16, device=device),
            "y": torch.empty((w.T, w.d), dtype=torch.bfloat16, device=device),
            "ws": torch.zeros(256, dtype=torch.uint8, device=device),
            "stream": torch.cuda.Stream(device=device),
        }

    def dense_fork(main):
        if dense is not None:
            dense["stream"].wait_stream(main)
            mb.moe_dense_ffn(dense["dm"], dense["x"], dense["W_g"], dense["W_u"], dense["W_d"],
                             dense["h"], dense["y"], dense["ws"], stream=dense["stream"])

    def dense_join(main):
        if dense is not None:
            main.wait_stream(dense["stream"])

    fw = None
    if args.fp8:
        log(f"[rank {rank}] quantising the expert weights to block-wise FP8")
        fw = mb.quantize_expert_weights_fp8(dm, wt["W_g"], wt["W_u"], wt["W_d"])

    def forward(x_in, y_out, c, ev=None, stream=None):
        if fw is not None:
            mb.moe_forward_fp8(dm, x_in, wt["W_r"], b, fw, y_out, c, ws, stream=stream,
                               events=ev)
        elif ev is None:
            mb.moe_forward(dm, x_in, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y_out, c, ws,
                           stream=stream)
        else:
            mb.moe_forward_timed(dm, x_in, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y_out,
                                 c, ws, ev, stream=stream)
    pid_state = torch.zeros(2, dtype=torch.float32, device=device)
    params = mb.PidParams(w.pid_target, *PID_GAINS, args.balance_gamma)
    n_steps = args.warmup + args.steps
    counts = torch.zeros((n_steps + args.steps, w.E), dtype=torch.int32, device=device)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(mb.NUM_STAGE_EVENTS)]
              for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    for ev in events:  # torch creates the CUDA event handle on first record
        for e in ev:
            e.record(stream)

    def step(i, ev=None):
        dense_fork(stream)
        forward(x, y, counts[i], ev)
        mb.moe_bias_update(dm, counts[i], b, pid_state, params)
        dense_join(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    scmoe = None
    if dense is not None:  # each branch alone, for the overlap report (outside the timed region)
        def alone(fn, n=5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n
        scratch_counts = torch.zeros(w.E, dtype=torch.int32, device=device)
        scmoe = {
            "I_dense": args.scmoe,
            "dense_ffn_ms_alone": round(alone(lambda: mb.moe_dense_ffn(
                dense["dm"], dense["x"], dense["W_g"], dense["W_u"], dense["W_d"], dense["h"],
                dense["y"], dense["ws"], stream=stream)), 4),
            "moe_forward_ms_alone": round(alone(lambda: forward(x, y, scratch_counts)), 4),
            "dense_flop_per_step": 6 * w.T * w.d * args.scmoe,
        }
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
    stage_ms = stage_durations(events)
    hist = counts[args.warmup:n_steps].cpu().numpy()
    tot_flops, tot_bytes, routing = step_work(w, hist, wb=1 if args.fp8 else 2,
                                              ab=1 if args.fp8_activations else 2)
    roof = roofline_of(w, stage_ms, tot_flops, tot_bytes, fp8=args.fp8,
                       fp8_act=args.fp8_activations)
    layer_flops = sum(tot_flops.values())
    if scmoe is not None:
        scmoe["step_ms"] = round(ms / args.steps, 4)
        layer_flops += scmoe["dense_flop_per_step"] * args.steps
    layer = layer_of(layer_flops, sum(tot_bytes.values()), ms, decode=w.name == "decode")
    layer["near_tie_tokens"] = near_tie_tokens(dm, x, wt["W_r"], b, ws)
    if not args.no_decode and w.name != "decode" and w.d == WORKLOADS["decode"].d and \
            w.N == WORKLOADS["decode"].N and w.I == WORKLOADS["decode"].I and not args.fp8:
        # The second target's workload on the same expert weights (decode shares every one),
        # and the same with FP8 weights and activations read by the tensor cores.
        layer["decode"] = decode_record(args, wt, device, rank, world)
        layer["decode_fp8"] = decode_record(args, wt, device, rank, world, fp8_act=True)
    if scmoe is not None:
        layer["scmoe"] = scmoe

    # ---------------------------------------------------------------- end to end, host buffers
    if args.no_e2e:
        return finish(args, w, world, rank, ms_max, routing, roof, layer, stage_ms,
                      clk, None, x, wt, b)
    # Pipelined like a serving loop: step i+1's input is copied host -> device on one copy
    # stream and step i-1's output device -> host on another while step i computes; every
    # step still moves its full input and output across the bus inside the timed region.
    x_host = torch.empty((w.T, w.d), dtype=torch.bfloat16).pin_memory()
    x_host.copy_(x.cpu())
    y_host = [torch.empty((w.T, w.d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    cs = torch.cuda.current_stream()
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    e2e_steps = args.steps

    def e2e_run(n):
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        hs.wait_stream(cs)
        ds.wait_stream(cs)
        with torch.cuda.stream(hs):
            x_dev[0].copy_(x_host, non_blocking=True)
            h2d_done[0].record(hs)
        for i in range(n):
            cur = i % 2
            if i + 1 < n:
                nxt = (i + 1) % 2
                if i >= 1:
                    hs.wait_event(comp_done[nxt])  # step i-1 has finished reading x_dev[nxt]
                with torch.cuda.stream(hs):
                    x_dev[nxt].copy_(x_host, non_blocking=True)
                    h2d_done[nxt].record(hs)
            cs.wait_event(h2d_done[cur])
            if i >= 2:
                cs.wait_event(d2h_done[cur])  # y_dev[cur] of step i-2 has left the device
            c = counts[n_steps + (i % args.steps)]
            dense_fork(cs)
            forward(x_dev[cur], y_dev[cur], c, stream=cs)
            mb.moe_bias_update(dm, c, b, pid_state, params, stream=cs)
            dense_join(cs)
            comp_done[cur].record(cs)
            ds.wait_event(comp_done[cur])
            with torch.cuda.stream(ds):
                y_host[cur].copy_(y_dev[cur], non_blocking=True)
                d2h_done[cur].record(ds)
        cs.wait_stream(ds)
        cs.wait_stream(hs)

    e2e_run(2)  # warm the copy path
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cs)
    e2e_run(e2e_steps)
    e1.record(cs)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
    e2e = {"value": round(job_throughput(world, w.T, e2e_steps, e2e_ms), 1), "unit": UNIT,
           "h2d_bytes_per_step": int(x_host.numel() * 2),
           "d2h_bytes_per_step": int(y_host[0].numel() * 2),
           "pipelined": "input and output copies on two copy streams, overlapped with compute"}
    return finish(args, w, world, rank, ms_max, routing, roof, layer, stage_ms, clk,
                  e2e, x, wt, b)


def finish(args, w, world, rank, ms_max, routing, roof, layer, stage_ms, clk, e2e, x, wt, b):
    A_steps, U_steps, load_ratio = routing
    near_ties = layer.pop("near_tie_tokens", None)
    decode = layer.pop("decode", None)
    decode_fp8 = layer.pop("decode_fp8", None)
    result = {
        "metric": METRIC, "value": round(job_throughput(world, w.T, args.steps, ms_max), 1),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> f32" if args.fp8_activations else "bf16",
        "data": "synthetic (seeded; x~N(0,1), weights~N(0,0.02^2) bf16, biases~U(-0.05,0.05))",
        "config": {
            "workload": w.name, "T": w.T, "d": w.d, "N": w.N, "Z": w.Z, "K": w.K, "I": w.I,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs larger than L2 (weights %.1f GB, x %.0f MB); no flush"
                  % (w.weight_bytes / 1e9, w.T * w.d * 2 / 1e6),
            "step": "moe_forward + moe_bias_update (PID target %.1f, kp=%g ki=%g kd=%g)"
                    % ((w.pid_target,) + PID_GAINS),
            "variant": {"renormalize_gates": bool(args.renormalize_gates),
                        "balance_gamma": args.balance_gamma,
                        "expert_weights": "fp8 e4m3, 128x128 blocks" if args.fp8 else "bf16",
                        "activations": "fp8 e4m3, 1x128 blocks (E4M3 x E4M3 MMAs)"
                                       if args.fp8_activations else "bf16",
                        "fused_combine": bool(args.fused_combine),
                        "scmoe_dense_ffn": args.scmoe or None},
            "mean_ffn_experts_per_token": round(float(np.mean(A_steps)) / w.T, 4),
            "distinct_ffn_experts": int(np.mean(U_steps)),
            "ffn_load_max_over_mean": round(float(np.mean(load_ratio)), 2),
        },
        "roofline": roof,
        "layer": layer,
        "near_tie_tokens": near_ties,
        "stages_ms": {k: round(v / args.steps, 4) for k, v in stage_ms.items()},
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": (LAUNCHES_PER_STEP + (2 if args.scmoe else 0) +
                         (1 if args.fp8_activations else 0)) * args.steps,
    }
    if decode is not None:
        result["decode"] = decode
    if decode_fp8 is not None:
        result["decode_fp8_activations"] = decode_fp8
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
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode (T=128) record on the same weights")
    ap.add_argument("--renormalize-gates", action="store_true",
                    help="variant: gates renormalised over the K selected experts")
    ap.add_argument("--scmoe", type=int, default=0, metavar="I_DENSE",
                    help="variant: a dense SwiGLU FFN of this intermediate width (the ScMoE "
                         "shortcut branch) on a second stream beside each step")
    ap.add_argument("--fp8", action="store_true",
                    help="variant: block-wise FP8 (E4M3) expert weights, quantised on the GPU")
    ap.add_argument("--fp8-activations", action="store_true",
                    help="variant (with --fp8): E4M3 activations too, 1x128 blocks, read by "
                         "E4M3 x E4M3 tensor-core MMAs")
    ap.add_argument("--fused-combine", action="store_true",
                    help="variant: the combine fused into the down projection's epilogue")
    ap.add_argument("--balance-gamma", type=float, default=0.0,
                    help="variant: step of the per-expert balancing term after the PID step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.fp8_activations and not args.fp8:
        ap.error("--fp8-activations needs --fp8")
    if args.fused_combine and args.fp8:
        ap.error("--fused-combine runs with bf16 weights only")
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
