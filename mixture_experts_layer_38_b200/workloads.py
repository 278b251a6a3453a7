"""Seeded synthetic workloads for the MoE layer with zero-computation experts.

This module only draws random inputs; it holds none of the layer's arithmetic, and both the
CUDA path's tests and the CPU oracle take their inputs from it.

The five workloads (tokens T, model width d, N SwiGLU FFN experts of intermediate width I,
Z zero-computation experts, K experts per token):

    tiny     T=64     d=128   N=8    I=256   Z=4    K=3    biases 0
    mid      T=4096   d=2048  N=64   I=1024  Z=32   K=6    biases ~ U(-0.05, 0.05)
    decode   T=128    d=6144  N=512  I=2048  Z=256  K=12   biases ~ U(-0.05, 0.05)
    prefill  T=16384  d=6144  N=512  I=2048  Z=256  K=12   biases ~ U(-0.05, 0.05)
    skewed   T=8192   d=6144  N=512  I=2048  Z=256  K=12   biases ~ U(-0.05, 0.05), plus a
             Zipf(s=1.1) per-expert router-logit offset; 50 PID steps toward 8 FFN experts/token

The expert pool size (512 FFN + 256 zero experts, K=12) and the ~8 activated experts follow
the LongCat-Flash descriptions ("美团LongCat-Flash：算力调度新纪元", §技术创新, caption (b)).
``pid_target`` is the set-point of the PID step the benchmark runs after every forward pass:
8 FFN experts per token at K=12, and the same 2/3 share of K for the small workloads.

Distributions: x ~ N(0, 1) and every weight ~ N(0, 0.02^2), rounded to bf16; biases fp32.
Weights come from one generator seeded with ``seed`` in the order W_r, b, then per expert
W_g[i], W_u[i], W_d[i]; tokens come from a second generator seeded from (seed, step), so a
PID run draws a fresh batch every step while the weights stay fixed.

The skewed workload realises its logit offset c_i = -s * ln(i + 1) (rank = expert index + 1,
so FFN experts hold the top ranks) inside the inputs themselves: feature 0 of every token is
set to 1 and column 0 of W_r to c_i, so x . W_r[i] carries c_i (rounded to bf16) and the layer
itself is unchanged.

Small workloads are drawn on the CPU (identical values on every machine); workloads whose
weights exceed 2 GB are drawn on the target CUDA device with torch's CUDA generator.
"""
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    N: int
    Z: int
    K: int
    I: int
    bias_range: float = 0.05
    zipf_s: float = 0.0
    pid_steps: int = 0
    pid_target: float = 8.0

    @property
    def E(self) -> int:
        return self.N + self.Z

    @property
    def expert_weight_bytes(self) -> int:
        """bf16 bytes of one FFN expert (W_g, W_u: I x d; W_d: d x I)."""
        return 3 * self.d * self.I * 2

    @property
    def weight_bytes(self) -> int:
        return self.N * self.expert_weight_bytes + self.E * self.d * 2

    def dims(self) -> dict:
        return dict(T=self.T, d=self.d, N=self.N, Z=self.Z, K=self.K, I=self.I)


WORKLOADS = {
    "tiny": Workload("tiny", T=64, d=128, N=8, Z=4, K=3, I=256, bias_range=0.0, pid_target=2.0),
    "mid": Workload("mid", T=4096, d=2048, N=64, Z=32, K=6, I=1024, pid_target=4.0),
    "decode": Workload("decode", T=128, d=6144, N=512, Z=256, K=12, I=2048),
    "prefill": Workload("prefill", T=16384, d=6144, N=512, Z=256, K=12, I=2048),
    "skewed": Workload("skewed", T=8192, d=6144, N=512, Z=256, K=12, I=2048, zipf_s=1.1,
                       pid_steps=50, pid_target=8.0),
    # The prefill layer's widths with a sixteenth of its experts and tokens (2.4 GB of weights,
    # still far above the L2): the small case for multi-pass profiler captures of the
    # 256-token-tile GEMMs.
    "prefill_small": Workload("prefill_small", T=1536, d=6144, N=32, Z=16, K=12, I=2048),
}

_GEN_ON_DEVICE_ABOVE = 2 * 10**9


def _gen_device(w: Workload, device) -> torch.device:
    device = torch.device(device)
    if device.type == "cuda" and w.weight_bytes > _GEN_ON_DEVICE_ABOVE:
        return device
    return torch.device("cpu")


def _normal_bf16(gen, shape, std, dev):
    return (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * std).to(
        torch.bfloat16)


def apply_zipf_router(w: Workload, W_r: torch.Tensor) -> torch.Tensor:
    """In place: column 0 of W_r becomes -s * ln(i + 1), the Zipf(s) logit offset of expert i
    (tokens of a Zipf workload carry a constant 1 in feature 0)."""
    ranks = torch.arange(1, W_r.shape[0] + 1, dtype=torch.float64, device=W_r.device)
    W_r[:, 0] = (-w.zipf_s * torch.log(ranks)).to(torch.bfloat16)
    return W_r


def make_weights(w: Workload, device="cpu", seed: int = 0) -> dict:
    """W_r [E,d], b [E] fp32, W_g/W_u [N,I,d], W_d [N,d,I] (bf16), all on ``device``."""
    gdev = _gen_device(w, device)
    gen = torch.Generator(device=gdev)
    gen.manual_seed(seed)
    W_r = _normal_bf16(gen, (w.E, w.d), 0.02, gdev)
    if w.bias_range > 0:
        b = (torch.rand((w.E,), generator=gen, device=gdev, dtype=torch.float32) * 2.0 - 1.0) \
            * w.bias_range
    else:
        b = torch.zeros((w.E,), dtype=torch.float32, device=gdev)
    if w.zipf_s > 0:
        apply_zipf_router(w, W_r)
    W_g = torch.empty((w.N, w.I, w.d), dtype=torch.bfloat16, device=device)
    W_u = torch.empty((w.N, w.I, w.d), dtype=torch.bfloat16, device=device)
    W_d = torch.empty((w.N, w.d, w.I), dtype=torch.bfloat16, device=device)
    for i in range(w.N):
        W_g[i].copy_(_normal_bf16(gen, (w.I, w.d), 0.02, gdev))
        W_u[i].copy_(_normal_bf16(gen, (w.I, w.d), 0.02, gdev))
        W_d[i].copy_(_normal_bf16(gen, (w.d, w.I), 0.02, gdev))
    return {"W_r": W_r.to(device), "b": b.to(device), "W_g": W_g, "W_u": W_u, "W_d": W_d}


def make_tokens(w: Workload, device="cpu", seed: int = 0, step: int = 0, T: int = None):
    """x [T, d] bf16 for PID step ``step`` (step 0 is the plain workload)."""
    T = w.T if T is None else T
    gdev = _gen_device(w, device)
    gen = torch.Generator(device=gdev)
    gen.manual_seed(1_000_003 * (seed + 1) + 7_919 * step)
    x = torch.randn((T, w.d), generator=gen, device=gdev, dtype=torch.float32).to(torch.bfloat16)
    if w.zipf_s > 0:
        x[:, 0] = 1.0
    return x.to(device)
