"""GPU parity at the full 512 + 256-expert size (d = 6144, I = 2048, K = 12), in the launch
configuration the benchmark times (moe_forward), on sampled tokens the oracle computes one by
one, plus properties that hold for every token: counts sum to T*K, the dispatch is exactly
the stable (expert, token) sort of the GPU's own routing, the staged calls reproduce
moe_forward bit for bit, and the PID run of the skewed workload settles at its set-point.

One weight set (38.7 GB, seed 0) serves decode, prefill and skewed: the three share every
expert weight and differ only in column 0 of W_r for the skewed (Zipf) workload.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import (WORKLOADS, apply_zipf_router, make_tokens,
                                                     make_weights)
from parity import Stages, assert_y_close, check_dispatch_properties, check_routing, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def big_weights():
    wt = make_weights(WORKLOADS["prefill"], DEV, seed=0)
    yield wt
    del wt
    torch.cuda.empty_cache()


def _fetch(wt):
    return lambda e: (wt["W_g"][e].cpu(), wt["W_u"][e].cpu(), wt["W_d"][e].cpu())


def _full_check(w, x, wt, n_sample, seed):
    st = Stages(w, x, wt)  # the weights are already on the GPU: no copies
    st.forward()
    y_fwd = st.y.clone()
    counts = to_np(st.counts)
    assert counts.sum() == w.T * w.K
    assert st.device_status() == 0
    # Staged calls: same kernels and launch configurations as moe_forward.
    st.route()
    st.dispatch()
    idx = to_np(st.topk_idx)
    check_dispatch_properties(idx, to_np(st.counts), to_np(st.offsets), to_np(st.perm_tok),
                              to_np(st.slot_pos), w.N, w.E)
    np.testing.assert_array_equal(to_np(st.counts), counts)
    ffn_per_tok = (idx < w.N).sum(axis=1)
    assert ((ffn_per_tok >= 0) & (ffn_per_tok <= w.K)).all()
    st.expert_ffn()
    st.combine()
    assert torch.equal(st.y, y_fwd)
    # Oracle on a seeded token sample.
    tokens = np.sort(np.random.default_rng(seed).choice(w.T, n_sample, replace=False))
    xs = x[torch.from_numpy(tokens).to(x.device)].cpu()
    W_r, b = wt["W_r"].cpu(), wt["b"].cpu()
    ref = oracle.router(xs, W_r, b, w.K, want_scores=True)
    near, differ = check_routing(idx[tokens], to_np(st.topk_gate)[tokens], ref, ref["scores"])
    out = oracle.forward_sampled(np.arange(n_sample), xs, W_r, b, w.N, w.Z, w.K, _fetch(wt),
                                 routing=ref)
    same = (idx[tokens] == ref["topk_idx"]).all(axis=1)
    y = oracle.bf16_to_f64(to_np(y_fwd))[tokens]
    rel = assert_y_close(y[same], out["y"][same], f"{w.name} y")
    print(f"{w.name}: mean FFN/token {ffn_per_tok.mean():.3f}, near-ties {near}/{n_sample}, "
          f"differing {differ}, y errors {rel}")
    return counts


def test_decode_full_size(big_weights):
    w = WORKLOADS["decode"]
    x = make_tokens(w, DEV, seed=0)
    _full_check(w, x, big_weights, n_sample=32, seed=1)


def test_prefill_full_size(big_weights):
    w = WORKLOADS["prefill"]
    x = make_tokens(w, DEV, seed=0)
    _full_check(w, x, big_weights, n_sample=24, seed=2)


def test_skewed_pid_full_size(big_weights):
    w = WORKLOADS["skewed"]
    wt = dict(big_weights)
    wt["W_r"] = apply_zipf_router(w, big_weights["W_r"].clone())
    x0 = make_tokens(w, DEV, seed=0, step=0)
    counts0 = _full_check(w, x0, wt, n_sample=16, seed=3)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = mb.alloc_workspace(dm, DEV)
    y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=DEV)
    b = wt["b"].clone()
    state = torch.zeros(2, dtype=torch.float32, device=DEV)
    counts = torch.zeros((w.pid_steps, w.E), dtype=torch.int32, device=DEV)
    params = mb.PidParams(w.pid_target, 0.005, 0.002, 0.0)
    for s in range(w.pid_steps):
        x = x0 if s == 0 else make_tokens(w, DEV, seed=0, step=s)
        mb.moe_forward(dm, x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], y, counts[s], ws)
        mb.moe_bias_update(dm, counts[s], b, state, params)
    assert mb.moe_last_device_error(ws) == 0
    c = counts.cpu().numpy()
    assert (c[0] == counts0).all()
    means = c[:, :w.N].sum(axis=1) / w.T
    print("skewed PID trajectory (mean FFN experts/token):", np.round(means, 3).tolist())
    assert means[0] > w.pid_target + 1.0  # the Zipf offset favours FFN experts at the start
    assert abs(means[-10:].mean() - w.pid_target) < 0.15
    assert (b[w.N:] == wt["b"][w.N:]).all()  # zero-expert biases never move


def test_decode_fp8_full_size(big_weights):
    # Block-wise FP8 expert weights at full size, in the launch configuration the benchmark's
    # --fp8 leg times (moe_forward_fp8): sampled tokens against the oracle run on the
    # dequantised weights (q * 2^e, exact in bf16).
    w = WORKLOADS["decode"]
    x = make_tokens(w, DEV, seed=0)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    fw = mb.quantize_expert_weights_fp8(dm, big_weights["W_g"], big_weights["W_u"],
                                        big_weights["W_d"])
    ws = mb.alloc_workspace(dm, DEV)
    y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=DEV)
    counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    mb.moe_forward_fp8(dm, x, big_weights["W_r"], big_weights["b"], fw, y, counts, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    assert int(counts.sum().item()) == w.T * w.K

    def fetch_deq(e):
        out = []
        for k in ("g", "u", "d"):
            bits = oracle.dequantize_fp8_blocks(fw["q_" + k][e:e + 1].cpu().numpy(),
                                                fw["s_" + k][e:e + 1].cpu().numpy())[0]
            out.append(bits)
        return tuple(out)
    n_sample = 24
    tokens = np.sort(np.random.default_rng(5).choice(w.T, n_sample, replace=False))
    xs = x[torch.from_numpy(tokens).to(DEV)].cpu()
    W_r, b = big_weights["W_r"].cpu(), big_weights["b"].cpu()
    ref = oracle.router(xs, W_r, b, w.K, want_scores=True)
    out = oracle.forward_sampled(np.arange(n_sample), xs, W_r, b, w.N, w.Z, w.K, fetch_deq,
                                 routing=ref)
    st = Stages(w, x, big_weights)
    st.route()
    idx = to_np(st.topk_idx)[tokens]
    check_routing(idx, to_np(st.topk_gate)[tokens], ref, ref["scores"])
    same = (idx == ref["topk_idx"]).all(axis=1)
    y_s = oracle.bf16_to_f64(to_np(y))[tokens]
    assert_y_close(y_s[same], out["y"][same], "decode fp8 y")
    del fw
