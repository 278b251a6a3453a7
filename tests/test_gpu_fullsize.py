"""GPU parity at the full 512 + 256-expert size (d = 6144, I = 2048, K = 12), in the launch
configuration the benchmark times (moe_forward).

For EVERY token of each batch (decode 128, prefill 16384, skewed 8192): the routing against the
oracle's router run on the whole batch (ids bit-exact wherever the oracle's gap exceeds 1e-4,
near-ties counted and eps-valid, every gate equal to the oracle's probability of the id chosen
up to the propagated error of the GPU's fp32 router logits, themselves within the fp32
accumulation bound), and the dispatch tables bit-exact against the oracle's dispatch of the
GPU's routing.  The layer output y on a seeded token sample plus the tokens the GPU routed
differently from the oracle (near-ties), against the oracle's layer run on the GPU's routing.
Besides: the staged calls reproduce moe_forward bit for bit, and the PID run of the skewed
workload settles at its set-point.

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
from parity import (Stages, assert_y_close, check_dispatch_vs_oracle,
                    check_gates_against_logits, check_routing_full, exact_logits,
                    gpu_routing_for_oracle, to_np)

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


def _full_check(w, x, wt, n_sample, seed, n_differ=8):
    st = Stages(w, x, wt)  # the weights are already on the GPU: no copies
    st.forward()
    y_fwd = st.y.clone()
    counts = to_np(st.counts)
    assert counts.sum() == w.T * w.K
    assert st.device_status() == 0
    # Staged calls: same kernels and launch configurations as moe_forward.
    st.route()
    logits = st.logits()
    st.dispatch()
    idx, gate = to_np(st.topk_idx), to_np(st.topk_gate)
    np.testing.assert_array_equal(to_np(st.counts), counts)
    st.expert_ffn()
    st.combine()
    assert torch.equal(st.y, y_fwd)
    # The combine fused into the down projection gives the same bits.
    fused = Stages(w, x, wt, flags=mb.FUSED_COMBINE)
    fused.forward()
    assert fused.device_status() == 0
    assert torch.equal(fused.y, y_fwd), "fused combine differs at full size"
    del fused
    # Whole-batch routing and dispatch against the oracle.
    W_r, b = wt["W_r"].cpu(), wt["b"].cpu()
    xc = x.cpu()
    ref = oracle.router(xc, W_r, b, w.K, want_probs=True, want_scores=True)
    stats = check_routing_full(idx, gate, ref, logits, xc, W_r)
    check_dispatch_vs_oracle(idx, gate, to_np(st.counts), to_np(st.offsets), to_np(st.perm_tok),
                             to_np(st.perm_gate), to_np(st.slot_pos), w.N, w.E)
    ffn_per_tok = (idx < w.N).sum(axis=1)
    assert ((ffn_per_tok >= 0) & (ffn_per_tok <= w.K)).all()
    # y: a seeded sample plus near-tie tokens the GPU routed differently, on the GPU's routing.
    differ = np.flatnonzero((idx != ref["topk_idx"]).any(axis=1))
    rng = np.random.default_rng(seed)
    tokens = np.union1d(rng.choice(w.T, n_sample, replace=False),
                        differ[rng.permutation(len(differ))[:n_differ]])
    out = oracle.forward_sampled(np.arange(len(tokens)), oracle.bf16_bits(xc)[tokens], W_r, b,
                                 w.N, w.Z, w.K, _fetch(wt),
                                 routing=gpu_routing_for_oracle(idx, ref, tokens))
    y = oracle.bf16_to_f64(to_np(y_fwd))[tokens]
    rel = assert_y_close(y, out["y"], f"{w.name} y")
    n_diff_in = int(np.isin(tokens, differ).sum())
    print(f"{w.name}: routing {stats}; mean FFN/token {ffn_per_tok.mean():.3f}; y errors "
          f"(max, L2) {rel} on {len(tokens)} tokens ({n_diff_in} routed differently)")
    return counts


def test_decode_full_size(big_weights):
    w = WORKLOADS["decode"]
    x = make_tokens(w, DEV, seed=0)
    _full_check(w, x, big_weights, n_sample=32, seed=1)


def test_prefill_full_size(big_weights):
    w = WORKLOADS["prefill"]
    x = make_tokens(w, DEV, seed=0)
    _full_check(w, x, big_weights, n_sample=24, seed=2)


@pytest.mark.parametrize("name", ["prefill", "skewed"])
def test_router_logits_and_gates_whole_batch(big_weights, name):
    """The router's fp32 logits (moe_router_logits) of every token against l = x W_r^T in fp64,
    within the fp32 accumulation bound, and every gate against the first-order propagation of
    those logit errors through the softmax (check_gates_against_logits).  The skewed
    workload's Zipf term is the first term every later accumulation step rounds against, so
    its logit and gate errors are the largest of the workloads."""
    w = WORKLOADS[name]
    wt = dict(big_weights)
    if name == "skewed":
        wt["W_r"] = apply_zipf_router(w, big_weights["W_r"].clone())
    x = make_tokens(w, DEV, seed=0)
    st = Stages(w, x, wt)
    st.route()
    logits = st.logits()
    l_ref, mag = exact_logits(x, wt["W_r"])
    ref = oracle.router(x.cpu(), wt["W_r"].cpu(), wt["b"].cpu(), w.K, want_probs=True,
                        want_scores=True)
    gate_err = check_gates_against_logits(to_np(st.topk_idx), to_np(st.topk_gate), logits, x,
                                          wt["W_r"], ref["probs"])
    delta = np.abs(logits - l_ref)
    print(f"{name} router logits at d={w.d}: max|l~ - l| = {delta.max():.3e} "
          f"= {(delta / mag).max() * 2 ** 24:.1f} u sum|xW| at most (bound "
          f"{2 * (w.d // 16 + 16)}); max |l| {np.abs(l_ref).max():.2f}; max gate rel err "
          f"{gate_err:.3e}")
    assert st.device_status() == 0


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
    W_r, b = big_weights["W_r"].cpu(), big_weights["b"].cpu()
    ref = oracle.router(x.cpu(), W_r, b, w.K, want_probs=True, want_scores=True)
    st = Stages(w, x, big_weights)
    st.route()
    idx = to_np(st.topk_idx)
    check_routing_full(idx, to_np(st.topk_gate), ref, st.logits(), x, big_weights["W_r"])
    differ = np.flatnonzero((idx != ref["topk_idx"]).any(axis=1))
    tokens = np.union1d(np.random.default_rng(5).choice(w.T, 24, replace=False), differ[:8])
    out = oracle.forward_sampled(np.arange(len(tokens)), oracle.bf16_bits(x.cpu())[tokens], W_r,
                                 b, w.N, w.Z, w.K, fetch_deq,
                                 routing=gpu_routing_for_oracle(idx, ref, tokens))
    y_s = oracle.bf16_to_f64(to_np(y))[tokens]
    assert_y_close(y_s, out["y"], "decode fp8 y")

    # FP8 activations too (the benchmark's --fp8 --fp8-activations leg): the same routing, the
    # oracle's FP8-activation experts on the same sampled tokens
    dm8 = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=mb.FP8_ACTIVATIONS)
    ws8 = mb.alloc_workspace(dm8, DEV)
    y8 = torch.empty_like(y)
    mb.moe_forward_fp8(dm8, x, big_weights["W_r"], big_weights["b"], fw, y8, None, ws8)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws8) == 0
    out8 = oracle.forward_sampled(np.arange(len(tokens)), oracle.bf16_bits(x.cpu())[tokens], W_r,
                                  b, w.N, w.Z, w.K, fetch_deq,
                                  routing=gpu_routing_for_oracle(idx, ref, tokens), fp8_act=True)
    y8_s = oracle.bf16_to_f64(to_np(y8))[tokens]
    assert_y_close(y8_s, out8["y"], "decode fp8-activation y")
    del ws8, fw
