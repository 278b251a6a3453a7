"""GPU parity of the optional variants against the CPU oracle, through the C ABI.

  * MOE_RENORMALIZE_GATES: gates divided by their sum over the K selected experts; routing
    (ids) unchanged, gates within the routing rule's rtol, the whole layer within the output
    tolerances, on tiny (every token) and mid (a token sample, several tiles and a ragged
    tail).
  * the per-expert balancing term of moe_bias_update (balance_gamma != 0): bit-exact with the
    oracle's PID step followed by its balancing step, over 20 steps of random loads.
Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 零計算專家.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import WORKLOADS, Workload, make_tokens, make_weights
from parity import (GAP_EPS, GATE_RTOL, Stages, assert_y_close, check_gates_against_logits,
                    gpu_routing_for_oracle, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(name, T=None, seed=0):
    w = WORKLOADS[name]
    wt = make_weights(w, seed=seed)
    x = make_tokens(w, seed=seed, T=T)
    if T is not None:
        w = Workload(w.name, T=T, d=w.d, N=w.N, Z=w.Z, K=w.K, I=w.I, bias_range=w.bias_range)
    return w, x, wt


@pytest.mark.parametrize("name,T", [("tiny", None), ("mid", None)])
def test_route_renormalized_matches_oracle(name, T):
    w, x, wt = _case(name, T=T)
    st = Stages(w, x, wt, flags=mb.RENORMALIZE_GATES)
    st.route()
    torch.cuda.synchronize()
    assert st.device_status() == 0
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K, want_probs=True, want_scores=True)
    gate, idx = to_np(st.topk_gate), to_np(st.topk_idx)
    clear = ref["gap"] > GAP_EPS
    np.testing.assert_array_equal(idx[clear], ref["topk_idx"][clear])
    check_gates_against_logits(idx, gate, st.logits(), x, wt["W_r"], ref["probs"],
                               renormalize=True)
    np.testing.assert_allclose(gate.astype(np.float64).sum(axis=1), 1.0, rtol=0, atol=4e-6)


@pytest.mark.parametrize("name,T,sample", [("tiny", None, None), ("mid", 333, 48)])
def test_forward_renormalized_matches_oracle(name, T, sample):
    w, x, wt = _case(name, T=T, seed=1)
    st = Stages(w, x, wt, flags=mb.RENORMALIZE_GATES)
    st.forward()
    torch.cuda.synchronize()
    assert st.device_status() == 0
    y = oracle.bf16_to_f64(to_np(st.y))
    # Whole-batch routing; y of a sample plus every token the GPU routed differently, against
    # the oracle run on the GPU's selection with the gates renormalised over that selection.
    r = oracle.router(x, wt["W_r"], wt["b"], w.K, want_probs=True, want_scores=True)
    st.route()
    idx = to_np(st.topk_idx)
    clear = r["gap"] > GAP_EPS
    np.testing.assert_array_equal(idx[clear], r["topk_idx"][clear])
    differ = np.flatnonzero((idx != r["topk_idx"]).any(axis=1))
    tokens = np.arange(w.T) if sample is None else np.union1d(
        np.random.default_rng(3).choice(w.T, sample, replace=False), differ[:16])
    routing = gpu_routing_for_oracle(idx, r, tokens)
    oracle.renormalize_gates(routing["topk_gate"])
    np.testing.assert_allclose(to_np(st.topk_gate)[tokens], routing["topk_gate"],
                               rtol=GATE_RTOL, atol=1e-30)
    ref = oracle.forward_sampled(np.arange(len(tokens)), oracle.bf16_bits(x)[tokens],
                                 wt["W_r"], wt["b"], w.N, w.Z, w.K,
                                 lambda e: (wt["W_g"][e], wt["W_u"][e], wt["W_d"][e]),
                                 routing=routing)
    assert_y_close(y[tokens], ref["y"], f"{name} renormalised y")


def test_renormalized_all_zero_expert_tokens_return_x():
    w, x, wt = _case("tiny", seed=2)
    b = torch.zeros(w.E)
    b[w.N:w.N + w.K] = 10.0  # every token picks the same K zero experts
    wt["b"] = b
    st = Stages(w, x, wt, flags=mb.RENORMALIZE_GATES)
    st.forward()
    torch.cuda.synchronize()
    assert st.device_status() == 0
    assert (to_np(st.counts)[:w.N] == 0).all()
    y = oracle.bf16_to_f64(to_np(st.y))
    xf = x.double().numpy()
    # (sum of K fp32 gates, which is 1 to a few ulps) * x, rounded once to bf16
    assert (np.abs(y - xf) <= 2.0 ** -8 * np.abs(xf) + 1e-6).all()


def test_pid_with_balancing_term_matches_oracle_bit_exact():
    w = WORKLOADS["skewed"]
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    rng = np.random.default_rng(11)
    b = (rng.uniform(-0.05, 0.05, w.E)).astype(np.float32)
    st = np.zeros(2, np.float32)
    b_gpu = torch.from_numpy(b.copy()).to(DEV)
    st_gpu = torch.zeros(2, dtype=torch.float32, device=DEV)
    gamma = 1e-3
    params = mb.PidParams(8.0, 0.005, 0.002, 0.001, gamma)
    for step in range(20):
        counts = rng.integers(0, 400, w.E).astype(np.int32)
        if step == 3:
            counts[:w.N] = 300  # a perfectly balanced load: the sign term is zero everywhere
        mb.moe_bias_update(dm, torch.from_numpy(counts).to(DEV), b_gpu, st_gpu, params)
        oracle.pid_step(counts, b, st, w.N, w.K, w.T, 8.0, 0.005, 0.002, 0.001)
        oracle.balance_step(counts, b, w.N, gamma)
        assert b_gpu.cpu().numpy().tobytes() == b.tobytes(), step
        assert st_gpu.cpu().numpy().tobytes() == st.tobytes(), step
