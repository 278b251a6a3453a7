"""Pins for the oracle's optional variants: renormalised gates and the per-expert balancing term.

Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 零計算專家 (softmax router R; the
expert-specific bias of the aux-loss-free scheme, adjusted from recent expert usage, which the
PID controller refines).  Pins used:
  * the worked examples in tests/golden/ (closed forms, exact in fp32);
  * scipy's softmax over the selected logits (renormalised softmax gates are the softmax of
    the selected logits alone);
  * invariants: renormalised gates sum to one, so all-zero-expert tokens return x; selecting
    every expert leaves p unchanged; a balanced load leaves the biases unchanged;
  * behaviour: the balancing term alone evens out a toy router's expert loads, and the same
    run with the sign flipped (a planted mistake) does not.
"""
import json
import math
import os

import numpy as np
import scipy.special
import torch

import oracle
from mixture_experts_layer_38_b200.workloads import WORKLOADS, make_tokens, make_weights

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------ renormalised gates
def test_renormalized_worked_example():
    with open(os.path.join(GOLDEN, "router_worked_example.json")) as f:
        ex = json.load(f)
    d, E, K = ex["d"], ex["N"] + ex["Z"], ex["K"]
    W = np.zeros((E, d), np.float32)
    W[:, 0] = ex["W_r_column0"]
    r = oracle.router(_bf16([ex["x"]]), _bf16(W), np.array(ex["b"], np.float32), K,
                      renormalize=True)
    assert r["topk_idx"][0].tolist() == ex["expected_topk_idx"]  # selection is unchanged
    e2 = math.exp(2)
    np.testing.assert_allclose(r["topk_gate"][0], [1 / (1 + e2), e2 / (1 + e2)], rtol=1e-14)


def test_renormalized_gates_are_softmax_of_selected_logits():
    g = torch.Generator().manual_seed(21)
    T, d, E, K = 64, 24, 20, 5
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    W_r = (torch.randn((E, d), generator=g) * 0.3).to(torch.bfloat16)
    b = ((torch.rand((E,), generator=g) * 2 - 1) * 0.05).float()
    r = oracle.router(x, W_r, b, K, renormalize=True)
    logits = (x.double() @ W_r.double().T).numpy()
    for t in range(T):
        sel = r["topk_idx"][t]
        np.testing.assert_allclose(r["topk_gate"][t], scipy.special.softmax(logits[t, sel]),
                                   rtol=1e-12)
    np.testing.assert_allclose(r["topk_gate"].sum(axis=1), 1.0, rtol=1e-14)


def test_renormalize_with_every_expert_selected_keeps_p():
    g = torch.Generator().manual_seed(5)
    x = torch.randn((8, 16), generator=g).to(torch.bfloat16)
    W_r = (torch.randn((6, 16), generator=g) * 0.3).to(torch.bfloat16)
    b = torch.zeros(6)
    plain = oracle.router(x, W_r, b, 6)
    renorm = oracle.router(x, W_r, b, 6, renormalize=True)
    np.testing.assert_allclose(renorm["topk_gate"], plain["topk_gate"], rtol=1e-14)


def test_renormalized_all_zero_expert_tokens_return_x():
    # Every token selects only zero experts (their biases dominate): y = (sum g) x = x.
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=3)
    x = make_tokens(w, seed=3)
    b = torch.zeros(w.E)
    b[w.N:w.N + w.K] = 10.0
    ref = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K,
                         renormalize=True)
    assert (ref["topk_idx"] >= w.N).all()
    np.testing.assert_allclose(ref["y"], x.double().numpy(), rtol=1e-14, atol=0)


def test_renormalized_forward_scales_each_token_by_its_gate_sum():
    # Renormalising divides every term of y_t by the same sum, so y_renorm = y / sum(g).
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=9)
    x = make_tokens(w, seed=9)
    b = (torch.rand(w.E, generator=torch.Generator().manual_seed(2)) * 0.02).float()
    plain = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    renorm = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K,
                            renormalize=True)
    assert (plain["topk_idx"] == renorm["topk_idx"]).all()
    s = plain["topk_gate"].sum(axis=1, keepdims=True)
    np.testing.assert_allclose(renorm["y"], plain["y"] / s, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------------------ per-expert balancing term
def test_balance_worked_example():
    with open(os.path.join(GOLDEN, "balance_worked_example.json")) as f:
        ex = json.load(f)
    b = np.array(ex["b_before"], np.float32)
    oracle.balance_step(np.array(ex["counts"], np.int32), b, ex["N"], ex["gamma"])
    assert b.tolist() == ex["b_after"]


def test_balance_balanced_load_and_zero_gamma_change_nothing():
    b = np.array([0.1, 0.2, 0.3, 0.4, 9.0], np.float32)
    before = b.copy()
    oracle.balance_step(np.array([4, 4, 4, 4, 100], np.int32), b, 4, 0.5)
    assert b.tobytes() == before.tobytes()
    oracle.balance_step(np.array([1, 9, 4, 4, 0], np.int32), b, 4, 0.0)
    assert b.tobytes() == before.tobytes()


def test_balance_sign_is_exact_when_the_mean_is_not_representable():
    # total 10 over N = 3: mean 3.333...; loads 3 and 4 straddle it, no load equals it.
    b = np.zeros(3, np.float32)
    oracle.balance_step(np.array([3, 4, 3], np.int32), b, 3, 1.0)
    assert b.tolist() == [1.0, -1.0, 1.0]


def _toy_balance_run(gamma, steps=60):
    """Router + dispatch + balancing term on a toy router that favours a few FFN experts."""
    N, Z, K, d, T = 8, 4, 2, 16, 256
    g = torch.Generator().manual_seed(31)
    W_r = torch.randn((N + Z, d), generator=g) * 0.2
    W_r[:3, 0] += 2.0  # experts 0-2 get much larger logits
    W_r = W_r.to(torch.bfloat16)
    b = np.zeros(N + Z, np.float32)
    b[N:] = -1.0  # keep the zero experts out of the way
    ratios = []
    for s in range(steps):
        x = torch.randn((T, d), generator=torch.Generator().manual_seed(500 + s))
        x[:, 0] = 1.0
        r = oracle.router(x.to(torch.bfloat16), W_r, b, K)
        c = oracle.dispatch(r["topk_idx"], N, N + Z)["counts"]
        ratios.append(c[:N].max() / (c[:N].sum() / N))
        oracle.balance_step(c, b, N, gamma)
    return ratios


def test_balance_evens_out_a_skewed_router_and_a_flipped_sign_does_not():
    good = _toy_balance_run(0.01)
    assert good[0] > 2.5  # three favoured experts carry most of the load at first
    assert np.mean(good[-10:]) < 1.5
    bad = _toy_balance_run(-0.01)  # planted mistake: the sign of the step flipped
    assert np.mean(bad[-10:]) > 2.5


def test_balance_after_pid_composes_in_order():
    # PID first (uniform shift u), then the sign term; both exact here, so the sum is exact.
    counts = np.array([6, 2, 4, 0, 0], np.int32)  # N = 3, total 12, mean 4, T = 4: m = 3
    b = np.zeros(5, np.float32)
    st = np.zeros(2, np.float32)
    oracle.pid_step(counts, b, st, 3, 2, 4, 2.0, 0.5, 0.0, 0.0)  # e = (2 - 3)/2, u = -0.25
    oracle.balance_step(counts, b, 3, 0.125)
    assert b.tolist() == [-0.375, -0.125, -0.25, 0.0, 0.0]
