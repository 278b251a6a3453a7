"""Pins for the CPU oracle, each against something other than the oracle itself.

Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 零計算專家 (softmax router R, per-expert bias
b_i steering selection only, K experts per token, zero-computation experts return their input,
a PID controller on the biases).  Pins used:
  * a worked example with a closed form (tests/golden/router_worked_example.json);
  * brute-force enumeration of every K-subset on tiny expert pools;
  * library routines: scipy's softmax, torch fp64 matmul / silu, numpy's stable lexsort;
  * invariants: gates sum with the rest of p to 1, bias shifts by a constant change nothing,
    per-token FFN counts lie in [0, K], all-zero-expert tokens return (sum g) x;
  * the PID's closed form on a constant load, its convergence on a toy load, and
    checkpoint/resume of its state.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mixture_experts_layer_38_b200.workloads import WORKLOADS, make_tokens, make_weights

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _rand_case(rng_seed, T, d, E, bias_scale=0.05, w_std=0.3):
    g = torch.Generator().manual_seed(rng_seed)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    W_r = (torch.randn((E, d), generator=g) * w_std).to(torch.bfloat16)
    b = (torch.rand((E,), generator=g) * 2 - 1) * bias_scale
    return x, W_r, b.float()


def _library_scores(x, W_r, b):
    """p and s from library routines: torch fp64 matmul, then scipy's softmax."""
    logits = (x.double() @ W_r.double().T).numpy()
    p = scipy.special.softmax(logits, axis=1)
    return p, p + b.double().numpy()[None, :]


# ------------------------------------------------------------------ worked example (closed form)
def test_router_worked_example():
    with open(os.path.join(GOLDEN, "router_worked_example.json")) as f:
        ex = json.load(f)
    d, E, K = ex["d"], ex["N"] + ex["Z"], ex["K"]
    x = _bf16([ex["x"]])
    W = np.zeros((E, d), np.float32)
    W[:, 0] = ex["W_r_column0"]
    r = oracle.router(x, _bf16(W), np.array(ex["b"], np.float32), K)
    S = 1 + math.exp(1) + math.exp(2) + math.exp(3)
    assert r["topk_idx"][0].tolist() == ex["expected_topk_idx"]
    np.testing.assert_allclose(r["topk_gate"][0], [1 / S, math.exp(2) / S], rtol=1e-14)
    b32 = np.array(ex["b"], np.float32).astype(np.float64)  # the fp32 biases, widened
    gap = (math.exp(2) / S + b32[2]) - (math.exp(3) / S + b32[3])
    assert abs(r["gap"][0] - gap) < 1e-14


# ------------------------------------------------------------------ brute force over K-subsets
@pytest.mark.parametrize("seed,E,K", [(s, E, K) for s in range(6) for E, K in
                                      [(4, 1), (6, 2), (8, 3), (12, 3), (12, 5), (12, 12)]])
def test_router_topk_matches_bruteforce(seed, E, K):
    T, d = 24, 16
    x, W_r, b = _rand_case(100 * seed + E + K, T, d, E)
    r = oracle.router(x, W_r, b, K, want_probs=True, want_scores=True)
    p_lib, s_lib = _library_scores(x, W_r, b)
    np.testing.assert_allclose(r["probs"], p_lib, rtol=1e-12, atol=1e-15)
    for t in range(T):
        s = s_lib[t]
        best = max(itertools.combinations(range(E), K),
                   key=lambda S: (sum(s[i] for i in S), [-i for i in S]))
        assert r["topk_idx"][t].tolist() == list(best), (t, r["topk_idx"][t], best)
        np.testing.assert_allclose(r["topk_gate"][t], p_lib[t, list(best)], rtol=1e-12)
        rest = [i for i in range(E) if i not in best]
        want_gap = min(s[i] for i in best) - max(s[i] for i in rest) if rest else math.inf
        if rest:
            assert abs(r["gap"][t] - want_gap) < 1e-12
        else:
            assert r["gap"][t] == math.inf


def test_router_exact_ties_go_to_lower_index():
    # Identical router rows and equal biases: every score ties, so the K lowest ids win.
    E, K, d = 10, 4, 8
    x = _bf16(np.ones((3, d)))
    W_r = _bf16(np.full((E, d), 0.25))
    r = oracle.router(x, W_r, np.zeros(E, np.float32), K)
    assert (r["topk_idx"] == np.arange(K)).all()
    assert (r["gap"] == 0).all()
    # Raising expert 7 by one ulp-sized bias makes it win one tie.
    b = np.zeros(E, np.float32)
    b[7] = 1e-6
    r = oracle.router(x, W_r, b, K)
    assert (r["topk_idx"] == [0, 1, 2, 7]).all()


def test_softmax_sums_to_one_and_gates_are_unrenormalised_p():
    x, W_r, b = _rand_case(7, 32, 64, 20)
    r = oracle.router(x, W_r, b, 5, want_probs=True)
    np.testing.assert_allclose(r["probs"].sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert ((r["probs"] >= 0) & (r["probs"] <= 1)).all()
    picked = np.take_along_axis(r["probs"], r["topk_idx"].astype(np.int64), axis=1)
    assert (picked == r["topk_gate"]).all()
    assert (r["topk_gate"].sum(axis=1) < 1.0).all()  # not renormalised over the K selected


def test_bias_shift_by_constant_changes_nothing():
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=3)
    x = make_tokens(w, seed=3)
    # Dyadic biases k/1024 with |k| <= 50: b + 0.5 is exact in fp32, so only the shift differs.
    b = torch.randint(-50, 51, (w.E,), generator=torch.Generator().manual_seed(1)).float() / 1024
    r0 = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    r1 = oracle.forward(x, wt["W_r"], b + 0.5, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    assert (r0["topk_idx"] == r1["topk_idx"]).all()
    assert (r0["topk_gate"] == r1["topk_gate"]).all()
    assert (r0["y"] == r1["y"]).all()


def test_bias_changes_selection_not_gate_weights():
    x, W_r, _ = _rand_case(11, 16, 32, 12, w_std=0.2)
    b0 = np.zeros(12, np.float32)
    b1 = np.zeros(12, np.float32)
    b1[[1, 5, 9]] = 1.0  # forces these three into every token's selection
    r0 = oracle.router(x, W_r, b0, 3, want_probs=True)
    r1 = oracle.router(x, W_r, b1, 3, want_probs=True)
    assert (r1["topk_idx"] == [1, 5, 9]).all()
    assert (r0["probs"] == r1["probs"]).all()  # the router's p ignores the bias
    np.testing.assert_array_equal(r1["topk_gate"], r0["probs"][:, [1, 5, 9]])


# ------------------------------------------------------------------ zero experts are identities
def test_all_zero_expert_tokens_return_sum_g_times_x():
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=5)
    x = make_tokens(w, seed=5)
    b = torch.zeros(w.E)
    b[w.N:] = 1.0  # every zero expert outranks every FFN expert; Z >= K
    r = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    assert (r["topk_idx"] >= w.N).all()
    want = r["topk_gate"].sum(axis=1, keepdims=True) * oracle.bf16_to_f64(oracle.bf16_bits(x))
    np.testing.assert_allclose(r["y"], want, rtol=1e-14, atol=1e-300)


def test_single_ffn_expert_reduces_to_swiglu():
    # N=1, Z=0, K=1: p = 1 for the only expert, so y = W_d (silu(W_g x) * W_u x).
    T, d, I = 9, 64, 128
    g = torch.Generator().manual_seed(2)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    W_r = (torch.randn((1, d), generator=g) * 0.02).to(torch.bfloat16)
    W_g = (torch.randn((1, I, d), generator=g) * 0.1).to(torch.bfloat16)
    W_u = (torch.randn((1, I, d), generator=g) * 0.1).to(torch.bfloat16)
    W_d = (torch.randn((1, d, I), generator=g) * 0.1).to(torch.bfloat16)
    r = oracle.forward(x, W_r, torch.zeros(1), W_g, W_u, W_d, 1, 0, 1)
    xd = x.double()
    want = (torch.nn.functional.silu(xd @ W_g[0].double().T) * (xd @ W_u[0].double().T)) \
        @ W_d[0].double().T
    assert (r["topk_gate"] == 1.0).all()
    np.testing.assert_allclose(r["y"], want.numpy(), rtol=1e-11, atol=1e-13)


def test_mixed_ffn_and_zero_slots_by_library():
    # y = p_0 E_0(x) + p_2 x for the worked example (expert 0 FFN, expert 2 zero).
    with open(os.path.join(GOLDEN, "router_worked_example.json")) as f:
        ex = json.load(f)
    d, N, Z, K, I = ex["d"], ex["N"], ex["Z"], ex["K"], 16
    g = torch.Generator().manual_seed(9)
    x = _bf16([ex["x"]])
    W = np.zeros((N + Z, d), np.float32)
    W[:, 0] = ex["W_r_column0"]
    W_g = (torch.randn((N, I, d), generator=g) * 0.5).to(torch.bfloat16)
    W_u = (torch.randn((N, I, d), generator=g) * 0.5).to(torch.bfloat16)
    W_d = (torch.randn((N, d, I), generator=g) * 0.5).to(torch.bfloat16)
    r = oracle.forward(x, _bf16(W), np.array(ex["b"], np.float32), W_g, W_u, W_d, N, Z, K)
    S = 1 + math.exp(1) + math.exp(2) + math.exp(3)
    xd = x.double()
    e0 = (torch.nn.functional.silu(xd @ W_g[0].double().T) * (xd @ W_u[0].double().T)) \
        @ W_d[0].double().T
    want = (1 / S) * e0 + (math.exp(2) / S) * xd
    np.testing.assert_allclose(r["y"], want.numpy(), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ counts and dispatch
def test_ffn_counts_per_token_in_range_and_total():
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=0)
    x = make_tokens(w, seed=0)
    r = oracle.router(x, wt["W_r"], wt["b"], w.K)
    per_tok = (r["topk_idx"] < w.N).sum(axis=1)
    assert ((per_tok >= 0) & (per_tok <= w.K)).all()
    dsp = oracle.dispatch(r["topk_idx"], w.N, w.E)
    assert dsp["counts"].sum() == w.T * w.K
    assert dsp["offsets"][-1] == per_tok.sum()


@pytest.mark.parametrize("seed", range(4))
def test_dispatch_matches_stable_lexsort(seed):
    rng = np.random.default_rng(seed)
    T, K, N, Z = 200, 5, 13, 7
    E = N + Z
    idx = np.stack([np.sort(rng.choice(E, K, replace=False)) for _ in range(T)]).astype(np.int32)
    dsp = oracle.dispatch(idx, N, E)
    tok = np.repeat(np.arange(T), K)
    ex = idx.reshape(-1)
    ffn = ex < N
    order = np.lexsort((tok[ffn], ex[ffn]))  # key: expert, then token (numpy, stable)
    np.testing.assert_array_equal(dsp["perm_tok"], tok[ffn][order])
    np.testing.assert_array_equal(dsp["counts"], np.bincount(ex, minlength=E))
    np.testing.assert_array_equal(dsp["offsets"],
                                  np.concatenate([[0], np.cumsum(np.bincount(ex[ffn],
                                                                             minlength=N))]))
    rows = np.full(T * K, -1)
    rows[np.flatnonzero(ffn)[order]] = np.arange(ffn.sum())
    np.testing.assert_array_equal(dsp["slot_pos"].reshape(-1), rows)


def test_dispatch_empty_and_all_zero():
    idx = np.zeros((0, 3), np.int32)
    dsp = oracle.dispatch(idx, 4, 6)
    assert dsp["counts"].sum() == 0 and dsp["perm_tok"].size == 0
    idx = np.tile(np.array([[4, 5]], np.int32), (7, 1))
    dsp = oracle.dispatch(idx, 4, 6)
    assert (dsp["slot_pos"] == -1).all() and (dsp["offsets"] == 0).all()


# ------------------------------------------------------------------ PID controller
def test_pid_closed_form_on_constant_load():
    N, Z, K, T = 6, 3, 4, 100
    counts = np.array([50, 50, 50, 50, 50, 50, 30, 30, 40], np.int32)  # m = 300/100 = 3
    target, kp, ki, kd = 2.0, 0.01, 0.004, 0.02
    b = np.zeros(N + Z, np.float32)
    st = np.zeros(2, np.float32)
    S = 12
    for _ in range(S):
        oracle.pid_step(counts, b, st, N, K, T, target, kp, ki, kd)
    e = (target - 3.0) / K
    want = S * kp * e + ki * e * S * (S + 1) / 2 + kd * e  # derivative acts on step 1 only
    np.testing.assert_allclose(b[:N], want, rtol=2e-6)
    assert (b[N:] == 0).all()  # zero-expert biases are never moved
    np.testing.assert_allclose(st, [S * e, e], rtol=2e-6)


def test_pid_sign_and_empty_batch():
    b = np.zeros(5, np.float32)
    st = np.zeros(2, np.float32)
    oracle.pid_step(np.array([9, 9, 9, 0, 0], np.int32), b, st, 3, 2, 10, 1.0, 0.1, 0.0, 0.0)
    assert (b[:3] < 0).all()  # too many FFN experts -> FFN biases go down
    b2 = np.zeros(5, np.float32)
    oracle.pid_step(np.array([1, 0, 0, 9, 9], np.int32), b2, st * 0, 3, 2, 10, 1.0, 0.1, 0.0, 0.0)
    assert (b2[:3] > 0).all()
    b3 = np.ones(5, np.float32)
    st3 = np.array([0.25, 0.5], np.float32)
    oracle.pid_step(np.zeros(5, np.int32), b3, st3, 3, 2, 0, 1.0, 0.1, 0.1, 0.1)
    assert (b3 == 1).all() and (st3 == [0.25, 0.5]).all()


def _toy_pid_run(steps, b, st, start=0):
    """Router + dispatch + PID on a toy layer whose FFN experts are favoured by the router."""
    w = WORKLOADS["tiny"]
    N, Z, K, d, T = w.N, w.Z, w.K, 32, 256
    g = torch.Generator().manual_seed(77)
    W_r = (torch.randn((N + Z, d), generator=g) * 0.2)
    W_r[:N, 0] += 1.0  # FFN experts get larger logits on average
    W_r = W_r.to(torch.bfloat16)
    means = []
    for s in range(start, start + steps):
        x = torch.randn((T, d), generator=torch.Generator().manual_seed(1000 + s))
        x[:, 0] = 1.0
        r = oracle.router(x.to(torch.bfloat16), W_r, b, K)
        dsp = oracle.dispatch(r["topk_idx"], N, N + Z)
        means.append(dsp["counts"][:N].sum() / T)
        oracle.pid_step(dsp["counts"], b, st, N, K, T, 1.5, 0.05, 0.02, 0.0)
    return means


def test_pid_drives_toy_load_to_setpoint():
    b = np.zeros(12, np.float32)
    st = np.zeros(2, np.float32)
    means = _toy_pid_run(50, b, st)
    assert means[0] > 2.4  # starts well above the set-point of 1.5
    assert abs(np.mean(means[-10:]) - 1.5) < 0.1
    assert abs(means[-1] - 1.5) < abs(means[0] - 1.5)


def test_pid_checkpoint_resume_is_bit_identical():
    b_a = np.zeros(12, np.float32)
    st_a = np.zeros(2, np.float32)
    _toy_pid_run(20, b_a, st_a)
    b_b = np.zeros(12, np.float32)
    st_b = np.zeros(2, np.float32)
    _toy_pid_run(10, b_b, st_b)
    saved = (b_b.tobytes(), st_b.tobytes())  # checkpoint = the flat fp32 state
    b_c = np.frombuffer(saved[0], np.float32).copy()
    st_c = np.frombuffer(saved[1], np.float32).copy()
    _toy_pid_run(10, b_c, st_c, start=10)
    assert b_c.tobytes() == b_a.tobytes() and st_c.tobytes() == st_a.tobytes()


# ------------------------------------------------------------------ a planted mistake is caught
def test_brute_force_pin_catches_a_planted_sign_error():
    # The pins above must be able to fail: flip the sign of the bias (a plausible mistake)
    # by handing the oracle -b and check that the brute force disagrees on some token.
    x, W_r, b = _rand_case(3, 40, 16, 12)
    _, s_lib = _library_scores(x, W_r, b)
    r_bad = oracle.router(x, W_r, -b, 3)
    mismatches = 0
    for t in range(40):
        best = sorted(np.argsort(-s_lib[t], kind="stable")[:3].tolist())
        mismatches += r_bad["topk_idx"][t].tolist() != best
    assert mismatches > 0


def test_combine_rows_agrees_with_whole_layer():
    # Two routes to the same y: the whole layer, and dispatch + per-expert outputs + the
    # weighted sum of given rows.  Both must agree with the single-expert library pin above.
    w = WORKLOADS["tiny"]
    wt = make_weights(w, seed=8)
    x = make_tokens(w, seed=8)
    b = (torch.rand(w.E, generator=torch.Generator().manual_seed(4)) * 0.02).float()
    ref = oracle.forward(x, wt["W_r"], b, wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    dsp = oracle.dispatch(ref["topk_idx"], w.N, w.E)
    xb = oracle.bf16_bits(x)
    rows = np.zeros((len(dsp["perm_tok"]), w.d))
    gates = np.zeros(len(dsp["perm_tok"]))
    for t in range(w.T):
        for k in range(w.K):
            if dsp["slot_pos"][t, k] >= 0:
                gates[dsp["slot_pos"][t, k]] = ref["topk_gate"][t, k]
    for e in range(w.N):
        lo, hi = dsp["offsets"][e], dsp["offsets"][e + 1]
        out = oracle.swiglu_expert(xb[dsp["perm_tok"][lo:hi]], wt["W_g"][e], wt["W_u"][e], wt["W_d"][e])
        rows[lo:hi] = gates[lo:hi, None] * out
    y = oracle.combine_rows(x, ref["topk_idx"], ref["topk_gate"], dsp["slot_pos"], rows, w.N)
    np.testing.assert_allclose(y, ref["y"], rtol=1e-12, atol=1e-14)
