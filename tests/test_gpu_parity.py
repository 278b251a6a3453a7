"""GPU parity: every stage of the CUDA path, called through the C ABI, against the CPU oracle.

Stage tests feed the GPU stage the oracle's own upstream results (never the other way round),
so each kernel is checked in isolation; end-to-end tests compare moe_forward with the oracle
on the same seeded inputs.  Workloads: tiny (whole batch), mid (sampled tokens), and edge
cases (T = 0, ragged T, one token, all-zero-expert routing, one expert holding every token,
K = N + Z, widths that are not multiples of the 128-row tiles).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import WORKLOADS, Workload, make_tokens, make_weights
from parity import (Stages, assert_y_close, check_dispatch_properties, check_dispatch_vs_oracle,
                    check_routing_full, gpu_routing_for_oracle, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(w, seed=0, bias=None, T=None):
    wt = make_weights(w, seed=seed)
    if bias is not None:
        wt["b"] = bias
    x = make_tokens(w, seed=seed, T=T)
    if T is not None:
        w = Workload(w.name, T=T, d=w.d, N=w.N, Z=w.Z, K=w.K, I=w.I, bias_range=w.bias_range)
    return w, x, wt


def _oracle_expert_rows(w, x, wt, ref_idx, ref_gate, dsp):
    """g_r * E_e(x_t) per grouped row, from the oracle (fp64)."""
    xb = oracle.bf16_bits(x)
    A = len(dsp["perm_tok"])
    gates = np.zeros(A)
    T, K = ref_idx.shape
    for t in range(T):
        for k in range(K):
            r = dsp["slot_pos"][t, k]
            if r >= 0:
                gates[r] = np.float32(ref_gate[t, k])  # the fp32 gate the GPU stage is given
    rows = np.zeros((A, w.d))
    for e in range(w.N):
        lo, hi = dsp["offsets"][e], dsp["offsets"][e + 1]
        if hi > lo:
            out = oracle.swiglu_expert(xb[dsp["perm_tok"][lo:hi]], wt["W_g"][e], wt["W_u"][e],
                                       wt["W_d"][e])
            rows[lo:hi] = gates[lo:hi, None] * out
    return rows, gates


# ---------------------------------------------------------------------------------- stages
@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_route_matches_oracle(name):
    # Whole batch (mid: all 4096 tokens): ids bit-exact wherever the oracle's gap exceeds 1e-4,
    # near-ties eps-valid, every gate the oracle's p of the chosen id up to the propagated
    # error of the GPU's fp32 logits (check_gates_against_logits).
    w = WORKLOADS[name]
    w, x, wt = _case(w)
    st = Stages(w, x, wt)
    st.route()
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K, want_probs=True, want_scores=True)
    stats = check_routing_full(to_np(st.topk_idx), to_np(st.topk_gate), ref, st.logits(), x,
                               wt["W_r"])
    gap = to_np(st.gap).astype(np.float64)
    np.testing.assert_allclose(gap, ref["gap"], rtol=0, atol=2e-6)
    assert st.device_status() == 0
    print(f"{name} routing: {stats}")


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_dispatch_matches_oracle(name):
    w = WORKLOADS[name]
    w, x, wt = _case(w, T=1000 if name == "mid" else None)
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K)
    dsp = oracle.dispatch(ref["topk_idx"], w.N, w.E)
    st = Stages(w, x, wt)
    st.topk_idx.copy_(torch.from_numpy(ref["topk_idx"]))
    st.topk_gate.copy_(torch.from_numpy(ref["topk_gate"].astype(np.float32)))
    st.dispatch()
    A = len(dsp["perm_tok"])
    np.testing.assert_array_equal(to_np(st.counts), dsp["counts"])
    np.testing.assert_array_equal(to_np(st.offsets), dsp["offsets"])
    np.testing.assert_array_equal(to_np(st.perm_tok)[:A], dsp["perm_tok"])
    np.testing.assert_array_equal(to_np(st.slot_pos), dsp["slot_pos"])
    assert (to_np(st.perm_tok)[A:] == -7).all()  # rows past A untouched
    g32 = ref["topk_gate"].astype(np.float32)
    want_gate = np.zeros(A, np.float32)
    ffn = dsp["slot_pos"] >= 0
    want_gate[dsp["slot_pos"][ffn]] = g32[ffn]
    np.testing.assert_array_equal(to_np(st.perm_gate)[:A], want_gate)
    np.testing.assert_array_equal(to_np(st.x_perm)[:A], oracle.bf16_bits(x)[dsp["perm_tok"]])
    assert st.device_status() == 0


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_expert_ffn_matches_oracle(name):
    w = WORKLOADS[name]
    w, x, wt = _case(w, T=256 if name == "mid" else None)
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K)
    dsp = oracle.dispatch(ref["topk_idx"], w.N, w.E)
    rows, gates = _oracle_expert_rows(w, x, wt, ref["topk_idx"], ref["topk_gate"], dsp)
    A = len(dsp["perm_tok"])
    st = Stages(w, x, wt)
    st.x_perm[:A].copy_(x[torch.from_numpy(dsp["perm_tok"]).long()])
    st.offsets.copy_(torch.from_numpy(dsp["offsets"]))
    st.perm_gate[:A].copy_(torch.from_numpy(gates.astype(np.float32)))
    st.expert_ffn()
    got = to_np(st.y_perm)[:A]
    assert_y_close(oracle.bf16_to_f64(got), rows, f"{name} y_perm")
    assert st.device_status() == 0


@pytest.mark.parametrize("I,counts", [
    (512, (520, 300, 256, 100, 17, 1, 0, 30)),
    (384, (520, 300, 256, 100, 17, 1, 0, 30)),
    (512, (192, 193, 65, 64, 384, 257, 0, 129)),
    (512, (224, 225, 33, 32, 448, 256, 0, 130)),
])
def test_expert_ffn_wide_tiles_matches_oracle(I, counts):
    # d = 4096 with >= 128 rows per expert selects the wide tiles: I = 512 runs them on CTA
    # pairs (I a multiple of 256, d of 512) with the two-pipeline kernel (192-row full tiles
    # and tails over 64 rows in one pipeline, tails of at most 64 rows in the other), I = 384
    # on single CTAs with 256-token tiles.  Ragged groups built directly: several full tiles
    # with and without tails, tail-only experts (100 / 30 / 17 / 1 rows), an empty expert; the
    # last case sits on the two-pipeline kernel's boundaries (224-row full tiles, tails of at
    # most 32 rows in the tail pipeline): 224 = one full tile, 225 = one full tile + a 1-row
    # tail, 33 = the smallest remainder kept in the full-tile pipeline, 32 = the largest in the
    # tail pipeline, 448, 256 = 224 + 32, 130.  Rows = K = 4 times the tokens.
    counts = np.array(counts)
    R = int(counts.sum())
    w = Workload("wide", T=R // 4, d=4096, N=8, Z=4, K=4, I=I)
    wt = make_weights(w, seed=5)
    xr = make_tokens(w, seed=5, T=R)
    gates = np.random.default_rng(5).uniform(0.05, 1.0, R).astype(np.float32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    xb = oracle.bf16_bits(xr)
    want = np.zeros((R, w.d))
    for e in range(w.N):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            want[lo:hi] = gates[lo:hi, None].astype(np.float64) * oracle.swiglu_expert(
                xb[lo:hi], wt["W_g"][e], wt["W_u"][e], wt["W_d"][e])
    st = Stages(w, xr[: w.T], wt)
    st.x_perm.copy_(xr)
    st.offsets.copy_(torch.from_numpy(offsets))
    st.perm_gate.copy_(torch.from_numpy(gates))
    st.expert_ffn()
    assert_y_close(oracle.bf16_to_f64(to_np(st.y_perm)), want, f"wide I={I} y_perm")
    assert st.device_status() == 0


@pytest.mark.parametrize("name,T", [("tiny", None), ("mid", 256), ("mid", 333)])
def test_expert_ffn_gather_matches_oracle_and_unfused(name, T):
    # The up-projection gathering token rows from x by perm_tok (no x_perm): against the
    # oracle's expert rows, and bit for bit against moe_expert_ffn on the gathered copy.
    w = WORKLOADS[name]
    w, x, wt = _case(w, T=T)
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K)
    dsp = oracle.dispatch(ref["topk_idx"], w.N, w.E)
    rows, gates = _oracle_expert_rows(w, x, wt, ref["topk_idx"], ref["topk_gate"], dsp)
    A = len(dsp["perm_tok"])
    st = Stages(w, x, wt)
    st.x_perm[:A].copy_(x[torch.from_numpy(dsp["perm_tok"]).long()])
    st.perm_tok[:A].copy_(torch.from_numpy(dsp["perm_tok"]))
    st.offsets.copy_(torch.from_numpy(dsp["offsets"]))
    st.perm_gate[:A].copy_(torch.from_numpy(gates.astype(np.float32)))
    st.expert_ffn()
    h_ref, y_ref = st.h[:A].clone(), st.y_perm[:A].clone()
    st.h.zero_()
    st.y_perm.zero_()
    mb.moe_expert_ffn_gather(st.dm, st.x, st.perm_tok, st.offsets, st.perm_gate, st.wt["W_g"],
                             st.wt["W_u"], st.wt["W_d"], st.h, st.y_perm, st.ws)
    torch.cuda.synchronize()
    assert st.device_status() == 0
    assert torch.equal(st.h[:A], h_ref) and torch.equal(st.y_perm[:A], y_ref)
    assert_y_close(oracle.bf16_to_f64(to_np(st.y_perm)[:A]), rows, f"{name} gathered y_perm")


def test_dispatch_row_copy_token_major():
    # Token rows of 64 MB or more are copied token-major (each x row read once, written to its
    # slots' rows); the grouped rows must equal x[perm_tok] exactly, as with the row gather.
    w = Workload("wide", T=8192, d=4096, N=8, Z=4, K=3, I=256)
    g = torch.Generator(device=DEV).manual_seed(9)
    x = torch.randn((w.T, w.d), generator=g, device=DEV).to(torch.bfloat16)
    W_r = (torch.randn((w.E, w.d), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    b = torch.zeros(w.E, device=DEV)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = mb.alloc_workspace(dm, DEV, scratch_only=True)
    R = w.T * w.K
    i32 = dict(dtype=torch.int32, device=DEV)
    idx, gate = torch.empty((w.T, w.K), **i32), torch.empty((w.T, w.K), dtype=torch.float32,
                                                            device=DEV)
    mb.moe_route(dm, x, W_r, b, idx, gate, None, ws)
    counts, offsets = torch.empty(w.E, **i32), torch.empty(w.N + 1, **i32)
    perm_tok, slot_pos = torch.empty(R, **i32), torch.empty((w.T, w.K), **i32)
    perm_gate = torch.empty(R, dtype=torch.float32, device=DEV)
    x_perm = torch.zeros((R, w.d), dtype=torch.bfloat16, device=DEV)
    mb.moe_dispatch(dm, x, idx, gate, counts, offsets, perm_tok, perm_gate, slot_pos, x_perm, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    A = int(offsets[-1].item())
    assert A > 0
    assert torch.equal(x_perm[:A], x[perm_tok[:A].long()])
    assert (x_perm[A:] == 0).all()  # rows past the groups are not written
    check_dispatch_vs_oracle(to_np(idx), to_np(gate), to_np(counts), to_np(offsets),
                             to_np(perm_tok), to_np(perm_gate), to_np(slot_pos), w.N, w.E)


def test_dispatch_without_gather_leaves_x_perm_alone():
    w, x, wt = _case(WORKLOADS["tiny"])
    st = Stages(w, x, wt)
    st.route()
    st.dispatch()
    tables = [t.clone() for t in (st.counts, st.offsets, st.perm_tok, st.perm_gate, st.slot_pos)]
    st.x_perm.fill_(3.0)
    mb.moe_dispatch(st.dm, st.x, st.topk_idx, st.topk_gate, st.counts, st.offsets, st.perm_tok,
                    st.perm_gate, st.slot_pos, None, st.ws)
    torch.cuda.synchronize()
    for a, b in zip(tables, (st.counts, st.offsets, st.perm_tok, st.perm_gate, st.slot_pos)):
        assert torch.equal(a, b)
    assert (st.x_perm == 3.0).all()


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_combine_matches_oracle(name):
    w = WORKLOADS[name]
    w, x, wt = _case(w, T=300 if name == "mid" else None)
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K)
    dsp = oracle.dispatch(ref["topk_idx"], w.N, w.E)
    A = len(dsp["perm_tok"])
    # Arbitrary seeded expert-output rows (combine does not care where they come from).
    g = torch.Generator().manual_seed(11)
    y_perm = torch.randn((w.T * w.K, w.d), generator=g).to(torch.bfloat16)
    st = Stages(w, x, wt)
    st.y_perm.copy_(y_perm)
    st.topk_idx.copy_(torch.from_numpy(ref["topk_idx"]))
    st.topk_gate.copy_(torch.from_numpy(ref["topk_gate"].astype(np.float32)))
    st.slot_pos.copy_(torch.from_numpy(dsp["slot_pos"]))
    st.combine()
    rows = oracle.bf16_to_f64(oracle.bf16_bits(y_perm))[:max(A, 1)]
    want = oracle.combine_rows(x, ref["topk_idx"], ref["topk_gate"].astype(np.float32),
                               dsp["slot_pos"], rows, w.N)
    got = oracle.bf16_to_f64(to_np(st.y))
    assert_y_close(got, want, f"{name} combine")
    # fp32 accumulation then one bf16 rounding: within 2^-8 relative of each element (+ abs eps)
    assert (np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-3 * np.abs(want).max()).all()


def test_pid_matches_oracle_bit_exact():
    w = WORKLOADS["skewed"]
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    rng = np.random.default_rng(5)
    b = (rng.uniform(-0.05, 0.05, w.E)).astype(np.float32)
    st = np.zeros(2, np.float32)
    b_gpu = torch.from_numpy(b.copy()).to(DEV)
    st_gpu = torch.zeros(2, dtype=torch.float32, device=DEV)
    params = mb.PidParams(8.0, 0.005, 0.002, 0.001)
    for step in range(20):
        counts = rng.integers(0, 400, w.E).astype(np.int32)
        mb.moe_bias_update(dm, torch.from_numpy(counts).to(DEV), b_gpu, st_gpu, params)
        oracle.pid_step(counts, b, st, w.N, w.K, w.T, 8.0, 0.005, 0.002, 0.001)
        assert b_gpu.cpu().numpy().tobytes() == b.tobytes(), step
        assert st_gpu.cpu().numpy().tobytes() == st.tobytes(), step


# ---------------------------------------------------------------------------------- end to end
def _forward_vs_oracle(w, x, wt, sample=None, seed=0):
    """moe_forward against the oracle: routing of the whole batch (check_routing_full), the
    per-expert counts against the oracle's dispatch of the GPU's routing, and y of every token
    (or a seeded sample plus every token whose GPU set differs from the oracle's) against the
    oracle's layer output on the GPU's routing, near-tie tokens included."""
    st = Stages(w, x, wt)
    st.forward()
    y = oracle.bf16_to_f64(to_np(st.y))
    counts = to_np(st.counts)
    assert counts.sum() == w.T * w.K
    st.route()  # same kernels and launch configuration as moe_forward's routing
    idx = to_np(st.topk_idx)
    ref = oracle.router(x, wt["W_r"], wt["b"], w.K, want_probs=True, want_scores=True)
    stats = check_routing_full(idx, to_np(st.topk_gate), ref, st.logits(), x, wt["W_r"])
    np.testing.assert_array_equal(counts, oracle.dispatch(idx, w.N, w.E)["counts"])
    differ = np.flatnonzero((idx != ref["topk_idx"]).any(axis=1))
    tokens = np.arange(w.T) if sample is None else np.union1d(
        np.random.default_rng(seed).choice(w.T, sample, replace=False), differ[:16])
    xs = oracle.bf16_bits(x)[tokens]
    out = oracle.forward_sampled(np.arange(len(tokens)), xs, wt["W_r"], wt["b"], w.N, w.Z, w.K,
                                 lambda e: (wt["W_g"][e], wt["W_u"][e], wt["W_d"][e]),
                                 routing=gpu_routing_for_oracle(idx, ref, tokens))
    assert_y_close(y[tokens], out["y"], f"{w.name} y")
    assert st.device_status() == 0
    print(f"{w.name}: {stats}, y checked on {len(tokens)} tokens")
    return st, stats["near_ties"], stats["differing"]


def test_forward_tiny_whole_batch():
    w, x, wt = _case(WORKLOADS["tiny"])
    _forward_vs_oracle(w, x, wt)


def test_forward_mid_sampled():
    w, x, wt = _case(WORKLOADS["mid"])
    _forward_vs_oracle(w, x, wt, sample=192)


def test_forward_is_deterministic():
    w, x, wt = _case(WORKLOADS["mid"], T=700)
    st = Stages(w, x, wt)
    st.forward()
    y0 = st.y.clone()
    c0 = st.counts.clone()
    st.y.zero_()
    st.forward()
    assert torch.equal(st.y, y0) and torch.equal(st.counts, c0)


def test_staged_calls_equal_forward():
    w, x, wt = _case(WORKLOADS["mid"], T=333)
    st = Stages(w, x, wt)
    st.forward()
    y_fwd = st.y.clone()
    st.route()
    st.dispatch()
    check_dispatch_properties(to_np(st.topk_idx), to_np(st.counts), to_np(st.offsets),
                              to_np(st.perm_tok), to_np(st.slot_pos), w.N, w.E)
    st.expert_ffn()
    st.combine()
    assert torch.equal(st.y, y_fwd)


# ---------------------------------------------------------------------------------- edge cases
def test_zero_tokens():
    w = Workload("t0", T=0, d=128, N=8, Z=4, K=3, I=256)
    wt = make_weights(w)
    x = torch.zeros((0, w.d), dtype=torch.bfloat16)
    st = Stages(w, x, wt)
    st.counts.fill_(5)
    st.forward()
    torch.cuda.synchronize()
    assert (st.counts == 0).all()
    assert st.device_status() == 0


def test_zero_tokens_gather_and_fp8_paths():
    w = Workload("t0", T=0, d=128, N=8, Z=4, K=3, I=256)
    wt = make_weights(w)
    x = torch.zeros((0, w.d), dtype=torch.bfloat16)
    st = Stages(w, x, wt)
    mb.moe_expert_ffn_gather(st.dm, st.x, st.perm_tok, st.offsets, st.perm_gate, st.wt["W_g"],
                             st.wt["W_u"], st.wt["W_d"], st.h, st.y_perm, st.ws)
    fw = mb.quantize_expert_weights_fp8(st.dm, st.wt["W_g"], st.wt["W_u"], st.wt["W_d"])
    st.counts.fill_(5)
    mb.moe_forward_fp8(st.dm, st.x, st.wt["W_r"], st.wt["b"], fw, st.y, st.counts, st.ws)
    torch.cuda.synchronize()
    assert (st.counts == 0).all()
    assert st.device_status() == 0


@pytest.mark.parametrize("T", [1, 77, 300])
def test_ragged_token_counts(T):
    w, x, wt = _case(WORKLOADS["tiny"], T=T, seed=T)
    _forward_vs_oracle(w, x, wt)


def test_all_zero_experts_return_sum_g_times_x():
    w = WORKLOADS["tiny"]
    b = torch.zeros(w.E)
    b[w.N:] = 1.0
    w, x, wt = _case(w, bias=b)
    st = Stages(w, x, wt)
    st.forward()
    ref = oracle.router(x, wt["W_r"], b, w.K)
    st.route()
    assert (to_np(st.topk_idx) >= w.N).all()
    assert (to_np(st.counts)[:w.N] == 0).all()
    want = ref["topk_gate"].sum(axis=1, keepdims=True) * oracle.bf16_to_f64(oracle.bf16_bits(x))
    assert_y_close(oracle.bf16_to_f64(to_np(st.y)), want, "zero-expert y")
    assert st.device_status() == 0


def test_one_expert_takes_every_token():
    # Expert 3 is selected by all 1000 tokens: one group of 1000 rows spans 8 token tiles.
    w = WORKLOADS["tiny"]
    b = torch.zeros(w.E)
    b[3] = 1.0
    w, x, wt = _case(w, bias=b, T=1000, seed=2)
    st, _, _ = _forward_vs_oracle(w, x, wt, sample=128)
    assert to_np(st.counts)[3] == 1000


def test_k_equals_all_experts():
    w = Workload("all", T=96, d=128, N=8, Z=4, K=12, I=256, bias_range=0.0)
    w, x, wt = _case(w)
    st, _, _ = _forward_vs_oracle(w, x, wt)
    st.route()
    assert torch.isinf(st.gap).all()


def test_widths_not_multiple_of_tiles():
    # d = 192 (GEMM2 weight tile half-used), I = 320 (partial up-projection tile), E = 9.
    w = Workload("odd", T=200, d=192, N=5, Z=4, K=3, I=320)
    w, x, wt = _case(w, seed=4)
    _forward_vs_oracle(w, x, wt)


# ---------------------------------------------------------------------------------- error paths
def test_device_status_codes():
    w, x, wt = _case(WORKLOADS["tiny"])
    st = Stages(w, x, wt)
    st.offsets.copy_(torch.tensor([0, 5, 3, 9, 9, 9, 9, 9, 9], dtype=torch.int32))
    st.y_perm.fill_(1.0)
    st.expert_ffn()
    assert st.device_status() == 0x300  # rows out of order: nothing computed, nothing faulted
    assert (st.y_perm == 1.0).all()
    assert st.device_status() == 0  # reading clears it
    bad = torch.tensor([[0, 1, 99]] * w.T, dtype=torch.int32)
    st.topk_idx.copy_(bad)
    st.dispatch()
    assert st.device_status() == 0x200  # expert id out of range, skipped
    assert int(st.counts.sum()) == 2 * w.T


def test_combine_reports_a_bad_slot_row():
    # An FFN slot whose grouped row lies outside [0, T*K): its term is skipped and the
    # workspace's status word says so (MOE_DEV_BAD_ROWS); nothing is read out of bounds.
    w, x, wt = _case(WORKLOADS["tiny"])
    st = Stages(w, x, wt)
    st.forward()
    assert st.device_status() == 0
    idx = to_np(st.topk_idx)
    t, k = map(int, np.argwhere(idx < w.N)[0])
    st.slot_pos[t, k] = w.T * w.K + 5
    st.combine()
    assert st.device_status() == 0x300
    st.slot_pos[t, k] = -3
    st.combine()
    assert st.device_status() == 0x300
    assert st.device_status() == 0


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    # The grouped GEMMs' bounded waits, made to run out: with a 64-cycle limit no pipeline wait
    # can succeed in time (a tile needs its TMA loads, hundreds of cycles at least), so every
    # GEMM of the step records MOE_DEV_WAIT_TIMEOUT, unwinds, drains its copies and MMAs and
    # frees its tensor memory.  tiny runs every GEMM on single CTAs with 128-token tiles.  The
    # next, normal step must reproduce the reference output bit for bit.
    w, x, wt = _case(WORKLOADS["tiny"])
    st = Stages(w, x, wt)
    st.forward()
    y_ref = st.y.clone()
    assert st.device_status() == 0
    mb.moe_debug_set_wait_limit(64)
    try:
        st.y.zero_()
        st.forward()
        code = st.device_status()
    finally:
        mb.moe_debug_set_wait_limit(0)
    assert code == 0x100
    for _ in range(2):
        st.y.zero_()
        st.forward()
        assert st.device_status() == 0
        assert torch.equal(st.y, y_ref)


def test_host_side_argument_errors():
    w, x, wt = _case(WORKLOADS["tiny"])
    st = Stages(w, x, wt)
    with pytest.raises(mb.MoeError) as e:
        mb.moe_forward(st.dm, st.x, wt["W_r"].to(DEV), wt["b"].to(DEV), wt["W_g"].to(DEV),
                       wt["W_u"].to(DEV), wt["W_d"].to(DEV), st.y, st.counts, st.ws[:1024])
    assert e.value.code == 4  # workspace too small
    bad_dm = mb.dims(w.T, 100, w.N, w.Z, w.K, w.I)
    assert mb.workspace_size(bad_dm) == 0
