"""GPU parity of the FP8 expert-weight path against the CPU oracle, through the C ABI.

  * moe_quantize_fp8: codes and scales bit-exact with the oracle's block quantisation
    (integer output), on random weights plus all-zero blocks, wide-range blocks, tiny values
    and exact rounding ties;
  * moe_expert_ffn_fp8 / moe_forward_fp8: within the output tolerances of the oracle run on
    the dequantised weights, and bit-identical to the bf16 path given those same dequantised
    weights (the E4M3 -> bf16 step is exact, the tensor-core path is shared).
FP8 activations (MOE_FP8_ACTIVATIONS: E4M3 x E4M3 on the tensor cores):
  * moe_quantize_fp8_rows: codes and block scales bit-exact with the oracle's 1 x 128 row
    quantisation, special blocks included;
  * moe_expert_ffn_fp8 / moe_forward_fp8 with the flag: within the output tolerances of the
    oracle's FP8-activation expert on the dequantised weights, over several token tiles per
    expert and ragged tails; and measurably different from the bf16-activation result, so the
    comparison sees the quantisation.
Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 系統級優化 (block-wise quantisation as in
DeepSeek-V3).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import WORKLOADS, Workload, make_tokens, make_weights
from parity import Stages, assert_y_close, gpu_routing_for_oracle, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _special_weights(G, R, C, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn((G, R, C), generator=g) * 0.02
    w[0, :128, :128] = 0                                  # an all-zero block
    if C >= 256:
        w[0, :128, 128:256] *= 3000                       # a wide-range block
    if R >= 256:
        w[0, 128:256, :128] *= 1e-30                      # tiny values (scale near 2^-126)
    # exact rounding ties after scaling: amax 1.0 (e = -8), then (1 + 1/16) * 2^k and
    # (1 + 3/16) * 2^k sit halfway between two E4M3 codes
    blk = w[G - 1, R - 128:, C - 128:]
    blk[:] = 0
    blk[0, 0] = 1.0
    for i, k in enumerate(range(-14, -5)):
        blk[1, i] = (1 + 1 / 16) * 2.0 ** k
        blk[2, i] = -(1 + 3 / 16) * 2.0 ** k
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("G,R,C", [(1, 128, 128), (3, 256, 384), (2, 1024, 2048)])
def test_quantize_bit_exact_with_oracle(G, R, C):
    w = _special_weights(G, R, C, seed=G * 7 + R)
    q = torch.empty((G, R, C), dtype=torch.uint8, device=DEV)
    s = torch.empty((G, R // 128, C // 128), dtype=torch.float32, device=DEV)
    mb.moe_quantize_fp8(w.to(DEV), q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_fp8_blocks(w)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


def _fp8_case(name, T=None, seed=0):
    w = WORKLOADS[name]
    wt = make_weights(w, seed=seed)
    x = make_tokens(w, seed=seed, T=T)
    if T is not None:
        w = Workload(w.name, T=T, d=w.d, N=w.N, Z=w.Z, K=w.K, I=w.I, bias_range=w.bias_range)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    fw = mb.quantize_expert_weights_fp8(dm, wt["W_g"].to(DEV), wt["W_u"].to(DEV),
                                        wt["W_d"].to(DEV))
    torch.cuda.synchronize()
    deq = {}
    for k in ("g", "u", "d"):
        bits = oracle.dequantize_fp8_blocks(fw["q_" + k].cpu().numpy(), fw["s_" + k].cpu().numpy())
        deq["W_" + k] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    wt_deq = dict(wt, **deq)
    return w, x, wt, fw, wt_deq


# several token tiles per expert and ragged tails (mid at T = 1500: 9000 rows over 64 experts)
@pytest.mark.parametrize("name,T", [("tiny", None), ("mid", 333), ("mid", 1500)])
def test_expert_ffn_fp8_matches_oracle_and_bf16_path(name, T):
    w, x, wt, fw, wt_deq = _fp8_case(name, T)
    st = Stages(w, x, wt_deq)
    st.route()
    st.dispatch()
    st.expert_ffn()  # bf16 path on the dequantised weights
    A = int(st.offsets[-1].item())
    h_ref, y_ref = st.h[:A].clone(), st.y_perm[:A].clone()
    st.h.zero_()
    st.y_perm.zero_()
    mb.moe_expert_ffn_fp8(st.dm, st.x_perm, st.offsets, st.perm_gate, fw, st.h, st.y_perm,
                          st.ws)
    torch.cuda.synchronize()
    assert st.device_status() == 0
    assert torch.equal(st.h[:A], h_ref) and torch.equal(st.y_perm[:A], y_ref)
    # and against the oracle's expert rows on the dequantised weights
    xb = oracle.bf16_bits(x)
    perm, offs, gates = to_np(st.perm_tok)[:A], to_np(st.offsets), to_np(st.perm_gate)[:A]
    rows = np.zeros((A, w.d))
    for e in range(w.N):
        lo, hi = offs[e], offs[e + 1]
        if hi > lo:
            rows[lo:hi] = gates[lo:hi, None].astype(np.float64) * oracle.swiglu_expert(
                xb[perm[lo:hi]], wt_deq["W_g"][e], wt_deq["W_u"][e], wt_deq["W_d"][e])
    assert_y_close(oracle.bf16_to_f64(to_np(st.y_perm)[:A]), rows, f"{name} fp8 y_perm")


def test_forward_fp8_tiny_matches_oracle():
    w, x, wt, fw, wt_deq = _fp8_case("tiny", seed=4)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = mb.alloc_workspace(dm, DEV)
    y = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device=DEV)
    counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    mb.moe_forward_fp8(dm, x.to(DEV), wt["W_r"].to(DEV), wt["b"].to(DEV), fw, y, counts, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    ref = oracle.forward(x, wt["W_r"], wt["b"], wt_deq["W_g"], wt_deq["W_u"], wt_deq["W_d"],
                         w.N, w.Z, w.K)
    assert_y_close(oracle.bf16_to_f64(to_np(y)), ref["y"], "tiny fp8 forward")
    # the same layer through the bf16 path on the dequantised weights: bit-identical
    y2 = torch.zeros_like(y)
    mb.moe_forward(dm, x.to(DEV), wt["W_r"].to(DEV), wt["b"].to(DEV), wt_deq["W_g"].to(DEV),
                   wt_deq["W_u"].to(DEV), wt_deq["W_d"].to(DEV), y2, None, ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


# ------------------------------------------------------------------ FP8 activations

def _special_rows(R, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((R, C), generator=g)
    x[0, :128] = 0                                        # an all-zero block
    if C >= 256:
        x[1, 128:256] *= 3000                             # a wide-range block
        x[2, 128:256] *= 1e-30                            # tiny values (scale near 2^-126)
    # exact rounding ties after scaling: amax 3 (e = -7), (1 + 1/16) * 2^k halfway between codes
    x[3, :128] = 0
    x[3, 0] = 3.0
    for i, k in enumerate(range(-16, -6)):
        x[3, 1 + i] = (1 + 1 / 16) * 2.0 ** k
        x[3, 20 + i] = -(1 + 3 / 16) * 2.0 ** k
    x[4, :] = -0.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("R,C", [(5, 128), (37, 384), (1139, 6144)])
def test_quantize_rows_bit_exact_with_oracle(R, C):
    x = _special_rows(R, C, seed=R + C)
    q = torch.empty((R, C), dtype=torch.uint8, device=DEV)
    s = torch.empty((C // 128, R), dtype=torch.float32, device=DEV)
    mb.moe_quantize_fp8_rows(x.to(DEV), q, s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_fp8_rows(x.double().numpy())
    np.testing.assert_array_equal(s.cpu().numpy().T, s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


def _fp8act_rows(w, st, x, wt_deq, A):
    xb = oracle.bf16_bits(x)
    perm, offs, gates = to_np(st.perm_tok)[:A], to_np(st.offsets), to_np(st.perm_gate)[:A]
    rows = np.zeros((A, w.d))
    for e in range(w.N):
        lo, hi = offs[e], offs[e + 1]
        if hi > lo:
            rows[lo:hi] = gates[lo:hi, None].astype(np.float64) * oracle.swiglu_expert(
                xb[perm[lo:hi]], wt_deq["W_g"][e], wt_deq["W_u"][e], wt_deq["W_d"][e],
                fp8_act=True)
    return rows


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# 64-token tiles: several per expert and ragged tails at mid T = 1500 (9000 rows, 64 experts),
# one partial tile per expert at T = 333 and tiny
@pytest.mark.parametrize("name,T", [("tiny", None), ("mid", 333), ("mid", 1500)])
def test_expert_ffn_fp8_activations_match_oracle(name, T):
    w, x, wt, fw, wt_deq = _fp8_case(name, T)
    st = Stages(w, x, wt_deq)
    st.route()
    st.dispatch()
    A = int(st.offsets[-1].item())
    mb.moe_expert_ffn_fp8(st.dm, st.x_perm, st.offsets, st.perm_gate, fw, st.h, st.y_perm,
                          st.ws)  # bf16 activations, for the contrast below
    torch.cuda.synchronize()
    y_bf16act = oracle.bf16_to_f64(to_np(st.y_perm)[:A])
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=mb.FP8_ACTIVATIONS)
    ws = mb.alloc_workspace(dm, DEV, scratch_only=True)
    y_perm = torch.zeros_like(st.y_perm)
    mb.moe_expert_ffn_fp8(dm, st.x_perm, st.offsets, st.perm_gate, fw, None, y_perm, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    got = oracle.bf16_to_f64(to_np(y_perm)[:A])
    ref = _fp8act_rows(w, st, x, wt_deq, A)
    assert_y_close(got, ref, f"{name} fp8-activation y_perm")
    # the activation quantisation is visible: the bf16-activation rows differ from the
    # reference far more than the tolerance the FP8-activation rows meet
    assert _rel_l2(y_bf16act, ref) > 10 * max(_rel_l2(got, ref), 1e-4)


def test_forward_fp8_activations_tiny_matches_oracle():
    w, x, wt, fw, wt_deq = _fp8_case("tiny", seed=5)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=mb.FP8_ACTIVATIONS)
    ws = mb.alloc_workspace(dm, DEV)
    y = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device=DEV)
    counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
    mb.moe_forward_fp8(dm, x.to(DEV), wt["W_r"].to(DEV), wt["b"].to(DEV), fw, y, counts, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    r = oracle.router(x, wt["W_r"], wt["b"], w.K)
    ref = oracle.combine_tokens(np.arange(w.T), x, r["topk_idx"], r["topk_gate"], wt_deq["W_g"],
                                wt_deq["W_u"], wt_deq["W_d"], w.N, fp8_act=True)
    assert int(counts.sum().item()) == w.T * w.K
    assert_y_close(oracle.bf16_to_f64(to_np(y)), ref, "tiny fp8-activation forward")


def test_fp8_activations_edge_inputs():
    # All-zero token rows (every block scale 1, codes 0), rows scaled by 2^12 and 2^-12 (block
    # exponents far from 0 both ways), a batch of one token, and experts left without tokens.
    # The 2^12 row's softmax underflows in fp32 for all but its top expert, so its lower slots
    # are near-ties decided differently in fp32 and fp64: y is compared on the GPU's routing
    # with the oracle's gates of those ids (the parity rule for every token).
    for T in (1, 40):
        w, x, wt, fw, wt_deq = _fp8_case("tiny", T=T, seed=6)
        x = x.float()
        if T > 1:
            x[0] = 0
            x[1] *= 2.0 ** 12
            x[2] *= 2.0 ** -12
        x = x.to(torch.bfloat16)
        dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=mb.FP8_ACTIVATIONS)
        ws = mb.alloc_workspace(dm, DEV)
        y = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device=DEV)
        counts = torch.zeros(w.E, dtype=torch.int32, device=DEV)
        mb.moe_forward_fp8(dm, x.to(DEV), wt["W_r"].to(DEV), wt["b"].to(DEV), fw, y, counts, ws)
        torch.cuda.synchronize()
        assert mb.moe_last_device_error(ws) == 0
        st = Stages(w, x, wt)
        st.route()
        idx = to_np(st.topk_idx)
        np.testing.assert_array_equal(to_np(counts), np.bincount(idx.reshape(-1), minlength=w.E))
        ref_r = oracle.router(x, wt["W_r"], wt["b"], w.K, want_probs=True)
        r = gpu_routing_for_oracle(idx, ref_r, np.arange(w.T))
        ref = oracle.combine_tokens(np.arange(w.T), x, r["topk_idx"], r["topk_gate"],
                                    wt_deq["W_g"], wt_deq["W_u"], wt_deq["W_d"], w.N, fp8_act=True)
        got = oracle.bf16_to_f64(to_np(y))
        if T > 1:
            assert np.all(got[0] == 0.0) and np.all(ref[0] == 0.0)
            # each scaled token against its own magnitude, so the 2^-12 row is checked too
            for t in (1, 2):
                assert_y_close(got[t:t + 1], ref[t:t + 1], f"fp8-activation token {t}")
        assert_y_close(got, ref, f"fp8-activation edge inputs T={T}")


def test_fp8_activations_with_renormalized_gates():
    w, x, wt, fw, wt_deq = _fp8_case("tiny", seed=7)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I,
                 flags=mb.FP8_ACTIVATIONS | mb.RENORMALIZE_GATES)
    ws = mb.alloc_workspace(dm, DEV)
    y = torch.zeros((w.T, w.d), dtype=torch.bfloat16, device=DEV)
    mb.moe_forward_fp8(dm, x.to(DEV), wt["W_r"].to(DEV), wt["b"].to(DEV), fw, y, None, ws)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    r = oracle.router(x, wt["W_r"], wt["b"], w.K, renormalize=True)
    ref = oracle.combine_tokens(np.arange(w.T), x, r["topk_idx"], r["topk_gate"], wt_deq["W_g"],
                                wt_deq["W_u"], wt_deq["W_d"], w.N, fp8_act=True)
    assert_y_close(oracle.bf16_to_f64(to_np(y)), ref, "tiny fp8-activation renormalised")
