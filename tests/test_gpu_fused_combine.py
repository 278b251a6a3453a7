"""GPU: the layer's combine fused into the down projection's epilogue (MOE_FUSED_COMBINE).

The fused form sums each token's block of y in the combine's fixed order from the same bf16
rows, so moe_forward with the flag must give y bit for bit equal to moe_forward without it --
whichever tile happens to complete a token -- and hence the same parity with the oracle.
Cases: tiny (against the oracle too), mid with one and several 128-token tiles per expert,
widths that leave partial weight tiles (d = 192, I = 320), tokens with no FFN slot mixed with
tokens that have some, one expert holding every token of a 1000-token batch, T = 1 and T = 0.
The variant follows the CSDN codearts article on LongCat-Flash, section 二、训练优化 (tiles
accumulated in a deterministic order, the addition fused into the GEMM epilogue).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import WORKLOADS, Workload, make_tokens, make_weights
from parity import Stages, assert_y_close, to_np

pytestmark = pytest.mark.gpu


def _case(w, seed=0, bias=None, T=None):
    wt = make_weights(w, seed=seed)
    if bias is not None:
        wt["b"] = bias
    x = make_tokens(w, seed=seed, T=T)
    if T is not None:
        w = Workload(w.name, T=T, d=w.d, N=w.N, Z=w.Z, K=w.K, I=w.I, bias_range=w.bias_range)
    return w, x, wt


def _fused_equals_unfused(w, x, wt):
    plain = Stages(w, x, wt)
    plain.forward()
    fused = Stages(w, x, wt, flags=mb.FUSED_COMBINE)
    fused.y.fill_(7.0)  # every element must be written
    fused.forward()
    torch.cuda.synchronize()
    assert plain.device_status() == 0 and fused.device_status() == 0
    assert torch.equal(plain.y, fused.y), "fused combine differs from the combine kernel"
    assert torch.equal(plain.counts, fused.counts)
    return fused


def test_fused_combine_tiny_matches_oracle_and_unfused():
    w, x, wt = _case(WORKLOADS["tiny"])
    st = _fused_equals_unfused(w, x, wt)
    ref = oracle.forward(x, wt["W_r"], wt["b"], wt["W_g"], wt["W_u"], wt["W_d"], w.N, w.Z, w.K)
    assert_y_close(oracle.bf16_to_f64(to_np(st.y)), ref["y"], "tiny fused-combine y")


@pytest.mark.parametrize("T", [1, 333, 1500])
def test_fused_combine_mid_equals_unfused(T):
    w, x, wt = _case(WORKLOADS["mid"], T=T, seed=1)
    _fused_equals_unfused(w, x, wt)


def test_fused_combine_partial_tiles_equal_unfused():
    w, x, wt = _case(Workload("odd", T=200, d=192, N=5, Z=4, K=3, I=320), seed=4)
    _fused_equals_unfused(w, x, wt)


def test_fused_combine_with_zero_only_tokens():
    # Two zero experts always win; the third slot is an FFN expert for some tokens and the
    # other zero experts for the rest, so both kinds of token are in the batch.
    w = WORKLOADS["tiny"]
    b = torch.zeros(w.E)
    b[w.N:w.N + 2] = 1.0
    w, x, wt = _case(w, bias=b, T=300, seed=3)
    st = _fused_equals_unfused(w, x, wt)
    st.route()
    nffn = (to_np(st.topk_idx) < w.N).sum(axis=1)
    assert (nffn == 0).any() and (nffn > 0).any()


def test_fused_combine_one_expert_over_many_tiles():
    w = WORKLOADS["tiny"]
    b = torch.zeros(w.E)
    b[3] = 1.0
    w, x, wt = _case(w, bias=b, T=1000, seed=2)
    _fused_equals_unfused(w, x, wt)


def test_fused_combine_zero_tokens():
    w = Workload("empty", T=0, d=128, N=8, Z=4, K=3, I=256)
    dm = mb.dims(0, w.d, w.N, w.Z, w.K, w.I, flags=mb.FUSED_COMBINE)
    wt = make_weights(WORKLOADS["tiny"], seed=0)
    g = {k: v.to("cuda") for k, v in wt.items()}
    ws = mb.alloc_workspace(dm, "cuda")
    x = torch.empty((0, w.d), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((0, w.d), dtype=torch.bfloat16, device="cuda")
    mb.moe_forward(dm, x, g["W_r"], g["b"], g["W_g"], g["W_u"], g["W_d"], y, None, ws)
    assert mb.moe_last_device_error(ws) == 0


def test_fused_combine_with_renormalized_gates():
    # The flags combine: renormalised gates change topk_gate, which the fused epilogue reads
    # for the zero-expert term and the combine pass uses alike.
    w, x, wt = _case(WORKLOADS["mid"], T=500, seed=5)
    plain = Stages(w, x, wt, flags=mb.RENORMALIZE_GATES)
    plain.forward()
    fused = Stages(w, x, wt, flags=mb.RENORMALIZE_GATES | mb.FUSED_COMBINE)
    fused.forward()
    torch.cuda.synchronize()
    assert plain.device_status() == 0 and fused.device_status() == 0
    assert torch.equal(plain.y, fused.y)
