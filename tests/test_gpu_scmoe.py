"""GPU parity of the dense SwiGLU FFN (the ScMoE shortcut branch) against the oracle, alone and
on a second stream beside the MoE layer.

Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 快捷連接 MoE (the previous block's dense
FFN runs in parallel with the current MoE layer).  The dense branch is the oracle's SwiGLU
expert applied to every token (pinned against torch fp64 in the oracle tests); running it
concurrently with moe_forward must not change either output by a single bit.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb
from mixture_experts_layer_38_b200.workloads import WORKLOADS, make_tokens, make_weights
from parity import assert_y_close, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dense_case(T, d, I, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    W_g = (torch.randn((I, d), generator=g) * 0.02).to(torch.bfloat16)
    W_u = (torch.randn((I, d), generator=g) * 0.02).to(torch.bfloat16)
    W_d = (torch.randn((d, I), generator=g) * 0.02).to(torch.bfloat16)
    return x, W_g, W_u, W_d


def _run_dense(x, W_g, W_u, W_d, stream=None):
    T, d = x.shape
    I = W_g.shape[0]
    dm = mb.dims(T, d, 1, 0, 1, I)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    h = torch.empty((T, I), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    mb.moe_dense_ffn(dm, x.to(DEV), W_g.to(DEV), W_u.to(DEV), W_d.to(DEV), h, y, ws, stream)
    return y, ws


# d = 4096 with T >= 128 selects 256-token tiles (one full tile and a 44-row tail at T = 300):
# on CTA pairs at I = 512, on single CTAs at I = 384.
@pytest.mark.parametrize("T,d,I", [(64, 128, 256), (1, 128, 256), (333, 2048, 1024),
                                   (700, 384, 640), (300, 4096, 512), (300, 4096, 384)])
def test_dense_ffn_matches_oracle(T, d, I):
    x, W_g, W_u, W_d = _dense_case(T, d, I, seed=T + d)
    y, ws = _run_dense(x, W_g, W_u, W_d)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0
    ref = oracle.swiglu_expert(x, W_g, W_u, W_d)
    assert_y_close(oracle.bf16_to_f64(to_np(y)), ref, f"dense T={T}")


def test_dense_ffn_zero_tokens():
    x, W_g, W_u, W_d = _dense_case(0, 128, 256, seed=1)
    y, ws = _run_dense(x, W_g, W_u, W_d)
    torch.cuda.synchronize()
    assert mb.moe_last_device_error(ws) == 0 and y.shape == (0, 128)


def test_dense_ffn_beside_moe_forward_on_two_streams():
    w = WORKLOADS["mid"]
    wt = {k: v.to(DEV) for k, v in make_weights(w, seed=0).items()}
    x = make_tokens(w, seed=0).to(DEV)
    dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = mb.alloc_workspace(dm, DEV)
    xd, W_g, W_u, W_d = (t.to(DEV) for t in _dense_case(w.T, w.d, 2 * w.I, seed=9))
    dmd = mb.dims(w.T, w.d, 1, 0, 1, 2 * w.I)
    wsd = torch.zeros(256, dtype=torch.uint8, device=DEV)
    hd = torch.empty((w.T, 2 * w.I), dtype=torch.bfloat16, device=DEV)

    def serial():
        y = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=DEV)
        yd = torch.empty((w.T, w.d), dtype=torch.bfloat16, device=DEV)
        mb.moe_forward(dm, x, wt["W_r"], wt["b"], wt["W_g"], wt["W_u"], wt["W_d"], y, None, ws)
        mb.moe_dense_ffn(dmd, xd, W_g, W_u, W_d, hd, yd, wsd)
        torch.cuda.synchronize()
        return y, yd

    y0, yd0 = serial()
    a = torch.cuda.current_stream()
    s2 = torch.cuda.Stream()
    y = torch.empty_like(y0)
    yd = torch.empty_like(yd0)
    for _ in range(3):  # the two calls overlap on the GPU; results must not change
        s2.wait_stream(a)
        mb.moe_dense_ffn(dmd, xd, W_g, W_u, W_d, hd, yd, wsd, stream=s2)
        mb.moe_forward(dm, x, wt["W_r"], wt["b"], wt["W_g"], wt["W_u"], wt["W_d"], y, None, ws)
        a.wait_stream(s2)
        torch.cuda.synchronize()
        assert torch.equal(y, y0) and torch.equal(yd, yd0)
    assert mb.moe_last_device_error(ws) == 0 and mb.moe_last_device_error(wsd) == 0
