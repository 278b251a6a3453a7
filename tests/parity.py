"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI and compare it
with the CPU oracle under the layer's parity rules.

Parity rules (from the layer's specification):
  * routing: for every token whose oracle gap s_(K) - s_(K+1) exceeds 1e-4 the selected ids
    are bit-exact; tokens at or below it are near-ties, counted, and the GPU's set must be
    eps-valid: min over selected oracle scores >= max over unselected oracle scores - 1e-4;
  * dispatch (counts, offsets, permutation, slot rows): bit-exact;
  * outputs: max|y - y_ref| <= 1e-2 * max|y_ref| and ||y - y_ref||_2 <= 5e-3 * ||y_ref||_2.
Gate values come from an fp32 softmax on the GPU and an fp64 one in the oracle.  The GPU's
logits are fp32 sums of d exact bf16 x bf16 products accumulated on the tensor cores; a gate's
relative error is, to first order, its logit's error minus the probability-weighted mean logit
error, plus a few 1e-6 of fp32 rounding in the softmax.  Where the GPU's logits are read back
(moe_router_logits), gates are checked against exactly that expansion and the logits against
the fp32 accumulation bound (check_gates_against_logits); the logit errors themselves depend
on the data (at d = 6144: ~6e-5 at prefill, ~1.6e-4 on the Zipf-skewed logits, whose large
first term every later accumulation step rounds against).  Elsewhere gates are compared with
rtol = 1e-4.
"""
import numpy as np
import torch

import oracle
from mixture_experts_layer_38_b200 import binding as mb

GAP_EPS = 1e-4
Y_MAX_TOL = 1e-2
Y_L2_TOL = 5e-3
GATE_RTOL = 1e-4       # gates of small cases checked without the GPU logits
GATE_PROP_TOL = 3e-6   # gate error minus its first-order logit-error part (fp32 softmax)


def y_errors(y, y_ref):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    max_ref = np.abs(y_ref).max()
    max_err = np.abs(y - y_ref).max()
    l2 = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    return max_err / max(max_ref, 1e-300), l2


def assert_y_close(y, y_ref, what="y"):
    rel_max, rel_l2 = y_errors(y, y_ref)
    assert rel_max <= Y_MAX_TOL and rel_l2 <= Y_L2_TOL, (
        f"{what}: max|err|/max|ref| = {rel_max:.3e} (<= {Y_MAX_TOL}), "
        f"relative L2 = {rel_l2:.3e} (<= {Y_L2_TOL})")
    return rel_max, rel_l2


def exact_logits(x, W_r):
    """l = x W_r^T and sum_j |x_j W_ij| in fp64 on the exactly widened bf16 inputs."""
    xs = oracle.bf16_to_f64(oracle.bf16_bits(x))
    W = oracle.bf16_to_f64(oracle.bf16_bits(W_r))
    return xs @ W.T, np.abs(xs) @ np.abs(W).T


def check_gates_against_logits(gpu_idx, gpu_gate, gpu_logits, x, W_r, probs, renormalize=False):
    """The GPU's gates, checked through the GPU's own fp32 router logits (moe_router_logits).

    1. Logits: the tensor cores add d exact bf16 products in d/16 MMA steps of fp32
       accumulation and the top-K kernel adds the S <= 16 split-K partials; each of these at
       most d/16 + 16 roundings is at most 2u (u = 2^-24) times a partial sum, itself at most
       sum_j |x_j W_ij|, so |l~_i - l_i| <= (d/16 + 16) * 2u * sum_j |x_j W_ij|.
    2. Gates: with delta = l~ - l, the fp32 softmax gives, to first order,
       g_i / p_i - 1 = delta_i - sum_k p_k delta_k (renormalised: delta_i minus the
       p-weighted mean of delta over the selected set) plus the fp32 roundings of the
       subtraction, expf, the tree sum and the division, together below 3e-6.  The measured
       gate errors must match that expansion to within 3e-6: nothing but the logits' fp32
       accumulation separates the GPU's gates from the oracle's.
    Returns the largest relative gate error."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_gate = np.asarray(gpu_gate, np.float64)
    l_ref, mag = exact_logits(x, W_r)
    d = oracle.bf16_bits(x).shape[1]
    delta = np.asarray(gpu_logits, np.float64) - l_ref
    bound = (d // 16 + 16) * 2.0 ** -23 * mag
    worst = np.abs(delta) / bound
    assert (worst <= 1.0).all(), f"router logit error beyond the fp32 accumulation bound ({worst.max():.2f}x)"
    p_sel = np.take_along_axis(probs, gpu_idx, axis=1)
    d_sel = np.take_along_axis(delta, gpu_idx, axis=1)
    if renormalize:
        want = p_sel / p_sel.sum(axis=1, keepdims=True)
        mean = (p_sel * d_sel).sum(axis=1, keepdims=True) / p_sel.sum(axis=1, keepdims=True)
    else:
        want = p_sel
        mean = (probs * delta).sum(axis=1, keepdims=True)
    measured = gpu_gate / want - 1.0
    resid = np.abs(measured - (d_sel - mean))
    assert resid.max() <= GATE_PROP_TOL, (
        f"gate error not explained by the logit error: residual {resid.max():.3e}")
    return float(np.abs(measured).max()) if measured.size else 0.0


def check_routing_full(gpu_idx, gpu_gate, ref, gpu_logits=None, x=None, W_r=None):
    """Whole-batch routing check against ``ref`` = oracle.router(..., want_probs=True,
    want_scores=True) over the same tokens.  Returns a dict of counts and the largest gate
    error.

    * every token whose oracle gap exceeds GAP_EPS: the GPU's ids equal the oracle's;
    * every token: ids ascending, distinct and in range; each GPU gate is the oracle's fp64
      probability of the id the GPU selected, up to the propagated fp32 logit error
      (check_gates_against_logits, given the GPU's logits) or within GATE_RTOL otherwise;
    * near-tie tokens whose GPU set differs: eps-valid under the oracle's scores."""
    gpu_idx = np.asarray(gpu_idx)
    gpu_gate = np.asarray(gpu_gate, np.float64)
    T, K = gpu_idx.shape
    E = ref["scores"].shape[1]
    assert ((gpu_idx >= 0) & (gpu_idx < E)).all()
    if K > 1:
        assert (np.diff(gpu_idx, axis=1) > 0).all(), "ids not strictly ascending"
    clear = ref["gap"] > GAP_EPS
    np.testing.assert_array_equal(gpu_idx[clear], ref["topk_idx"][clear])
    if gpu_logits is not None:
        gate_err = check_gates_against_logits(gpu_idx, gpu_gate, gpu_logits, x, W_r,
                                              ref["probs"])
    else:
        p_sel = np.take_along_axis(ref["probs"], gpu_idx, axis=1)
        np.testing.assert_allclose(gpu_gate, p_sel, rtol=GATE_RTOL, atol=1e-30)
        gate_err = float((np.abs(gpu_gate - p_sel) / np.maximum(p_sel, 1e-300)).max()) \
            if p_sel.size else 0.0
    differ = np.flatnonzero((gpu_idx != ref["topk_idx"]).any(axis=1))
    if len(differ):
        s = ref["scores"][differ]
        sel = np.zeros(s.shape, bool)
        np.put_along_axis(sel, gpu_idx[differ], True, axis=1)
        min_sel = np.where(sel, s, np.inf).min(axis=1)
        max_unsel = np.where(sel, -np.inf, s).max(axis=1)
        bad = differ[min_sel < max_unsel - GAP_EPS]
        assert len(bad) == 0, f"GPU top-K sets not eps-valid for tokens {bad[:10]}"
    return {"tokens": int(T), "near_ties": int((~clear).sum()), "differing": int(len(differ)),
            "max_gate_rel_err": gate_err}


def gpu_routing_for_oracle(gpu_idx, ref, rows):
    """The routing the GPU took for ``rows``, with the oracle's fp64 gates of those ids: the
    input under which the oracle's layer output is compared for every token (it equals the
    oracle's own routing wherever the sets agree, which every non-near-tie token does)."""
    idx = np.ascontiguousarray(np.asarray(gpu_idx)[rows], dtype=np.int32)
    gate = np.take_along_axis(ref["probs"][rows], idx, axis=1)
    return {"topk_idx": idx, "topk_gate": np.ascontiguousarray(gate), "gap": ref["gap"][rows]}


def check_dispatch_vs_oracle(gpu_idx, gpu_gate, counts, offsets, perm_tok, perm_gate, slot_pos,
                             N, E):
    """The GPU's dispatch tables bit-exact against oracle.dispatch fed the GPU's own routing
    (every token); perm_gate carries each slot's fp32 gate unchanged."""
    gpu_idx = np.asarray(gpu_idx)
    dsp = oracle.dispatch(gpu_idx, N, E)
    A = len(dsp["perm_tok"])
    np.testing.assert_array_equal(counts, dsp["counts"])
    np.testing.assert_array_equal(offsets, dsp["offsets"])
    np.testing.assert_array_equal(np.asarray(perm_tok)[:A], dsp["perm_tok"])
    np.testing.assert_array_equal(slot_pos, dsp["slot_pos"])
    ffn = dsp["slot_pos"] >= 0
    want_gate = np.zeros(A, np.float32)
    want_gate[dsp["slot_pos"][ffn]] = np.asarray(gpu_gate, np.float32)[ffn]
    np.testing.assert_array_equal(np.asarray(perm_gate)[:A], want_gate)
    return dsp


def check_dispatch_properties(idx, counts, offsets, perm_tok, slot_pos, N, E):
    """The GPU dispatch must be exactly the stable (expert, token) sort of its own routing."""
    idx = np.asarray(idx)
    T, K = idx.shape
    np.testing.assert_array_equal(counts, np.bincount(idx.reshape(-1), minlength=E))
    ex = idx.reshape(-1)
    tok = np.repeat(np.arange(T), K)
    ffn = ex < N
    order = np.lexsort((tok[ffn], ex[ffn]))
    A = int(ffn.sum())
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts[:N])]))
    np.testing.assert_array_equal(perm_tok[:A], tok[ffn][order])
    rows = np.full(T * K, -1)
    rows[np.flatnonzero(ffn)[order]] = np.arange(A)
    np.testing.assert_array_equal(np.asarray(slot_pos).reshape(-1), rows)


def to_np(t):
    if t.dtype == torch.bfloat16:
        return oracle.bf16_bits(t)
    return t.detach().cpu().numpy()


class Stages:
    """Device buffers for running the staged C-ABI calls on one workload."""

    def __init__(self, w, x, wt, device="cuda", flags=0):
        self.w = w
        self.dm = mb.dims(w.T, w.d, w.N, w.Z, w.K, w.I, flags=flags)
        R = w.T * w.K
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.x = x.to(device)
        self.wt = {k: v.to(device) for k, v in wt.items()}
        self.ws = mb.alloc_workspace(self.dm, device)
        self.topk_idx = torch.zeros((w.T, w.K), **i32)
        self.topk_gate = torch.zeros((w.T, w.K), **f32)
        self.gap = torch.zeros((w.T,), **f32)
        self.counts = torch.zeros((w.E,), **i32)
        self.offsets = torch.zeros((w.N + 1,), **i32)
        self.perm_tok = torch.full((R,), -7, **i32)
        self.perm_gate = torch.zeros((R,), **f32)
        self.slot_pos = torch.zeros((w.T, w.K), **i32)
        self.x_perm = torch.zeros((R, w.d), **bf)
        self.h = torch.zeros((R, w.I), **bf)
        self.y_perm = torch.zeros((R, w.d), **bf)
        self.y = torch.zeros((w.T, w.d), **bf)

    def route(self, b=None):
        mb.moe_route(self.dm, self.x, self.wt["W_r"], self.wt["b"] if b is None else b,
                     self.topk_idx, self.topk_gate, self.gap, self.ws)

    def logits(self):
        """The fp32 router logits of the last routing call on this workspace (host copy)."""
        out = torch.empty((self.w.T, self.w.E), dtype=torch.float32, device=self.x.device)
        mb.moe_router_logits(self.dm, self.ws, out)
        return out.cpu().numpy()

    def dispatch(self):
        mb.moe_dispatch(self.dm, self.x, self.topk_idx, self.topk_gate, self.counts, self.offsets,
                        self.perm_tok, self.perm_gate, self.slot_pos, self.x_perm, self.ws)

    def expert_ffn(self):
        mb.moe_expert_ffn(self.dm, self.x_perm, self.offsets, self.perm_gate, self.wt["W_g"],
                          self.wt["W_u"], self.wt["W_d"], self.h, self.y_perm, self.ws)

    def combine(self):
        mb.moe_combine(self.dm, self.x, self.y_perm, self.topk_idx, self.topk_gate,
                       self.slot_pos, self.y, self.ws)

    def forward(self, b=None, counts=None):
        mb.moe_forward(self.dm, self.x, self.wt["W_r"], self.wt["b"] if b is None else b,
                       self.wt["W_g"], self.wt["W_u"], self.wt["W_d"], self.y,
                       self.counts if counts is None else counts, self.ws)

    def device_status(self):
        return mb.moe_last_device_error(self.ws)
