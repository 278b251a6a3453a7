"""CPU oracle for the LongCat-Flash MoE layer with zero-computation experts.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  It shares nothing with
the CUDA library and never imports it.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64 on exactly-widened bf16 inputs); this
module only marshals numpy arrays into it.  For layers whose weights do not fit in host memory
(d = 6144, 512 experts), :func:`forward_sampled` routes a sample of tokens and fetches one
expert's weights at a time through a caller-supplied accessor.

Pages cited (title, then section): P1 = "衝上熱搜！美團大模型，靠「快」火了", §零計算專家
(softmax router R, per-expert bias b_i, K selected experts, zero-computation experts return
their input, PID-tuned biases).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _lib.oracle_router.argtypes = [_i64, _i64, _i64, _i64, _ptr, _ptr, _ptr,
                                       _ptr, _ptr, _ptr, _ptr, _ptr]
        _lib.oracle_dispatch.argtypes = [_i64, _i64, _i64, _i64, _ptr, _ptr, _ptr, _ptr, _ptr]
        _lib.oracle_swiglu_expert.argtypes = [_i64, _i64, _i64, _ptr, _ptr, _ptr, _ptr, _ptr]
        _lib.oracle_combine_tokens.argtypes = [_i64, _i64, _i64, _i64, _i64, _ptr, _ptr, _ptr,
                                               _ptr, _ptr, _ptr, _ptr, _ptr]
        _lib.oracle_forward.argtypes = [_i64, _i64, _i64, _i64, _i64, _i64, _ptr, _ptr, _ptr,
                                        _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr]
        _lib.oracle_combine_rows.argtypes = [_i64, _i64, _i64, _i64, _ptr, _ptr, _ptr, _ptr,
                                             _ptr, _ptr]
        _lib.oracle_pid_step.argtypes = [_i64, _i64, _i64, _ptr, _ptr, _ptr, ctypes.c_float,
                                         ctypes.c_float, ctypes.c_float, ctypes.c_float]
        _lib.oracle_renormalize_gates.argtypes = [_i64, _i64, _ptr]
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_decode.restype = ctypes.c_double
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        _lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        _lib.oracle_quantize_fp8_blocks.argtypes = [_i64, _i64, _i64, _ptr, _ptr, _ptr]
        _lib.oracle_quantize_fp8_blocks.restype = None
        _lib.oracle_dequantize_fp8_blocks.argtypes = [_i64, _i64, _i64, _ptr, _ptr, _ptr]
        _lib.oracle_dequantize_fp8_blocks.restype = None
        _lib.oracle_balance_step.argtypes = [_i64, _ptr, _ptr, ctypes.c_float]
        _lib.oracle_quantize_fp8_rows.argtypes = [_i64, _i64, _ptr, _ptr, _ptr]
        _lib.oracle_swiglu_expert_fp8act.argtypes = list(_lib.oracle_swiglu_expert.argtypes)
        _lib.oracle_combine_tokens_fp8act.argtypes = list(_lib.oracle_combine_tokens.argtypes)
        for f in ("oracle_router", "oracle_dispatch", "oracle_swiglu_expert",
                  "oracle_combine_tokens", "oracle_combine_rows", "oracle_forward",
                  "oracle_pid_step", "oracle_renormalize_gates", "oracle_balance_step",
                  "oracle_quantize_fp8_rows", "oracle_swiglu_expert_fp8act",
                  "oracle_combine_tokens_fp8act"):
            getattr(_lib, f).restype = None
    return _lib


def bf16_bits(a):
    """bf16 data as a contiguous numpy uint16 array of bit patterns (torch tensor or numpy)."""
    if hasattr(a, "detach"):  # torch.Tensor
        import torch
        a = a.detach().to("cpu").contiguous()
        assert a.dtype == torch.bfloat16, a.dtype
        return a.view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _f32(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_to_f64(bits):
    """Exact widening of bf16 bit patterns to fp64 (the oracle's view of every input)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def router(x, W_r, b, K, want_probs=False, want_scores=False, renormalize=False):
    """Softmax router R and biased top-K (P1 §零計算專家).

    x: [T, d] bf16, W_r: [E, d] bf16, b: [E] fp32.  Returns a dict with ``topk_idx`` [T, K]
    int32 in ascending expert id, ``topk_gate`` [T, K] fp64 (= p_i, not renormalised unless
    ``renormalize``: then p_i over the sum of the K selected p), ``gap`` [T] fp64
    (= s_(K) - s_(K+1)), and optionally ``probs`` / ``scores`` [T, E] fp64.
    """
    x, W_r, b = bf16_bits(x), bf16_bits(W_r), _f32(b)
    T, d = x.shape
    E = W_r.shape[0]
    assert W_r.shape[1] == d and b.shape == (E,) and 1 <= K <= E
    out = {
        "topk_idx": np.zeros((T, K), np.int32),
        "topk_gate": np.zeros((T, K), np.float64),
        "gap": np.zeros((T,), np.float64),
        "probs": np.zeros((T, E), np.float64) if want_probs else None,
        "scores": np.zeros((T, E), np.float64) if want_scores else None,
    }
    _load().oracle_router(T, d, E, K, _p(x), _p(W_r), _p(b), _p(out["topk_idx"]),
                          _p(out["topk_gate"]), _p(out["gap"]), _p(out["probs"]),
                          _p(out["scores"]))
    if renormalize:
        renormalize_gates(out["topk_gate"])
    return out


def renormalize_gates(topk_gate):
    """In place: each token's K gates divided by their sum (the renormalised-gate variant)."""
    assert topk_gate.dtype == np.float64 and topk_gate.flags.c_contiguous
    T, K = topk_gate.shape
    _load().oracle_renormalize_gates(T, K, _p(topk_gate))
    return topk_gate


def dispatch(topk_idx, N, E):
    """Stable counting sort of the FFN slots by (expert, token); zero-expert slots get -1."""
    topk_idx = _i32(topk_idx)
    T, K = topk_idx.shape
    assert topk_idx.size == 0 or (topk_idx.min() >= 0 and topk_idx.max() < E)
    counts = np.zeros((E,), np.int32)
    offsets = np.zeros((N + 1,), np.int32)
    A = int((topk_idx < N).sum())
    perm_tok = np.zeros((max(A, 1),), np.int32)
    slot_pos = np.zeros((T, K), np.int32)
    _load().oracle_dispatch(T, K, N, E, _p(topk_idx), _p(counts), _p(offsets), _p(perm_tok),
                            _p(slot_pos))
    return {"counts": counts, "offsets": offsets, "perm_tok": perm_tok[:A], "slot_pos": slot_pos}


def swiglu_expert(xrows, W_g, W_u, W_d, fp8_act=False):
    """E(x) = W_d (silu(W_g x) * (W_u x)) for each row of xrows, in fp64.

    With ``fp8_act`` the token rows and h are quantised to E4M3 in 1 x 128 blocks (see
    :func:`quantize_fp8_rows`) before the products; d and I must be multiples of 128."""
    xrows, W_g, W_u, W_d = bf16_bits(xrows), bf16_bits(W_g), bf16_bits(W_u), bf16_bits(W_d)
    R, d = xrows.shape
    I = W_g.shape[0]
    assert W_g.shape == (I, d) and W_u.shape == (I, d) and W_d.shape == (d, I)
    if fp8_act:
        assert d % 128 == 0 and I % 128 == 0
    out = np.zeros((R, d), np.float64)
    if R:
        fn = _load().oracle_swiglu_expert_fp8act if fp8_act else _load().oracle_swiglu_expert
        fn(d, I, R, _p(xrows), _p(W_g), _p(W_u), _p(W_d), _p(out))
    return out


def combine_tokens(tokens, x, topk_idx, topk_gate, W_g, W_u, W_d, N, fp8_act=False):
    """y_t = sum_k g_{t,k} E_{i_{t,k}}(x_t) for the listed tokens (weights all in host memory).

    ``fp8_act``: the FFN experts quantise their activations (see :func:`swiglu_expert`)."""
    x, W_g, W_u, W_d = bf16_bits(x), bf16_bits(W_g), bf16_bits(W_u), bf16_bits(W_d)
    topk_idx = _i32(topk_idx)
    topk_gate = np.ascontiguousarray(topk_gate, dtype=np.float64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    T, d = x.shape
    K = topk_idx.shape[1]
    I = W_g.shape[1]
    if fp8_act:
        assert d % 128 == 0 and I % 128 == 0
    y = np.zeros((len(tokens), d), np.float64)
    fn = _load().oracle_combine_tokens_fp8act if fp8_act else _load().oracle_combine_tokens
    fn(d, N, K, I, len(tokens), _p(tokens), _p(x), _p(topk_idx), _p(topk_gate), _p(W_g),
       _p(W_u), _p(W_d), _p(y))
    return y


def combine_rows(x, topk_idx, topk_gate, slot_pos, rows, N):
    """y_t = sum_k (FFN slot: rows[slot_pos[t,k]], zero slot: g_{t,k} x_t); rows are already gated."""
    x = bf16_bits(x)
    topk_idx, slot_pos = _i32(topk_idx), _i32(slot_pos)
    topk_gate = np.ascontiguousarray(topk_gate, dtype=np.float64)
    rows = np.ascontiguousarray(rows, dtype=np.float64)
    T, d = x.shape
    K = topk_idx.shape[1]
    assert rows.ndim == 2 and rows.shape[1] == d
    ffn = topk_idx < N
    assert (slot_pos[ffn] >= 0).all() and (slot_pos[ffn] < max(len(rows), 1)).all()
    y = np.zeros((T, d), np.float64)
    _load().oracle_combine_rows(T, d, N, K, _p(x), _p(topk_idx), _p(topk_gate), _p(slot_pos),
                                _p(rows), _p(y))
    return y


def forward(x, W_r, b, W_g, W_u, W_d, N, Z, K, renormalize=False):
    """The whole layer for every token: router, biased top-K, experts, weighted sum (fp64).

    With ``renormalize`` the gates are renormalised over the selected set before the sum."""
    x, W_r, b = bf16_bits(x), bf16_bits(W_r), _f32(b)
    W_g, W_u, W_d = bf16_bits(W_g), bf16_bits(W_u), bf16_bits(W_d)
    T, d = x.shape
    I = W_g.shape[1]
    assert W_r.shape == (N + Z, d) and W_g.shape == (N, I, d) and W_d.shape == (N, d, I)
    if renormalize:
        r = router(x, W_r, b, K, renormalize=True)
        y = combine_tokens(np.arange(T), x, r["topk_idx"], r["topk_gate"], W_g, W_u, W_d, N)
        return {"y": y, "topk_idx": r["topk_idx"], "topk_gate": r["topk_gate"], "gap": r["gap"]}
    y = np.zeros((T, d), np.float64)
    idx = np.zeros((T, K), np.int32)
    gate = np.zeros((T, K), np.float64)
    gap = np.zeros((T,), np.float64)
    _load().oracle_forward(T, d, N, Z, K, I, _p(x), _p(W_r), _p(b), _p(W_g), _p(W_u), _p(W_d),
                           _p(y), _p(idx), _p(gate), _p(gap))
    return {"y": y, "topk_idx": idx, "topk_gate": gate, "gap": gap}


def forward_sampled(tokens, x, W_r, b, N, Z, K, fetch_expert, routing=None, fp8_act=False):
    """The layer's output for a sample of tokens when the weights live elsewhere.

    ``fetch_expert(i)`` returns (W_g[i], W_u[i], W_d[i]) as bf16 arrays ([I,d], [I,d], [d,I]).
    Routing (router + biased top-K) is computed here for the sampled rows unless ``routing``
    (a dict like :func:`router`'s, for exactly these rows) is given.  Each distinct FFN expert
    is fetched once and applied to all sampled rows that selected it; the K slot terms of each
    token are then summed in slot order, as in oracle_combine_tokens.  ``fp8_act`` as in
    :func:`swiglu_expert`.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    xs = bf16_bits(x)[tokens] if not hasattr(x, "detach") else bf16_bits(x[tokens])
    if routing is None:
        routing = router(xs, W_r, b, K)
    idx, gate = routing["topk_idx"], routing["topk_gate"]
    n, d = xs.shape
    terms = np.zeros((n, K, d), np.float64)
    xs64 = bf16_to_f64(xs)
    for k in range(K):
        zero = idx[:, k] >= N
        terms[zero, k, :] = xs64[zero]
    for i in np.unique(idx[idx < N]):
        rows, slots = np.nonzero(idx == i)
        W_g, W_u, W_d = fetch_expert(int(i))
        terms[rows, slots, :] = swiglu_expert(xs[rows], W_g, W_u, W_d, fp8_act=fp8_act)
    y = np.zeros((n, d), np.float64)
    for k in range(K):
        y += gate[:, k:k + 1] * terms[:, k, :]
    return {"y": y, **routing}


def pid_step(counts, b, state, N, K, T, target, kp, ki, kd):
    """One PID update of the FFN experts' biases (P1 §零計算專家, last paragraph), in place.

    b: float32 [E] numpy array, state: float32 [2] numpy array {integral, e_prev}.
    """
    counts = _i32(counts)
    assert b.dtype == np.float32 and b.flags.c_contiguous
    assert state.dtype == np.float32 and state.shape == (2,)
    _load().oracle_pid_step(N, K, T, _p(counts), _p(b), _p(state), target, kp, ki, kd)


def balance_step(counts, b, N, gamma):
    """Per-expert balancing term, in place: b_i += gamma * sign(mean FFN load - counts_i), i < N.

    b: float32 [E] numpy array.  Applied after :func:`pid_step` when both are used."""
    counts = _i32(counts)
    assert b.dtype == np.float32 and b.flags.c_contiguous
    _load().oracle_balance_step(N, _p(counts), _p(b), gamma)


def e4m3_decode(code):
    """Value of an E4M3 code (NaN for S.1111.111)."""
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode(v):
    """E4M3 code of v: nearest, ties to even mantissa, saturating at +-448."""
    return int(_load().oracle_e4m3_encode(float(v)))


def quantize_fp8_blocks(w):
    """Block-wise FP8 of bf16 weights [G, R, C] (R, C multiples of 128): returns (q uint8
    [G, R, C], scale float32 [G, R/128, C/128]), one power-of-two scale per 128 x 128 block."""
    w = bf16_bits(w)
    if w.ndim == 2:
        w = w[None]
    G, R, C = w.shape
    assert R % 128 == 0 and C % 128 == 0
    q = np.zeros((G, R, C), np.uint8)
    scale = np.zeros((G, R // 128, C // 128), np.float32)
    _load().oracle_quantize_fp8_blocks(G, R, C, _p(np.ascontiguousarray(w)), _p(q), _p(scale))
    return q, scale


def dequantize_fp8_blocks(q, scale):
    """q * (its block's scale) as bf16 bit patterns [G, R, C] (the weights the FP8 variant uses)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    G, R, C = q.shape
    w = np.zeros((G, R, C), np.uint16)
    _load().oracle_dequantize_fp8_blocks(G, R, C, _p(q), _p(scale), _p(w))
    return w


def quantize_fp8_rows(v):
    """FP8 activations: rows of v [R, C] (C a multiple of 128; float values, fp64 exact) ->
    (q uint8 [R, C], scale float32 [R, C/128]), one power-of-two scale per 1 x 128 block by
    the weights' rule (smallest 2^e with max|v| <= 448 * 2^e, e >= -126, 1 for an all-zero
    block; q = E4M3(v / 2^e), nearest, ties to even)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    if v.ndim == 1:
        v = v[None]
    R, C = v.shape
    assert C % 128 == 0
    q = np.zeros((R, C), np.uint8)
    scale = np.zeros((R, C // 128), np.float32)
    if R and C:
        _load().oracle_quantize_fp8_rows(R, C, _p(v), _p(q), _p(scale))
    return q, scale
