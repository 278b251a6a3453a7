"""Thin ctypes binding over libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: each function checks dtypes, shapes and devices of the torch
tensors it is given, passes their device pointers and the current CUDA stream to the C entry
point of the same name, and raises :class:`MoeError` on a non-zero return code.  Every step of
the layer runs in the library's CUDA kernels; there is no fallback of any kind, and using any
entry point without the built library raises immediately.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

# Every symbol declared in include/moe.h.
EXPORTS = (
    "moe_strerror", "moe_workspace_size", "moe_scratch_size", "moe_route", "moe_dispatch",
    "moe_expert_ffn", "moe_combine", "moe_bias_update", "moe_forward", "moe_forward_timed",
    "moe_last_device_error", "moe_dispatch_noalloc", "moe_expert_ffn_gather",
    "moe_quantize_fp8", "moe_expert_ffn_fp8", "moe_forward_fp8", "moe_dense_ffn",
    "moe_router_logits", "moe_debug_set_wait_limit", "moe_quantize_fp8_rows",
)
NUM_STAGE_EVENTS = 7
STAGE_NAMES = ("router_gemm", "route_topk", "dispatch", "ffn_up_gemm", "ffn_down_gemm",
               "combine")

MOE_DEV_CODES = {0: "ok", 0x100: "bounded wait timed out", 0x200: "expert id out of range",
                 0x300: "row offsets / indices out of range"}


class MoeError(RuntimeError):
    def __init__(self, fn, code, text):
        super().__init__(f"{fn} failed with code {code}: {text}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("Z", ctypes.c_int32), ("K", ctypes.c_int32), ("I", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]

    def __repr__(self):
        return (f"Dims(T={self.T}, d={self.d}, N={self.N}, Z={self.Z}, K={self.K}, I={self.I}, "
                f"flags={self.flags})")


class PidParams(ctypes.Structure):
    _fields_ = [("target", ctypes.c_float), ("kp", ctypes.c_float), ("ki", ctypes.c_float),
                ("kd", ctypes.c_float), ("balance_gamma", ctypes.c_float)]


_lib = None
_P = ctypes.c_void_p
_S = ctypes.c_size_t
_DP = ctypes.POINTER(Dims)


def lib():
    """The loaded library; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m "
                "mixture_experts_layer_38_b200.build` (nvcc, sm_100a); there is no fallback")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_strerror.restype = ctypes.c_char_p
        L.moe_strerror.argtypes = [ctypes.c_int]
        L.moe_workspace_size.restype = _S
        L.moe_workspace_size.argtypes = [_DP]
        L.moe_scratch_size.restype = _S
        L.moe_scratch_size.argtypes = [_DP]
        L.moe_route.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_dispatch.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_expert_ffn.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_combine.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_router_logits.argtypes = [_DP, _P, _S, _P, _P]
        L.moe_debug_set_wait_limit.argtypes = [ctypes.c_int64]
        L.moe_bias_update.argtypes = [_DP, _P, _P, _P, ctypes.POINTER(PidParams), _P]
        L.moe_forward.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_forward_timed.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S,
                                        ctypes.POINTER(ctypes.c_void_p), _P]
        L.moe_last_device_error.argtypes = [_P, _P]
        L.moe_dispatch_noalloc.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_expert_ffn_gather.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        _I64 = ctypes.c_int64
        L.moe_quantize_fp8.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
        L.moe_quantize_fp8_rows.argtypes = [_P, _I64, _I64, _P, _P, _P]
        L.moe_dense_ffn.argtypes = [_DP, _P, _P, _P, _P, _P, _P, _P, _S, _P]
        L.moe_expert_ffn_fp8.argtypes = [_DP] + [_P] * 11 + [_P, _S, _P]
        L.moe_forward_fp8.argtypes = [_DP] + [_P] * 11 + [_P, _S,
                                                          ctypes.POINTER(ctypes.c_void_p), _P]
        for f in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine",
                  "moe_bias_update", "moe_forward", "moe_forward_timed",
                  "moe_last_device_error", "moe_dispatch_noalloc", "moe_expert_ffn_gather",
                  "moe_quantize_fp8", "moe_expert_ffn_fp8", "moe_forward_fp8",
                  "moe_dense_ffn", "moe_router_logits", "moe_debug_set_wait_limit",
                  "moe_quantize_fp8_rows"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


RENORMALIZE_GATES = 1  # MOE_RENORMALIZE_GATES
FP8_ACTIVATIONS = 2  # MOE_FP8_ACTIVATIONS
FUSED_COMBINE = 4  # MOE_FUSED_COMBINE


def dims(T, d, N, Z, K, I, flags=0) -> Dims:
    return Dims(int(T), int(d), int(N), int(Z), int(K), int(I), int(flags))


def strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def _check(fn, rc):
    if rc != 0:
        raise MoeError(fn, rc, strerror(rc))


def _ptr(t, dtype, shape=None, name="tensor", nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(dm: Dims) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(dm)))


def scratch_size(dm: Dims) -> int:
    return int(lib().moe_scratch_size(ctypes.byref(dm)))


def alloc_workspace(dm: Dims, device="cuda", scratch_only=False) -> torch.Tensor:
    """A workspace for moe_forward (or, with scratch_only, for the staged calls); the status
    word at its start is zeroed."""
    n = scratch_size(dm) if scratch_only else workspace_size(dm)
    if n == 0:
        raise ValueError(f"unsupported dims {dm!r}")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def _ws(ws):
    return _ptr(ws, torch.uint8, name="ws"), ws.numel()


def moe_route(dm, x, W_r, b, topk_idx, topk_gate, gap, ws, stream=None):
    E = dm.N + dm.Z
    w, n = _ws(ws)
    rc = lib().moe_route(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(W_r, torch.bfloat16, (E, dm.d), "W_r"), _ptr(b, torch.float32, (E,), "b"),
        _ptr(topk_idx, torch.int32, (dm.T, dm.K), "topk_idx"),
        _ptr(topk_gate, torch.float32, (dm.T, dm.K), "topk_gate"),
        _ptr(gap, torch.float32, (dm.T,), "gap", nullable=True), w, n, _stream(stream))
    _check("moe_route", rc)


def moe_dispatch(dm, x, topk_idx, topk_gate, counts, offsets, perm_tok, perm_gate, slot_pos,
                 x_perm, ws, stream=None):
    E, R = dm.N + dm.Z, dm.T * dm.K
    w, n = _ws(ws)
    rc = lib().moe_dispatch(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(topk_idx, torch.int32, (dm.T, dm.K), "topk_idx"),
        _ptr(topk_gate, torch.float32, (dm.T, dm.K), "topk_gate"),
        _ptr(counts, torch.int32, (E,), "counts"), _ptr(offsets, torch.int32, (dm.N + 1,), "offsets"),
        _ptr(perm_tok, torch.int32, (R,), "perm_tok"), _ptr(perm_gate, torch.float32, (R,), "perm_gate"),
        _ptr(slot_pos, torch.int32, (dm.T, dm.K), "slot_pos"),
        _ptr(x_perm, torch.bfloat16, (R, dm.d), "x_perm", nullable=True), w, n, _stream(stream))
    _check("moe_dispatch", rc)


def moe_dispatch_noalloc(dm, x, topk_idx, topk_gate, counts, offsets, perm_tok, perm_gate,
                         slot_pos, x_perm, stream=None):
    """moe_dispatch without a workspace, for callers that cannot hand the library device
    memory; its scratch is a fixed array inside the library (see include/moe.h)."""
    E, R = dm.N + dm.Z, dm.T * dm.K
    rc = lib().moe_dispatch_noalloc(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(topk_idx, torch.int32, (dm.T, dm.K), "topk_idx"),
        _ptr(topk_gate, torch.float32, (dm.T, dm.K), "topk_gate"),
        _ptr(counts, torch.int32, (E,), "counts"), _ptr(offsets, torch.int32, (dm.N + 1,), "offsets"),
        _ptr(perm_tok, torch.int32, (R,), "perm_tok"), _ptr(perm_gate, torch.float32, (R,), "perm_gate"),
        _ptr(slot_pos, torch.int32, (dm.T, dm.K), "slot_pos"),
        _ptr(x_perm, torch.bfloat16, (R, dm.d), "x_perm", nullable=True), _stream(stream))
    _check("moe_dispatch_noalloc", rc)


def moe_expert_ffn(dm, x_perm, offsets, perm_gate, W_g, W_u, W_d, h, y_perm, ws, stream=None):
    R = dm.T * dm.K
    w, n = _ws(ws)
    rc = lib().moe_expert_ffn(
        ctypes.byref(dm), _ptr(x_perm, torch.bfloat16, (R, dm.d), "x_perm"),
        _ptr(offsets, torch.int32, (dm.N + 1,), "offsets"),
        _ptr(perm_gate, torch.float32, (R,), "perm_gate"),
        _ptr(W_g, torch.bfloat16, (dm.N, dm.I, dm.d), "W_g"),
        _ptr(W_u, torch.bfloat16, (dm.N, dm.I, dm.d), "W_u"),
        _ptr(W_d, torch.bfloat16, (dm.N, dm.d, dm.I), "W_d"),
        _ptr(h, torch.bfloat16, (R, dm.I), "h"), _ptr(y_perm, torch.bfloat16, (R, dm.d), "y_perm"),
        w, n, _stream(stream))
    _check("moe_expert_ffn", rc)


def moe_expert_ffn_gather(dm, x, perm_tok, offsets, perm_gate, W_g, W_u, W_d, h, y_perm, ws,
                          stream=None):
    R = dm.T * dm.K
    w, n = _ws(ws)
    rc = lib().moe_expert_ffn_gather(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(perm_tok, torch.int32, (R,), "perm_tok"),
        _ptr(offsets, torch.int32, (dm.N + 1,), "offsets"),
        _ptr(perm_gate, torch.float32, (R,), "perm_gate"),
        _ptr(W_g, torch.bfloat16, (dm.N, dm.I, dm.d), "W_g"),
        _ptr(W_u, torch.bfloat16, (dm.N, dm.I, dm.d), "W_u"),
        _ptr(W_d, torch.bfloat16, (dm.N, dm.d, dm.I), "W_d"),
        _ptr(h, torch.bfloat16, (R, dm.I), "h"), _ptr(y_perm, torch.bfloat16, (R, dm.d), "y_perm"),
        w, n, _stream(stream))
    _check("moe_expert_ffn_gather", rc)


def moe_combine(dm, x, y_perm, topk_idx, topk_gate, slot_pos, y, ws, stream=None):
    R = dm.T * dm.K
    w, n = _ws(ws)
    rc = lib().moe_combine(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(y_perm, torch.bfloat16, (R, dm.d), "y_perm"),
        _ptr(topk_idx, torch.int32, (dm.T, dm.K), "topk_idx"),
        _ptr(topk_gate, torch.float32, (dm.T, dm.K), "topk_gate"),
        _ptr(slot_pos, torch.int32, (dm.T, dm.K), "slot_pos"),
        _ptr(y, torch.bfloat16, (dm.T, dm.d), "y"), w, n, _stream(stream))
    _check("moe_combine", rc)


def moe_router_logits(dm, ws, logits, stream=None):
    """The fp32 router logits [T, N+Z] of the last routing call on ``ws`` (same dims)."""
    w, n = _ws(ws)
    rc = lib().moe_router_logits(
        ctypes.byref(dm), w, n, _ptr(logits, torch.float32, (dm.T, dm.N + dm.Z), "logits"),
        _stream(stream))
    _check("moe_router_logits", rc)


def moe_debug_set_wait_limit(cycles: int):
    """Testing hook: the grouped GEMMs' per-wait limit in SM cycles (0 = the default)."""
    _check("moe_debug_set_wait_limit", lib().moe_debug_set_wait_limit(int(cycles)))


def moe_bias_update(dm, counts, b, pid_state, params: PidParams, stream=None):
    E = dm.N + dm.Z
    rc = lib().moe_bias_update(
        ctypes.byref(dm), _ptr(counts, torch.int32, (E,), "counts"),
        _ptr(b, torch.float32, (E,), "b"), _ptr(pid_state, torch.float32, (2,), "pid_state"),
        ctypes.byref(params), _stream(stream))
    _check("moe_bias_update", rc)


def moe_forward(dm, x, W_r, b, W_g, W_u, W_d, y, counts, ws, stream=None):
    E = dm.N + dm.Z
    w, n = _ws(ws)
    rc = lib().moe_forward(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(W_r, torch.bfloat16, (E, dm.d), "W_r"), _ptr(b, torch.float32, (E,), "b"),
        _ptr(W_g, torch.bfloat16, (dm.N, dm.I, dm.d), "W_g"),
        _ptr(W_u, torch.bfloat16, (dm.N, dm.I, dm.d), "W_u"),
        _ptr(W_d, torch.bfloat16, (dm.N, dm.d, dm.I), "W_d"),
        _ptr(y, torch.bfloat16, (dm.T, dm.d), "y"),
        _ptr(counts, torch.int32, (E,), "counts", nullable=True), w, n, _stream(stream))
    _check("moe_forward", rc)


def moe_forward_timed(dm, x, W_r, b, W_g, W_u, W_d, y, counts, ws, events, stream=None):
    """moe_forward recording ``events`` (NUM_STAGE_EVENTS torch.cuda.Event, timing enabled)
    at the stage boundaries; durations are ``events[i].elapsed_time(events[i + 1])``."""
    E = dm.N + dm.Z
    if len(events) != NUM_STAGE_EVENTS:
        raise ValueError(f"need {NUM_STAGE_EVENTS} events")
    arr = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[ctypes.c_void_p(ev.cuda_event) for ev in events])
    w, n = _ws(ws)
    rc = lib().moe_forward_timed(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(W_r, torch.bfloat16, (E, dm.d), "W_r"), _ptr(b, torch.float32, (E,), "b"),
        _ptr(W_g, torch.bfloat16, (dm.N, dm.I, dm.d), "W_g"),
        _ptr(W_u, torch.bfloat16, (dm.N, dm.I, dm.d), "W_u"),
        _ptr(W_d, torch.bfloat16, (dm.N, dm.d, dm.I), "W_d"),
        _ptr(y, torch.bfloat16, (dm.T, dm.d), "y"),
        _ptr(counts, torch.int32, (E,), "counts", nullable=True), w, n, arr, _stream(stream))
    _check("moe_forward_timed", rc)


def moe_last_device_error(ws, stream=None) -> int:
    return int(lib().moe_last_device_error(_ptr(ws, torch.uint8, name="ws"), _stream(stream)))


def moe_quantize_fp8(w, q, scale, stream=None):
    """Block-wise E4M3 codes and power-of-two scales of bf16 weights [G, R, C] (or [R, C])."""
    shape = tuple(w.shape) if w.dim() == 3 else (1,) + tuple(w.shape)
    G, R, C = shape
    rc = lib().moe_quantize_fp8(
        _ptr(w, torch.bfloat16, tuple(w.shape), "w"), G, R, C,
        _ptr(q, torch.uint8, tuple(w.shape), "q"),
        _ptr(scale, torch.float32, (G, R // 128, C // 128) if w.dim() == 3 else
             (R // 128, C // 128), "scale"), _stream(stream))
    _check("moe_quantize_fp8", rc)


def moe_quantize_fp8_rows(x, q, scale, stream=None):
    """E4M3 codes of bf16 rows x [R, C] with one power-of-two scale per 1 x 128 block;
    scale is block-major [C/128, R]."""
    R, C = x.shape
    rc = lib().moe_quantize_fp8_rows(
        _ptr(x, torch.bfloat16, (R, C), "x"), R, C, _ptr(q, torch.uint8, (R, C), "q"),
        _ptr(scale, torch.float32, (C // 128, R), "scale"), _stream(stream))
    _check("moe_quantize_fp8_rows", rc)


def quantize_expert_weights_fp8(dm, W_g, W_u, W_d, stream=None):
    """All three expert weight tensors quantised on the device: a dict of codes and scales."""
    out = {}
    for name, w in (("g", W_g), ("u", W_u), ("d", W_d)):
        G, R, C = w.shape
        out["q_" + name] = torch.empty((G, R, C), dtype=torch.uint8, device=w.device)
        out["s_" + name] = torch.empty((G, R // 128, C // 128), dtype=torch.float32,
                                       device=w.device)
        moe_quantize_fp8(w, out["q_" + name], out["s_" + name], stream)
    return out


def _fp8_args(dm, fw):
    I, d, N = dm.I, dm.d, dm.N
    return (_ptr(fw["q_g"], torch.uint8, (N, I, d), "q_g"),
            _ptr(fw["s_g"], torch.float32, (N, I // 128, d // 128), "s_g"),
            _ptr(fw["q_u"], torch.uint8, (N, I, d), "q_u"),
            _ptr(fw["s_u"], torch.float32, (N, I // 128, d // 128), "s_u"),
            _ptr(fw["q_d"], torch.uint8, (N, d, I), "q_d"),
            _ptr(fw["s_d"], torch.float32, (N, d // 128, I // 128), "s_d"))


def moe_expert_ffn_fp8(dm, x_perm, offsets, perm_gate, fw, h, y_perm, ws, stream=None):
    R = dm.T * dm.K
    w, n = _ws(ws)
    rc = lib().moe_expert_ffn_fp8(
        ctypes.byref(dm), _ptr(x_perm, torch.bfloat16, (R, dm.d), "x_perm"),
        _ptr(offsets, torch.int32, (dm.N + 1,), "offsets"),
        _ptr(perm_gate, torch.float32, (R,), "perm_gate"), *_fp8_args(dm, fw),
        _ptr(h, torch.bfloat16, (R, dm.I), "h", nullable=bool(dm.flags & FP8_ACTIVATIONS)),
        _ptr(y_perm, torch.bfloat16, (R, dm.d), "y_perm"), w, n, _stream(stream))
    _check("moe_expert_ffn_fp8", rc)


def moe_forward_fp8(dm, x, W_r, b, fw, y, counts, ws, stream=None, events=None):
    w, n = _ws(ws)
    ev = None
    if events is not None:
        assert len(events) == NUM_STAGE_EVENTS
        ev = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    rc = lib().moe_forward_fp8(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(W_r, torch.bfloat16, (dm.N + dm.Z, dm.d), "W_r"),
        _ptr(b, torch.float32, (dm.N + dm.Z,), "b"), *_fp8_args(dm, fw),
        _ptr(y, torch.bfloat16, (dm.T, dm.d), "y"),
        _ptr(counts, torch.int32, (dm.N + dm.Z,), "counts", nullable=True), w, n, ev,
        _stream(stream))
    _check("moe_forward_fp8", rc)


def moe_dense_ffn(dm, x, W_g, W_u, W_d, h, y, ws, stream=None):
    """Dense SwiGLU FFN of all T tokens (dm.T, dm.d, dm.I; W_g, W_u [I, d], W_d [d, I])."""
    w, n = _ws(ws)
    rc = lib().moe_dense_ffn(
        ctypes.byref(dm), _ptr(x, torch.bfloat16, (dm.T, dm.d), "x"),
        _ptr(W_g, torch.bfloat16, (dm.I, dm.d), "W_g"), _ptr(W_u, torch.bfloat16, (dm.I, dm.d), "W_u"),
        _ptr(W_d, torch.bfloat16, (dm.d, dm.I), "W_d"), _ptr(h, torch.bfloat16, (dm.T, dm.I), "h"),
        _ptr(y, torch.bfloat16, (dm.T, dm.d), "y"), w, n, _stream(stream))
    _check("moe_dense_ffn", rc)
