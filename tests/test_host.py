"""Host-side tests (no GPU): the C-ABI library loads and exports every entry point the header
declares, argument errors return the documented codes before any CUDA call, the
multi-process replica timing of bench.py reduces to the maximum over ranks (gloo, 2 ranks), and
the benchmark's algorithmic work model and GEMM source hash behave as its roofline needs.
"""
import ctypes
import os
import re

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_38_b200 import binding as mb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, re.M)))


def test_library_exports_every_declared_entry_point():
    names = header_functions()
    assert "moe_forward" in names and "moe_route" in names and len(names) >= 10
    lib = mb.lib()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(mb.EXPORTS) == names


def test_strerror_and_sizes():
    for code in range(8):
        assert mb.strerror(code)
    assert "unknown" in mb.strerror(99)
    dm = mb.dims(16384, 6144, 512, 256, 12, 2048)
    ws = mb.workspace_size(dm)
    rows = 16384 * 12
    assert ws >= rows * (2 * 6144 + 2048) * 2
    assert ws < rows * (2 * 6144 + 2048) * 2 * 1.02 + 64e6
    assert 0 < mb.scratch_size(dm) < ws
    # invalid dims give 0
    for bad in [(64, 100, 8, 4, 3, 256), (64, 128, 8, 4, 0, 256), (64, 128, 8, 4, 13, 256),
                (64, 128, 800, 300, 3, 256), (-1, 128, 8, 4, 3, 256), (64, 128, 8, 4, 33, 256),
                (64, 128, 0, 0, 1, 256), (64, 128, 8, 4, 3, 96)]:
        assert mb.workspace_size(mb.dims(*bad)) == 0, bad


P = ctypes.c_void_p


def _fwd(dm, x=0x10000, W_r=0x20000, b=0x30000, W_g=0x40000, W_u=0x50000, W_d=0x60000,
         y=0x70000, counts=None, ws=0x100000, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = mb.workspace_size(dm)
    return mb.lib().moe_forward(ctypes.byref(dm), P(x), P(W_r), P(b), P(W_g), P(W_u), P(W_d),
                                P(y), P(counts), P(ws), ws_bytes, None)


def test_argument_errors_are_reported_before_any_device_work():
    dm = mb.dims(64, 128, 8, 4, 3, 256)
    assert _fwd(mb.dims(64, 100, 8, 4, 3, 256)) == 2          # MOE_ERR_SHAPE
    assert mb.lib().moe_forward(None, P(1), P(1), P(1), P(1), P(1), P(1), P(1), None, P(1), 0,
                                None) == 1                     # NULL dims
    assert _fwd(dm, x=0) == 1                                  # NULL tensor: MOE_ERR_ARG
    assert _fwd(dm, W_g=0x40008) == 3                          # misaligned: MOE_ERR_ALIGN
    assert _fwd(dm, ws=0x100010) == 3                          # workspace not 256-aligned
    assert _fwd(dm, ws_bytes=mb.workspace_size(dm) - 1) == 4   # MOE_ERR_WORKSPACE
    assert _fwd(dm, counts=0x90004) == 3
    # Everything valid: the first CUDA call happens and fails on a machine without a GPU.
    if not torch.cuda.is_available():
        assert _fwd(dm) == 5                                   # MOE_ERR_CUDA
        # An empty batch accepts NULL token buffers (validation passes, then the CUDA call).
        assert _fwd(mb.dims(0, 128, 8, 4, 3, 256), x=0, y=0) == 5
    lib = mb.lib()
    assert lib.moe_route(ctypes.byref(dm), P(0x10000), P(0x20000), P(0x30000), P(0x40000),
                         P(0x50000), P(0x60008), P(0x100000), mb.scratch_size(dm), None) == 3
    assert lib.moe_dispatch(ctypes.byref(dm), *[P(0x10000)] * 9, P(0x100000),
                            mb.scratch_size(dm) - 256, None) == 4
    params = mb.PidParams(8.0, 0.1, 0.0, 0.0)
    assert lib.moe_bias_update(ctypes.byref(dm), P(0x10000), P(0x20000), P(0x30000), None,
                               None) == 1
    assert lib.moe_bias_update(ctypes.byref(dm), P(0x10000), P(0), P(0x30000),
                               ctypes.byref(params), None) == 1
    assert lib.moe_last_device_error(None, None) == 1


def test_combine_logits_and_wait_limit_argument_errors():
    lib = mb.lib()
    dm = mb.dims(64, 128, 8, 4, 3, 256)
    bufs = [P(0x10000 * (i + 1)) for i in range(6)]  # x, y_perm, topk_idx, topk_gate, slot_pos, y
    assert lib.moe_combine(ctypes.byref(dm), *bufs, None, 256, None) == 1        # no workspace
    assert lib.moe_combine(ctypes.byref(dm), *bufs, P(0x100000), 255, None) == 4  # < status word
    assert lib.moe_combine(ctypes.byref(dm), *bufs, P(0x100010), 256, None) == 3  # misaligned
    assert lib.moe_combine(ctypes.byref(mb.dims(64, 100, 8, 4, 3, 256)), *bufs, P(0x100000), 256,
                           None) == 2
    assert lib.moe_router_logits(ctypes.byref(dm), P(0x100000), mb.scratch_size(dm), P(0),
                                 None) == 1                                     # NULL logits
    assert lib.moe_router_logits(ctypes.byref(dm), P(0x100000), mb.scratch_size(dm) - 1,
                                 P(0x10000), None) == 4
    assert lib.moe_router_logits(ctypes.byref(dm), P(0x100000), mb.scratch_size(dm),
                                 P(0x10008), None) == 3
    assert lib.moe_debug_set_wait_limit(-1) == 1
    assert lib.moe_debug_set_wait_limit(0) == 0


def test_fp8_shape_errors_before_device_work():
    lib = mb.lib()
    # R or C not a multiple of 128
    assert lib.moe_quantize_fp8(P(0x10000), 1, 100, 128, P(0x20000), P(0x30000), None) == 2
    assert lib.moe_quantize_fp8(P(0x10000), 1, 128, 192, P(0x20000), P(0x30000), None) == 2
    assert lib.moe_quantize_fp8(None, 0, 128, 128, None, None, None) == 0  # nothing to do
    assert lib.moe_quantize_fp8(P(0x10000), 1 << 40, 1 << 30, 128, P(0x20000), P(0x30000),
                                None) == 2  # too many blocks (and no overflow in the check)
    # d = 192 is a valid bf16 width but not a whole number of 128-wide scale blocks
    dm = mb.dims(64, 192, 8, 4, 3, 256)
    args = [P(0x10000 * (i + 1)) for i in range(10)]  # x, W_r, b, 6 FP8 tensors, y
    assert lib.moe_forward_fp8(ctypes.byref(dm), *args, None, P(0x1000000),
                               mb.workspace_size(dm), None, None) == 2
    dm2 = mb.dims(64, 128, 8, 4, 3, 256)
    args[3] = P(0)  # NULL codes
    assert lib.moe_forward_fp8(ctypes.byref(dm2), *args, None, P(0x1000000),
                               mb.workspace_size(dm2), None, None) == 1


def test_fp8_activation_flag_layout_and_errors():
    lib = mb.lib()
    T, d, N, Z, K, I = 64, 256, 8, 4, 3, 384
    plain = mb.dims(T, d, N, Z, K, I)
    dm = mb.dims(T, d, N, Z, K, I, flags=mb.FP8_ACTIVATIONS)
    # the scratch grows by the codes and block scales of x_perm and h (256-byte aligned regions)
    rows = T * K
    extra = sum(-(-b // 256) * 256 for b in (rows * d, rows * d // 128 * 4, rows * I,
                                             rows * I // 128 * 4))
    assert mb.scratch_size(dm) == mb.scratch_size(plain) + extra
    assert mb.workspace_size(dm) == mb.workspace_size(plain) + extra
    # widths that are not whole 128-channel blocks are rejected with the flag only
    assert mb.workspace_size(mb.dims(T, 192, N, Z, K, I)) > 0
    assert mb.workspace_size(mb.dims(T, 192, N, Z, K, I, flags=mb.FP8_ACTIVATIONS)) == 0
    assert mb.workspace_size(mb.dims(T, d, N, Z, K, 320, flags=mb.FP8_ACTIVATIONS)) == 0
    # the bf16 entry points refuse the flag (MOE_ERR_ARG), before any device work
    assert _fwd(dm) == 1
    assert lib.moe_expert_ffn(ctypes.byref(dm), *[P(0x10000 * (i + 1)) for i in range(8)],
                              P(0x1000000), mb.scratch_size(dm), None) == 1
    # the FP8 stage call takes h = NULL with the flag, and needs the larger scratch
    args = [P(0x10000 * (i + 1)) for i in range(9)]  # x_perm, offsets, perm_gate, 6 FP8 tensors
    assert lib.moe_expert_ffn_fp8(ctypes.byref(dm), *args, None, P(0x200000), P(0x1000000),
                                  mb.scratch_size(dm) - 256, None) == 4
    assert lib.moe_expert_ffn_fp8(ctypes.byref(plain), *args, None, P(0x200000), P(0x1000000),
                                  mb.scratch_size(plain), None) == 1  # h required without it
    # the row quantiser's shape checks
    assert lib.moe_quantize_fp8_rows(P(0x10000), 4, 192, P(0x20000), P(0x30000), None) == 2
    assert lib.moe_quantize_fp8_rows(P(0x10000), -1, 128, P(0x20000), P(0x30000), None) == 2
    assert lib.moe_quantize_fp8_rows(None, 0, 128, None, None, None) == 0  # nothing to do
    assert lib.moe_quantize_fp8_rows(P(0x10000), 1 << 40, 1 << 20, P(0x20000), P(0x30000),
                                     None) == 2  # too many warps for one grid
    assert lib.moe_quantize_fp8_rows(P(0x10008), 4, 128, P(0x20000), P(0x30000), None) == 3


def test_fused_combine_flag_layout_and_errors():
    lib = mb.lib()
    T, d, N, Z, K, I = 64, 320, 8, 4, 3, 256
    plain = mb.dims(T, d, N, Z, K, I)
    dm = mb.dims(T, d, N, Z, K, I, flags=mb.FUSED_COMBINE)
    # counters: 4 feature blocks per 256-feature m-tile of the down projection, per token
    blocks = 4 * -(-d // 256)
    assert mb.workspace_size(dm) == mb.workspace_size(plain) + -(-(T * blocks * 4) // 256) * 256
    assert mb.scratch_size(dm) == mb.scratch_size(plain)
    # every entry point other than moe_forward(_timed) refuses it (MOE_ERR_ARG) before device work
    ws = mb.workspace_size(dm)
    assert lib.moe_expert_ffn(ctypes.byref(dm), *[P(0x10000 * (i + 1)) for i in range(8)],
                              P(0x1000000), ws, None) == 1
    assert lib.moe_expert_ffn_gather(ctypes.byref(dm), *[P(0x10000 * (i + 1)) for i in range(9)],
                                     P(0x1000000), ws, None) == 1
    fp8 = mb.dims(T, 384, N, Z, K, I, flags=mb.FUSED_COMBINE)
    args = [P(0x10000 * (i + 1)) for i in range(10)]
    assert lib.moe_forward_fp8(ctypes.byref(fp8), *args, None, P(0x1000000),
                               mb.workspace_size(fp8), None, None) == 1
    assert lib.moe_expert_ffn_fp8(ctypes.byref(fp8), *args[:9], P(0x200000), P(0x200000),
                                  P(0x1000000), mb.scratch_size(fp8), None) == 1
    # moe_forward takes it, and checks the larger workspace
    assert _fwd(dm, ws_bytes=mb.workspace_size(plain)) == 4


def test_dense_ffn_argument_errors():
    lib = mb.lib()
    for bad in [(64, 100, 1, 0, 1, 256), (64, 128, 1, 0, 1, 96), (-1, 128, 1, 0, 1, 256)]:
        dm = mb.dims(*bad)
        assert lib.moe_dense_ffn(ctypes.byref(dm), *[P(0x10000)] * 6, P(0x100000), 256,
                                 None) == 2
    dm = mb.dims(64, 128, 1, 0, 1, 256)
    assert lib.moe_dense_ffn(ctypes.byref(dm), P(0x10000), P(0), P(0x10000), P(0x10000),
                             P(0x10000), P(0x10000), P(0x100000), 256, None) == 1
    assert lib.moe_dense_ffn(ctypes.byref(dm), *[P(0x10000)] * 6, P(0x100000), 128,
                             None) == 4  # workspace smaller than its 256-byte status region


def test_variant_switches_are_validated():
    lib = mb.lib()
    dm = mb.dims(64, 128, 8, 4, 3, 256, flags=mb.RENORMALIZE_GATES)
    assert mb.workspace_size(dm) == mb.workspace_size(mb.dims(64, 128, 8, 4, 3, 256))
    assert mb.workspace_size(mb.dims(64, 128, 8, 4, 3, 256, flags=8)) == 0  # unknown flag
    assert _fwd(mb.dims(64, 128, 8, 4, 3, 256, flags=0x80)) == 2            # MOE_ERR_SHAPE
    for gamma in (float("nan"), float("inf")):
        params = mb.PidParams(8.0, 0.1, 0.0, 0.0, gamma)
        assert lib.moe_bias_update(ctypes.byref(dm), P(0x10000), P(0x20000), P(0x30000),
                                   ctypes.byref(params), None) == 1          # MOE_ERR_ARG
    assert ctypes.sizeof(mb.Dims) == 28 and ctypes.sizeof(mb.PidParams) == 20


def _replica_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [12.5, 17.25][rank]
    m = bench.max_over_ranks(ms, world)
    tput = bench.job_throughput(world, 16384, 10, m)
    out.put((rank, m, tput))
    dist.barrier()
    dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_replica_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, tput in res:
        assert m == 17.25
        assert tput == pytest.approx(2 * 16384 * 10 / 0.01725)


def _bench():
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    return bench


def test_work_model_per_unit_figures():
    # The roofline's algorithmic work, on a routing small enough to count by hand: T = 4 tokens,
    # d = 8, I = 16, N = 3 FFN experts + Z = 1 zero expert, K = 2; counts 3, 0, 2 on the FFN
    # experts (A = 5 slots, U = 2 experts used) and 3 on the zero expert.
    from mixture_experts_layer_38_b200.workloads import Workload
    w = Workload("hand", T=4, d=8, N=3, Z=1, K=2, I=16)
    A, U, flops, nbytes = _bench().work_model(w, [3, 0, 2, 3])
    assert (A, U) == (5, 2)
    assert flops == {"router_gemm": 256, "ffn_up_gemm": 2560, "ffn_down_gemm": 1280}
    assert nbytes == {"router_gemm": 192, "ffn_up_gemm": 1264, "ffn_down_gemm": 752,
                      "dispatch": 144, "combine": 208}
    _, _, _, nbytes8 = _bench().work_model(w, [3, 0, 2, 3], wb=1)  # E4M3 weight codes
    assert nbytes8["ffn_up_gemm"] == 512 + 80 + 160 and nbytes8["ffn_down_gemm"] == 256 + 240
    # FP8 activations: one byte per x_perm and h element in the GEMMs, plus the up stage's row
    # quantiser (2 bytes read + 1 written per element of the A x d token rows); y_perm stays bf16
    _, _, flops8a, nbytes8a = _bench().work_model(w, [3, 0, 2, 3], wb=1, ab=1)
    assert flops8a == flops
    assert nbytes8a["ffn_up_gemm"] == 512 + 40 + 80 + 120
    assert nbytes8a["ffn_down_gemm"] == 256 + 80 + 80


def test_gemm_source_hash_ignores_comments_only():
    # The recorded DRAM traffic is reported only while the GEMM sources hash to the captured
    # version: comment edits must keep the hash, any code edit must change it.
    bench = _bench()

    def real(path):
        with open(os.path.join(ROOT, path), encoding="utf-8") as f:
            return f.read()
    h0 = bench.gemm_source_hash()
    assert bench.gemm_source_hash(real) == h0
    assert bench.gemm_source_hash(lambda p: real(p) + "\n// note\n/* block\n note */\n") == h0
    assert bench.gemm_source_hash(
        lambda p: real(p).replace("constexpr int kBK = 64;", "constexpr int kBK = 32;")) != h0
