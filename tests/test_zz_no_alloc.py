"""The allocation-free dispatch entry point gives the same results as the regular one.

moe_dispatch_noalloc exists for callers that cannot give this library device memory, such as
a plugin whose host process owns all GPU memory through its own pool, or a deployment whose
memory budget allows no allocation after start-up.  Its scratch lives in a fixed array inside
the library instead of a caller workspace, and that array keeps whatever the previous call
left in it.  This test therefore makes two calls in a row with different routings (the second
call must not see the first call's histogram) and compares every output of each call with
moe_dispatch on the same inputs.  Dispatch outputs are integers and row copies, so the
comparison is exact.  It also checks that requests beyond the fixed capacity are refused.

This file is named so pytest collects it after every other test file.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_38_b200 import binding as mb

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _routing(T, K, E, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([np.sort(rng.choice(E, K, replace=False)) for _ in range(T)]).astype(np.int32)
    gate = rng.random((T, K)).astype(np.float32)
    return torch.from_numpy(idx).to(DEV), torch.from_numpy(gate).to(DEV)


def _outputs(T, K, N, E, d):
    R = T * K
    return dict(
        counts=torch.full((E,), -1, dtype=torch.int32, device=DEV),
        offsets=torch.full((N + 1,), -1, dtype=torch.int32, device=DEV),
        perm_tok=torch.full((R,), -1, dtype=torch.int32, device=DEV),
        perm_gate=torch.zeros((R,), dtype=torch.float32, device=DEV),
        slot_pos=torch.full((T, K), -9, dtype=torch.int32, device=DEV),
        x_perm=torch.zeros((R, d), dtype=torch.bfloat16, device=DEV),
    )


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    T, d, N, Z, K, I = 1000, 256, 64, 32, 6, 128
    E = N + Z
    dm = mb.dims(T, d, N, Z, K, I)
    ws = mb.alloc_workspace(dm, DEV, scratch_only=True)
    x = torch.randn((T, d), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(DEV)
    for call, seed in enumerate((11, 12)):
        idx, gate = _routing(T, K, E, seed)
        want = _outputs(T, K, N, E, d)
        got = _outputs(T, K, N, E, d)
        mb.moe_dispatch(dm, x, idx, gate, want["counts"], want["offsets"], want["perm_tok"],
                        want["perm_gate"], want["slot_pos"], want["x_perm"], ws)
        mb.moe_dispatch_noalloc(dm, x, idx, gate, got["counts"], got["offsets"], got["perm_tok"],
                                got["perm_gate"], got["slot_pos"], got["x_perm"])
        torch.cuda.synchronize()
        for name in want:
            assert torch.equal(got[name], want[name]), (call, name)
        assert int(got["counts"].sum()) == T * K
    assert mb.moe_last_device_error(ws) == 0


def test_noalloc_dispatch_without_the_row_copy():
    # x_perm = NULL skips the gathered copy (the fused-gather up-projection reads x itself),
    # exactly as moe_dispatch does: the tables match and x_perm's memory is not touched.
    T, d, N, Z, K, I = 300, 128, 8, 4, 3, 256
    E = N + Z
    dm = mb.dims(T, d, N, Z, K, I)
    ws = mb.alloc_workspace(dm, DEV, scratch_only=True)
    x = torch.randn((T, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).to(DEV)
    idx, gate = _routing(T, K, E, 13)
    want = _outputs(T, K, N, E, d)
    got = _outputs(T, K, N, E, d)
    got["x_perm"].fill_(3.0)
    mb.moe_dispatch(dm, x, idx, gate, want["counts"], want["offsets"], want["perm_tok"],
                    want["perm_gate"], want["slot_pos"], None, ws)
    mb.moe_dispatch_noalloc(dm, x, idx, gate, got["counts"], got["offsets"], got["perm_tok"],
                            got["perm_gate"], got["slot_pos"], None)
    torch.cuda.synchronize()
    for name in ("counts", "offsets", "perm_tok", "perm_gate", "slot_pos"):
        assert torch.equal(got[name], want[name]), name
    assert (got["x_perm"] == 3.0).all()


def test_noalloc_dispatch_refuses_requests_beyond_its_capacity():
    # ceil(T/256) * (N+Z) must stay within 262144 counters: N+Z = 1024 allows T <= 65536.
    T, d, N, Z, K, I = 70000, 64, 512, 512, 1, 64
    dm = mb.dims(T, d, N, Z, K, I)
    x = torch.zeros((T, d), dtype=torch.bfloat16, device=DEV)
    idx = torch.zeros((T, K), dtype=torch.int32, device=DEV)
    gate = torch.zeros((T, K), dtype=torch.float32, device=DEV)
    out = _outputs(T, K, N, N + Z, d)
    with pytest.raises(mb.MoeError) as e:
        mb.moe_dispatch_noalloc(dm, x, idx, gate, out["counts"], out["offsets"],
                                out["perm_tok"], out["perm_gate"], out["slot_pos"],
                                out["x_perm"])
    assert e.value.code == 4  # MOE_ERR_WORKSPACE: the fixed scratch is too small
