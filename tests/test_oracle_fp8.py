"""Pins for the oracle's FP8 (E4M3) block quantisation of expert weights.

Page cited: "衝上熱搜！美團大模型，靠「快」火了", section 系統級優化 (fine-grained block-wise
quantisation as in DeepSeek-V3: one scale per 128 x 128 weight block).  Pins used:
  * torch's float8_e4m3fn dtype (a library routine) for the value of every code and for
    round-to-nearest-even encoding inside the finite range;
  * brute force: the encoder's code is the nearest of all 254 finite codes (ties to the even
    mantissa), and saturation at +-448 past the range;
  * a block worked by hand (tests/golden/fp8_block_worked_example.json);
  * invariants: scales are powers of two and minimal, dequantised weights are exact in bf16,
    the error is within half an E4M3 step of each weight.
"""
import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_decode_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        v = oracle.e4m3_decode(c)
        assert (math.isnan(v) and math.isnan(ref[c])) or v == ref[c], c


def _nearest_code(v):
    """Brute force: nearest finite code, ties to the code with an even mantissa (LSB 0)."""
    best, bd = None, None
    for c in FINITE:
        d = abs(oracle.e4m3_decode(c) - v)
        if bd is None or d < bd or (d == bd and (c & 1) == 0 and (best & 1) == 1):
            best, bd = c, d
    if v == 0 and math.copysign(1.0, v) < 0:
        return 0x80
    return best


def test_encode_is_nearest_code_brute_force():
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(300) * 30) + list(rng.uniform(-1e-3, 1e-3, 100))
    # every midpoint between adjacent positive codes (exact ties) and its neighbours
    pos = sorted(oracle.e4m3_decode(c) for c in FINITE if c < 0x80)
    for a, b in zip(pos, pos[1:]):
        m = (a + b) / 2
        vals += [m, -m, np.nextafter(m, 0), np.nextafter(m, 1e9)]
    for v in vals:
        got = oracle.e4m3_encode(v)
        want = _nearest_code(v)
        assert oracle.e4m3_decode(got) == oracle.e4m3_decode(want), (v, got, want)


def test_encode_matches_torch_in_range_and_saturates_beyond():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(2000) * 50, rng.uniform(-463.9, 463.9, 2000)])
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(np.float32(x))) for x in v], np.uint8)
    np.testing.assert_array_equal(ours, t)
    for big in (464.0, 500.0, 1e30, float("inf")):
        assert oracle.e4m3_encode(big) == 0x7E and oracle.e4m3_encode(-big) == 0xFE
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def test_block_worked_example():
    with open(os.path.join(GOLDEN, "fp8_block_worked_example.json")) as f:
        ex = json.load(f)
    w = np.zeros((128, 128), np.float32)
    for r, c, v in ex["entries"]:
        w[r, c] = v
    q, s = oracle.quantize_fp8_blocks(torch.from_numpy(w).to(torch.bfloat16))
    assert s.shape == (1, 1, 1) and s[0, 0, 0] == ex["expected_scale"]
    for r, c, code in ex["expected_codes"]:
        assert q[0, r, c] == code, (r, c, q[0, r, c])
    deq = oracle.bf16_to_f64(oracle.dequantize_fp8_blocks(q, s))
    for r, c, v in ex["expected_dequantized"]:
        assert deq[0, r, c] == v
    assert np.count_nonzero(q[0]) == 4


def test_block_invariants_on_random_weights():
    g = torch.Generator().manual_seed(5)
    w = (torch.randn((2, 256, 384), generator=g) * 0.02).to(torch.bfloat16)
    w[1, 128:, :128] = 0  # an all-zero block
    w[0, :128, 128:256] *= 1000  # a block with a much larger range
    q, s = oracle.quantize_fp8_blocks(w)
    assert q.shape == (2, 256, 384) and s.shape == (2, 2, 3)
    wf = w.double().numpy()
    deq = oracle.bf16_to_f64(oracle.dequantize_fp8_blocks(q, s))
    for gi in range(2):
        for rb in range(2):
            for cb in range(3):
                blk = wf[gi, rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]
                sc = float(s[gi, rb, cb])
                e = math.frexp(sc)[1] - 1
                assert sc == 2.0 ** e  # a power of two
                amax = np.abs(blk).max()
                if amax == 0:
                    assert sc == 1.0
                    continue
                assert amax <= 448 * sc and amax > 448 * sc / 2  # the smallest such power
                d = deq[gi, rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]
                # half an E4M3 step: 2^-4 relative in the normal range, 2^-10 * sc below it
                tol = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * sc)
                assert (np.abs(d - blk) <= tol).all()
    # dequantised values are exact in bf16: re-rounding changes nothing
    deq_bits = oracle.dequantize_fp8_blocks(q, s)
    again = torch.from_numpy(oracle.bf16_to_f64(deq_bits)).to(torch.bfloat16)
    assert (oracle.bf16_bits(again) == deq_bits).all()
