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
FP8 activations (the optional variant that quantises the expert GEMMs' inputs, one scale per
token per 128 channels, read from the same DeepSeek-V3 scheme):
  * a token row worked by hand (tests/golden/fp8_row_worked_example.json);
  * codes against torch's float8_e4m3fn cast, scales against a search over the integers;
  * a row repeated 128 times quantised by the 128 x 128 block rule gives the same scales and
    codes (the two granularities share the rule, not the indexing);
  * the expert restated with torch's fp64 matmuls and float8 casts;
  * zero experts stay exact identities.
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


# ------------------------------------------------------------------ FP8 activations

def _exponent_by_search(amax):
    """The scale rule by direct search: the smallest integer e >= -126 with amax <= 448 * 2^e
    (0 for an all-zero block)."""
    if amax == 0:
        return 0
    e = -126
    while amax > 448.0 * 2.0 ** e:
        e += 1
    return e


def _torch_quant_dequant_rows(v):
    """q * 2^e per 1 x 128 block of each row, with torch's float8_e4m3fn cast doing the
    rounding (v / 2^e is exact; the cast goes through fp32, as v is fp32-exact or the double
    rounding is immaterial at fp64 accuracy)."""
    v = np.asarray(v, np.float64)
    out = np.empty_like(v)
    for r in range(v.shape[0]):
        for cb in range(v.shape[1] // 128):
            blk = v[r, cb * 128:(cb + 1) * 128]
            s = 2.0 ** _exponent_by_search(float(np.abs(blk).max()))
            q = torch.from_numpy(blk / s).to(torch.float32).to(torch.float8_e4m3fn)
            out[r, cb * 128:(cb + 1) * 128] = q.double().numpy() * s
    return out


def test_row_worked_example():
    with open(os.path.join(GOLDEN, "fp8_row_worked_example.json")) as f:
        ex = json.load(f)
    v = np.zeros((1, ex["C"]), np.float64)
    for c, x in ex["entries"]:
        v[0, c] = x
    q, s = oracle.quantize_fp8_rows(v)
    assert s.shape == (1, ex["C"] // 128)
    assert s[0].tolist() == ex["expected_scale"]
    for c, code in ex["expected_codes"]:
        assert q[0, c] == code, (c, q[0, c])
    listed = {c for c, _ in ex["expected_codes"]}
    assert all(q[0, c] == 0 for c in range(ex["C"]) if c not in listed)
    for c, x in ex["expected_dequantized"]:
        got = oracle.e4m3_decode(int(q[0, c])) * float(s[0, c // 128])
        assert got == x and math.copysign(1.0, got) == math.copysign(1.0, x), (c, got, x)


def test_rows_match_torch_float8_and_the_scale_search():
    g = torch.Generator().manual_seed(11)
    R, C = 7, 640
    x = torch.randn((R, C), generator=g)
    # block magnitudes from 2^-20 to 2^20, an all-zero block, a block with one nonzero value
    mags = 2.0 ** torch.randint(-20, 21, (R, C // 128), generator=g).double()
    x = (x.double() * mags.repeat_interleave(128, dim=1)).to(torch.bfloat16)
    x[2, 128:256] = 0
    x[3, 256:384] = 0
    x[3, 300] = -5.5
    v = x.double().numpy()
    q, s = oracle.quantize_fp8_rows(v)
    assert q.shape == (R, C) and s.shape == (R, C // 128)
    for r in range(R):
        for cb in range(C // 128):
            blk = v[r, cb * 128:(cb + 1) * 128]
            sc = 2.0 ** _exponent_by_search(float(np.abs(blk).max()))
            assert float(s[r, cb]) == sc, (r, cb)
            want = torch.from_numpy((blk / sc).astype(np.float32)).to(torch.float8_e4m3fn)
            np.testing.assert_array_equal(q[r, cb * 128:(cb + 1) * 128],
                                          want.view(torch.uint8).numpy())


def test_rows_follow_the_block_rule_on_repeated_rows():
    g = torch.Generator().manual_seed(12)
    row = (torch.randn((1, 384), generator=g) * 0.3).to(torch.bfloat16)
    row[0, 128:256] *= 64
    qr, sr = oracle.quantize_fp8_rows(row.double().numpy())
    qb, sb = oracle.quantize_fp8_blocks(row.repeat(128, 1))
    np.testing.assert_array_equal(sb[0, 0], sr[0])
    for r in range(128):
        np.testing.assert_array_equal(qb[0, r], qr[0])


def _expert_case(seed, R, d, I):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((R, d), generator=g).to(torch.bfloat16)
    W_g = (torch.randn((I, d), generator=g) * 0.05).to(torch.bfloat16)
    W_u = (torch.randn((I, d), generator=g) * 0.05).to(torch.bfloat16)
    W_d = (torch.randn((d, I), generator=g) * 0.05).to(torch.bfloat16)
    return x, W_g, W_u, W_d


def test_expert_fp8act_matches_a_torch_restatement():
    x, W_g, W_u, W_d = _expert_case(13, 6, 256, 384)
    got = oracle.swiglu_expert(x, W_g, W_u, W_d, fp8_act=True)
    xq = torch.from_numpy(_torch_quant_dequant_rows(x.double().numpy()))
    a = xq @ W_g.double().T
    u = xq @ W_u.double().T
    h = a / (1.0 + torch.exp(-a)) * u
    hq = torch.from_numpy(_torch_quant_dequant_rows(h.numpy()))
    want = (hq @ W_d.double().T).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    # and the quantisation is visible: the bf16-activation expert differs by far more
    plain = oracle.swiglu_expert(x, W_g, W_u, W_d)
    assert np.linalg.norm(plain - got) > 1e-3 * np.linalg.norm(plain)


def test_combine_fp8act_zero_experts_stay_identities_and_ffn_slots_use_the_expert():
    x, W_g, W_u, W_d = _expert_case(14, 5, 128, 128)
    N = 2
    Wg = torch.stack([W_g, W_g.flip(0)])
    Wu = torch.stack([W_u, W_u.flip(1)])
    Wd = torch.stack([W_d, -W_d])
    gate = np.array([[0.25, 0.5], [0.125, 0.75], [0.5, 0.25], [1.0, 0.0], [0.3, 0.6]])
    idx_zero = np.array([[2, 3]] * 5, np.int32)
    y = oracle.combine_tokens(np.arange(5), x, idx_zero, gate, Wg, Wu, Wd, N, fp8_act=True)
    xv = x.double().numpy()
    want = np.zeros_like(xv)
    for k in range(2):
        want += gate[:, k:k + 1] * xv
    np.testing.assert_array_equal(y, want)
    idx = np.array([[0, 2], [1, 3], [0, 1], [1, 2], [0, 3]], np.int32)
    y = oracle.combine_tokens(np.arange(5), x, idx, gate, Wg, Wu, Wd, N, fp8_act=True)
    want = np.zeros_like(xv)
    for t in range(5):
        for k in range(2):
            i = idx[t, k]
            term = xv[t] if i >= N else oracle.swiglu_expert(
                x[t:t + 1], Wg[i], Wu[i], Wd[i], fp8_act=True)[0]
            want[t] += gate[t, k] * term
    np.testing.assert_allclose(y, want, rtol=1e-13, atol=1e-15)
