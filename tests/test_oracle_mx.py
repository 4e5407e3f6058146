"""Pins of the oracle's MX (power-of-two scale) FP8 quantisation.

MegaMoE walk-through §2.3 / §5.1: E4M3 activations with one scale per token
per 128 elements and weights with one scale per 128x128 block, the scales
folded into the GEMM.  The MX variant keeps those groups and rounds each
scale up to a power of two, s = 2^p with p the smallest integer such that
448 * 2^p >= amax, so that an 8-bit exponent (UE8M0) carries it and the
tensor core applies it.  Checked against a brute-force search for p, hand
boundary values, the fp32-scale quantiser where the two must agree, and the
FFN's group-wise rule for h.
"""
import numpy as np
import pytest

import oracle
from oracle import fp8


def _brute_p(amax: float) -> int:
    if amax == 0:
        return 0
    p = -140
    while 448.0 * 2.0 ** p < amax:
        p += 1
    return max(-127, min(127, p))


def test_pow2_scale_is_the_smallest_power_of_two_covering_amax():
    rng = np.random.default_rng(0)
    amax = np.concatenate([
        np.float32(rng.lognormal(0, 8, size=3000)),
        np.float32([448.0, 224.0, 896.0, 1.0, 2.0 ** -20 * 448]),
        np.nextafter(np.float32([448.0, 224.0, 896.0]), np.float32(np.inf)),
        np.nextafter(np.float32([448.0, 224.0, 896.0]), np.float32(0)),
    ]).astype(np.float32)
    s = fp8.pow2_scale_of(amax)
    for a, v in zip(amax.tolist(), s.tolist()):
        assert v == 2.0 ** _brute_p(a), (a, v)
        m, _ = np.frexp(v)
        assert m == 0.5  # an exact power of two
        if 2.0 ** -120 < a < 2.0 ** 120:
            assert 448.0 * v >= a > 224.0 * v


def test_pow2_scale_boundaries():
    f = lambda a: float(fp8.pow2_scale_of(np.float32([a]))[0])  # noqa: E731
    assert f(0.0) == 1.0
    assert f(448.0) == 1.0
    assert f(float(np.nextafter(np.float32(448.0), np.float32(1e9)))) == 2.0
    assert f(224.0) == 0.5
    assert f(float(np.nextafter(np.float32(224.0), np.float32(1e9)))) == 1.0
    assert f(1e-40) == 2.0 ** -127     # clamped to the 8-bit exponent range
    assert f(3.0e38) == 2.0 ** 120     # 448 * 2^119 < 3e38 <= 448 * 2^120


def test_pow2_quantisation_equals_the_fp32_scale_one_when_amax_is_448_times_a_power_of_two():
    rng = np.random.default_rng(1)
    a = rng.normal(size=(6, 256)).astype(np.float32)
    for r in range(6):
        for g in range(2):
            blk = a[r, 128 * g:128 * g + 128]
            top = np.float32(448.0 * 2.0 ** (r - 3))
            blk *= np.float32(0.9) * top / np.abs(blk).max()
            blk[int(np.argmax(np.abs(blk)))] = -top if g else top  # amax exactly 448 * 2^(r-3)
    q1, s1 = fp8.quantize_1x128(a)
    q2, s2 = fp8.quantize_1x128(a, pow2=True)
    assert np.array_equal(s1, s2) and np.array_equal(q1, q2)


def test_pow2_codes_stay_within_half_a_step_and_use_the_upper_half_range():
    rng = np.random.default_rng(2)
    a = (rng.normal(size=(16, 384)) * rng.uniform(1e-3, 1e3, size=(16, 1))).astype(np.float32)
    q, s = fp8.quantize_1x128(a, pow2=True)
    v = a.astype(np.float64) / np.repeat(s, 128, axis=1)
    d = fp8.e4m3_decode(q)
    half = np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-9)
    assert np.all(np.abs(d - v) <= half)
    big = np.abs(v).reshape(16, 3, 128).max(axis=2)
    assert np.all((big > 224.0) & (big <= 448.0))
    # and the product of the dequantised operands is the blockwise GEMM with these scales
    W = (rng.normal(size=(128, 384)) * 0.05).astype(np.float32)
    qw, sw = fp8.quantize_128x128(W, pow2=True)
    ref = fp8.dequantize_1x128(q, s) @ fp8.dequantize_128x128(qw, sw).T
    assert np.allclose(fp8.fp8_gemm(q, s, qw, sw), ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_mx_ffn_requantises_h_with_power_of_two_groups():
    rng = np.random.default_rng(3)
    I, d, T = 256, 256, 8
    x = oracle.bf16_round(rng.normal(size=(T, d))).astype(np.float32)
    W1 = (rng.normal(size=(2 * I, d)) * 0.05).astype(np.float32)
    W1[128:256] *= 20.0            # the second group of gate rows is much larger
    W1[I + 128:] *= 20.0
    W2 = (rng.normal(size=(d, I)) * 0.05).astype(np.float32)
    xq, sx = fp8.quantize_1x128(x, pow2=True)
    W1q, s1 = fp8.quantize_128x128(W1, pow2=True)
    W2q, s2 = fp8.quantize_128x128(W2, pow2=True)
    r = fp8.swiglu_ffn_fp8(xq, sx, W1q, s1, W2q, s2, pow2=True)
    h32 = r["h"].astype(np.float32)
    for m in range(T):
        for gi in range(I // 128):
            amax = float(np.abs(h32[m, 128 * gi:128 * gi + 128]).max())
            assert r["sh"][m, gi] == 2.0 ** _brute_p(amax)
    assert np.all(r["sh"][:, 1] > 64 * r["sh"][:, 0])
    want = fp8.e4m3_encode((h32 / np.repeat(r["sh"], 128, axis=1)).astype(np.float32))
    assert np.array_equal(r["hq"], want)
    H = fp8.dequantize_1x128(r["hq"], r["sh"])
    assert np.allclose(r["y"], H @ fp8.dequantize_128x128(W2q, s2).T, rtol=1e-12, atol=1e-14)


def test_mx_forward_identical_experts_closed_form():
    rng = np.random.default_rng(5)
    T, d, E, I = 16, 256, 4, 128
    x = oracle.bf16_round(rng.normal(size=(T, d)))
    Wr = rng.normal(size=(E, d)) * 0.05
    W1 = np.repeat(rng.normal(size=(1, 2 * I, d)) * 0.05, E, axis=0)
    W2 = np.repeat(rng.normal(size=(1, d, I)) * 0.05, E, axis=0)
    r = fp8.moe_forward_fp8(x, Wr, None, W1, W2, k=2, pow2=True)
    psum = np.take_along_axis(r["p"], r["idx"], axis=1).sum(axis=1)
    xq, sx = fp8.quantize_1x128(x.astype(np.float32), pow2=True)
    dense = fp8.swiglu_ffn_fp8(xq, sx, *fp8.quantize_expert(W1[0], W2[0], pow2=True), pow2=True)["y"]
    assert np.allclose(r["out"], psum[:, None] * dense, rtol=1e-12, atol=1e-12)
    ref = oracle.moe_forward(x, Wr, None, W1, W2, k=2)["out"]
    assert np.linalg.norm(r["out"] - ref) / np.linalg.norm(ref) < 1e-1
