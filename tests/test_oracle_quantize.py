"""Pins for the oracle's quantize + pack (asymmetric INT-b, group 128, RTN).

Each check is an independent route to what the format fixes:
  * codes lie in [0, 2^b - 1] and each group fills exactly 4b words;
  * every code is the brute-force nearest grid point (ties to even) of the
    binary32 quotient w / s, and the zero point is the brute-force nearest
    integer to -min / s, clamped (round-to-nearest, the RTN baseline of the
    reddit excerpt);
  * the stored fp16 scale is numpy's own fp16 rounding of the binary32 step
    (max - min) / (2^b - 1) and lies within half an fp16 ulp of the exact step;
  * every element whose code is not clamped reconstructs within s/2;
  * an independent numpy bit-stream unpacker reads the same codes back;
  * b = 8 groups holding the integers 0..255 have s = 1, z = 0, q = w exactly;
  * the gamma^2 law of the pages (gamma = 1.2 -> +44% noise) holds for the
    oracle's asymmetric grid against a symmetric grid.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from pinlib import fp16_bits_to_f64, nearest_int_ties_even_bruteforce, unpack_bitstream

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = [2, 3, 4, 5, 6, 7, 8]


def _f32(bits16):
    return synth.bf16_bits_to_f32(bits16)


@pytest.mark.parametrize("bits", BITS)
def test_shapes_ranges_and_bitstream(bits):
    N, K = 5, 384
    w = synth.weights(N, K, seed=11 + bits)
    packed, scales, zeros, flags = oracle.quantize(w, bits)
    assert flags == 0
    assert packed.shape == (N, K * bits // 32)
    assert packed.shape[1] == (K // 128) * 4 * bits  # 4b words per group
    codes = unpack_bitstream(packed, K, bits)
    assert codes.min() >= 0 and codes.max() <= 2**bits - 1
    assert zeros.max() <= 2**bits - 1
    # the oracle's own reader agrees with the independent unpacker
    for n, k in [(0, 0), (1, 127), (2, 128), (4, K - 1), (3, 200)]:
        assert oracle.code_at(packed, K, bits, n, k) == codes[n, k]


@pytest.mark.parametrize("bits", BITS)
def test_codes_and_zero_are_bruteforce_nearest(bits):
    N, K = 3, 256
    w = synth.weights(N, K, seed=100 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    codes = unpack_bitstream(packed, K, bits)
    wf = _f32(w)
    maxq = 2**bits - 1
    for n in range(N):
        for g in range(K // 128):
            sl = slice(128 * g, 128 * g + 128)
            s = np.float32(fp16_bits_to_f64(scales[n, g:g + 1])[0])
            mn = wf[n, sl].min()
            z = int(zeros[n, g])
            zt = np.float32(-mn) / s
            assert z == nearest_int_ties_even_bruteforce(zt, 0, maxq)
            for k in range(0, 128, 7 if bits > 3 else 3):
                t = np.float32(wf[n, sl][k]) / s  # IEEE binary32 quotient
                want = nearest_int_ties_even_bruteforce(t, -z, maxq - z) + z
                assert codes[n, sl][k] == want


def test_ties_go_to_even():
    # s = 1 exactly (range 0..15 at b=4); values k + 0.5 are exact ties.
    bits = 4
    vals = np.zeros(128)
    vals[0], vals[1] = 0.0, 15.0
    vals[2:16] = np.arange(14) + 0.5
    vals[16:] = 7.0
    w = synth.to_bf16_bits(vals.reshape(1, 128))
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    assert fp16_bits_to_f64(scales[0, 0]) == 1.0 and zeros[0, 0] == 0
    codes = unpack_bitstream(packed, 128, bits)[0]
    for i in range(14):
        t = i + 0.5
        want = i if i % 2 == 0 else i + 1  # the even neighbour
        assert codes[2 + i] == want


def test_zero_point_tie_goes_to_even():
    bits = 4
    vals = np.linspace(-2.5, 12.5, 128)
    vals[0], vals[-1] = -2.5, 12.5  # s = 15/15 = 1, -min/s = 2.5 -> 2
    w = synth.to_bf16_bits(vals.reshape(1, 128))
    _, scales, zeros, _ = oracle.quantize(w, bits)
    assert fp16_bits_to_f64(scales[0, 0]) == 1.0
    assert zeros[0, 0] == 2


@pytest.mark.parametrize("bits", BITS)
def test_scale_is_fp16_of_binary32_step(bits):
    N, K = 4, 512
    w = synth.weights(N, K, seed=200 + bits)
    _, scales, _, _ = oracle.quantize(w, bits)
    wf = _f32(w).reshape(N, K // 128, 128)
    mn, mx = wf.min(axis=2), wf.max(axis=2)
    step32 = (mx - mn).astype(np.float32) / np.float32(2**bits - 1)
    assert np.array_equal(scales, step32.astype(np.float16).view(np.uint16))
    exact = (mx.astype(np.float64) - mn.astype(np.float64)) / (2**bits - 1)
    s = fp16_bits_to_f64(scales)
    ulp = np.spacing(s.astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(s - exact) <= 0.5 * ulp * (1 + 1e-6) + 1e-12)


@pytest.mark.parametrize("bits", BITS)
def test_in_range_elements_reconstruct_within_half_step(bits):
    N, K = 8, 1024
    w = synth.weights(N, K, seed=300 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    codes = unpack_bitstream(packed, K, bits)
    wf = _f32(w).astype(np.float64)
    s = np.repeat(fp16_bits_to_f64(scales), 128, axis=1)
    z = np.repeat(zeros.astype(np.int64), 128, axis=1)
    maxq = 2**bits - 1
    t = (wf / s)
    unclamped = (np.rint(t) + z >= 0) & (np.rint(t) + z <= maxq)
    err = np.abs(wf - s * (codes - z))
    bound = s / 2 + np.abs(wf) * 2.0**-23
    assert np.all(err[unclamped] <= bound[unclamped])
    # clamping only happens at the two ends of the grid
    assert np.all((codes[~unclamped] == 0) | (codes[~unclamped] == maxq))
    # and the clamped ones are still within one step of their value
    assert np.all(err <= 1.5 * s + np.abs(wf) * 2.0**-23)


def test_degenerate_groups():
    bits = 4
    K = 128 * 5
    vals = np.zeros((1, K))
    vals[0, 128:256] = 0.75        # constant positive group
    vals[0, 256:384] = -3.0        # constant negative group
    vals[0, 384:512] = np.linspace(1.0, 2.0, 128)   # min > 0
    vals[0, 512:640] = np.linspace(-2.0, -1.0, 128)  # max < 0
    w = synth.to_bf16_bits(vals)
    packed, scales, zeros, flags = oracle.quantize(w, bits)
    assert flags == 0
    codes = unpack_bitstream(packed, K, bits)[0]
    s = fp16_bits_to_f64(scales[0])
    # all zeros: scale 1.0, zero 0, codes 0
    assert s[0] == 1.0 and zeros[0, 0] == 0 and np.all(codes[:128] == 0)
    # constant groups reconstruct to themselves within one fp16 rounding step
    rec1 = s[1] * (codes[128:256] - zeros[0, 1])
    assert np.allclose(rec1, 0.75, rtol=2**-10)
    rec2 = s[2] * (codes[256:384] - zeros[0, 2])
    assert np.allclose(rec2, -3.0, rtol=2**-10)
    # min > 0: zero clamps to 0; max < 0: zero clamps to 2^b - 1
    assert zeros[0, 3] == 0
    assert zeros[0, 4] == 15


def test_b8_integer_groups_are_exact():
    bits = 8
    ints = np.tile(np.arange(256, dtype=np.float64), 2).reshape(2, 256)
    rng = np.random.default_rng(5)
    for r in range(2):
        for g in range(2):
            seg = ints[r, 128 * g:128 * g + 128]
            perm = rng.permutation(128)
            seg[:] = seg[perm]
    # make every group span exactly 0..255
    ints[:, 0], ints[:, 1], ints[:, 128], ints[:, 129] = 0, 255, 0, 255
    w = synth.to_bf16_bits(ints)
    assert np.array_equal(synth.bf16_bits_to_f32(w), ints.astype(np.float32))
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    assert np.all(fp16_bits_to_f64(scales) == 1.0) and np.all(zeros == 0)
    assert np.array_equal(unpack_bitstream(packed, 256, bits), ints.astype(np.int64))


def test_flags_nonfinite_and_scale_overflow():
    K = 256
    vals = np.zeros((1, K))
    vals[0, :128] = np.linspace(-1, 1, 128)
    vals[0, 5] = np.inf
    w = synth.to_bf16_bits(vals)
    _, _, _, flags = oracle.quantize(w, 4)
    assert flags & oracle.FLAG_NONFINITE
    vals = np.zeros((1, K))
    vals[0, :128] = np.linspace(-3e38, 3e38, 128)
    _, scales, _, flags = oracle.quantize(synth.to_bf16_bits(vals), 4)
    assert flags & oracle.FLAG_SCALE_OVERFLOW and not flags & oracle.FLAG_NONFINITE
    assert scales[0, 0] == 0x7BFF
    vals = np.zeros((1, K))
    vals[0, :128] = np.linspace(0, 1e-12, 128)  # step far below fp16 range
    _, scales, _, flags = oracle.quantize(synth.to_bf16_bits(vals), 4)
    assert flags == 0 and scales[0, 0] == 0x0001


def _symmetric_mse(w, bits):
    """Symmetric RTN grid -M + i * 2M/(2^b - 1), computed here independently."""
    M = np.abs(w).max(axis=1, keepdims=True)
    step = 2 * M / (2**bits - 1)
    i = np.clip(np.rint((w + M) / step), 0, 2**bits - 1)
    return ((w - (-M + i * step)) ** 2).mean(axis=1)


def _asym_mse_oracle(w, bits):
    wb = synth.to_bf16_bits(w)
    wf = synth.bf16_bits_to_f32(wb).astype(np.float64)
    packed, scales, zeros, _ = oracle.quantize(wb.reshape(1, -1), bits)
    rec = oracle.dequantize(packed, scales, zeros, wb.size, bits).reshape(w.shape)
    return wf, ((wf - rec) ** 2).mean(axis=1)


@pytest.mark.parametrize("bits", [4, 5])
def test_gamma_squared_law(bits):
    """Symmetric/asymmetric noise-variance ratio = gamma^2 within 5 percent."""
    rng = np.random.default_rng(17 + bits)
    for gamma in [1.0, 1.2, 1.5, 2.0]:
        R = np.exp(rng.uniform(np.log(0.01), np.log(0.1), size=(400, 1)))
        c = (gamma - 1.0) * R / 2  # centre offset so that 2 max|w| / R = gamma
        w = c + R * (rng.random((400, 128)) - 0.5)
        wf, mse_a = _asym_mse_oracle(w, bits)
        g = 2 * np.abs(wf).max(axis=1) / (wf.max(axis=1) - wf.min(axis=1))
        mse_s = _symmetric_mse(wf, bits)
        ratio = mse_s.sum() / (g**2 * mse_a).sum()
        assert abs(ratio - 1.0) < 0.05, (gamma, ratio)


def test_gamma_law_worked_example_from_the_pages():
    with open(os.path.join(GOLDEN, "gamma_law.json")) as f:
        gold = json.load(f)
    gamma, want = gold["gamma"], gold["noise_variance_ratio"]
    rng = np.random.default_rng(3)
    R = np.exp(rng.uniform(np.log(0.01), np.log(0.1), size=(600, 1)))
    w = (gamma - 1.0) * R / 2 + R * (rng.random((600, 128)) - 0.5)
    ratios = []
    for bits in (4, 5):
        wf, mse_a = _asym_mse_oracle(w, bits)
        ratios.append(_symmetric_mse(wf, bits).sum() / mse_a.sum())
    for r in ratios:
        assert abs(r / want - 1.0) < 0.05, ratios
