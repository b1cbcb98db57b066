"""Pins for the oracle's dequantize and weight-only GEMM.

  * one-hot rows of X pick out single dequantized weights, which must equal
    an independent dequantization (numpy bit stream + numpy fp16 decode);
  * random X against numpy's matmul of that independent dequantization;
  * b = 8 with s = 1, z = 0 reduces to an exact integer matmul;
  * sampled rows equal the corresponding rows of the full product.
"""
import numpy as np
import pytest

import oracle
import synth
from pinlib import dequant_independent


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_dequantize_matches_independent_reader(bits):
    N, K = 6, 384
    w = synth.weights(N, K, seed=400 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    ours = oracle.dequantize(packed, scales, zeros, K, bits)
    ref = dequant_independent(packed, scales, zeros, K, bits)
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_one_hot_rows_select_weights(bits):
    N, K = 9, 256
    w = synth.weights(N, K, seed=500 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    ks = np.array([0, 1, 77, 127, 128, 200, 255])
    x = np.zeros((len(ks), K))
    x[np.arange(len(ks)), ks] = 1.0
    y = oracle.gemm(synth.to_bf16_bits(x), packed, scales, zeros, K, bits)
    ref = dequant_independent(packed, scales, zeros, K, bits)
    assert np.array_equal(y, ref[:, ks].T)


@pytest.mark.parametrize("bits", [2, 5, 7])
def test_random_x_matches_numpy_matmul(bits):
    M, N, K = 7, 33, 512
    w = synth.weights(N, K, seed=600 + bits)
    x = synth.activations(M, K, seed=601)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    y = oracle.gemm(x, packed, scales, zeros, K, bits)
    xd = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = xd @ dequant_independent(packed, scales, zeros, K, bits).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_b8_unit_scale_is_integer_matmul():
    rng = np.random.default_rng(9)
    N, K, M = 4, 256, 3
    ints = rng.integers(0, 256, size=(N, K)).astype(np.float64)
    ints[:, 0], ints[:, 1], ints[:, 128], ints[:, 129] = 0, 255, 0, 255
    packed, scales, zeros, _ = oracle.quantize(synth.to_bf16_bits(ints), 8)
    xi = rng.integers(-8, 9, size=(M, K)).astype(np.float64)
    y = oracle.gemm(synth.to_bf16_bits(xi), packed, scales, zeros, K, 8)
    assert np.array_equal(y, (xi.astype(np.int64) @ ints.astype(np.int64).T).astype(np.float64))


def test_sampled_rows_equal_full_rows():
    M, N, K, bits = 12, 20, 256, 4
    w = synth.weights(N, K, seed=700)
    x = synth.activations(M, K, seed=701)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    full = oracle.gemm(x, packed, scales, zeros, K, bits)
    rows = np.array([11, 0, 5])
    part = oracle.gemm(x, packed, scales, zeros, K, bits, rows=rows)
    assert np.array_equal(part, full[rows])


# ---------------------------------------------------------------------------
# bf16 fake-quantized weights (the exported checkpoint's form)
# ---------------------------------------------------------------------------
def _bf16_nearest_brute(v):
    """Nearest bf16 to each binary64 value by comparing the two bf16 numbers
    that bracket it (ties to the even significand)."""
    out = np.empty(v.shape, dtype=np.uint16)
    for i, x in enumerate(v.ravel()):
        f = np.float32(x)
        t = int(np.array([f]).view(np.uint32)[0]) >> 16  # truncated toward zero
        cands = [t, t + 1]
        vals = [float(np.array([c << 16], dtype=np.uint32).view(np.float32)[0]) for c in cands]
        d = [abs(val - x) for val in vals]
        if d[0] < d[1] or (d[0] == d[1] and cands[0] % 2 == 0):
            out.ravel()[i] = cands[0]
        else:
            out.ravel()[i] = cands[1]
    return out


def test_bf16_rn_matches_brute_force_and_ties():
    rng = np.random.default_rng(11)
    v = (rng.standard_normal(3000) * 2.0 ** rng.integers(-20, 20, 3000)).astype(np.float32).astype(np.float64)
    assert np.array_equal(oracle.bf16_rn(v), _bf16_nearest_brute(v))
    # Ties: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7 -> even (1.0);
    # 1 + 3 * 2^-8 halfway between 1 + 2^-7 and 1 + 2^-6 -> even (1 + 2^-6).
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])
    assert list(oracle.bf16_rn(ties)) == [0x3F80, 0x3F82, 0xBF80]
    # Values already in bf16 are unchanged.
    exact = np.array([0.0, 1.0, -2.5, 2.0 ** -130, 3.0 * 2.0 ** 100])
    back = (oracle.bf16_rn(exact).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(back, exact)


@pytest.mark.parametrize("bits", [2, 4, 5, 8])
def test_fake_quant_rounds_each_dequantized_weight(bits):
    N, K = 7, 384
    w = synth.weights(N, K, seed=610 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    fq = oracle.fake_quant_bf16(packed, scales, zeros, K, bits)
    exact = dequant_independent(packed, scales, zeros, K, bits)
    assert np.array_equal(fq, _bf16_nearest_brute(exact))
    # Within half a bf16 ulp of the exact weight: the unit roundoff of an
    # 8-bit significand is 2^-8.
    back = (fq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(back - exact) <= 2.0 ** -8 * np.abs(exact))


def test_fake_quant_is_exact_for_power_of_two_scales():
    # s = 2^e makes every s (q - z) a bf16 number: no rounding at all.
    N, K, bits = 4, 256, 8
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 256, size=(N, K))
    packed = np.zeros((N, K * bits // 32), dtype=np.uint32)
    for n in range(N):
        for k in range(K):
            packed[n, k // 4] |= np.uint32(int(codes[n, k]) << (8 * (k % 4)))
    scales = np.full((N, K // 128), 0x2C00, dtype=np.uint16)  # fp16 2^-4
    zeros = rng.integers(0, 256, size=(N, K // 128)).astype(np.uint8)
    fq = oracle.fake_quant_bf16(packed, scales, zeros, K, bits)
    back = (fq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = (codes - np.repeat(zeros.astype(np.int64), 128, axis=1)) * 2.0 ** -4
    assert np.array_equal(back, ref)


@pytest.mark.parametrize("bits", [3, 6])
def test_gemm_fake_quant_one_hot_and_error_bound(bits):
    N, K = 11, 512
    w = synth.weights(N, K, seed=620 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    ks = np.array([0, 5, 127, 128, 300, 511])
    x1 = np.zeros((len(ks), K))
    x1[np.arange(len(ks)), ks] = 1.0
    y1 = oracle.gemm_fake_quant(synth.to_bf16_bits(x1), packed, scales, zeros, K, bits)
    fq = oracle.fake_quant_bf16(packed, scales, zeros, K, bits)
    back = (fq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(y1, back[:, ks].T)
    # Against the exact product: each weight moves by at most 2^-8 of itself.
    x = synth.activations(5, K, seed=621)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y = oracle.gemm_fake_quant(x, packed, scales, zeros, K, bits)
    y_exact = oracle.gemm(x, packed, scales, zeros, K, bits)
    bound = 2.0 ** -8 * (np.abs(xf) @ np.abs(dequant_independent(packed, scales, zeros, K, bits)).T)
    assert np.all(np.abs(y - y_exact) <= bound * (1 + 1e-12))
    rows = np.array([4, 0, 2])
    assert np.array_equal(oracle.gemm_fake_quant(x, packed, scales, zeros, K, bits, rows=rows), y[rows])
