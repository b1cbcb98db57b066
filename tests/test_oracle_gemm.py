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
