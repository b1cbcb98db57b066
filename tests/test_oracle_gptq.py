"""Pins for the oracle's GPTQ encoder (the pages' layer-wise GPTQ, asymmetric
INT, group 128: GitHub README "Pipeline" and "1. Quantize").

GPTQ (Frantar et al.) fixes one column of W at a time and moves the row's
later columns to absorb the error, using the upper Cholesky factor of
(X^T X + damping)^-1.  Each pin checks the oracle against something other
than its own code:

  * a diagonal X^T X has nothing to spread the error over: the result is
    the plain RTN encode, bit for bit;
  * an independent route: the explicit-inverse form of the same procedure
    (at step k, the remaining block of H inverted by numpy.linalg.inv,
    update -(w_k - d_k) / [H_F^-1]_kk * [H_F^-1]_{:,k}) gives the same codes;
  * on correlated inputs the layer's output error is far below RTN's;
  * invariances: permuting rows permutes the result, one row alone equals
    its row of the batch, scaling X by 2 changes nothing;
  * the first group's scale and zero are RTN's (no update has reached it);
  * an input that is always zero leaves its weight at zero.
"""
import numpy as np
import pytest

import oracle
import synth


def _corr_x(T, K, seed, rho=0.9):
    """Calibration rows whose neighbouring inputs are correlated (AR(1))."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, K))
    x = np.empty_like(z)
    x[:, 0] = z[:, 0]
    for k in range(1, K):
        x[:, k] = rho * x[:, k - 1] + np.sqrt(1 - rho**2) * z[:, k]
    return synth.to_bf16_bits(x)


def _f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _out_err(xb, wb, enc, bits):
    packed, scales, zeros = enc[:3]
    dq = oracle.dequantize(packed, scales, zeros, wb.shape[1], bits)
    return float(np.sum((_f64(xb) @ (_f64(wb) - dq).T) ** 2))


def _same(a, b):
    return all(np.array_equal(u, v) for u, v in zip(a[:3], b[:3]))


@pytest.mark.parametrize("bits", [2, 4, 7])
def test_diagonal_hessian_is_rtn(bits):
    K = 256
    wb = synth.weights(16, K, seed=20 + bits)
    rng = np.random.default_rng(bits)
    d = 2.0 ** rng.integers(-2, 3, size=K)  # unequal diagonal entries, exact in bf16
    xb = synth.to_bf16_bits(np.diag(d))
    assert _same(oracle.gptq(wb, xb, bits), oracle.quantize(wb, bits))


def _rtn_params(w32, bits):
    """The format's group rule on binary32 values (pinned separately for the
    RTN oracle): fp16 scale of (max - min) / (2^b - 1), zero rne(-min / s)."""
    L = np.float32(2**bits - 1)
    lo, hi = w32.min(), w32.max()
    assert hi > lo
    s16 = np.float16(np.float32(hi - lo) / L)
    s = np.float32(s16)
    z = np.clip(np.rint(np.float32(-lo) / s), 0, L)
    return s16, s, z


def _gptq_explicit_inverse(wb, xb, bits, damp=0.01):
    """GPTQ in its explicit-inverse form (no Cholesky): H_F^-1 of the columns
    not yet fixed is recomputed with numpy.linalg.inv at every step."""
    w = _f64(wb).copy()
    x = _f64(xb)
    N, K = w.shape
    h = x.T @ x
    h[np.diag_indices(K)] += damp * np.mean(np.diag(h))
    L = 2**bits - 1
    codes = np.zeros((N, K), dtype=np.int64)
    scales = np.zeros((N, K // 128), dtype=np.float16)
    zeros = np.zeros((N, K // 128), dtype=np.int64)
    for k in range(K):
        if k % 128 == 0:
            g = k // 128
            for n in range(N):
                s16, _, z = _rtn_params(w[n, k:k + 128].astype(np.float32), bits)
                scales[n, g], zeros[n, g] = s16, int(z)
        g = k // 128
        s = scales[:, g].astype(np.float32)
        q = np.clip(np.rint(w[:, k].astype(np.float32) / s) + zeros[:, g], 0, L).astype(np.int64)
        codes[:, k] = q
        d = scales[:, g].astype(np.float64) * (q - zeros[:, g])
        hinv = np.linalg.inv(h[k:, k:])
        w[:, k:] -= np.outer((w[:, k] - d) / hinv[0, 0], hinv[:, 0])
    return codes, scales, zeros


@pytest.mark.parametrize("bits", [3, 4])
def test_matches_explicit_inverse_form(bits):
    K, N = 256, 6
    wb = synth.weights(N, K, seed=60 + bits)
    xb = _corr_x(384, K, seed=61 + bits)
    packed, scales, zeros, _ = oracle.gptq(wb, xb, bits)
    codes = np.array([[oracle.code_at(packed, K, bits, n, k) for k in range(K)] for n in range(N)])
    c_ref, s_ref, z_ref = _gptq_explicit_inverse(wb, xb, bits)
    assert np.array_equal(scales, s_ref.view(np.uint16))
    assert np.array_equal(zeros, z_ref)
    assert np.array_equal(codes, c_ref)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
def test_beats_rtn_on_correlated_inputs(bits):
    K = 256
    wb = synth.weights(32, K, seed=3)
    xb = _corr_x(512, K, seed=4)
    ratio = _out_err(xb, wb, oracle.gptq(wb, xb, bits), bits) / _out_err(xb, wb, oracle.quantize(wb, bits), bits)
    assert ratio < 0.5, ratio


def test_rows_are_independent():
    K, bits = 256, 4
    wb = synth.weights(8, K, seed=8)
    xb = _corr_x(300, K, seed=9)
    full = oracle.gptq(wb, xb, bits)
    perm = np.array([5, 2, 7, 0, 1, 6, 3, 4])
    permuted = oracle.gptq(np.ascontiguousarray(wb[perm]), xb, bits)
    assert all(np.array_equal(a[perm], b) for a, b in zip(full[:3], permuted[:3]))
    one = oracle.gptq(np.ascontiguousarray(wb[3:4]), xb, bits)
    assert all(np.array_equal(a[3:4], b) for a, b in zip(full[:3], one[:3]))


def test_scaling_the_inputs_changes_nothing():
    K, bits = 256, 3
    wb = synth.weights(8, K, seed=12)
    xb = _corr_x(300, K, seed=13)
    assert _same(oracle.gptq(wb, xb, bits), oracle.gptq(wb, synth.to_bf16_bits(2.0 * _f64(xb)), bits))


def test_first_group_parameters_are_rtn():
    K, bits = 384, 5
    wb = synth.weights(8, K, seed=14)
    g = oracle.gptq(wb, _corr_x(300, K, seed=15), bits)
    r = oracle.quantize(wb, bits)
    assert np.array_equal(g[1][:, 0], r[1][:, 0]) and np.array_equal(g[2][:, 0], r[2][:, 0])
    assert not np.array_equal(g[1], r[1])  # later groups were moved by the updates


def test_dead_input_leaves_weight_at_zero():
    K, bits, dead = 256, 4, 37
    wb = synth.weights(8, K, seed=16)
    x = _f64(_corr_x(300, K, seed=17))
    x[:, dead] = 0.0
    packed, scales, zeros, _ = oracle.gptq(wb, synth.to_bf16_bits(x), bits)
    dq = oracle.dequantize(packed, scales, zeros, K, bits)
    s = np.array([oracle.f16_bits_to_f64(int(v)) for v in scales[:, dead // 128]])
    assert np.all(np.abs(dq[:, dead]) <= s / 2)


def test_rejects_bad_arguments():
    wb = synth.weights(2, 256, seed=1)
    xb = _corr_x(16, 256, seed=2)
    for bits in (1, 9):
        with pytest.raises(ValueError):
            oracle.gptq(wb, xb, bits)
    with pytest.raises(ValueError):
        oracle.gptq(wb, xb, 4, damp=-1.0)
