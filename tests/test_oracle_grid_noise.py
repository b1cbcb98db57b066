"""Pins for the oracle's grid-noise measurement (symmetric vs asymmetric grid).

The gamma^2 variance law of the pages (wispaper.ai blog, section on the
gamma^2 law; gist.science summary, Methodology section 1): with
gamma = 2 max|w| / (max w - min w), a symmetric grid over [-max|w|, max|w|]
adds gamma^2 times the rounding-noise variance of an asymmetric grid over
[min w, max w].  oracle.grid_noise gives, per 128-group, gamma and the squared
error of each grid.  Each pin below checks it against something other than
its own formula:

  * brute force: every error equals the distance to the nearest of all 2^b
    grid points, found by exhaustive search (not by rounding a position);
  * closed forms of gamma on groups built from exact values;
  * a group symmetric about 0 has gamma = 1 and the two grids coincide;
  * the law itself, and the pages' worked example gamma = 1.2 -> +44 %;
  * exact scaling by powers of two; degenerate groups.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float64))


def _as_f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _brute_sse(w, start, stop, levels):
    """Sum over w of the squared distance to the nearest of the levels + 1
    evenly spaced points from start to stop, by exhaustive search."""
    pts = np.linspace(start, stop, levels + 1)
    d = (w[:, None] - pts[None, :]) ** 2
    return d.min(axis=1).sum()


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
def test_matches_exhaustive_nearest_point(bits):
    wb = synth.weights(6, 384, seed=40 + bits)
    gamma, sse_a, sse_s = oracle.grid_noise(wb, bits)
    wf = _as_f64(wb)
    L = 2**bits - 1
    for n in range(wf.shape[0]):
        for g in range(wf.shape[1] // 128):
            w = wf[n, 128 * g:128 * (g + 1)]
            lo, hi, m = w.min(), w.max(), np.abs(w).max()
            assert gamma[n, g] == pytest.approx(2 * m / (hi - lo), rel=1e-15)
            assert sse_a[n, g] == pytest.approx(_brute_sse(w, lo, hi, L), rel=1e-9, abs=1e-300)
            assert sse_s[n, g] == pytest.approx(_brute_sse(w, -m, m, L), rel=1e-9, abs=1e-300)


def test_gamma_closed_forms():
    base = np.linspace(-1.0, 3.0, 128)  # min -1, max 3: M = 3, R = 4
    rows = [base, -base, np.linspace(-2.0, 2.0, 128), np.linspace(0.5, 1.0, 128)]
    gamma, _, _ = oracle.grid_noise(_bf16(np.stack(rows)), 4)
    # bf16 keeps -1, 3, -2, 2, 0.5 and 1.0 exact.
    assert gamma[:, 0].tolist() == [1.5, 1.5, 1.0, 4.0]


@pytest.mark.parametrize("bits", [2, 4, 7])
def test_symmetric_group_grids_coincide(bits):
    rng = np.random.default_rng(5 + bits)
    half = rng.normal(0, 0.02, size=(8, 64))
    w = np.concatenate([half, -half], axis=1)  # min = -max, so R = 2M
    gamma, sse_a, sse_s = oracle.grid_noise(_bf16(w), bits)
    assert np.all(gamma == 1.0)
    assert np.array_equal(sse_a, sse_s)


def _skewed_groups(rng, gamma, rows):
    R = np.exp(rng.uniform(np.log(0.01), np.log(0.1), size=(rows, 1)))
    return (gamma - 1.0) * R / 2 + R * (rng.random((rows, 128)) - 0.5)


@pytest.mark.parametrize("bits", [4, 5])
def test_gamma_squared_law(bits):
    rng = np.random.default_rng(70 + bits)
    for target in (1.2, 1.5, 2.0):
        gamma, sse_a, sse_s = oracle.grid_noise(_bf16(_skewed_groups(rng, target, 500)), bits)
        ratio = sse_s.sum() / (gamma**2 * sse_a).sum()
        assert abs(ratio - 1.0) < 0.05, (target, ratio)


def test_worked_example_from_the_pages():
    with open(os.path.join(GOLDEN, "gamma_law.json")) as f:
        gold = json.load(f)
    rng = np.random.default_rng(11)
    w = _bf16(_skewed_groups(rng, gold["gamma"], 800))
    for bits in (4, 5):
        _, sse_a, sse_s = oracle.grid_noise(w, bits)
        assert abs(sse_s.sum() / sse_a.sum() / gold["noise_variance_ratio"] - 1.0) < 0.05


def test_power_of_two_scaling_is_exact():
    wb = synth.weights(4, 256, seed=9)
    w = _as_f64(wb)
    g1, a1, s1 = oracle.grid_noise(wb, 4)
    g2, a2, s2 = oracle.grid_noise(_bf16(4.0 * w), 4)
    assert np.array_equal(g1, g2)
    assert np.array_equal(a2, 16.0 * a1) and np.array_equal(s2, 16.0 * s1)


def test_degenerate_groups():
    rows = [np.full(128, 0.375), np.full(128, -0.375), np.zeros(128)]
    gamma, sse_a, sse_s = oracle.grid_noise(_bf16(np.stack(rows)), 3)
    assert gamma[:, 0].tolist() == [1.0, 1.0, 1.0]
    assert sse_a[:, 0].tolist() == [0.0, 0.0, 0.0]
    # A constant c sits on the symmetric grid's end point +-|c| (up to the
    # rounding of -M + L * (2M / L)); zero has the zero-width grid.
    assert sse_s[1, 0] == 0.0 and sse_s[2, 0] == 0.0
    assert sse_s[0, 0] <= 128 * (0.375 * 2.0**-50) ** 2


def test_rejects_bad_arguments():
    w = synth.weights(2, 256, seed=1)
    for bits in (1, 9):
        with pytest.raises(ValueError):
            oracle.grid_noise(w, bits)
    with pytest.raises(ValueError):
        oracle.grid_noise(w[:, :200], 4)
