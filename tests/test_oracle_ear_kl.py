"""Pins for the oracle's EAR and KL(p || q).

  * scipy's softmax and scipy.stats.entropy (a library KL) on the same rows;
  * EAR = 1 - TV with TV = 0.5 * sum |p - q| (the coupling identity behind
    'maximum token-agreement probability under optimal coupling');
  * a speculative-sampling simulation: draft from q, accept with probability
    min(1, p/q); the acceptance rate estimates EAR (the metric is named after
    it: Expected Acceptance Rate);
  * EAR(p, p) = 1 and KL(p, p) = 0; disjoint supports give EAR = 0;
  * shifting all logits of a row by a constant changes nothing;
  * V = 2 closed forms with the logistic function;
  * temperature divides the logits (tau = 0.5 equals doubled logits).
"""
import math

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import entropy

import oracle
import synth


def _vals(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_matches_scipy(tau):
    a, b = synth.logits(6, 3000, seed=1, noise_seed=2)
    ear, kl = oracle.ear_kl(a, b, tau)
    for t in range(6):
        p = softmax(_vals(a[t]) / tau)
        q = softmax(_vals(b[t]) / tau)
        assert abs(ear[t] - np.minimum(p, q).sum()) < 1e-12
        assert abs(kl[t] - entropy(p, q)) < 1e-12
        assert abs(ear[t] - (1 - 0.5 * np.abs(p - q).sum())) < 1e-12
        assert kl[t] >= 0


def test_speculative_acceptance_rate_estimates_ear():
    rng = np.random.default_rng(4)
    la = rng.normal(0, 1.0, size=(1, 6))
    lb = la + rng.normal(0, 0.6, size=(1, 6))
    a, b = synth.to_bf16_bits(la), synth.to_bf16_bits(lb)
    ear, _ = oracle.ear_kl(a, b, 1.0)
    p, q = softmax(_vals(a[0])), softmax(_vals(b[0]))
    n = 400000
    draft = rng.choice(6, size=n, p=q)
    accept = rng.random(n) < np.minimum(1.0, p[draft] / q[draft])
    rate = accept.mean()
    sd = math.sqrt(ear[0] * (1 - ear[0]) / n)
    assert abs(rate - ear[0]) < 5 * sd


def test_identity_disjoint_shift():
    a, _ = synth.logits(3, 1000, seed=5)
    ear, kl = oracle.ear_kl(a, a, 1.0)
    assert np.all(np.abs(ear - 1) < 1e-12) and np.all(np.abs(kl) < 1e-12)
    # disjoint supports: each row puts all its mass where the other has none
    la = np.full((2, 64), -1e4)
    lb = np.full((2, 64), -1e4)
    la[:, :32] = 0.0
    lb[:, 32:] = 0.0
    ear, kl = oracle.ear_kl(synth.to_bf16_bits(la), synth.to_bf16_bits(lb), 1.0)
    assert np.all(ear < 1e-300) and np.all(kl > 1e3)
    # shift invariance with exactly representable integer logits
    rng = np.random.default_rng(6)
    li = rng.integers(-20, 21, size=(2, 300)).astype(np.float64)
    ear, kl = oracle.ear_kl(synth.to_bf16_bits(li), synth.to_bf16_bits(li + 3.0), 0.7)
    assert np.all(np.abs(ear - 1) < 1e-12) and np.all(np.abs(kl) < 1e-12)


def test_two_token_closed_form():
    rng = np.random.default_rng(8)
    la = rng.normal(0, 2, size=(20, 2))
    lb = rng.normal(0, 2, size=(20, 2))
    a, b = synth.to_bf16_bits(la), synth.to_bf16_bits(lb)
    for tau in (1.0, 0.7):
        ear, kl = oracle.ear_kl(a, b, tau)
        va, vb = _vals(a) / tau, _vals(b) / tau
        p = 1 / (1 + np.exp(-(va[:, 0] - va[:, 1])))
        q = 1 / (1 + np.exp(-(vb[:, 0] - vb[:, 1])))
        assert np.allclose(ear, 1 - np.abs(p - q), atol=1e-13)
        want = p * np.log(p / q) + (1 - p) * np.log((1 - p) / (1 - q))
        assert np.allclose(kl, want, atol=1e-12)


def test_temperature_divides_logits():
    a, b = synth.logits(3, 500, seed=9)
    va, vb = _vals(a), _vals(b)
    a2, b2 = synth.to_bf16_bits(2 * va), synth.to_bf16_bits(2 * vb)  # exact doubling
    e1, k1 = oracle.ear_kl(a, b, 0.5)
    e2, k2 = oracle.ear_kl(a2, b2, 1.0)
    assert np.allclose(e1, e2, atol=1e-14) and np.allclose(k1, k2, atol=1e-14)


def test_sampled_rows_and_single_token_vocab():
    a, b = synth.logits(5, 700, seed=10)
    ear, kl = oracle.ear_kl(a, b, 1.0)
    e2, k2 = oracle.ear_kl(a, b, 1.0, rows=[4, 1])
    assert np.array_equal(e2, ear[[4, 1]]) and np.array_equal(k2, kl[[4, 1]])
    one = synth.to_bf16_bits(np.array([[3.0], [-2.0]]))
    two = synth.to_bf16_bits(np.array([[1.0], [5.0]]))
    ear, kl = oracle.ear_kl(one, two, 1.0)
    assert np.all(ear == 1.0) and np.all(kl == 0.0)


# ---------------------------------------------------------------------------
# Top-K form (T = the K largest reference logits, ties to the lower index;
# EAR over T with full softmaxes; KL between p and q renormalized over T).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_topk_with_k_equal_v_is_the_full_metric(tau):
    a, b = synth.logits(4, 777, seed=21)
    e, k, top = oracle.ear_kl_topk(a, b, 777, tau)
    E, K = oracle.ear_kl(a, b, tau)
    assert np.allclose(e, E, rtol=0, atol=1e-12) and np.allclose(k, K, rtol=0, atol=1e-12)
    assert all(sorted(r) == list(range(777)) for r in top)


@pytest.mark.parametrize("K", [1, 3, 10, 32])
@pytest.mark.parametrize("tau", [1.0, 0.7])
def test_topk_matches_scipy_on_the_selected_set(K, tau):
    a, b = synth.logits(5, 1500, seed=31 + K)
    e, k, top = oracle.ear_kl_topk(a, b, K, tau)
    for i in range(a.shape[0]):
        x, y = _vals(a[i]), _vals(b[i])
        order = np.argsort(-x, kind="stable")[:K]  # stable: ties keep the lower index first
        assert np.array_equal(top[i], order)
        p, q = softmax(x / tau), softmax(y / tau)
        assert abs(e[i] - np.minimum(p[order], q[order]).sum()) <= 1e-12
        pt, qt = p[order] / p[order].sum(), q[order] / q[order].sum()
        assert abs(k[i] - entropy(pt, qt)) <= 1e-12


def test_topk_ties_take_the_lower_index():
    x = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, -1.0, 2.0, 2.0]])
    bits = synth.to_bf16_bits(x)
    _, _, top = oracle.ear_kl_topk(bits, bits, 5, 1.0)
    assert top[0].tolist() == [1, 2, 4, 3, 6]


def test_topk_invariants():
    a, b = synth.logits(6, 900, seed=41)
    for K in (1, 2, 10):
        e_aa, k_aa, top = oracle.ear_kl_topk(a, a, K, 1.0)
        p_mass = np.array([softmax(_vals(a[i]))[top[i]].sum() for i in range(a.shape[0])])
        assert np.allclose(e_aa, p_mass, atol=1e-12)  # EAR(p, p) over T = p(T)
        assert np.abs(k_aa).max() <= 1e-12  # KL(p, p) = 0
    # K = 1: min(p_top, q_top); the renormalized one-point distributions agree.
    e1, k1, top1 = oracle.ear_kl_topk(a, b, 1, 1.0)
    for i in range(a.shape[0]):
        v = top1[i, 0]
        assert abs(e1[i] - min(softmax(_vals(a[i]))[v], softmax(_vals(b[i]))[v])) <= 1e-12
    assert np.abs(k1).max() <= 1e-15
    # EAR over T grows with K and stays below the full EAR.
    E, _ = oracle.ear_kl(a, b, 1.0)
    prev = np.zeros(a.shape[0])
    for K in (1, 2, 5, 10, 50, 900):
        e, _, _ = oracle.ear_kl_topk(a, b, K, 1.0)
        assert np.all(e >= prev - 1e-15) and np.all(e <= E + 1e-12)
        prev = e
