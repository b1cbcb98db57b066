"""Pins for the oracle's hand-written number-format conversions.

The binary32 -> binary16 rounding is checked against numpy's independent
implementation (round to nearest even, subnormals kept, overflow to inf), and
the binary16 decoder against numpy on every one of the 65536 bit patterns.
"""
import numpy as np

import oracle


def _numpy_f16_bits(x32: np.ndarray) -> np.ndarray:
    return x32.astype(np.float16).view(np.uint16)


def test_f32_to_f16_matches_numpy_on_random_bit_patterns():
    rng = np.random.default_rng(7)
    u = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    x = u.view(np.float32)
    x = x[np.isfinite(x)]
    ours = np.array([oracle.f32_to_f16_bits(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(ours, _numpy_f16_bits(x))


def test_f32_to_f16_boundaries_ties_subnormals_overflow():
    vals = []
    # every binade of binary16 and its neighbourhood, incl. subnormal range
    for e in range(-30, 18):
        base = np.float32(2.0) ** e
        for frac in np.linspace(1.0, 2.0, 257, dtype=np.float32):
            v = np.float32(base * frac)
            vals += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(np.inf))]
    # exact ties between binary16 neighbours: midpoints of consecutive halves
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    mids = (h[:-1].astype(np.float64) + h[1:].astype(np.float64)) / 2
    vals += list(mids.astype(np.float32))
    vals += [np.float32(65504.0), np.float32(65519.99), np.float32(65520.0), np.float32(1e30),
             np.float32(2.0**-24), np.float32(2.0**-25), np.float32(2.0**-25 * 1.0000001),
             np.float32(1e-40), np.float32(0.0), np.float32(np.inf)]
    x = np.array(vals, dtype=np.float32)
    x = np.concatenate([x, -x])
    ours = np.array([oracle.f32_to_f16_bits(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(ours, _numpy_f16_bits(x))


def test_f16_decoder_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    ours = np.array([oracle.f16_bits_to_f64(int(v)) for v in h])
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isinf(ours), np.isinf(ref))
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
