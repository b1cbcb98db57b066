"""Independent checking helpers for the oracle pins.

Nothing here calls the oracle or the CUDA library: these are second,
differently-written implementations (numpy bit streams, numpy's own fp16
conversion, brute-force searches) that the oracle is checked against.
"""
import numpy as np


def unpack_bitstream(packed_rows: np.ndarray, K: int, bits: int) -> np.ndarray:
    """Codes [N, K] from LSB-first per-row bitstreams (numpy unpackbits)."""
    packed_rows = np.ascontiguousarray(packed_rows, dtype="<u4")
    N = packed_rows.shape[0]
    stream = np.unpackbits(packed_rows.view(np.uint8).reshape(N, -1), axis=1,
                           bitorder="little")
    assert stream.shape[1] == K * bits
    fields = stream.reshape(N, K, bits).astype(np.int64)
    return (fields << np.arange(bits, dtype=np.int64)).sum(axis=2)


def fp16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


def dequant_independent(packed, scales, zeros, K: int, bits: int) -> np.ndarray:
    codes = unpack_bitstream(packed, K, bits).astype(np.float64)
    s = np.repeat(fp16_bits_to_f64(scales), 128, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=np.float64), 128, axis=1)
    return s * (codes - z)


def nearest_int_ties_even_bruteforce(t: float, lo: int, hi: int) -> int:
    """argmin over integers i in [lo, hi] of |t - i|; equal distances go to the
    even integer.  Brute force over the whole range."""
    best, best_d = None, None
    for i in range(lo, hi + 1):
        d = abs(float(t) - i)
        if best is None or d < best_d or (d == best_d and i % 2 == 0):
            best, best_d = i, d
    return best
