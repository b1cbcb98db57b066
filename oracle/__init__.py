"""CPU oracle for the SLQ weight format -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow reference the CUDA library is checked
against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline/reference leg may import it; the product path
(``weight_only_mixed_b200``) never does, and the two share no code.

The arithmetic lives in ``slq_oracle.c`` (plain C, binary32 encode decisions,
binary64 dequantize/GEMM/EAR/KL, GPTQ error feedback and grid-noise sums);
this module only compiles it with gcc and marshals numpy arrays through
ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "slq_oracle.c")
_HDR = os.path.join(_HERE, "slq_oracle.h")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libslq_oracle.so")

GROUP = 128
FLAG_NONFINITE = 1
FLAG_SCALE_OVERFLOW = 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest_src:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
             "-Wall", "-Wextra", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"],
            check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_f32_to_f16_rn.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16_rn.restype = ctypes.c_uint16
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_quantize.argtypes = [P, I64, I64, ctypes.c_int, P, P, P, P]
        lib.oracle_quantize.restype = ctypes.c_int
        lib.oracle_code_at.argtypes = [P, I64, ctypes.c_int, I64, I64]
        lib.oracle_code_at.restype = ctypes.c_uint32
        lib.oracle_dequantize.argtypes = [P, P, P, I64, I64, ctypes.c_int, P]
        lib.oracle_dequantize.restype = ctypes.c_int
        lib.oracle_gemm.argtypes = [P, P, I64, I64, I64, ctypes.c_int, P, P, P, P]
        lib.oracle_gemm.restype = ctypes.c_int
        lib.oracle_ear_kl.argtypes = [P, P, P, I64, I64, ctypes.c_double, P, P]
        lib.oracle_ear_kl.restype = ctypes.c_int
        lib.oracle_ear_kl_topk.argtypes = [P, P, P, I64, I64, I64, ctypes.c_double, P, P, P]
        lib.oracle_ear_kl_topk.restype = ctypes.c_int
        lib.oracle_gptq.argtypes = [P, I64, I64, ctypes.c_int, P, I64, ctypes.c_double, P, P, P, P]
        lib.oracle_gptq.restype = ctypes.c_int
        lib.oracle_grid_noise.argtypes = [P, I64, I64, ctypes.c_int, P, P, P]
        lib.oracle_grid_noise.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16/fp16 data is passed as raw uint16 bits"
    return a


def f32_to_f16_bits(x: float) -> int:
    """binary32 -> binary16 bits, round to nearest even (hand-written)."""
    return int(_load().oracle_f32_to_f16_rn(ctypes.c_float(x)))


def f16_bits_to_f64(h: int) -> float:
    return float(_load().oracle_f16_to_f64(ctypes.c_uint16(h)))


def packed_words(N: int, K: int, bits: int) -> int:
    return N * K * bits // 32


def quantize(w_bf16: np.ndarray, bits: int):
    """Quantize W ([N, K] bf16 bits) -> (packed u32 [N, K*b/32], scales fp16
    bits [N, K/128], zeros u8 [N, K/128], flags)."""
    w = _u16(w_bf16)
    N, K = w.shape
    packed = np.zeros((N, K * bits // 32), dtype=np.uint32)
    scales = np.zeros((N, K // GROUP), dtype=np.uint16)
    zeros = np.zeros((N, K // GROUP), dtype=np.uint8)
    flags = np.zeros(1, dtype=np.uint32)
    rc = _load().oracle_quantize(_ptr(w), N, K, bits, _ptr(packed), _ptr(scales),
                                 _ptr(zeros), _ptr(flags))
    if rc != 0:
        raise ValueError(f"oracle_quantize rejected N={N} K={K} bits={bits}")
    return packed, scales, zeros, int(flags[0])


def code_at(packed: np.ndarray, K: int, bits: int, n: int, k: int) -> int:
    p = np.ascontiguousarray(packed, dtype=np.uint32)
    return int(_load().oracle_code_at(_ptr(p), K, bits, n, k))


def dequantize(packed, scales, zeros, K: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = _u16(scales)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    N = scales.shape[0]
    out = np.empty((N, K), dtype=np.float64)
    rc = _load().oracle_dequantize(_ptr(packed), _ptr(scales), _ptr(zeros), N, K, bits,
                                   _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequantize rejected its arguments")
    return out


def gemm(x_bf16, packed, scales, zeros, K: int, bits: int, rows=None) -> np.ndarray:
    """y = X[rows] W'^T in binary64 ([len(rows), N])."""
    x = _u16(x_bf16)
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = _u16(scales)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    N = scales.shape[0]
    if rows is None:
        n_rows = x.shape[0]
        rows_arr = None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.shape[0]
    y = np.empty((n_rows, N), dtype=np.float64)
    rc = _load().oracle_gemm(_ptr(x), None if rows_arr is None else _ptr(rows_arr), n_rows,
                             N, K, bits, _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_gemm rejected its arguments")
    return y


def ear_kl(a_bf16, b_bf16, tau: float, rows=None):
    """Per-token (EAR, KL) in binary64 for the selected rows."""
    a = _u16(a_bf16)
    b = _u16(b_bf16)
    assert a.shape == b.shape and a.ndim == 2
    T, V = a.shape
    if rows is None:
        n_rows, rows_arr = T, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.shape[0]
    ear = np.empty(n_rows, dtype=np.float64)
    kl = np.empty(n_rows, dtype=np.float64)
    rc = _load().oracle_ear_kl(_ptr(a), _ptr(b), None if rows_arr is None else _ptr(rows_arr),
                               n_rows, V, float(tau), _ptr(ear), _ptr(kl))
    if rc != 0:
        raise ValueError("oracle_ear_kl rejected its arguments")
    return ear, kl


def ear_kl_topk(a_bf16, b_bf16, k: int, tau: float, rows=None):
    """Per-token top-K (EAR, KL, selected indices) in binary64."""
    a = _u16(a_bf16)
    b = _u16(b_bf16)
    assert a.shape == b.shape and a.ndim == 2
    T, V = a.shape
    if rows is None:
        n_rows, rows_arr = T, None
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = rows_arr.shape[0]
    ear = np.empty(n_rows, dtype=np.float64)
    kl = np.empty(n_rows, dtype=np.float64)
    top = np.empty((n_rows, k), dtype=np.int64)
    rc = _load().oracle_ear_kl_topk(_ptr(a), _ptr(b), None if rows_arr is None else _ptr(rows_arr),
                                    n_rows, V, int(k), float(tau), _ptr(ear), _ptr(kl), _ptr(top))
    if rc != 0:
        raise ValueError("oracle_ear_kl_topk rejected its arguments")
    return ear, kl, top


def grid_noise(w_bf16, bits: int):
    """Per-group (gamma, sse_asym, sse_sym), each [N, K/128] binary64: the
    gamma^2-law ablation of an asymmetric grid over [min, max] against a
    symmetric grid over [-max|w|, max|w|] (see oracle_grid_noise)."""
    w = _u16(w_bf16)
    assert w.ndim == 2
    N, K = w.shape
    G = K // 128
    gamma = np.empty((N, G), dtype=np.float64)
    sse_a = np.empty((N, G), dtype=np.float64)
    sse_s = np.empty((N, G), dtype=np.float64)
    rc = _load().oracle_grid_noise(_ptr(w), N, K, int(bits), _ptr(gamma), _ptr(sse_a), _ptr(sse_s))
    if rc != 0:
        raise ValueError("oracle_grid_noise rejected its arguments")
    return gamma, sse_a, sse_s


def gptq(w_bf16: np.ndarray, x_bf16: np.ndarray, bits: int, damp: float = 0.01):
    """GPTQ encode of bf16 W [N, K] with calibration rows X [T, K] (bf16 bits):
    (packed, scales, zeros, flags) in the format of quantize()."""
    w = _u16(w_bf16)
    x = _u16(x_bf16)
    assert w.ndim == 2 and x.ndim == 2 and x.shape[1] == w.shape[1]
    N, K = w.shape
    packed = np.zeros((N, K * bits // 32), dtype=np.uint32)
    scales = np.zeros((N, K // 128), dtype=np.uint16)
    zeros = np.zeros((N, K // 128), dtype=np.uint8)
    flags = ctypes.c_uint32(0)
    rc = _load().oracle_gptq(_ptr(w), N, K, int(bits), _ptr(x), x.shape[0], float(damp),
                             _ptr(packed), _ptr(scales), _ptr(zeros), ctypes.byref(flags))
    if rc != 0:
        raise ValueError(f"oracle_gptq failed ({rc})")
    return packed, scales, zeros, int(flags.value)
