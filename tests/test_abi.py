"""Host-side checks of the C ABI that need no GPU.

  * libslq.so loads and exports every function include/slq.h declares, and
    the binding gives each one its ctypes signature;
  * the header carries no torch or CUDA types in its signatures;
  * argument validation rejects bad calls with SLQ_ERR_INVALID_ARGUMENT
    before touching CUDA (fake, never-dereferenced pointers are used);
  * with no CUDA device, a valid call reports SLQ_ERR_UNSUPPORTED_DEVICE;
  * host helpers (packed_words, gemm_select, status strings).
"""
import ctypes
import re
import subprocess

import pytest
import torch

import weight_only_mixed_b200 as slq

L = slq.lib()
FAKE = 0x7f0000100000  # 16-byte aligned, never dereferenced by validation


def test_every_declared_symbol_is_exported():
    names = slq.declared_symbols()
    assert {"slq_quantize", "slq_gemm", "slq_ear_kl"} <= set(names)
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", slq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (slq_\w+)", out))
    assert set(names) <= exported


def test_binding_declares_every_signature():
    # Without argtypes ctypes passes Python ints as C int, which would cut
    # 64-bit sizes and pointers; every declared function gets its signature.
    for n in slq.declared_symbols():
        assert getattr(L, n).argtypes is not None, n


def test_header_is_plain_c():
    with open(slq.HEADER_PATH) as f:
        text = f.read()
    code = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    for bad in ("torch", "at::", "cudaStream_t", "#include <cuda", "std::"):
        assert bad not in code
    assert 'extern "C"' in code


def test_status_strings_and_version():
    assert slq.status_string(0) == "SLQ_OK"
    assert "INVALID" in slq.status_string(1)
    assert slq.version() >= 100


def test_packed_words():
    for b in range(2, 9):
        assert slq.packed_words(4096, 4096, b) == 4096 * 4096 * b // 32
        assert slq.packed_words(3, 128, b) == 3 * 4 * b  # 4b words per group
    assert slq.packed_words(10, 100, 4) == 0
    assert slq.packed_words(10, 128, 9) == 0
    assert slq.packed_words(10, 128, 1) == 0


def test_gemm_select():
    assert slq.gemm_select(1, 4096, 4096, 4) == "gemv"
    assert slq.gemm_select(16, 4096, 4096, 4) == "gemv"
    assert slq.gemm_select(17, 4096, 4096, 4) == "tiled"
    assert slq.gemm_select(4096, 8192, 8192, 2) == "tiled"


def _q(N=8, K=256, bits=4, W=FAKE, packed=FAKE + (1 << 24), scales=FAKE + (2 << 24),
       zeros=FAKE + (3 << 24), flags=None):
    return L.slq_quantize(W, N, K, bits, packed, scales, zeros, flags, None)


def test_quantize_validation():
    bad = [dict(bits=1), dict(bits=9), dict(K=100), dict(K=0), dict(K=-128), dict(N=-1),
           dict(W=None), dict(packed=None), dict(scales=None), dict(zeros=None),
           dict(W=FAKE + 8), dict(packed=FAKE + (1 << 24) + 4), dict(scales=FAKE + (2 << 24) + 1),
           dict(flags=FAKE + (4 << 24) + 2), dict(N=1 << 31),
           # output overlapping the input
           dict(packed=FAKE + 64)]
    for kw in bad:
        assert _q(**kw) == slq.SLQ_ERR_INVALID_ARGUMENT, kw
    assert _q(N=0) == slq.SLQ_OK  # empty: nothing to do, nothing launched


WS = FAKE + (6 << 24)


def _g(M=4, N=8, K=256, bits=4, X=FAKE, packed=FAKE + (1 << 24), scales=FAKE + (2 << 24),
       zeros=FAKE + (3 << 24), Y=FAKE + (4 << 24), dtype=0, path=0, ws=WS, ws_bytes=1 << 24,
       flags=None):
    return L.slq_gemm_ex(X, M, N, K, bits, packed, scales, zeros, Y, dtype, path, ws, ws_bytes,
                         flags, None)


def test_gemm_validation():
    bad = [dict(bits=1), dict(bits=9), dict(K=64), dict(K=129), dict(M=-1), dict(N=-1),
           dict(X=None), dict(Y=None), dict(packed=None), dict(scales=None), dict(zeros=None),
           dict(X=FAKE + 2), dict(Y=FAKE + (4 << 24) + 8), dict(packed=FAKE + (1 << 24) + 4),
           dict(dtype=2), dict(path=4), dict(path=1, M=17), dict(path=3, M=17), dict(Y=FAKE + 16),  # Y overlaps X
           dict(M=1 << 31)]
    for kw in bad:
        assert _g(**kw) == slq.SLQ_ERR_INVALID_ARGUMENT, kw
    assert _g(M=0) == slq.SLQ_OK and _g(N=0) == slq.SLQ_OK


def test_slq_gemm_takes_no_workspace():
    # slq_gemm(X, M, N, K, bits, packed, scales, zeros, Y, y_dtype, flags, stream):
    # the kernels it selects use no memory beyond their arguments.
    def g(M=4, N=8, K=256, bits=4, X=FAKE, Y=FAKE + (4 << 24), dtype=0):
        return L.slq_gemm(X, M, N, K, bits, FAKE + (1 << 24), FAKE + (2 << 24), FAKE + (3 << 24), Y,
                          dtype, None, None)
    assert len(L.slq_gemm.argtypes) == 12
    for bad in [dict(bits=9), dict(K=100), dict(X=None), dict(Y=FAKE + 16), dict(dtype=2)]:
        assert g(**bad) == slq.SLQ_ERR_INVALID_ARGUMENT, bad
    assert g(M=0) == slq.SLQ_OK
    assert g() in (slq.SLQ_OK, slq.SLQ_ERR_UNSUPPORTED_DEVICE)
    assert g(M=300, N=4096, K=4096, X=FAKE, Y=FAKE + (8 << 24)) in (slq.SLQ_OK,
                                                                      slq.SLQ_ERR_UNSUPPORTED_DEVICE)


def test_gemm_workspace_rules():
    # A layer whose row tiles are split over several CTAs needs a workspace.
    M, N, K, b = 4, 4096, 4096, 4
    need = slq.gemm_workspace_bytes(M, N, K, b)
    assert need > 0
    assert slq.gemm_workspace_bytes(17, N, K, b) == 0  # tiled kernel: none
    assert slq.gemm_workspace_bytes(4, N, 100, b) == 0  # invalid K
    kw = dict(M=M, N=N, K=K, bits=b, path=1)  # the stream-K decode kernel
    big = dict(packed=FAKE + (1 << 28), scales=FAKE + (2 << 28), zeros=FAKE + (3 << 28),
               Y=FAKE + (4 << 28), ws=FAKE + (5 << 28))
    for bad in [dict(ws=None), dict(ws_bytes=need - 1), dict(ws=FAKE + (5 << 28) + 16),
                dict(ws=FAKE + 256)]:  # misaligned, overlapping X
        args = {**kw, **big, "ws_bytes": need, **bad}
        assert _g(**args) == slq.SLQ_ERR_INVALID_ARGUMENT, bad
    # The tiled and GEMV kernels (and AUTO, which picks them) take none.
    for path in (0, 2, 3):
        assert _g(**{**kw, **big, "ws": None, "ws_bytes": 0, "path": path}) != slq.SLQ_ERR_INVALID_ARGUMENT


def _e(T=4, V=1000, tau=1.0, a=FAKE, b=FAKE + (1 << 24), ear=FAKE + (2 << 24),
       kl=FAKE + (3 << 24), em=None, km=None, flags=None):
    return L.slq_ear_kl(a, b, T, V, tau, ear, kl, em, km, flags, None)


def test_ear_kl_validation():
    bad = [dict(V=0), dict(T=-1), dict(tau=0.0), dict(tau=-1.0), dict(tau=float("inf")),
           dict(tau=float("nan")), dict(a=None), dict(b=None), dict(ear=None), dict(kl=None),
           dict(a=FAKE + 2), dict(ear=FAKE + (2 << 24) + 2), dict(em=FAKE + (5 << 24) + 4),
           dict(ear=FAKE + 8)]  # output overlaps the input
    for kw in bad:
        assert _e(**kw) == slq.SLQ_ERR_INVALID_ARGUMENT, kw
    assert _e(T=0) == slq.SLQ_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_valid_calls_without_a_device_are_refused():
    assert _q() == slq.SLQ_ERR_UNSUPPORTED_DEVICE
    assert _g() == slq.SLQ_ERR_UNSUPPORTED_DEVICE
    assert _e() == slq.SLQ_ERR_UNSUPPORTED_DEVICE


def _layer(X=FAKE, N=8, K=256, bits=4, off=0):
    base = FAKE + ((1 + 8 * off) << 24)
    return slq.GemmLayer(X, N, K, bits, base, base + (1 << 24), base + (2 << 24), base + (3 << 24))


def _grp(layers, M=4, dtype=0, flags=None):
    arr = (slq.GemmLayer * max(1, len(layers)))(*layers)
    return L.slq_gemm_group(arr if layers else None, len(layers), M, dtype, flags, None)


def test_gemm_group_validation():
    assert L.slq_gemm_group_max() == 8
    ok = [_layer(off=0), _layer(X=FAKE + (100 << 24), N=16, K=512, bits=7, off=1)]
    # Valid arguments reach the device check (no GPU here) or run.
    assert _grp(ok) in (slq.SLQ_OK, slq.SLQ_ERR_UNSUPPORTED_DEVICE)
    assert _grp(ok, M=0) == slq.SLQ_OK
    bad = [
        _grp([]),                                               # no layers
        _grp([_layer(off=i) for i in range(9)]),                # more than 8
        _grp(ok, M=17),                                         # decode sizes only
        _grp(ok, dtype=2),
        _grp([_layer(K=100)]),                                  # K % 128
        _grp([_layer(bits=9)]),
        _grp([_layer(X=FAKE + 8)]),                             # misaligned X
        # layer 1's Y lands on layer 0's packed weights
        _grp([_layer(off=0), slq.GemmLayer(FAKE + (100 << 24), 8, 256, 4, FAKE + (9 << 24),
                                           FAKE + (10 << 24), FAKE + (11 << 24), FAKE + (1 << 24))]),
        # two layers write the same Y
        _grp([_layer(off=0), slq.GemmLayer(FAKE + (100 << 24), 8, 256, 4, FAKE + (9 << 24),
                                           FAKE + (10 << 24), FAKE + (11 << 24), FAKE + (4 << 24))]),
    ]
    assert all(r == slq.SLQ_ERR_INVALID_ARGUMENT for r in bad), bad


def test_ear_kl_topk_validation():
    assert L.slq_ear_kl_topk_max() == 16

    def call(T=4, V=1000, k=10, tau=1.0, a=FAKE, b=FAKE + (1 << 24), ear=FAKE + (2 << 24),
             kl=FAKE + (3 << 24)):
        return L.slq_ear_kl_topk(a, b, T, V, k, tau, ear, kl, None, None, None, None)

    for bad in [dict(k=0), dict(k=17), dict(V=5, k=6), dict(tau=0.0), dict(a=None), dict(ear=FAKE + 8),
                dict(a=FAKE + 2)]:
        assert call(**bad) == slq.SLQ_ERR_INVALID_ARGUMENT, bad
    assert call(T=0) == slq.SLQ_OK
    assert call() in (slq.SLQ_OK, slq.SLQ_ERR_UNSUPPORTED_DEVICE)


def test_grid_noise_validation():
    def call(W=FAKE, N=4, K=256, bits=4, g=FAKE + (1 << 24), a=FAKE + (2 << 24), s=FAKE + (3 << 24),
             flags=None):
        return L.slq_grid_noise(W, N, K, bits, g, a, s, flags, None)

    for bad in [dict(N=-1), dict(K=0), dict(K=200), dict(bits=1), dict(bits=9), dict(W=None),
                dict(g=None), dict(a=None), dict(s=None), dict(W=FAKE + 8), dict(g=FAKE + (1 << 24) + 2),
                dict(flags=FAKE + (4 << 24) + 1),
                dict(g=FAKE + 1024),                # output overlaps W
                dict(N=1 << 31)]:
        assert call(**bad) == slq.SLQ_ERR_INVALID_ARGUMENT, bad
    assert call(N=0) == slq.SLQ_OK
    assert call() in (slq.SLQ_OK, slq.SLQ_ERR_UNSUPPORTED_DEVICE)


def test_gptq_validation():
    need = slq.gptq_workspace_bytes(64, 256)
    assert need == L.slq_gptq_workspace_bytes(64, 256) and need > 3 * 256 * 256 * 8
    assert L.slq_gptq_workspace_bytes(64, 100) == 0
    assert L.slq_gptq_workspace_bytes(64, 16384 + 128) == 0

    def call(W=FAKE, N=64, K=256, bits=4, X=FAKE + (1 << 24), T=32, damp=0.01, p=FAKE + (2 << 24),
             s=FAKE + (3 << 24), z=FAKE + (4 << 24), ws=FAKE + (5 << 24), wsb=need, flags=None):
        return L.slq_gptq(W, N, K, bits, X, T, damp, p, s, z, ws, wsb, flags, None)

    for bad in [dict(N=-1), dict(K=200), dict(K=16384 + 128), dict(bits=9), dict(T=0), dict(damp=-1.0),
                dict(damp=float("nan")), dict(damp=float("inf")), dict(W=None), dict(X=None),
                dict(ws=None), dict(wsb=need - 1), dict(ws=FAKE + (5 << 24) + 8), dict(p=FAKE + 2),
                dict(p=FAKE + 16)]:                    # output overlaps W
        assert call(**bad) == slq.SLQ_ERR_INVALID_ARGUMENT, bad
    assert call(N=0) == slq.SLQ_OK
    assert call() in (slq.SLQ_OK, slq.SLQ_ERR_UNSUPPORTED_DEVICE)
