"""GPU test of slq_gemm_decode_static, the decode GEMM that allocates nothing.

Some callers cannot hand the library a workspace: a plugin inside a host engine
that owns all device memory, or a decode loop that must not call cudaMalloc
once it runs.  For them the library keeps the split-K scratch in a fixed
per-device array.  This file checks, through the C ABI, that the call gives
the same result as slq_gemm with a caller workspace, on two calls in a row,
and that layers too large for the array are refused.  It is collected last so
that a stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import weight_only_mixed_b200 as slq
from gpu_util import gemm_errors

pytestmark = pytest.mark.gpu
MAX_TOL = 1e-2
FROB_TOL = 4e-3


def _static_call(X, qw, y, dtype):
    L = slq.lib()
    return L.slq_gemm_decode_static(
        ctypes.c_void_p(X.data_ptr()), X.shape[0], qw.N, qw.K, qw.bits,
        ctypes.c_void_p(qw.packed.data_ptr()), ctypes.c_void_p(qw.scales.data_ptr()),
        ctypes.c_void_p(qw.zeros.data_ptr()), ctypes.c_void_p(y.data_ptr()), dtype, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("N,K,bits,M", [(4096, 4096, 5, 16), (12288, 4096, 4, 1), (1024, 8192, 8, 7),
                                        (300, 128 * 35, 3, 4)])
def test_static_matches_workspace_call_twice(N, K, bits, M):
    assert slq.gemm_workspace_bytes(M, N, K, bits) <= slq.DECODE_STATIC_SCRATCH_BYTES
    qw = slq.quantize(synth.weights_torch(N, K, seed=4100 + bits), bits)
    X = synth.activations_torch(M, K, seed=4200 + M)
    ref = slq.gemm(X, qw, out_dtype=torch.float32, path="decode").double().cpu().numpy()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _static_call(X, qw, y, slq.SLQ_DTYPE_F32) == slq.SLQ_OK
        torch.cuda.synchronize()
        mx, fro = gemm_errors(y.cpu().numpy(), ref)
        assert mx <= MAX_TOL and fro <= FROB_TOL, (mx, fro)
    yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _static_call(X, qw, yb, slq.SLQ_DTYPE_BF16) == slq.SLQ_OK
    torch.cuda.synchronize()
    mx, fro = gemm_errors(yb.float().cpu().numpy(), ref)
    assert fro <= FROB_TOL, fro


def test_static_refuses_oversize_and_large_m():
    # A layer whose split-K scratch would exceed the fixed array is refused
    # before anything is launched; so is a batch above the decode range.
    N, K, bits = 131072, 8192, 2
    assert slq.gemm_workspace_bytes(8, N, K, bits) > slq.DECODE_STATIC_SCRATCH_BYTES
    L = slq.lib()
    fake = 0x7f0000100000
    rc = L.slq_gemm_decode_static(fake, 8, N, K, bits, fake + (1 << 32), fake + (2 << 32),
                                  fake + (3 << 32), fake + (4 << 32), 0, None, None)
    assert rc == slq.SLQ_ERR_INVALID_ARGUMENT
    rc = L.slq_gemm_decode_static(fake, 17, 64, 256, 4, fake + (1 << 32), fake + (2 << 32),
                                  fake + (3 << 32), fake + (4 << 32), 0, None, None)
    assert rc == slq.SLQ_ERR_INVALID_ARGUMENT
