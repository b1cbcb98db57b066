"""GPU test of slq_gemm_decode_static, the decode GEMM that allocates nothing.

Some callers cannot hand the library a workspace: a plugin inside a host engine
that owns all device memory, or a decode loop that must not call cudaMalloc
once it runs.  For them the library keeps the split-K scratch in a fixed
per-device array.  This file checks, through the C ABI, that two calls in a
row match the oracle's binary64 GEMM within the library's tolerances (the
same bounds as every GEMM test: max |y - y_ref| <= 1e-2 rms on fp32 output,
relative Frobenius <= 4e-3 on bf16 output), give identical bits, agree with
the call that takes a caller workspace, and that layers too large for the
array are refused.  It is collected last so that a stop-at-first-failure run
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import bf16_rn_of_f32, gemm_errors, to_dev_u16, to_host_u16

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
def test_static_matches_oracle_twice(N, K, bits, M):
    assert slq.gemm_workspace_bytes(M, N, K, bits) <= slq.DECODE_STATIC_SCRATCH_BYTES
    # Weights quantized and packed by the oracle, activations seeded on the host.
    w = synth.weights(N, K, seed=4100 + bits)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    qw = slq.QuantizedWeight(packed=torch.from_numpy(packed.view(np.int32).copy()).cuda(),
                             scales=to_dev_u16(scales, torch.float16),
                             zeros=torch.from_numpy(zeros.copy()).cuda(), bits=bits, N=N, K=K)
    x = synth.activations(M, K, seed=4200 + M)
    X = to_dev_u16(x)
    y_ref = oracle.gemm(x, packed, scales, zeros, K, bits)
    outs = []
    for _ in range(2):
        y32 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        y16 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _static_call(X, qw, y32, slq.SLQ_DTYPE_F32) == slq.SLQ_OK
        assert _static_call(X, qw, y16, slq.SLQ_DTYPE_BF16) == slq.SLQ_OK
        torch.cuda.synchronize()
        g32, g16 = y32.cpu().numpy(), to_host_u16(y16)
        mx, _ = gemm_errors(g32, y_ref)
        _, fro = gemm_errors(synth.bf16_bits_to_f32(g16), y_ref)
        assert mx <= MAX_TOL, mx
        assert fro <= FROB_TOL, fro
        assert np.array_equal(g16, bf16_rn_of_f32(g32))
        outs.append(g32)
    assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))
    # The same kernel with a caller workspace gives the same bits.
    y_ws = slq.gemm(X, qw, out_dtype=torch.float32, path="decode").cpu().numpy()
    assert np.array_equal(outs[0].view(np.uint32), y_ws.view(np.uint32))


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
