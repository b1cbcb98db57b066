"""GPU parity: slq_gptq against oracle.gptq, bit for bit.

GPTQ (the pages' encoder: GitHub README, "Pipeline" and "1. Quantize";
Frantar et al.) decides each code from weights that earlier columns have
moved, so a change in the last bit of any intermediate could flip a code at a
near-tie.  The kernels form every value with the same sequence of correctly
rounded binary64 operations as the oracle's definition (binary32 for the
encode decisions), so the codes, scales, zeros and flags must be identical,
not merely close.  Larger layers, beyond the oracle's reach in a test, are
checked through properties that hold exactly at any size: rows are encoded
independently (a subset of rows gives the same bits), and a diagonal X^T X
reduces GPTQ to the RTN encode.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import to_dev_u16, to_host_u16, to_host_u32

pytestmark = pytest.mark.gpu


def _gpu(wb, xb, bits, damp=0.01):
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = slq.gptq(to_dev_u16(wb), to_dev_u16(xb), bits, damp=damp, flags=flags)
    torch.cuda.synchronize()
    return to_host_u32(q.packed), to_host_u16(q.scales), q.zeros.cpu().numpy(), int(flags.item())


def _assert_same(got, want):
    assert np.array_equal(got[1], want[1]), "scales differ"
    assert np.array_equal(got[2], want[2]), "zeros differ"
    assert np.array_equal(got[0], want[0]), "codes differ"
    assert got[3] == want[3], "flags differ"


@pytest.mark.parametrize("N,K,T,bits", [(64, 256, 96, 4), (33, 384, 200, 3), (40, 512, 128, 2),
                                        (17, 256, 64, 5), (20, 384, 150, 6), (9, 512, 300, 7),
                                        (24, 1024, 256, 8), (16, 1024, 512, 4)])
def test_gptq_matches_oracle(N, K, T, bits):
    wb = synth.weights(N, K, seed=300 + bits + N)
    xb = synth.calibration(T, K, seed=400 + bits + K)
    _assert_same(_gpu(wb, xb, bits), oracle.gptq(wb, xb, bits))


def test_dead_inputs_constant_groups_and_damping():
    # T > K, so that X^T X is positive definite even without damping.
    N, K, T, bits = 12, 384, 512, 4
    wb = synth.weights(N, K, seed=7).copy()
    wb[3, 128:256] = synth.to_bf16_bits(np.full(128, 0.25))   # constant group
    wb[5, 0:128] = 0                                          # all-zero group
    xb = synth.calibration(T, K, seed=8).copy()
    xb[:, 5] = 0                                              # an input that is always zero
    xb[:, 300:302] = 0
    for damp in (0.0, 0.01, 0.5):
        _assert_same(_gpu(wb, xb, bits, damp), oracle.gptq(wb, xb, bits, damp))


def test_singular_hessian_is_flagged():
    # Fewer calibration rows than inputs and no damping: X^T X is singular, the
    # definition stops at a non-positive Cholesky pivot, and the kernel raises
    # SLQ_FLAG_NOT_POSITIVE_DEFINITE at the same pivot.
    wb = synth.weights(8, 256, seed=70)
    xb = synth.calibration(16, 256, seed=71)
    with pytest.raises(ValueError):
        oracle.gptq(wb, xb, 4, damp=0.0)
    assert _gpu(wb, xb, 4, damp=0.0)[3] & slq.SLQ_FLAG_NOT_POSITIVE_DEFINITE


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_diagonal_hessian_is_rtn(bits):
    # Nothing to spread the error over: GPTQ is the RTN encode (slq_quantize).
    K = 512
    wb = synth.weights(40, K, seed=50 + bits)
    d = 2.0 ** np.random.default_rng(bits).integers(-2, 3, size=K)
    xb = synth.to_bf16_bits(np.diag(d))
    got = _gpu(wb, xb, bits)
    rtn = slq.quantize(to_dev_u16(wb), bits)
    assert np.array_equal(got[0], to_host_u32(rtn.packed))
    assert np.array_equal(got[1], to_host_u16(rtn.scales))
    assert np.array_equal(got[2], rtn.zeros.cpu().numpy())


@pytest.mark.parametrize("N,K,T,bits", [(1024, 4096, 512, 4), (512, 2048, 256, 3)])
def test_large_layer_rows_are_independent(N, K, T, bits):
    # Each row's encode depends only on that row and on X: encoding a subset
    # of rows gives the same bits as those rows of the whole layer.
    W = synth.weights_torch(N, K, seed=60 + bits)
    X = to_dev_u16(synth.calibration(T, K, seed=61 + bits))
    full = slq.gptq(W, X, bits)
    rows = torch.tensor([0, 1, 7, N // 2, N - 1], device="cuda")
    part = slq.gptq(W.index_select(0, rows).contiguous(), X, bits)
    torch.cuda.synchronize()
    for a, b in ((full.packed, part.packed), (full.scales, part.scales), (full.zeros, part.zeros)):
        assert torch.equal(a.index_select(0, rows), b)
    # And GPTQ lowers the layer's output error on the calibration rows below RTN's.
    rtn = slq.quantize(W, bits)
    xf = X.float()

    def out_err(q):
        g = torch.arange(K, device="cuda") // 128
        codes = _unpack(q.packed, K, bits).float()
        deq = q.scales.float()[:, g] * (codes - q.zeros.float()[:, g])
        return float(((xf @ (W.float() - deq).T) ** 2).sum())
    assert out_err(full) < 0.5 * out_err(rtn)


def _unpack(packed, K, bits):
    words = packed.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    k = torch.arange(K, device=packed.device)
    pos = k * bits
    lo = words[:, pos // 32] >> (pos % 32)
    hi = torch.where((pos % 32 + bits) > 32, words[:, torch.clamp(pos // 32 + 1, max=words.shape[1] - 1)]
                     << (32 - pos % 32), torch.zeros_like(lo))
    return (lo | hi) & ((1 << bits) - 1)


def test_empty_layer():
    W = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    X = to_dev_u16(synth.calibration(8, 256, seed=1))
    with pytest.raises(ValueError):
        slq.gptq(W, X, 4)  # QuantizedWeight needs N >= 1; the C entry returns OK for N = 0
    L = slq.lib()
    assert L.slq_gptq(None, 0, 256, 4, None, 8, 0.01, None, None, None, None, 0, None, None) == slq.SLQ_OK
