"""GPU parity: slq_quantize against the oracle, bit-exact (codes, scales,
zeros, flags), on small ragged shapes, adversarial groups and sampled rows of
the full-size layers."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import Guarded, to_dev_u16, to_host_u16, to_host_u32

pytestmark = pytest.mark.gpu
BITS = [2, 3, 4, 5, 6, 7, 8]


def _gpu_quantize(w_bits: np.ndarray, bits: int):
    N, K = w_bits.shape
    W = to_dev_u16(w_bits)
    packed = Guarded((N, K * bits // 32), torch.int32)
    scales = Guarded((N, K // 128), torch.float16)
    zeros = Guarded((N, K // 128), torch.uint8)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    qw = slq.QuantizedWeight(packed.t, scales.t, zeros.t, bits, N, K)
    slq.quantize(W, bits, out=qw, flags=flags)
    torch.cuda.synchronize()
    assert packed.intact() and scales.intact() and zeros.intact()
    return (to_host_u32(qw.packed), to_host_u16(qw.scales), qw.zeros.cpu().numpy(),
            int(flags.item()))


def _assert_same(w_bits, bits):
    got = _gpu_quantize(w_bits, bits)
    want = oracle.quantize(w_bits, bits)
    assert np.array_equal(got[1], want[1]), "scales differ"
    assert np.array_equal(got[2], want[2]), "zeros differ"
    assert np.array_equal(got[0], want[0]), "packed codes differ"
    assert got[3] == want[3], "flags differ"


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N,K", [(1, 128), (3, 384), (17, 1024), (100, 4096), (33, 128 * 13)])
def test_quantize_matches_oracle(bits, N, K):
    _assert_same(synth.weights(N, K, seed=10 * N + K + bits), bits)


def _adversarial(K=128 * 12) -> np.ndarray:
    rng = np.random.default_rng(99)
    rows = []
    v = np.zeros(K)
    v[0:128] = 0.0                                   # all zero
    v[128:256] = 0.75                                # constant > 0
    v[256:384] = -3.0                                # constant < 0
    v[384:512] = np.linspace(1.0, 2.0, 128)          # min > 0
    v[512:640] = np.linspace(-2.0, -1.0, 128)        # max < 0
    v[640:768] = np.arange(128) * 0.5 - 20.0         # many exact ties
    v[768:896] = np.linspace(0, 1e-12, 128)          # step below fp16 range
    v[896:1024] = rng.normal(0, 1e-3, 128) * (rng.random(128) < 0.01) * 1000
    v[1024:1152] = np.where(rng.random(128) < 0.5, -0.0, 0.0)   # signed zeros
    v[1152:1280] = rng.normal(0, 1, 128) * 2.0**-130           # bf16 subnormals
    v[1280:1408] = np.linspace(-2.5, 12.5, 128)      # zero-point tie
    v[1408:1536] = rng.normal(3, 0.01, 128)          # narrow range far from 0
    rows.append(v)
    rows.append(-v)
    rows.append(rng.standard_normal(K) * np.exp(rng.uniform(-20, 20, K)))
    return synth.to_bf16_bits(np.array(rows))


@pytest.mark.parametrize("bits", BITS)
def test_adversarial_groups(bits):
    _assert_same(_adversarial(), bits)


@pytest.mark.parametrize("bits", [2, 4, 7])
def test_flags(bits):
    K = 256
    v = np.zeros((2, K))
    v[0, :128] = np.linspace(-3e38, 3e38, 128)  # range beyond fp16: overflow flag
    _assert_same(synth.to_bf16_bits(v), bits)
    v[1, 200] = np.inf
    got = _gpu_quantize(synth.to_bf16_bits(v), bits)
    assert got[3] & slq.SLQ_FLAG_NONFINITE and got[3] & slq.SLQ_FLAG_SCALE_OVERFLOW


@pytest.mark.parametrize("N,K,bits", [(28672, 8192, 6), (8192, 28672, 6), (12288, 4096, 4),
                                      (1024, 4096, 8), (8192, 8192, 2), (8192, 8192, 3)])
def test_full_size_sampled_rows(N, K, bits):
    W = synth.weights_torch(N, K, seed=1000 + bits)
    qw = slq.quantize(W, bits)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(N + K + bits).choice(N, size=48, replace=False))
    rows = np.concatenate([[0, N - 1], rows])
    idx = torch.from_numpy(rows).cuda()
    w_rows = to_host_u16(W.index_select(0, idx))
    want = oracle.quantize(w_rows, bits)
    assert np.array_equal(to_host_u16(qw.scales.index_select(0, idx)), want[1])
    assert np.array_equal(qw.zeros.index_select(0, idx).cpu().numpy(), want[2])
    assert np.array_equal(to_host_u32(qw.packed.index_select(0, idx)), want[0])


def _near_tie_groups(bits: int, n_groups: int = 96, seed: int = 0) -> np.ndarray:
    """Groups whose elements sit exactly on half-integer multiples of the step,
    or one bf16 ulp to either side: the cases where a quotient computed any
    other way than the IEEE division would round differently."""
    rng = np.random.default_rng(seed + bits)
    maxq = 2**bits - 1
    rows = []
    for _ in range(n_groups):
        e = int(rng.integers(-12, 5))
        s = 2.0**e
        k = rng.integers(0, min(maxq, 127), size=126)
        v = (k + 0.5) * s
        bits16 = synth.to_bf16_bits(v)
        nudge = rng.integers(-1, 2, size=126).astype(np.int32)  # -1, 0, +1 ulp
        bits16 = (bits16.astype(np.int32) + nudge).astype(np.uint16)
        vals = synth.bf16_bits_to_f32(bits16).astype(np.float64)
        g = np.concatenate([[0.0, maxq * s], vals])  # pins the range: scale = s exactly
        rows.append(g)
    return synth.to_bf16_bits(np.array(rows).reshape(1, -1))


@pytest.mark.parametrize("bits", BITS)
def test_near_ties_are_bit_exact(bits):
    _assert_same(_near_tie_groups(bits), bits)
