"""GPU parity: slq_grid_noise against oracle.grid_noise.

Per 128-group the kernel gives gamma = 2 max|w| / (max w - min w) and the
rounding SSE of the asymmetric grid over [min w, max w] and of the symmetric
grid over [-max|w|, max|w|] (the gamma^2 law of the wispaper.ai blog and the
gist.science summary, Methodology section 1).  Tolerances follow from the
kernel's arithmetic:

  * gamma is computed from the same binary64 operations as the oracle and
    rounded once to binary32: bit-exact against float32(oracle).
  * each error is one rounding of an exact binary32 fma (L e = L d - i R), or
    for long asymmetric spans e with the step carried as two binary32 terms
    (relative error about 2^-23 per e^2), summed in binary32 over 128 terms
    (at most 34 roundings on a path, most terms far smaller than the sum): |sse - sse_ref| <= 1e-5 sse_ref plus an
    absolute floor of 1e-9 * 128 step^2 (1.2e-8 of a typical group's SSE),
    which covers groups whose points sit on the grid and whose exact SSE is
    zero.  Results below the binary32 range compare as float32(oracle).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import to_dev_u16, to_host_u16

pytestmark = pytest.mark.gpu
BITS = [2, 3, 4, 5, 6, 7, 8]
RTOL = 1e-5
FLOOR = 1e-9 * 128


def _gpu(w_bits: np.ndarray, bits: int):
    W = to_dev_u16(w_bits)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    g, a, s = slq.grid_noise(W, bits, flags=flags)
    torch.cuda.synchronize()
    return g.cpu().numpy(), a.cpu().numpy(), s.cpu().numpy(), int(flags.item())


def _steps(w_bits: np.ndarray, bits: int):
    w = synth.bf16_bits_to_f32(w_bits).astype(np.float64)
    N, K = w.shape
    g = w.reshape(N, K // 128, 128)
    L = 2**bits - 1
    return (g.max(-1) - g.min(-1)) / L, 2 * np.abs(g).max(-1) / L


def _check(w_bits: np.ndarray, bits: int, got=None, skip=None):
    if got is None:
        got = _gpu(w_bits, bits)
    gamma, sa, ss, _ = got
    rg, ra, rs = oracle.grid_noise(w_bits, bits)
    step_a, step_s = _steps(w_bits, bits)
    keep = np.ones(rg.shape, bool) if skip is None else ~skip
    with np.errstate(over="ignore"):
        assert np.array_equal(gamma[keep].view(np.uint32), rg[keep].astype(np.float32).view(np.uint32)), \
            "gamma differs"
        for name, mine, ref, step in (("sse_asym", sa, ra, step_a), ("sse_sym", ss, rs, step_s)):
            ref32 = ref.astype(np.float32).astype(np.float64)
            m = mine.astype(np.float64)
            inf = np.isinf(ref32) & keep
            assert np.array_equal(m[inf], ref32[inf]), f"{name}: overflow differs"
            fin = keep & ~inf
            tol = RTOL * np.abs(ref32[fin]) + FLOOR * step[fin] ** 2 + 1e-44
            err = np.abs(m[fin] - ref32[fin])
            worst = np.argmax(err - tol) if err.size else 0
            assert np.all(err <= tol), (name, err.flat[worst], ref32[fin].flat[worst])


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("N,K", [(1, 128), (3, 384), (17, 1024), (100, 4096), (33, 128 * 13)])
def test_grid_noise_matches_oracle(bits, N, K):
    w = synth.weights(N, K, seed=20 * N + K + bits)
    got = _gpu(w, bits)
    assert got[3] == 0
    _check(w, bits, got)


def _adversarial(K=128 * 14) -> np.ndarray:
    rng = np.random.default_rng(7)
    v = np.zeros(K)
    v[0:128] = 0.0                                   # all zero: gamma 1, both SSE 0
    v[128:256] = 0.75                                # constant > 0
    v[256:384] = -3.0                                # constant < 0
    v[384:512] = np.linspace(1.0, 2.0, 128)          # min > 0 (gamma = 4)
    v[512:640] = np.linspace(-2.0, -1.0, 128)        # max < 0
    v[640:768] = np.arange(128) * 0.5 - 20.0         # points on and between grid points
    v[768:896] = np.linspace(0, 1e-12, 128)          # tiny range
    v[896:1024] = rng.normal(0, 1e-3, 128) * (rng.random(128) < 0.01) * 1000
    v[1024:1152] = np.where(rng.random(128) < 0.5, -0.0, 0.0)   # signed zeros
    v[1152:1280] = rng.normal(0, 1, 128) * 2.0**-130           # bf16 subnormals
    v[1280:1408] = np.linspace(-2.5, 12.5, 128)
    v[1408:1536] = rng.normal(3, 0.01, 128)          # narrow range far from 0
    v[1536:1664] = rng.normal(0, 1, 128) * 1e18      # SSE near the top of binary32
    v[1664:1792] = np.linspace(-3e38, 3e38, 128)     # SSE beyond binary32 (inf)
    rows = [v, -v, rng.standard_normal(K) * np.exp(rng.uniform(-20, 20, K))]
    return synth.to_bf16_bits(np.array(rows))


@pytest.mark.parametrize("bits", BITS)
def test_adversarial_groups(bits):
    w = _adversarial()
    got = _gpu(w, bits)
    assert got[3] == 0
    _check(w, bits, got)


@pytest.mark.parametrize("bits", [2, 8])
def test_nonfinite_flag(bits):
    K = 384
    v = synth.weights(2, K, seed=3).copy()
    v[0, 5] = synth.to_bf16_bits(np.array([np.inf]))[0]
    v[1, 300] = synth.to_bf16_bits(np.array([np.nan]))[0]
    got = _gpu(v, bits)
    assert got[3] == slq.SLQ_FLAG_NONFINITE
    skip = np.zeros((2, 3), bool)
    skip[0, 0] = skip[1, 2] = True
    _check(v, bits, got, skip=skip)   # the finite groups are still exact


def test_empty_rows_launch_nothing():
    W = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    g, a, s = slq.grid_noise(W, 4)
    assert g.shape == a.shape == s.shape == (0, 2)


@pytest.mark.parametrize("N,K,bits", [(28672, 8192, 4), (8192, 28672, 2), (4096, 4096, 8)])
def test_full_size_sampled_rows(N, K, bits):
    W = synth.weights_torch(N, K, seed=2000 + bits)
    gamma, sa, ss = slq.grid_noise(W, bits)
    rows = np.sort(np.random.default_rng(N + K).choice(N, size=40, replace=False))
    rows = np.concatenate([[0, N - 1], rows])
    idx = torch.from_numpy(rows).cuda()
    w_rows = to_host_u16(W.index_select(0, idx))
    got = tuple(t.index_select(0, idx).cpu().numpy() for t in (gamma, sa, ss)) + (0,)
    _check(w_rows, bits, got)
    # Whole-layer properties at full size: gamma >= 1 (2 max|w| >= max w - min w),
    # and no weight is farther than half a step from its grid's nearest point.
    assert float(gamma.min()) >= 1.0
    g = W.view(N, K // 128, 128).float()
    L = 2**bits - 1
    step_a = (g.amax(-1) - g.amin(-1)) / L
    step_s = 2 * g.abs().amax(-1) / L
    assert bool(torch.all(sa <= 32 * step_a**2 * (1 + 1e-3)))
    assert bool(torch.all(ss <= 32 * step_s**2 * (1 + 1e-3)))
