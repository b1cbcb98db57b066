"""GPU parity: slq_gemm against the oracle's binary64 GEMM.

Tolerance (the library's contract): on the fp32 output,
max |y - y_ref| <= 1e-2 * rms(y_ref); on the bf16 output, relative Frobenius
error <= 4e-3; and the bf16 output equals round-to-nearest-even of the fp32
output bit for bit (same kernel, same reduction order).  One-hot rows of X
must reproduce the dequantized weights exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import Guarded, bf16_rn_of_f32, gemm_errors, to_dev_u16, to_host_u16

pytestmark = pytest.mark.gpu
BITS = [2, 3, 4, 5, 6, 7, 8]
MAX_TOL = 1e-2
FROB_TOL = 4e-3


def _layer(N, K, bits, seed):
    w = synth.weights(N, K, seed=seed)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    qw = slq.QuantizedWeight(
        packed=torch.from_numpy(packed.view(np.int32).copy()).cuda(),
        scales=to_dev_u16(scales, torch.float16),
        zeros=torch.from_numpy(zeros.copy()).cuda(), bits=bits, N=N, K=K)
    return (packed, scales, zeros), qw


def _run(x_bits, qw, path):
    M = x_bits.shape[0]
    X = to_dev_u16(x_bits)
    y32 = Guarded((M, qw.N), torch.float32)
    y16 = Guarded((M, qw.N), torch.bfloat16)
    slq.gemm(X, qw, out=y32.t, path=path)
    slq.gemm(X, qw, out=y16.t, path=path)
    torch.cuda.synchronize()
    assert y32.intact() and y16.intact()
    return y32.t.cpu().numpy(), to_host_u16(y16.t)


def _check(x_bits, host_layer, qw, path):
    packed, scales, zeros = host_layer
    y_ref = oracle.gemm(x_bits, packed, scales, zeros, qw.K, qw.bits)
    y32, y16 = _run(x_bits, qw, path)
    mx, _ = gemm_errors(y32, y_ref)
    _, fro = gemm_errors(synth.bf16_bits_to_f32(y16), y_ref)
    assert mx <= MAX_TOL, mx
    assert fro <= FROB_TOL, fro
    assert np.array_equal(y16, bf16_rn_of_f32(y32))
    return mx


DECODE_SHAPES = [(1, 1, 128), (2, 7, 256), (3, 33, 384), (5, 100, 1152), (8, 1000, 1024),
                 (9, 64, 2048), (15, 48, 128 * 9), (16, 256, 4096), (4, 300, 128 * 35)]


@pytest.mark.parametrize("path", ["gemv", "decode"])
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_decode_matches_oracle(bits, M, N, K, path):
    host, qw = _layer(N, K, bits, seed=M * 7 + N + K + bits)
    x = synth.activations(M, K, seed=M + K)
    _check(x, host, qw, path)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("path", ["gemv", "decode", "tiled"])
def test_one_hot_rows_are_exact(bits, path):
    N, K = 40, 512
    host, qw = _layer(N, K, bits, seed=77 + bits)
    ks = np.array([0, 1, 31, 32, 127, 128, 255, 300, 511, 64, 65, 96, 97, 200, 400, 401])
    x = np.zeros((len(ks), K))
    x[np.arange(len(ks)), ks] = 1.0
    y32, _ = _run(synth.to_bf16_bits(x), qw, path)
    wdq = oracle.dequantize(*host, K, bits)
    assert np.array_equal(y32.astype(np.float64), wdq[:, ks].T)


def _sampled_layer_check(N, K, bits, Ms, path="auto", n_sample=192):
    """Full-size layer on the GPU; oracle on all M rows for a sample of
    output columns (rows of W are independent)."""
    W = synth.weights_torch(N, K, seed=5000 + N + bits)
    qw = slq.quantize(W, bits)
    cols = np.sort(np.random.default_rng(N + K + bits).choice(N, size=min(N, n_sample), replace=False))
    cols = np.unique(np.concatenate([[0, N - 1], cols]))
    idx = torch.from_numpy(cols).cuda()
    from gpu_util import to_host_u32
    sub = (to_host_u32(qw.packed.index_select(0, idx)), to_host_u16(qw.scales.index_select(0, idx)),
           qw.zeros.index_select(0, idx).cpu().numpy())
    for M in Ms:
        X = synth.activations_torch(M, K, seed=6000 + M)
        y32 = slq.gemm(X, qw, out_dtype=torch.float32, path=path)
        y16 = slq.gemm(X, qw, out_dtype=torch.bfloat16, path=path)
        torch.cuda.synchronize()
        y_ref = oracle.gemm(to_host_u16(X), *sub, K, bits)
        g32 = y32.index_select(1, idx).cpu().numpy()
        g16 = to_host_u16(y16.index_select(1, idx))
        mx, _ = gemm_errors(g32, y_ref)
        _, fro = gemm_errors(synth.bf16_bits_to_f32(g16), y_ref)
        assert mx <= MAX_TOL and fro <= FROB_TOL, (M, mx, fro)
        assert np.array_equal(g16, bf16_rn_of_f32(g32))


def test_config0_single_linear_full():
    host, qw = _layer(1024, 1024, 4, seed=synth.SEED_WEIGHTS)
    x = synth.activations(8, 1024, seed=synth.SEED_X)
    _check(x, host, qw, "auto")


QWEN3_8B = [(4096, 4096, 5), (1024, 4096, 8), (1024, 4096, 8), (4096, 4096, 5),
            (12288, 4096, 4), (12288, 4096, 4), (4096, 12288, 4)]
LLAMA_70B = [(8192, 8192, 7), (1024, 8192, 8), (1024, 8192, 8), (8192, 8192, 7),
             (28672, 8192, 6), (28672, 8192, 6), (8192, 28672, 6)]


@pytest.mark.parametrize("N,K,bits", sorted(set(QWEN3_8B)))
def test_qwen3_8b_block_decode(N, K, bits):
    _sampled_layer_check(N, K, bits, Ms=[1, 4, 16])


@pytest.mark.parametrize("bits", BITS)
def test_sweep_8192_decode(bits):
    _sampled_layer_check(8192, 8192, bits, Ms=[1, 16], n_sample=96)


@pytest.mark.parametrize("N,K,bits", sorted(set(LLAMA_70B)))
def test_llama_70b_block_decode(N, K, bits):
    _sampled_layer_check(N, K, bits, Ms=[1, 16], n_sample=64)


# ---------------------------------------------------------------------------
# Tiled tensor-core path (TMA + dequant-to-smem + tcgen05.mma, TMEM accumulators)
# ---------------------------------------------------------------------------
TILED_SHAPES = [(17, 1, 128), (40, 130, 256), (64, 128, 384), (65, 257, 1024), (128, 100, 640),
                (129, 384, 512), (200, 64, 1152), (256, 256, 2048), (300, 200, 768), (1, 50, 256),
                (16, 129, 128 * 5)]


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("M,N,K", TILED_SHAPES)
def test_tiled_matches_oracle(bits, M, N, K):
    host, qw = _layer(N, K, bits, seed=M * 13 + N + K + bits)
    x = synth.activations(M, K, seed=M + K + 1)
    _check(x, host, qw, "tiled")


def _sampled_prefill_check(N, K, bits, Ms, n_rows=48, n_cols=160, path="auto"):
    W = synth.weights_torch(N, K, seed=7000 + N + bits)
    qw = slq.quantize(W, bits)
    del W
    from gpu_util import to_host_u32
    rng = np.random.default_rng(N + K + bits)
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(N, n_cols), replace=False)]))
    cidx = torch.from_numpy(cols).cuda()
    sub = (to_host_u32(qw.packed.index_select(0, cidx)), to_host_u16(qw.scales.index_select(0, cidx)),
           qw.zeros.index_select(0, cidx).cpu().numpy())
    for M in Ms:
        X = synth.activations_torch(M, K, seed=8000 + M)
        y32 = slq.gemm(X, qw, out_dtype=torch.float32, path=path)
        y16 = slq.gemm(X, qw, out_dtype=torch.bfloat16, path=path)
        torch.cuda.synchronize()
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, size=min(M, n_rows), replace=False)]))
        ridx = torch.from_numpy(rows).cuda()
        y_ref = oracle.gemm(to_host_u16(X.index_select(0, ridx)), *sub, K, bits)
        g32 = y32.index_select(0, ridx).index_select(1, cidx).cpu().numpy()
        g16 = to_host_u16(y16.index_select(0, ridx).index_select(1, cidx))
        mx, _ = gemm_errors(g32, y_ref)
        _, fro = gemm_errors(synth.bf16_bits_to_f32(g16), y_ref)
        assert mx <= MAX_TOL and fro <= FROB_TOL, (M, mx, fro)
        assert np.array_equal(g16, bf16_rn_of_f32(g32))


@pytest.mark.parametrize("bits", BITS)
def test_sweep_8192_prefill(bits):
    _sampled_prefill_check(8192, 8192, bits, Ms=[64, 256, 1024, 4096])


@pytest.mark.parametrize("N,K,bits", sorted(set(LLAMA_70B)))
def test_llama_70b_block_prefill(N, K, bits):
    _sampled_prefill_check(N, K, bits, Ms=[64, 2048])


# ---------------------------------------------------------------------------
# Decode kernel: stream-K split, workspace contract, determinism
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,bits,M", [(4096, 4096, 4, 16), (1024, 4096, 8, 1), (300, 128 * 37, 3, 5),
                                        (12288, 4096, 2, 4)])
def test_decode_workspace_left_zero_and_repeatable(N, K, bits, M):
    W = synth.weights_torch(N, K, seed=321 + bits)
    qw = slq.quantize(W, bits)
    X = synth.activations_torch(M, K, seed=322)
    need = slq.gemm_workspace_bytes(M, N, K, bits)
    ws = torch.zeros(max(need, 256) + 4096, dtype=torch.uint8, device="cuda")
    y1 = slq.gemm(X, qw, out_dtype=torch.float32, path="decode", workspace=ws)
    torch.cuda.synchronize()
    # Partial sums may stay behind; the per-tile counters must be zero again.
    ncnt = (N + 127) // 128
    assert int(ws[:4 * ncnt].count_nonzero()) == 0, "tile counters not reset"
    for _ in range(3):
        y2 = slq.gemm(X, qw, out_dtype=torch.float32, path="decode", workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    assert int(ws[:4 * ncnt].count_nonzero()) == 0


def test_decode_flags_stay_clear():
    N, K, bits = 2048, 8192, 5
    qw = slq.quantize(synth.weights_torch(N, K, seed=5), bits)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    for M in (1, 7, 16):
        slq.gemm(synth.activations_torch(M, K, seed=M), qw, flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0


@pytest.mark.parametrize("N,K,bits,M", [(8192, 8192, 5, 16), (4096, 12288, 4, 16), (8192, 8192, 8, 9)])
def test_decode_repeated_calls_identical(N, K, bits, M):
    """Twenty calls on one layer give identical bits, each on a freshly zeroed
    workspace and on a reused one (catches races on the staged buffers and on
    the cross-CTA partial sums)."""
    qw = slq.quantize(synth.weights_torch(N, K, seed=900 + bits), bits)
    X = synth.activations_torch(M, K, seed=901)
    need = slq.gemm_workspace_bytes(M, N, K, bits)
    ref = slq.gemm(X, qw, out_dtype=torch.float32, path="decode")
    reused = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    for i in range(20):
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda") if i % 2 else reused
        y = slq.gemm(X, qw, out_dtype=torch.float32, path="decode", workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int32), ref.view(torch.int32)), i


def test_decode_workspace_reused_across_layer_sizes():
    """One workspace serves layers of different N and K in any order: a
    layer's partial sums never land on another layer's tile counters."""
    layers = [(2048, 8192, 5, 7), (12288, 4096, 4, 1), (1024, 8192, 8, 16), (28672, 1024, 6, 3),
              (4096, 4096, 2, 16)]
    need = max(slq.gemm_workspace_bytes(M, N, K, b) for N, K, b, M in layers)
    shared = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for i, (N, K, b, M) in enumerate(layers):
            qw = slq.quantize(synth.weights_torch(N, K, seed=77 + i), b)
            X = synth.activations_torch(M, K, seed=78 + i)
            fresh = torch.zeros(need, dtype=torch.uint8, device="cuda")
            y_ref = slq.gemm(X, qw, out_dtype=torch.float32, path="decode", workspace=fresh)
            y = slq.gemm(X, qw, out_dtype=torch.float32, path="decode", workspace=shared)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int32), y_ref.view(torch.int32)), (rep, N, K, b, M)
