"""GPU parity of slq_gemm_group (several decode layers in one launch)
against the oracle, and against single-layer calls of the same kernel."""
import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_mixed_b200 as slq
from gpu_util import bf16_rn_of_f32, gemm_errors, to_dev_u16, to_host_u16, to_host_u32

pytestmark = pytest.mark.gpu
MAX_TOL = 1e-2
FROB_TOL = 4e-3


def _host_layer(N, K, bits, seed):
    w = synth.weights(N, K, seed=seed)
    packed, scales, zeros, _ = oracle.quantize(w, bits)
    qw = slq.QuantizedWeight(
        packed=torch.from_numpy(packed.view(np.int32).copy()).cuda(),
        scales=to_dev_u16(scales, torch.float16),
        zeros=torch.from_numpy(zeros.copy()).cuda(), bits=bits, N=N, K=K)
    return (packed, scales, zeros), qw


GROUPS = [
    [(33, 256, 5), (7, 384, 8), (100, 1152, 3)],
    [(1, 128, 2), (48, 1024, 4), (64, 2048, 6), (17, 640, 7), (200, 256, 8)],
    [(256, 4096, 5), (64, 4096, 8), (64, 4096, 8)],          # a QKV-like group
    [(40, 512, b) for b in range(2, 9)] + [(3, 128, 4)],       # 8 layers, every b
]


@pytest.mark.parametrize("M", [1, 5, 8, 16])
@pytest.mark.parametrize("gi", range(len(GROUPS)))
def test_group_matches_oracle(gi, M):
    layers = [_host_layer(N, K, b, seed=100 * gi + 7 * i + b) for i, (N, K, b) in enumerate(GROUPS[gi])]
    xs = [synth.activations(M, K, seed=M + K + i) for i, (N, K, b) in enumerate(GROUPS[gi])]
    items = [(to_dev_u16(x), qw) for x, (_, qw) in zip(xs, layers)]
    y32 = slq.gemm_group(items, out_dtype=torch.float32)
    y16 = slq.gemm_group(items, out_dtype=torch.bfloat16)
    y32b = slq.gemm_group(items, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for i, (x, (host, qw), a, b16, again) in enumerate(zip(xs, layers, y32, y16, y32b)):
        y_ref = oracle.gemm(x, *host, qw.K, qw.bits)
        g32 = a.cpu().numpy()
        mx, _ = gemm_errors(g32, y_ref)
        _, fro = gemm_errors(synth.bf16_bits_to_f32(to_host_u16(b16)), y_ref)
        assert mx <= MAX_TOL and fro <= FROB_TOL, (mx, fro)
        assert np.array_equal(to_host_u16(b16), bf16_rn_of_f32(g32))
        assert torch.equal(a, again)  # repeatable bit for bit
        single = slq.gemm(items[i][0], qw, out_dtype=torch.float32, path="gemv")
        rms = float(np.sqrt(np.mean(y_ref ** 2))) or 1.0
        assert float((single - a).abs().max()) <= 1e-5 * rms


def test_group_one_hot_rows_exact():
    K = 512
    layers = [_host_layer(40, K, b, seed=900 + b) for b in (3, 4, 8)]
    ks = np.array([0, 1, 31, 32, 127, 128, 255, 300, 511, 64, 65, 96, 97, 200, 400, 401])
    x = np.zeros((len(ks), K))
    x[np.arange(len(ks)), ks] = 1.0
    X = to_dev_u16(synth.to_bf16_bits(x))
    ys = slq.gemm_group([(X, qw) for _, qw in layers], out_dtype=torch.float32)
    torch.cuda.synchronize()
    for (host, qw), y in zip(layers, ys):
        wdq = oracle.dequantize(*host, K, qw.bits)
        assert np.array_equal(y.cpu().numpy().astype(np.float64), wdq[:, ks].T)


@pytest.mark.parametrize("M", [1, 16])
def test_qwen3_8b_fused_projections_sampled(M):
    """q, k, v (b5, b8, b8) in one launch and gate, up (b4) in another, at
    full size; the oracle on sampled output columns of each layer."""
    for shapes in ([(4096, 4096, 5), (1024, 4096, 8), (1024, 4096, 8)],
                   [(12288, 4096, 4), (12288, 4096, 4)]):
        qws = [slq.quantize(synth.weights_torch(N, K, seed=7000 + 10 * i + b), b)
               for i, (N, K, b) in enumerate(shapes)]
        xs = [synth.activations_torch(M, K, seed=8000 + i + M) for i, (N, K, b) in enumerate(shapes)]
        ys = slq.gemm_group(list(zip(xs, qws)), out_dtype=torch.float32)
        torch.cuda.synchronize()
        for i, ((N, K, b), qw, x, y) in enumerate(zip(shapes, qws, xs, ys)):
            cols = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(i + M).choice(N, 64, replace=False)]))
            idx = torch.from_numpy(cols).cuda()
            sub = (to_host_u32(qw.packed.index_select(0, idx)), to_host_u16(qw.scales.index_select(0, idx)),
                   qw.zeros.index_select(0, idx).cpu().numpy())
            y_ref = oracle.gemm(to_host_u16(x), *sub, K, b)
            mx, fro = gemm_errors(y.index_select(1, idx).cpu().numpy(), y_ref)
            assert mx <= MAX_TOL and fro <= FROB_TOL, (shapes[i], mx, fro)
