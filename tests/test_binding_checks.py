"""The Python binding refuses what it cannot hand to the library safely.

The C ABI takes raw pointers, so the binding is where a tensor's device,
dtype, shape and layout are checked.  Each case here fails before any CUDA
call, so it runs on a machine without a GPU.
"""
import pytest
import torch

import weight_only_mixed_b200 as slq


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_quantize_refuses_host_tensor():
    with pytest.raises(ValueError, match="CUDA"):
        slq.quantize(_bf16(4, 128), 4)


def test_quantize_refuses_wrong_dtype_and_layout():
    with pytest.raises(TypeError, match="dtype"):
        slq.quantize(torch.zeros((4, 128), dtype=torch.float16), 4)
    with pytest.raises(ValueError, match="contiguous"):
        slq.quantize(_bf16(128, 8).t(), 4)
    with pytest.raises(ValueError, match="dimensions"):
        slq.quantize(_bf16(4, 2, 128), 4)


@pytest.mark.parametrize("bits,K", [(1, 128), (9, 128), (4, 100)])
def test_quantize_refuses_bits_and_ragged_k(bits, K):
    with pytest.raises(ValueError, match="bits"):
        slq.quantize(_bf16(4, K), bits)


def test_weight_record_is_checked_when_made():
    N, K, b = 8, 256, 4
    good = dict(packed=torch.zeros((N, K * b // 32), dtype=torch.int32),
                scales=torch.zeros((N, K // 128), dtype=torch.float16),
                zeros=torch.zeros((N, K // 128), dtype=torch.uint8), bits=b, N=N, K=K)
    with pytest.raises(ValueError, match="CUDA"):
        slq.QuantizedWeight(**good)
    with pytest.raises(ValueError, match="shape"):
        slq.QuantizedWeight(**dict(good, packed=torch.zeros((N, 1), dtype=torch.int32)))
    with pytest.raises(TypeError, match="dtype"):
        slq.QuantizedWeight(**dict(good, scales=torch.zeros((N, K // 128), dtype=torch.float32)))
    with pytest.raises(TypeError, match="dtype"):
        slq.QuantizedWeight(**dict(good, zeros=torch.zeros((N, K // 128), dtype=torch.int8)))
    with pytest.raises(ValueError, match="bits"):
        slq.QuantizedWeight(**dict(good, bits=9))
    with pytest.raises(ValueError, match="bits"):
        slq.QuantizedWeight(**dict(good, K=200))


def test_gemm_refuses_bad_arguments():
    with pytest.raises(ValueError, match="path"):
        slq.gemm(_bf16(1, 128), None, path="fast")
    with pytest.raises(TypeError, match="QuantizedWeight"):
        slq.gemm(_bf16(1, 128), None)
    with pytest.raises(TypeError, match="dtype"):
        slq.gemm(torch.zeros((1, 128)), None)
    with pytest.raises(ValueError, match="contiguous"):
        slq.gemm(_bf16(128, 2).t(), None)


def test_gemm_group_refuses_empty_and_mismatched():
    with pytest.raises(ValueError, match="no layers"):
        slq.gemm_group([])
    with pytest.raises(ValueError, match="outputs"):
        slq.gemm_group([(_bf16(1, 128), None)], outs=[])
    with pytest.raises(TypeError, match="QuantizedWeight"):
        slq.gemm_group([(_bf16(1, 128), None)])


def test_ear_kl_refuses_bad_arguments():
    with pytest.raises(ValueError, match="CUDA"):
        slq.ear_kl(_bf16(2, 64), _bf16(2, 64))
    with pytest.raises(TypeError, match="dtype"):
        slq.ear_kl(torch.zeros((2, 64)), _bf16(2, 64))
    with pytest.raises(ValueError, match="dimensions"):
        slq.ear_kl(_bf16(64), _bf16(64))
    with pytest.raises(ValueError, match="shape"):
        slq.ear_kl(_bf16(2, 64), _bf16(2, 32))
    with pytest.raises(ValueError, match="contiguous"):
        slq.ear_kl(_bf16(64, 2).t(), _bf16(2, 64))


def test_weight_record_is_immutable():
    assert slq.QuantizedWeight.__dataclass_params__.frozen


def test_flags_and_output_dtype_checks():
    with pytest.raises(TypeError, match="dtype"):
        slq.quantize(_bf16(4, 128), 4, flags=torch.zeros(1, dtype=torch.float32))
    with pytest.raises(ValueError, match="32-bit word"):
        slq.quantize(_bf16(4, 128), 4, flags=torch.zeros(0, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        slq.quantize(_bf16(4, 128), 4, flags=torch.zeros(1, dtype=torch.int32))
