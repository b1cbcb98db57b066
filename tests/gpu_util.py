"""Helpers for the GPU tests: moving raw bf16/fp16 bit arrays to and from the
device, guard-banded output buffers, and the GEMM tolerance check."""
import numpy as np
import torch

GUARD = 4096  # bytes of sentinel before and after guarded outputs
SENTINEL = 0x5A


def to_dev_u16(bits: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    a = np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(a.copy()).view(dtype).cuda()


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_host_u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint32)


class Guarded:
    """A device buffer with sentinel bytes on both sides of the payload."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.raw[:GUARD] == SENTINEL).all()) and bool((self.raw[-GUARD:] == SENTINEL).all())


def gemm_errors(y: np.ndarray, y_ref: np.ndarray):
    """(max |y - y_ref| / rms(y_ref), ||y - y_ref||_F / ||y_ref||_F)."""
    d = y.astype(np.float64) - y_ref
    rms = np.sqrt(np.mean(y_ref ** 2))
    return float(np.abs(d).max() / rms), float(np.linalg.norm(d) / np.linalg.norm(y_ref))


def bf16_rn_of_f32(y32: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(y32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
