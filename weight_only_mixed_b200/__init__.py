"""Python binding of libslq.so, the sm_100a library for the SLQ weight format.

This module only marshals arguments: it checks each tensor's dtype, shape,
layout and device, allocates outputs with PyTorch, passes raw device pointers
and the CUDA stream through the C ABI declared in ``include/slq.h``, and turns
status codes into exceptions.  Every
step of quantize, dequantize-GEMM and EAR/KL runs in the library's CUDA
kernels; there is no CPU path and no fallback.  If the library has not been
built, importing this package fails.

Format (pages on "Statistically-Lossless Quantization of Large Language
Models"): asymmetric INT-b, b in 2..8 per layer, group size 128 along K,
fp16 scale and uint8 zero point per group, codes packed LSB-first into one
bit stream per row (a 128-code group fills exactly 4b uint32 words).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libslq.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "slq.h")

GROUP = 128

SLQ_OK = 0
SLQ_ERR_INVALID_ARGUMENT = 1
SLQ_ERR_UNSUPPORTED_DEVICE = 2
SLQ_ERR_CUDA = 3
SLQ_ERR_TIMEOUT = 4

SLQ_DTYPE_BF16 = 0
SLQ_DTYPE_F32 = 1

SLQ_FLAG_NONFINITE = 1
SLQ_FLAG_SCALE_OVERFLOW = 2
SLQ_FLAG_TIMEOUT = 4
SLQ_FLAG_NOT_POSITIVE_DEFINITE = 8

SLQ_GEMM_AUTO = 0
SLQ_GEMM_DECODE = 1
SLQ_GEMM_TILED = 2
SLQ_GEMM_GEMV = 3

_PATHS = {"auto": SLQ_GEMM_AUTO, "decode": SLQ_GEMM_DECODE, "tiled": SLQ_GEMM_TILED,
          "gemv": SLQ_GEMM_GEMV}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python weight_only_mixed_b200/build.py` "
        "(nvcc, sm_100a).  There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int

_lib.slq_version.argtypes = []
_lib.slq_version.restype = _I
_lib.slq_status_string.argtypes = [_I]
_lib.slq_status_string.restype = ctypes.c_char_p
_lib.slq_packed_words.argtypes = [_I64, _I64, _I]
_lib.slq_packed_words.restype = ctypes.c_size_t
_lib.slq_gemm_select.argtypes = [_I64, _I64, _I64, _I]
_lib.slq_gemm_select.restype = _I
_lib.slq_quantize.argtypes = [_P, _I64, _I64, _I, _P, _P, _P, _P, _P]
_lib.slq_quantize.restype = _I
_SZ = ctypes.c_size_t
_lib.slq_gemm_workspace_bytes.argtypes = [_I64, _I64, _I64, _I]
_lib.slq_gemm_workspace_bytes.restype = _SZ
_lib.slq_gemm.argtypes = [_P, _I64, _I64, _I64, _I, _P, _P, _P, _P, _I, _P, _P]
_lib.slq_gemm.restype = _I
_lib.slq_gemm_ex.argtypes = [_P, _I64, _I64, _I64, _I, _P, _P, _P, _P, _I, _I, _P, _SZ, _P, _P]
_lib.slq_gemm_ex.restype = _I
_lib.slq_gemm_decode_static.argtypes = [_P, _I64, _I64, _I64, _I, _P, _P, _P, _P, _I, _P, _P]
_lib.slq_gemm_decode_static.restype = _I
_lib.slq_ear_kl.argtypes = [_P, _P, _I64, _I64, ctypes.c_float, _P, _P, _P, _P, _P, _P]
_lib.slq_ear_kl.restype = _I


class GemmLayer(ctypes.Structure):
    """slq_gemm_layer: one layer of slq_gemm_group."""
    _fields_ = [("X_bf16", _P), ("N", _I64), ("K", _I64), ("bits", _I), ("packed", _P),
                ("scales_f16", _P), ("zeros", _P), ("Y", _P)]


_lib.slq_gemm_group.argtypes = [ctypes.POINTER(GemmLayer), _I, _I64, _I, _P, _P]
_lib.slq_gemm_group.restype = _I
_lib.slq_gemm_group_max.argtypes = []
_lib.slq_gemm_group_max.restype = _I
_lib.slq_ear_kl_topk.argtypes = [_P, _P, _I64, _I64, _I, ctypes.c_float, _P, _P, _P, _P, _P, _P]
_lib.slq_ear_kl_topk.restype = _I
_lib.slq_ear_kl_topk_max.argtypes = []
_lib.slq_ear_kl_topk_max.restype = _I
_lib.slq_grid_noise.argtypes = [_P, _I64, _I64, _I, _P, _P, _P, _P, _P]
_lib.slq_grid_noise.restype = _I
_lib.slq_gptq.argtypes = [_P, _I64, _I64, _I, _P, _I64, ctypes.c_double, _P, _P, _P, _P, _SZ, _P, _P]
_lib.slq_gptq.restype = _I
_lib.slq_gptq_workspace_bytes.argtypes = [_I64, _I64]
_lib.slq_gptq_workspace_bytes.restype = _SZ


def lib() -> ctypes.CDLL:
    """The loaded C library (for callers that pass raw pointers)."""
    return _lib


def declared_symbols() -> list[str]:
    """Names of the functions include/slq.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(slq_[a-z0-9_]+)\s*\(", text)))


class SLQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def status_string(status: int) -> str:
    return _lib.slq_status_string(status).decode()


def version() -> int:
    return _lib.slq_version()


def packed_words(N: int, K: int, bits: int) -> int:
    return int(_lib.slq_packed_words(N, K, bits))


def gemm_select(M: int, N: int, K: int, bits: int) -> str:
    return {SLQ_GEMM_DECODE: "decode", SLQ_GEMM_TILED: "tiled",
            SLQ_GEMM_GEMV: "gemv"}[_lib.slq_gemm_select(M, N, K, bits)]


def gemm_workspace_bytes(M: int, N: int, K: int, bits: int) -> int:
    """Device workspace bytes slq_gemm needs on the current device."""
    return int(_lib.slq_gemm_workspace_bytes(M, N, K, bits))


# One zero-filled workspace per (device, stream), grown on demand.  The
# library leaves it zero after every call, and calls on one stream never
# overlap, so a stream can reuse its buffer.  Growing it allocates, so a
# CUDA-graph capture should be preceded by an eager call of the largest size.
_workspaces: dict = {}


def workspace_for(nbytes: int, stream=None):
    import torch
    if nbytes == 0:
        return None
    s = stream if stream is not None else torch.cuda.current_stream()
    key = (s.device.index, int(s.cuda_stream))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=s.device)
        _workspaces[key] = ws
    return ws


def _check(status: int, what: str):
    if status != SLQ_OK:
        raise SLQError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


# ---------------------------------------------------------------------------
# Argument checks.  The library reads and writes whole row-major arrays
# through raw device pointers, so a host tensor, a strided view, a wrong dtype
# or a short output would hand a kernel the wrong memory: every such case is
# refused here, before the call.  Each public call first checks types,
# shapes and layouts, then that everything is on one CUDA device (so the
# host-only tests reach every check).
# ---------------------------------------------------------------------------
def _word_dtypes():
    import torch
    u32 = getattr(torch, "uint32", None)
    return (torch.int32,) if u32 is None else (torch.int32, u32)


def _require(t, name: str, dtypes, shape=None, ndim=None):
    """`t` is a dense tensor of one of `dtypes` (and of `ndim` / `shape`)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dimensions, got shape {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (row-major, no strides)")
    return t


def _require_cuda(device=None, **tensors):
    """All `tensors` (None entries skipped) are CUDA tensors on one device,
    `device` if given; returns that device."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: must be a CUDA tensor (the library has no CPU path)")
        if device is None:
            device = t.device
        elif t.device != device:
            raise ValueError(f"{name} is on {t.device}, the call's inputs on {device}")
    return device


def _require_flags(flags):
    if flags is None:
        return
    _require(flags, "flags", _word_dtypes())
    if flags.numel() < 1:
        raise ValueError("flags: needs at least one 32-bit word")


def _require_weight(qw, name: str = "qw"):
    if not isinstance(qw, QuantizedWeight):
        raise TypeError(f"{name}: expected a QuantizedWeight, got {type(qw).__name__}")


def _require_bits_k(bits: int, K: int):
    if not 2 <= bits <= 8 or K < 1 or K % GROUP:
        raise ValueError(f"bits {bits}, K {K}: bits in 2..8, K a positive multiple of {GROUP}")


def _y_dtype(out_dtype):
    import torch
    dt = out_dtype or torch.bfloat16
    if dt not in (torch.bfloat16, torch.float32):
        raise TypeError(f"output dtype {dt}: the library writes bf16 or fp32")
    return dt


def _require_out(out, out_dtype, M: int, N: int, name: str = "out"):
    """The caller's output, if any: bf16 or fp32 [M, N], dense, of out_dtype."""
    import torch
    _y_dtype(out_dtype)
    if out is None:
        return
    _require(out, name, (torch.bfloat16, torch.float32), (M, N))
    if out_dtype is not None and out.dtype != out_dtype:
        raise TypeError(f"{name}: dtype {out.dtype}, but out_dtype is {out_dtype}")


def _require_x(X, qw, name: str = "X"):
    """bf16 X [M, K] for the packed layer qw; returns M."""
    import torch
    _require(X, name, (torch.bfloat16,), ndim=2)
    _require_weight(qw)
    M, K = X.shape
    if K != qw.K:
        raise ValueError(f"{name}: K = {K}, the layer's K = {qw.K}")
    if M < 1:
        raise ValueError(f"{name}: M = {M}")
    return M


def _stream_ptr(stream, device) -> int:
    """The call's stream: `stream`, or the current stream of the inputs' device."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(device)
    if s.device != device:
        raise ValueError(f"stream is on {s.device}, the call's inputs on {device}")
    return int(s.cuda_stream)


def _on(device):
    """Make the inputs' device current for the call (the library launches on
    the current device); a no-op when it already is."""
    import contextlib
    import torch
    if device.index is None or device.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(device)


@dataclasses.dataclass(frozen=True)
class QuantizedWeight:
    """Packed layer: codes [N, K*b/32] (int32 storage of uint32 words),
    scales [N, K/128] fp16, zeros [N, K/128] uint8, all dense CUDA tensors on
    one device.  Checked once here and immutable afterwards, so the calls
    that take it only check that its device matches theirs."""
    packed: "object"
    scales: "object"
    zeros: "object"
    bits: int
    N: int
    K: int

    def __post_init__(self):
        import torch
        _require_bits_k(self.bits, self.K)
        if self.N < 1:
            raise ValueError(f"N = {self.N}")
        _require(self.packed, "packed", _word_dtypes(), (self.N, self.K * self.bits // 32))
        _require(self.scales, "scales", (torch.float16,), (self.N, self.K // GROUP))
        _require(self.zeros, "zeros", (torch.uint8,), (self.N, self.K // GROUP))
        _require_cuda(packed=self.packed, scales=self.scales, zeros=self.zeros)

    @property
    def device(self):
        return self.packed.device

    @property
    def nbytes(self) -> int:
        """Bytes the GEMM streams: codes + scales + zeros."""
        return self.N * self.K * self.bits // 8 + self.N * (self.K // GROUP) * 3


def empty_quantized(N: int, K: int, bits: int, device="cuda") -> QuantizedWeight:
    import torch
    _require_bits_k(bits, K)
    return QuantizedWeight(
        packed=torch.empty((N, K * bits // 32), dtype=torch.int32, device=device),
        scales=torch.empty((N, K // GROUP), dtype=torch.float16, device=device),
        zeros=torch.empty((N, K // GROUP), dtype=torch.uint8, device=device),
        bits=bits, N=N, K=K)


def quantize(W, bits: int, out: QuantizedWeight | None = None, flags=None, stream=None) -> QuantizedWeight:
    """Quantize a [N, K] bf16 CUDA tensor to the `bits`-bit packed format."""
    import torch
    _require(W, "W", (torch.bfloat16,), ndim=2)
    N, K = W.shape
    _require_bits_k(bits, K)
    if out is not None:
        _require_weight(out, "out")
        if (out.N, out.K, out.bits) != (N, K, bits):
            raise ValueError(f"out: a ({out.N}, {out.K}, {out.bits}-bit) layer, "
                             f"expected ({N}, {K}, {bits}-bit)")
    _require_flags(flags)
    dev = _require_cuda(W=W, flags=flags, out=None if out is None else out.packed)
    with _on(dev):
        q = out if out is not None else empty_quantized(N, K, bits, dev)
        _check(_lib.slq_quantize(_ptr(W), N, K, bits, _ptr(q.packed), _ptr(q.scales), _ptr(q.zeros),
                                 _ptr(flags), _stream_ptr(stream, dev)), "slq_quantize")
    return q


def gemm(X, qw: QuantizedWeight, out_dtype=None, path: str = "auto", out=None, flags=None,
         stream=None, workspace=None):
    """Y = X W^T for bf16 X [M, K] and a packed layer; Y is bf16 or fp32 [M, N].

    `workspace` (a zero-filled uint8 CUDA tensor) defaults to the stream's
    cached buffer."""
    import torch
    if path not in _PATHS:
        raise ValueError(f"path {path!r}: one of {sorted(_PATHS)}")
    M = _require_x(X, qw)
    K = qw.K
    _require_out(out, out_dtype, M, qw.N)
    _require_flags(flags)
    if workspace is not None:
        _require(workspace, "workspace", (torch.uint8,))
    dev = _require_cuda(X=X, qw=qw.packed, out=out, flags=flags, workspace=workspace)
    with _on(dev):
        y = out if out is not None else torch.empty((M, qw.N), dtype=_y_dtype(out_dtype), device=dev)
        dt = SLQ_DTYPE_F32 if y.dtype == torch.float32 else SLQ_DTYPE_BF16
        need = gemm_workspace_bytes(M, qw.N, K, qw.bits) if path == "decode" else 0
        ws = workspace if workspace is not None else workspace_for(need, stream)
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
        _check(_lib.slq_gemm_ex(_ptr(X), M, qw.N, K, qw.bits, _ptr(qw.packed), _ptr(qw.scales),
                                _ptr(qw.zeros), _ptr(y), dt, _PATHS[path], _ptr(ws), ws_bytes,
                                _ptr(flags), _stream_ptr(stream, dev)), "slq_gemm")
    return y


DECODE_STATIC_SCRATCH_BYTES = 8 << 20


def gemm_group(items, out_dtype=None, outs=None, flags=None, stream=None):
    """One launch for several decode-step layers: items = [(X, qw), ...] with
    bf16 X [M, K_i] (one M <= 16 for all) and packed layers of any b.
    Returns the list of Y_i [M, N_i] (bf16 unless out_dtype says fp32)."""
    import torch
    items = list(items)
    if not items:
        raise ValueError("gemm_group: no layers")
    if outs is not None and len(outs) != len(items):
        raise ValueError(f"outs: {len(outs)} outputs for {len(items)} layers")
    Ms = [_require_x(X, qw, f"items[{i}].X") for i, (X, qw) in enumerate(items)]
    M = Ms[0]
    if any(m != M for m in Ms):
        raise ValueError(f"items: M = {Ms}; all layers of one call take the same M")
    for i, (_, qw) in enumerate(items):
        _require_out(None if outs is None else outs[i], out_dtype, M, qw.N, f"outs[{i}]")
    if outs is not None and any(y.dtype != outs[0].dtype for y in outs):
        raise TypeError("outs: one call writes one output dtype")
    _require_flags(flags)
    tensors = {f"items[{i}].X": X for i, (X, _) in enumerate(items)}
    tensors.update({f"items[{i}].qw": qw.packed for i, (_, qw) in enumerate(items)})
    if outs is not None:
        tensors.update({f"outs[{i}]": y for i, y in enumerate(outs)})
    dev = _require_cuda(flags=flags, **tensors)
    with _on(dev):
        ys = outs if outs is not None else [
            torch.empty((M, qw.N), dtype=_y_dtype(out_dtype), device=dev) for _, qw in items]
        arr = (GemmLayer * len(items))()
        for i, ((X, qw), y) in enumerate(zip(items, ys)):
            arr[i] = GemmLayer(_ptr(X), qw.N, qw.K, qw.bits, _ptr(qw.packed), _ptr(qw.scales),
                               _ptr(qw.zeros), _ptr(y))
        dt = SLQ_DTYPE_F32 if ys[0].dtype == torch.float32 else SLQ_DTYPE_BF16
        _check(_lib.slq_gemm_group(arr, len(items), M, dt, _ptr(flags), _stream_ptr(stream, dev)),
               "slq_gemm_group")
    return ys


def gemm_decode_static(X, qw: QuantizedWeight, out_dtype=None, out=None, flags=None, stream=None):
    """Y = X W^T for M <= 16 without a workspace (the library's fixed per-device
    scratch array is used; calls must not overlap on the GPU)."""
    import torch
    M = _require_x(X, qw)
    _require_out(out, out_dtype, M, qw.N)
    _require_flags(flags)
    dev = _require_cuda(X=X, qw=qw.packed, out=out, flags=flags)
    with _on(dev):
        y = out if out is not None else torch.empty((M, qw.N), dtype=_y_dtype(out_dtype), device=dev)
        dt = SLQ_DTYPE_F32 if y.dtype == torch.float32 else SLQ_DTYPE_BF16
        _check(_lib.slq_gemm_decode_static(_ptr(X), M, qw.N, qw.K, qw.bits, _ptr(qw.packed),
                                           _ptr(qw.scales), _ptr(qw.zeros), _ptr(y), dt, _ptr(flags),
                                           _stream_ptr(stream, dev)), "slq_gemm_decode_static")
    return y


def ear_kl(a, b, temperature: float = 1.0, means: bool = True, flags=None, stream=None,
           top_k: int | None = None):
    """Per-token EAR and KL(p || q) of two [T, V] bf16 logit tensors; with
    top_k, the top-K form (slq_ear_kl_topk).

    Returns (ear_tok, kl_tok, ear_mean, kl_mean); the means are 0-d float64
    tensors on the device (None when means=False)."""
    import torch
    _require(a, "a", (torch.bfloat16,), ndim=2)
    _require(b, "b", (torch.bfloat16,), tuple(a.shape))
    _require_flags(flags)
    dev = _require_cuda(a=a, b=b, flags=flags)
    T, V = a.shape
    with _on(dev):
        ear = torch.empty(T, dtype=torch.float32, device=dev)
        kl = torch.empty(T, dtype=torch.float32, device=dev)
        em = torch.empty((), dtype=torch.float64, device=dev) if means else None
        km = torch.empty((), dtype=torch.float64, device=dev) if means else None
        if top_k is not None:
            _check(_lib.slq_ear_kl_topk(_ptr(a), _ptr(b), T, V, int(top_k), float(temperature),
                                        _ptr(ear), _ptr(kl), _ptr(em), _ptr(km), _ptr(flags),
                                        _stream_ptr(stream, dev)), "slq_ear_kl_topk")
        else:
            _check(_lib.slq_ear_kl(_ptr(a), _ptr(b), T, V, float(temperature), _ptr(ear), _ptr(kl),
                                   _ptr(em), _ptr(km), _ptr(flags), _stream_ptr(stream, dev)),
                   "slq_ear_kl")
    return ear, kl, em, km


def grid_noise(W, bits: int, flags=None, stream=None):
    """Per 128-weight group of a [N, K] bf16 CUDA tensor: gamma = 2 max|w| /
    (max w - min w) and the rounding SSE of the asymmetric and the symmetric
    continuous b-bit grids (slq_grid_noise).  Returns (gamma, sse_asym,
    sse_sym), fp32 [N, K/128] each."""
    import torch
    _require(W, "W", (torch.bfloat16,), ndim=2)
    N, K = W.shape
    _require_bits_k(bits, K)
    _require_flags(flags)
    dev = _require_cuda(W=W, flags=flags)
    with _on(dev):
        outs = [torch.empty((N, K // GROUP), dtype=torch.float32, device=dev) for _ in range(3)]
        _check(_lib.slq_grid_noise(_ptr(W), N, K, bits, _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                   _ptr(flags), _stream_ptr(stream, dev)), "slq_grid_noise")
    return tuple(outs)


def gptq_workspace_bytes(N: int, K: int) -> int:
    return int(_lib.slq_gptq_workspace_bytes(N, K))


def gptq(W, X, bits: int, damp: float = 0.01, out: QuantizedWeight | None = None, flags=None,
         stream=None, workspace=None) -> QuantizedWeight:
    """GPTQ encode (slq_gptq) of a [N, K] bf16 CUDA tensor with [T, K] bf16
    calibration rows X into the packed format of quantize().  `workspace` (a
    uint8 CUDA tensor of gptq_workspace_bytes(N, K) bytes or more) is
    allocated for the call when not given."""
    import torch
    _require(W, "W", (torch.bfloat16,), ndim=2)
    N, K = W.shape
    _require_bits_k(bits, K)
    _require(X, "X", (torch.bfloat16,), ndim=2)
    if X.shape[1] != K:
        raise ValueError(f"X: {tuple(X.shape)}, expected [T, {K}]")
    if out is not None:
        _require_weight(out, "out")
        if (out.N, out.K, out.bits) != (N, K, bits):
            raise ValueError(f"out: a ({out.N}, {out.K}, {out.bits}-bit) layer, "
                             f"expected ({N}, {K}, {bits}-bit)")
    _require_flags(flags)
    if workspace is not None:
        _require(workspace, "workspace", (torch.uint8,))
    dev = _require_cuda(W=W, X=X, flags=flags, workspace=workspace,
                        out=None if out is None else out.packed)
    with _on(dev):
        q = out if out is not None else empty_quantized(N, K, bits, dev)
        need = gptq_workspace_bytes(N, K)
        ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=dev)
        _check(_lib.slq_gptq(_ptr(W), N, K, bits, _ptr(X), X.shape[0], float(damp), _ptr(q.packed),
                             _ptr(q.scales), _ptr(q.zeros), _ptr(ws), ws.numel(), _ptr(flags),
                             _stream_ptr(stream, dev)), "slq_gptq")
    return q
