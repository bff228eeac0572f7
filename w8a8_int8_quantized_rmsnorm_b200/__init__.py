"""ConvRot W8A8 / W4A8 INT8 linear layers for NVIDIA B200 (sm_100a).

A thin Python binding over libconvrot.so (include/convrot.h).  Each function
has the name of the C entry point it calls and only marshals arguments:
PyTorch supplies device memory and the current CUDA stream; every step of the
method runs in the library's CUDA kernels.  There is no CPU fallback: calls
raise if the library or a CUDA device is missing.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _capi

__all__ = [
    "ConvRotError", "lib", "convrot_version", "convrot_device_status",
    "convrot_quantize_weight", "convrot_quantize_weight_w4", "convrot_smoothquant_calibrate",
    "convrot_rotate_quant_act", "convrot_linear_workspace_bytes", "convrot_int8_linear",
    "convrot_w4a8_linear", "convrot_int8_linear_noalloc", "convrot_int8_gemm_s32", "convrot_w4a8_gemm_s32",
    "Workspace", "ConvRotLinear",
]


class ConvRotError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {_capi.STATUS.get(status, status)}")


def lib():
    return _capi.load()


def _check(fn: str, status: int):
    if status != 0:
        raise ConvRotError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, dim: Optional[int] = None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU fallback)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")


def convrot_version() -> int:
    return lib().convrot_version()


def convrot_device_status(device=None) -> int:
    """Synchronises the current stream and returns/clears the device error word."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    detail = ctypes.c_uint32(0)
    st = lib().convrot_device_status(_stream(dev), ctypes.byref(detail))
    if st not in (0, 6):
        _check("convrot_device_status", st)
    return int(detail.value)


# ---------------------------------------------------------------- weights
def convrot_quantize_weight(W: torch.Tensor, group: int = 256,
                            col_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    _need(W, torch.bfloat16, "W", 2)
    if col_scale is not None:
        _need(col_scale, torch.float32, "col_scale", 1)
    N, K = W.shape
    Wq = torch.empty(N, K, dtype=torch.int8, device=W.device)
    s_row = torch.empty(N, dtype=torch.float32, device=W.device)
    _check("convrot_quantize_weight", lib().convrot_quantize_weight(
        _ptr(W), N, K, group, _ptr(col_scale), _ptr(Wq), _ptr(s_row), _stream(W.device)))
    return Wq, s_row


def convrot_quantize_weight_w4(W: torch.Tensor, group: int = 256,
                               col_scale: Optional[torch.Tensor] = None, clip_lo: float = 0.80,
                               clip_hi: float = 1.00, clip_steps: int = 21):
    _need(W, torch.bfloat16, "W", 2)
    if col_scale is not None:
        _need(col_scale, torch.float32, "col_scale", 1)
    N, K = W.shape
    Wq4 = torch.empty(N, K // 2, dtype=torch.uint8, device=W.device)
    s_row = torch.empty(N, dtype=torch.float32, device=W.device)
    _check("convrot_quantize_weight_w4", lib().convrot_quantize_weight_w4(
        _ptr(W), N, K, group, _ptr(col_scale), clip_lo, clip_hi, clip_steps, _ptr(Wq4),
        _ptr(s_row), _stream(W.device)))
    return Wq4, s_row


def convrot_smoothquant_calibrate(x: torch.Tensor, norm_w: torch.Tensor, W: torch.Tensor,
                                  eps: float = 1e-6, alpha: float = 0.5):
    _need(x, torch.bfloat16, "x", 2)
    _need(W, torch.bfloat16, "W", 2)
    _need(norm_w, torch.float32, "norm_w", 1)
    M, K = x.shape
    N = W.shape[0]
    smooth = torch.empty(K, dtype=torch.float32, device=x.device)
    folded = torch.empty(K, dtype=torch.float32, device=x.device)
    _check("convrot_smoothquant_calibrate", lib().convrot_smoothquant_calibrate(
        _ptr(x), M, K, _ptr(norm_w), eps, _ptr(W), N, alpha, _ptr(smooth), _ptr(folded),
        _stream(x.device)))
    return smooth, folded


# ---------------------------------------------------------------- activations
def convrot_rotate_quant_act(x: torch.Tensor, group: int = 256,
                             norm_w: Optional[torch.Tensor] = None, eps: float = 1e-6,
                             out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    _need(x, torch.bfloat16, "x", 2)
    if norm_w is not None:
        _need(norm_w, torch.float32, "norm_w", 1)
    M, K = x.shape
    if out is None:
        Xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
        s_tok = torch.empty(M, dtype=torch.float32, device=x.device)
    else:
        Xq, s_tok = out
    _check("convrot_rotate_quant_act", lib().convrot_rotate_quant_act(
        _ptr(x), M, K, group, _ptr(norm_w), eps, _ptr(Xq), _ptr(s_tok), _stream(x.device)))
    return Xq, s_tok


# ---------------------------------------------------------------- GEMM
def convrot_linear_workspace_bytes(M: int, N: int, K: int, weight_bits: int = 8) -> int:
    return int(lib().convrot_linear_workspace_bytes(M, N, K, weight_bits))


class Workspace:
    """Device workspace for the GEMM's split tiles, grown on demand.

    It starts zero-filled; the library keeps its tile counters at zero after
    every successful call, so it is reused without clearing.  One Workspace
    must not be used by calls that run concurrently on different streams.
    """

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int) -> Tuple[Optional[int], int]:
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf.data_ptr(), self.buf.numel()


_default_ws = {}


def _workspace(dev: torch.device, nbytes: int, ws: Optional[Workspace]):
    if ws is None:
        key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(dev.index)
    p, n = ws.get(nbytes)
    return (ctypes.c_void_p(p) if p else None), n


def _gemm_check(Xq, Wq, w4: bool):
    _need(Xq, torch.int8, "Xq", 2)
    _need(Wq, torch.uint8 if w4 else torch.int8, "Wq4" if w4 else "Wq", 2)
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] * (2 if w4 else 1) != K:
        raise ValueError("weight and activation disagree on K")
    return M, N, K


def convrot_int8_linear(Xq, s_tok, Wq, s_row, out=None, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq, False)
    _need(s_tok, torch.float32, "s_tok", 1)
    _need(s_row, torch.float32, "s_row", 1)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq.device) if out is None else out
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 8), workspace)
    _check("convrot_int8_linear", lib().convrot_int8_linear(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq), _ptr(s_row), M, N, K, _ptr(Y), ws, wn,
        _stream(Xq.device)))
    return Y


def convrot_int8_linear_noalloc(Xq, s_tok, Wq, s_row, out=None):
    """convrot_int8_linear without a caller workspace: the library's fixed
    24 MiB per-device array serves as the split-tile workspace (for callers
    that cannot allocate device memory where they run the layer).  Calls that
    overlap on the GPU race on that array."""
    M, N, K = _gemm_check(Xq, Wq, False)
    _need(s_tok, torch.float32, "s_tok", 1)
    _need(s_row, torch.float32, "s_row", 1)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq.device) if out is None else out
    _check("convrot_int8_linear_noalloc", lib().convrot_int8_linear_noalloc(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq), _ptr(s_row), M, N, K, _ptr(Y), _stream(Xq.device)))
    return Y


def convrot_w4a8_linear(Xq, s_tok, Wq4, s_row, out=None, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq4, True)
    _need(s_tok, torch.float32, "s_tok", 1)
    _need(s_row, torch.float32, "s_row", 1)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq.device) if out is None else out
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 4), workspace)
    _check("convrot_w4a8_linear", lib().convrot_w4a8_linear(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq4), _ptr(s_row), M, N, K, _ptr(Y), ws, wn,
        _stream(Xq.device)))
    return Y


def convrot_int8_gemm_s32(Xq, Wq, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq, False)
    acc = torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 8), workspace)
    _check("convrot_int8_gemm_s32", lib().convrot_int8_gemm_s32(
        _ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), ws, wn, _stream(Xq.device)))
    return acc


def convrot_w4a8_gemm_s32(Xq, Wq4, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq4, True)
    acc = torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 4), workspace)
    _check("convrot_w4a8_gemm_s32", lib().convrot_w4a8_gemm_s32(
        _ptr(Xq), _ptr(Wq4), M, N, K, _ptr(acc), ws, wn, _stream(Xq.device)))
    return acc


class ConvRotLinear:
    """A quantised linear layer: prepared weights plus the per-token forward.

    forward(x) = convrot_rotate_quant_act (optionally with the fused RMSNorm)
    followed by convrot_int8_linear / convrot_w4a8_linear.
    """

    def __init__(self, W: torch.Tensor, *, weight_bits: int = 8, group: int = 256,
                 norm_w: Optional[torch.Tensor] = None, col_scale: Optional[torch.Tensor] = None,
                 eps: float = 1e-6):
        self.group = group
        self.weight_bits = weight_bits
        self.eps = eps
        self.norm_w = norm_w
        self.N, self.K = W.shape
        if weight_bits == 8:
            self.Wq, self.s_row = convrot_quantize_weight(W, group, col_scale)
        elif weight_bits == 4:
            self.Wq, self.s_row = convrot_quantize_weight_w4(W, group, col_scale)
        else:
            raise ValueError("weight_bits must be 8 or 4")
        self.workspace = Workspace(W.device.index)

    @classmethod
    def with_smoothquant(cls, W, x_calib, norm_w, *, weight_bits=8, group=256, eps=1e-6, alpha=0.5):
        smooth, folded = convrot_smoothquant_calibrate(x_calib, norm_w, W, eps, alpha)
        return cls(W, weight_bits=weight_bits, group=group, norm_w=folded, col_scale=smooth, eps=eps)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        Xq, s_tok = convrot_rotate_quant_act(x, self.group, self.norm_w, self.eps)
        if self.weight_bits == 8:
            return convrot_int8_linear(Xq, s_tok, self.Wq, self.s_row, out, self.workspace)
        return convrot_w4a8_linear(Xq, s_tok, self.Wq, self.s_row, out, self.workspace)

    __call__ = forward
