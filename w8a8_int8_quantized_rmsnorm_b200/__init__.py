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
    "convrot_swiglu_workspace_bytes", "convrot_int8_linear_swiglu", "convrot_w4a8_linear_swiglu",
    "convrot_interleave_gate_up", "convrot_fold_row_scales",
    "convrot_rotate_act_bf16", "convrot_weight_only_workspace_bytes", "convrot_weight_only_linear",
    "convrot_weight_only_gemm_f32",
    "Workspace", "ConvRotLinear", "ConvRotFusedLinear", "ConvRotMLP",
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


def _need(t: torch.Tensor, dtype, name: str, dim: Optional[int] = None, shape=None):
    """dtype, contiguity and shape of one operand.  The device is checked
    afterwards, for all operands of a call together (_on_device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _on_device(**operands) -> torch.device:
    """Every operand is a CUDA tensor on one device, and that device is the
    current one: the library launches on the current device, on that device's
    current stream.  None entries (optional operands) are skipped."""
    dev = None
    for name, t in operands.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU fallback)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}; the other operands are on {dev}")
    cur = torch.cuda.current_device()
    if dev.index != cur:
        raise ValueError(f"the operands are on {dev} but the current device is cuda:{cur}")
    return dev


def convrot_version() -> int:
    return lib().convrot_version()


# Device timeouts reported so far.  A kernel that gave up on a bounded wait may
# leave partial sums and tile counters in its split-tile workspace; every
# Workspace zero-fills itself again before its next use once this has moved.
_timeouts_reported = 0


def _note_status(st: int) -> None:
    global _timeouts_reported
    if st == 6:  # CONVROT_ERR_DEVICE_TIMEOUT
        _timeouts_reported += 1


def convrot_device_status(device=None) -> int:
    """Synchronises the current stream and returns/clears the device error word.

    A non-zero word means a kernel gave up on a bounded wait; every Workspace
    is then zero-filled again before its next use."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    detail = ctypes.c_uint32(0)
    st = lib().convrot_device_status(_stream(dev), ctypes.byref(detail))
    if st not in (0, 6):
        _check("convrot_device_status", st)
    _note_status(st)
    return int(detail.value)


# ---------------------------------------------------------------- weights
def convrot_quantize_weight(W: torch.Tensor, group: int = 256,
                            col_scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    _need(W, torch.bfloat16, "W", 2)
    N, K = W.shape
    if col_scale is not None:
        _need(col_scale, torch.float32, "col_scale", shape=(K,))
    _on_device(W=W, col_scale=col_scale)
    Wq = torch.empty(N, K, dtype=torch.int8, device=W.device)
    s_row = torch.empty(N, dtype=torch.float32, device=W.device)
    _check("convrot_quantize_weight", lib().convrot_quantize_weight(
        _ptr(W), N, K, group, _ptr(col_scale), _ptr(Wq), _ptr(s_row), _stream(W.device)))
    return Wq, s_row


def convrot_quantize_weight_w4(W: torch.Tensor, group: int = 256,
                               col_scale: Optional[torch.Tensor] = None, clip_lo: float = 0.80,
                               clip_hi: float = 1.00, clip_steps: int = 21):
    _need(W, torch.bfloat16, "W", 2)
    N, K = W.shape
    if col_scale is not None:
        _need(col_scale, torch.float32, "col_scale", shape=(K,))
    _on_device(W=W, col_scale=col_scale)
    Wq4 = torch.empty(N, K // 2, dtype=torch.uint8, device=W.device)
    s_row = torch.empty(N, dtype=torch.float32, device=W.device)
    _check("convrot_quantize_weight_w4", lib().convrot_quantize_weight_w4(
        _ptr(W), N, K, group, _ptr(col_scale), clip_lo, clip_hi, clip_steps, _ptr(Wq4),
        _ptr(s_row), _stream(W.device)))
    return Wq4, s_row


def convrot_smoothquant_calibrate(x: torch.Tensor, norm_w: Optional[torch.Tensor], W: torch.Tensor,
                                  eps: float = 1e-6, alpha: float = 0.5):
    """SmoothQuant scales of the linear W fed by x (norm_w None: x reaches W as
    it is, and the second result is scratch)."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    _need(W, torch.bfloat16, "W", 2)
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("x and W disagree on K")
    if norm_w is not None:
        _need(norm_w, torch.float32, "norm_w", shape=(K,))
    _on_device(x=x, W=W, norm_w=norm_w)
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
    M, K = x.shape
    if norm_w is not None:
        _need(norm_w, torch.float32, "norm_w", shape=(K,))
    if out is None:
        Xq = s_tok = None
    else:
        Xq, s_tok = out
        _need(Xq, torch.int8, "Xq", shape=(M, K))
        _need(s_tok, torch.float32, "s_tok", shape=(M,))
    _on_device(x=x, norm_w=norm_w, Xq=Xq, s_tok=s_tok)
    if out is None:
        Xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
        s_tok = torch.empty(M, dtype=torch.float32, device=x.device)
    _check("convrot_rotate_quant_act", lib().convrot_rotate_quant_act(
        _ptr(x), M, K, group, _ptr(norm_w), eps, _ptr(Xq), _ptr(s_tok), _stream(x.device)))
    return Xq, s_tok


# ---------------------------------------------------------------- GEMM
def convrot_linear_workspace_bytes(M: int, N: int, K: int, weight_bits: int = 8) -> int:
    return int(lib().convrot_linear_workspace_bytes(M, N, K, weight_bits))


class Workspace:
    """Device workspace for the GEMM's split tiles, grown on demand.

    It starts zero-filled; the library leaves it zero after every call whose
    kernels complete, so it is reused without clearing.  After
    convrot_device_status has reported a device timeout (an aborted call may
    leave partial sums behind) it is zero-filled again before its next use.
    One Workspace must not be used by calls that run concurrently on
    different streams.
    """

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.buf: Optional[torch.Tensor] = None
        self.epoch = _timeouts_reported

    def get(self, nbytes: int) -> Tuple[Optional[int], int]:
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
            self.epoch = _timeouts_reported
        elif self.epoch != _timeouts_reported:
            self.buf.zero_()
            self.epoch = _timeouts_reported
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


def _linear_operands(Xq, s_tok, Wq, s_row, out, w4: bool, out_cols=None):
    """Checks the operands of a W8A8 / W4A8 linear; returns (M, N, K, Y) with
    Y the caller's `out` or a new bf16 [M, out_cols] tensor."""
    M, N, K = _gemm_check(Xq, Wq, w4)
    cols = N if out_cols is None else out_cols
    _need(s_tok, torch.float32, "s_tok", shape=(M,))
    _need(s_row, torch.float32, "s_row", shape=(N,))
    if out is not None:
        _need(out, torch.bfloat16, "out", shape=(M, cols))
    dev = _on_device(Xq=Xq, s_tok=s_tok, Wq=Wq, s_row=s_row, out=out)
    Y = torch.empty(M, cols, dtype=torch.bfloat16, device=dev) if out is None else out
    return M, N, K, Y


def convrot_int8_linear(Xq, s_tok, Wq, s_row, out=None, workspace: Optional[Workspace] = None):
    M, N, K, Y = _linear_operands(Xq, s_tok, Wq, s_row, out, False)
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
    M, N, K, Y = _linear_operands(Xq, s_tok, Wq, s_row, out, False)
    _check("convrot_int8_linear_noalloc", lib().convrot_int8_linear_noalloc(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq), _ptr(s_row), M, N, K, _ptr(Y), _stream(Xq.device)))
    return Y


def convrot_w4a8_linear(Xq, s_tok, Wq4, s_row, out=None, workspace: Optional[Workspace] = None):
    M, N, K, Y = _linear_operands(Xq, s_tok, Wq4, s_row, out, True)
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 4), workspace)
    _check("convrot_w4a8_linear", lib().convrot_w4a8_linear(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq4), _ptr(s_row), M, N, K, _ptr(Y), ws, wn,
        _stream(Xq.device)))
    return Y


def convrot_int8_gemm_s32(Xq, Wq, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq, False)
    _on_device(Xq=Xq, Wq=Wq)
    acc = torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 8), workspace)
    _check("convrot_int8_gemm_s32", lib().convrot_int8_gemm_s32(
        _ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), ws, wn, _stream(Xq.device)))
    return acc


def convrot_w4a8_gemm_s32(Xq, Wq4, workspace: Optional[Workspace] = None):
    M, N, K = _gemm_check(Xq, Wq4, True)
    _on_device(Xq=Xq, Wq4=Wq4)
    acc = torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    ws, wn = _workspace(Xq.device, convrot_linear_workspace_bytes(M, N, K, 4), workspace)
    _check("convrot_w4a8_gemm_s32", lib().convrot_w4a8_gemm_s32(
        _ptr(Xq), _ptr(Wq4), M, N, K, _ptr(acc), ws, wn, _stream(Xq.device)))
    return acc


# ---------------------------------------------------------------- weight-only path
def convrot_rotate_act_bf16(x: torch.Tensor, group: int = 256, norm_w: Optional[torch.Tensor] = None,
                            eps: float = 1e-6, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Xr = bf16([RMSNorm] x rotated by the group Hadamard), not quantised."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    if norm_w is not None:
        _need(norm_w, torch.float32, "norm_w", shape=(K,))
    if out is not None:
        _need(out, torch.bfloat16, "out", shape=(M, K))
    _on_device(x=x, norm_w=norm_w, out=out)
    Xr = torch.empty(M, K, dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("convrot_rotate_act_bf16", lib().convrot_rotate_act_bf16(
        _ptr(x), M, K, group, _ptr(norm_w), eps, _ptr(Xr), _stream(x.device)))
    return Xr


def _wo_check(Xr, Wq):
    _need(Xr, torch.bfloat16, "Xr", 2)
    _need(Wq, torch.int8, "Wq", 2)
    if Xr.shape[1] != Wq.shape[1]:
        raise ValueError("weight and activation disagree on K")
    return Xr.shape[0], Wq.shape[0], Xr.shape[1]


def convrot_weight_only_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().convrot_weight_only_workspace_bytes(M, N, K))


def convrot_weight_only_linear(Xr, Wq, s_row, out=None, workspace: Optional[Workspace] = None):
    """Y = bf16(s_row * (Xr @ Wq^T)) on rotated bf16 activations, int8 weights."""
    M, N, K = _wo_check(Xr, Wq)
    _need(s_row, torch.float32, "s_row", shape=(N,))
    if out is not None:
        _need(out, torch.bfloat16, "out", shape=(M, N))
    _on_device(Xr=Xr, Wq=Wq, s_row=s_row, out=out)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xr.device) if out is None else out
    ws, wn = _workspace(Xr.device, convrot_weight_only_workspace_bytes(M, N, K), workspace)
    _check("convrot_weight_only_linear", lib().convrot_weight_only_linear(
        _ptr(Xr), _ptr(Wq), _ptr(s_row), M, N, K, _ptr(Y), ws, wn, _stream(Xr.device)))
    return Y


def convrot_weight_only_gemm_f32(Xr, Wq, workspace: Optional[Workspace] = None):
    M, N, K = _wo_check(Xr, Wq)
    _on_device(Xr=Xr, Wq=Wq)
    acc = torch.empty(M, N, dtype=torch.float32, device=Xr.device)
    ws, wn = _workspace(Xr.device, convrot_weight_only_workspace_bytes(M, N, K), workspace)
    _check("convrot_weight_only_gemm_f32", lib().convrot_weight_only_gemm_f32(
        _ptr(Xr), _ptr(Wq), M, N, K, _ptr(acc), ws, wn, _stream(Xr.device)))
    return acc


# ---------------------------------------------------------------- MLP boundary
def convrot_swiglu_workspace_bytes(M: int, I: int, K: int, weight_bits: int = 8) -> int:
    return int(lib().convrot_swiglu_workspace_bytes(M, I, K, weight_bits))


def _swiglu(fn, Xq, s_tok, Wq_gu, s_row_gu, w4, out, workspace):
    M, N2, K = _gemm_check(Xq, Wq_gu, w4)
    if N2 % 2:
        raise ValueError("the gate/up weight must have an even number of rows")
    I = N2 // 2
    M, N2, K, H = _linear_operands(Xq, s_tok, Wq_gu, s_row_gu, out, w4, out_cols=I)
    ws, wn = _workspace(Xq.device, convrot_swiglu_workspace_bytes(M, I, K, 4 if w4 else 8), workspace)
    _check(fn, getattr(lib(), fn)(
        _ptr(Xq), _ptr(s_tok), _ptr(Wq_gu), _ptr(s_row_gu), M, I, K, _ptr(H), ws, wn,
        _stream(Xq.device)))
    return H


def convrot_int8_linear_swiglu(Xq, s_tok, Wq_gu, s_row_gu, out=None,
                               workspace: Optional[Workspace] = None):
    """H = bf16(SiLU(gate) * up) from interleaved gate/up rows (I = rows / 2)."""
    return _swiglu("convrot_int8_linear_swiglu", Xq, s_tok, Wq_gu, s_row_gu, False, out, workspace)


def convrot_w4a8_linear_swiglu(Xq, s_tok, Wq4_gu, s_row_gu, out=None,
                               workspace: Optional[Workspace] = None):
    return _swiglu("convrot_w4a8_linear_swiglu", Xq, s_tok, Wq4_gu, s_row_gu, True, out, workspace)


def convrot_interleave_gate_up(Wg: torch.Tensor, Wu: torch.Tensor) -> torch.Tensor:
    """Rows of gate and up in alternating blocks of 16 (any dtype, 1-D or 2-D)."""
    if Wg.shape != Wu.shape or Wg.dtype != Wu.dtype or Wg.device != Wu.device:
        raise ValueError("gate and up must match in shape, dtype and device")
    if not (Wg.is_contiguous() and Wu.is_contiguous()):
        raise ValueError("gate and up must be contiguous")
    _on_device(Wg=Wg, Wu=Wu)
    I = Wg.shape[0]
    row_bytes = Wg.numel() // max(I, 1) * Wg.element_size()
    out = torch.empty((2 * I,) + tuple(Wg.shape[1:]), dtype=Wg.dtype, device=Wg.device)
    _check("convrot_interleave_gate_up", lib().convrot_interleave_gate_up(
        _ptr(Wg), _ptr(Wu), I, row_bytes, _ptr(out), _stream(Wg.device)))
    return out


def convrot_fold_row_scales(s_row: torch.Tensor, smooth: torch.Tensor) -> torch.Tensor:
    """s_row /= smooth in place (a SmoothQuant scale folded into weight rows)."""
    _need(s_row, torch.float32, "s_row", 1)
    _need(smooth, torch.float32, "smooth", shape=tuple(s_row.shape))
    _on_device(s_row=s_row, smooth=smooth)
    _check("convrot_fold_row_scales", lib().convrot_fold_row_scales(
        _ptr(s_row), _ptr(smooth), s_row.numel(), _stream(s_row.device)))
    return s_row


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
    def from_checkpoint(cls, layer: dict, *, device=None, norm_w: Optional[torch.Tensor] = None,
                        eps: float = 1e-6):
        """A linear from an entry of checkpoint.load_quantized_layers (the stored
        codes and row scales are used as they are; nothing is re-quantised)."""
        self = cls.__new__(cls)
        dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
        self.group, self.weight_bits, self.eps, self.norm_w = int(layer["group"]), int(layer["bits"]), eps, norm_w
        self.Wq = torch.from_numpy(layer["Wq"]).to(dev)
        self.s_row = torch.from_numpy(layer["s_row"]).to(dev)
        self.N = self.Wq.shape[0]
        self.K = self.Wq.shape[1] * (2 if self.weight_bits == 4 else 1)
        self.workspace = Workspace(dev.index)
        return self

    def to_checkpoint(self) -> dict:
        """The layer's stored form for checkpoint.save_quantized_layers."""
        return {"Wq": self.Wq.cpu().numpy(), "s_row": self.s_row.cpu().numpy(),
                "group": self.group, "bits": self.weight_bits}

    @classmethod
    def with_smoothquant(cls, W, x_calib, norm_w, *, weight_bits=8, group=256, eps=1e-6, alpha=0.5):
        smooth, folded = convrot_smoothquant_calibrate(x_calib, norm_w, W, eps, alpha)
        return cls(W, weight_bits=weight_bits, group=group, norm_w=folded, col_scale=smooth, eps=eps)

    def forward_weight_only(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The same layer with bf16 activations: rotate (no quantisation), then the
        bf16 tensor-core GEMM over the int8 weight codes (int8 weights only)."""
        if self.weight_bits != 8:
            raise ValueError("the weight-only path takes int8 weights")
        Xr = convrot_rotate_act_bf16(x, self.group, self.norm_w, self.eps)
        return convrot_weight_only_linear(Xr, self.Wq, self.s_row, out, self.workspace)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        Xq, s_tok = convrot_rotate_quant_act(x, self.group, self.norm_w, self.eps)
        if self.weight_bits == 8:
            return convrot_int8_linear(Xq, s_tok, self.Wq, self.s_row, out, self.workspace)
        return convrot_w4a8_linear(Xq, s_tok, self.Wq, self.s_row, out, self.workspace)

    __call__ = forward


class ConvRotFusedLinear:
    """Several linears that read the same input, run as ONE GEMM over their
    concatenated output rows: a fused projection set such as q/k/v of an
    attention block, or a gated-DeltaNet input projection together with its
    small-N companion (the MOSS-Image card quantises attention, gated-DeltaNet
    projections and MLP linears).  Every row is quantised on its own, so the
    fused layer's codes, scales and outputs are those of the separate layers;
    one launch replaces several, and small-N members no longer under-fill the
    GPU.  A shared SmoothQuant scale (with a norm) is calibrated over all
    members' columns, since they share the input.
    """

    def __init__(self, weights, *, weight_bits: int = 8, group: int = 256,
                 norm_w: Optional[torch.Tensor] = None, x_calib: Optional[torch.Tensor] = None,
                 eps: float = 1e-6, alpha: float = 0.5):
        W = torch.cat(list(weights))
        self.sizes = [int(w.shape[0]) for w in weights]
        col = None
        if x_calib is not None and norm_w is not None:
            col, norm_w = convrot_smoothquant_calibrate(x_calib, norm_w, W, eps, alpha)
        self.col_scale = col
        self.linear = ConvRotLinear(W, weight_bits=weight_bits, group=group, norm_w=norm_w,
                                    col_scale=col, eps=eps)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None):
        """One output per member, as column views of the fused [M, sum N] result."""
        return torch.split(self.linear(x, out), self.sizes, dim=1)

    __call__ = forward


class ConvRotMLP:
    """The MLP block down(SiLU(gate(x)) * up(x)) of the quantised decoder layer.

    forward(x) = rotate-quantise (with the fused RMSNorm) -> one gate/up GEMM
    whose epilogue writes H = SiLU(g) * u -> rotate-quantise H -> down_proj.
    With calibration input, SmoothQuant scales are folded into the norm
    weight (gate/up input) and into up_proj's row scales (down_proj input),
    as the MOSS-Image card's "How it was made" describes.
    """

    def __init__(self, Wg: torch.Tensor, Wu: torch.Tensor, Wd: torch.Tensor, *,
                 norm_w: Optional[torch.Tensor] = None, x_calib: Optional[torch.Tensor] = None,
                 group: int = 256, eps: float = 1e-6, alpha: float = 0.5):
        self.group, self.eps = group, eps
        self.I, self.H = Wg.shape
        self.workspace = Workspace(Wg.device.index)
        col = None
        self.norm_w = norm_w
        if x_calib is not None and norm_w is not None:
            col, self.norm_w = convrot_smoothquant_calibrate(x_calib, norm_w, torch.cat([Wg, Wu]), eps, alpha)
        Wq_g, s_g = convrot_quantize_weight(Wg, group, col)
        Wq_u, s_u = convrot_quantize_weight(Wu, group, col)
        self.Wq_gu = convrot_interleave_gate_up(Wq_g, Wq_u)
        s_gu = convrot_interleave_gate_up(s_g, s_u)
        smooth_d = None
        if x_calib is not None:
            Xq, s_tok = convrot_rotate_quant_act(x_calib, group, self.norm_w, eps)
            h = convrot_int8_linear_swiglu(Xq, s_tok, self.Wq_gu, s_gu, workspace=self.workspace)
            smooth_d, _ = convrot_smoothquant_calibrate(h, None, Wd, eps, alpha)
            convrot_fold_row_scales(s_u, smooth_d)
            s_gu = convrot_interleave_gate_up(s_g, s_u)
        self.s_gu = s_gu
        self.Wq_d, self.s_d = convrot_quantize_weight(Wd, group, smooth_d)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        Xq, s_tok = convrot_rotate_quant_act(x, self.group, self.norm_w, self.eps)
        h = convrot_int8_linear_swiglu(Xq, s_tok, self.Wq_gu, self.s_gu, workspace=self.workspace)
        Hq, s_h = convrot_rotate_quant_act(h, self.group, None, self.eps)
        return convrot_int8_linear(Hq, s_h, self.Wq_d, self.s_d, out, self.workspace)

    __call__ = forward
