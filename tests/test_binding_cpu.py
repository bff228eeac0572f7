"""Argument checks of the Python binding that need no GPU.

Every wrapper checks dtype, contiguity and shape of each operand, including a
caller-given `out` and the lengths of the scale vectors, before it looks at
the device; a CUDA library launch with a too-short output or scale vector
would read or write past the caller's allocation.  The device check comes
last, so on a CPU-only machine a call with well-formed CPU tensors still
fails with "must be a CUDA tensor" (there is no CPU fallback)."""
import pytest
import torch

import w8a8_int8_quantized_rmsnorm_b200 as cr

M, N, K = 4, 32, 512


def i8(*shape):
    return torch.zeros(*shape, dtype=torch.int8)


def f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _raises(match, fn, *args, **kw):
    with pytest.raises((ValueError, TypeError), match=match):
        fn(*args, **kw)


@pytest.mark.parametrize("fn", [cr.convrot_int8_linear, cr.convrot_int8_linear_noalloc])
def test_int8_linear_operand_shapes(fn):
    _raises("s_tok must have shape", fn, i8(M, K), f32(M - 1), i8(N, K), f32(N))
    _raises("s_row must have shape", fn, i8(M, K), f32(M), i8(N, K), f32(N - 8))
    _raises("out must have shape", fn, i8(M, K), f32(M), i8(N, K), f32(N), out=bf16(M, N - 8))
    _raises("out must have shape", fn, i8(M, K), f32(M), i8(N, K), f32(N), out=bf16(M - 1, N))
    _raises("out must be torch.bfloat16", fn, i8(M, K), f32(M), i8(N, K), f32(N), out=f32(M, N))
    _raises("disagree on K", fn, i8(M, K), f32(M), i8(N, K - 16), f32(N))
    _raises("must be a CUDA tensor", fn, i8(M, K), f32(M), i8(N, K), f32(N), out=bf16(M, N))


def test_w4a8_and_swiglu_operand_shapes():
    w4 = torch.zeros(N, K // 2, dtype=torch.uint8)
    _raises("s_row must have shape", cr.convrot_w4a8_linear, i8(M, K), f32(M), w4, f32(N // 2))
    _raises("must be a CUDA tensor", cr.convrot_w4a8_linear, i8(M, K), f32(M), w4, f32(N))
    # SwiGLU writes N / 2 columns
    _raises("out must have shape", cr.convrot_int8_linear_swiglu, i8(M, K), f32(M), i8(N, K), f32(N),
            out=bf16(M, N))
    _raises("s_tok must have shape", cr.convrot_w4a8_linear_swiglu, i8(M, K), f32(2 * M), w4, f32(N))
    _raises("must be a CUDA tensor", cr.convrot_int8_linear_swiglu, i8(M, K), f32(M), i8(N, K), f32(N),
            out=bf16(M, N // 2))


def test_activation_and_weight_operand_shapes():
    _raises("Xq must have shape", cr.convrot_rotate_quant_act, bf16(M, K), out=(i8(M, K - 16), f32(M)))
    _raises("s_tok must have shape", cr.convrot_rotate_quant_act, bf16(M, K), out=(i8(M, K), f32(M + 1)))
    _raises("norm_w must have shape", cr.convrot_rotate_quant_act, bf16(M, K), 256, f32(K - 16))
    _raises("out must have shape", cr.convrot_rotate_act_bf16, bf16(M, K), out=bf16(M, K // 2))
    _raises("col_scale must have shape", cr.convrot_quantize_weight, bf16(N, K), 256, f32(K // 2))
    _raises("col_scale must have shape", cr.convrot_quantize_weight_w4, bf16(N, K), 256, f32(K + 16))
    _raises("norm_w must have shape", cr.convrot_smoothquant_calibrate, bf16(M, K), f32(K - 16), bf16(N, K))
    _raises("disagree on K", cr.convrot_smoothquant_calibrate, bf16(M, K), f32(K), bf16(N, K - 16))
    _raises("must be a CUDA tensor", cr.convrot_rotate_quant_act, bf16(M, K), out=(i8(M, K), f32(M)))


def test_weight_only_operand_shapes():
    _raises("s_row must have shape", cr.convrot_weight_only_linear, bf16(M, K), i8(N, K), f32(N + 8))
    _raises("out must have shape", cr.convrot_weight_only_linear, bf16(M, K), i8(N, K), f32(N),
            out=bf16(N, M))
    _raises("must be a CUDA tensor", cr.convrot_weight_only_linear, bf16(M, K), i8(N, K), f32(N))


def test_workspace_is_cleared_after_a_reported_timeout(monkeypatch):
    """A kernel that gave up on a bounded wait may leave partial sums in its
    workspace: once the device status has reported a timeout, a Workspace
    zero-fills itself before its next use (here on a CPU buffer, with the
    status call's result given directly)."""
    ws = cr.Workspace.__new__(cr.Workspace)
    ws.device = torch.device("cpu")
    ws.buf = None
    ws.epoch = cr._timeouts_reported
    ws.get(64)
    ws.buf.fill_(7)                  # what an aborted call could leave behind
    ws.get(64)
    assert int(ws.buf.sum()) == 7 * 64   # no timeout reported: reused as it is
    cr._note_status(0)
    ws.get(32)
    assert int(ws.buf.sum()) == 7 * 64
    cr._note_status(6)               # CONVROT_ERR_DEVICE_TIMEOUT
    ws.get(32)
    assert int(ws.buf.sum()) == 0
    ws.buf.fill_(1)
    ws.get(64)                       # cleared once per report, not on every call
    assert int(ws.buf.sum()) == 64
