"""End-to-end parity of the ConvRot linear: every step on the GPU through the
C ABI (SmoothQuant calibration, weight preparation, rotate-quantise with the
fused RMSNorm, W8A8 / W4A8 GEMM) against the oracle run independently on the
same seeded inputs.  Tolerance: |y - y_ref| <= 2^-7 |y_ref| + 1e-3 max|y_ref row|.

Small workloads are compared on every output; the full-size workloads run
through the kernels at full size (the launch configuration the bench times)
and are compared on sampled tokens x sampled output rows, which the oracle
computes one by one (tokens and weight rows are independent)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import convrot_ref as ref
from tests import _tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cr():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_quantized_rmsnorm_b200 as m
    m.lib()
    return m


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _gpu_linear(cr, x, W, nw, weight_bits, group=256):
    xd, Wd = x.cuda(), W.cuda()
    col = None
    nwd = None
    if nw is not None:
        col, nwd = cr.convrot_smoothquant_calibrate(xd, nw.cuda(), Wd, 1e-6, 0.5)
    if weight_bits == 8:
        Wq, s_row = cr.convrot_quantize_weight(Wd, group, col)
    else:
        Wq, s_row = cr.convrot_quantize_weight_w4(Wd, group, col)
    Xq, s_tok = cr.convrot_rotate_quant_act(xd, group, nwd, 1e-6)
    if weight_bits == 8:
        Y = cr.convrot_int8_linear(Xq, s_tok, Wq, s_row)
    else:
        Y = cr.convrot_w4a8_linear(Xq, s_tok, Wq, s_row)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    return Y


def _oracle_linear(x, W, nw, weight_bits, rows=None, cols=None, group=256):
    x64, W64 = _f64(x), _f64(W)
    col = nwf = None
    if nw is not None:
        col, nwf = ref.smoothquant_scales(x64, nw.double().numpy(), 1e-6, W64, 0.5)
        # the library stores both in fp32
        col = col.astype(np.float32).astype(np.float64)
        nwf = nwf.astype(np.float32).astype(np.float64)
    if rows is not None:
        x64 = x64[rows]
    if cols is not None:
        W64 = W64[cols]
    Xq, s_tok, _ = ref.rotate_quant_act(x64, group, nwf, 1e-6)
    if weight_bits == 8:
        Wq, s_row, _ = ref.quantize_weight(W64, group, col)
        yb, y, _ = ref.int8_linear(Xq, s_tok, Wq, s_row)
    else:
        o = ref.quantize_weight_w4(W64, group, col)
        yb, y, _ = ref.w4a8_linear(Xq, s_tok, o["packed"], o["s_row"])
    return yb, y


def _assert_close(Y, y_ref, what):
    got = _f64(Y) if isinstance(Y, torch.Tensor) else Y
    tol = _tol.output_tol(y_ref)
    err = np.abs(got - y_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} outputs out of tolerance, worst "
                           f"{(err - tol).max():.3e}")


def test_single_linear_m32_all_outputs(cr):
    w = workloads.WORKLOADS["single_linear_m32"]
    x, W, nw = workloads.workload_inputs(w, w.linears[0])
    Y = _gpu_linear(cr, x, W, nw, 8)
    yb, _ = _oracle_linear(x, W, nw, 8)
    _assert_close(Y, yb, "single linear")


def test_single_linear_group0_fallback(cr):
    w = workloads.WORKLOADS["single_linear_m32"]
    x, W, _ = workloads.workload_inputs(w, w.linears[0])
    Y = _gpu_linear(cr, x, W, None, 8, group=0)
    yb, _ = _oracle_linear(x, W, None, 8, group=0)
    _assert_close(Y, yb, "group 0")


def test_down_proj_m512_with_norm_all_outputs(cr):
    w = workloads.WORKLOADS["down_proj_m512"]
    x, W, nw = workloads.workload_inputs(w, w.linears[0])
    Y = _gpu_linear(cr, x, W, nw, 8)
    yb, _ = _oracle_linear(x, W, nw, 8)
    _assert_close(Y, yb, "down_proj with RMSNorm + SmoothQuant")


def _sampled(cr, wname, lin, M=None, weight_bits=8, layer=0, nrows=24, ncols=160):
    w = workloads.WORKLOADS[wname]
    x, W, nw = workloads.workload_inputs(w, lin, M=M, layer=layer)
    Y = _gpu_linear(cr, x, W, nw, weight_bits)
    rng = np.random.default_rng(lin.N + lin.K + x.shape[0])
    m = x.shape[0]
    rows = np.unique(np.concatenate([rng.choice(m, min(nrows, m), replace=False), [0, m - 1]]))
    cols = np.unique(np.concatenate([rng.choice(lin.N, min(ncols, lin.N), replace=False),
                                     [0, lin.N - 1]]))
    yb, _ = _oracle_linear(x, W, nw, weight_bits, rows, cols)
    _assert_close(_f64(Y)[np.ix_(rows, cols)], yb, f"{wname}/{lin.name}")


@pytest.mark.parametrize("lin", workloads.WORKLOADS["decoder_layer_m2048"].linears,
                         ids=lambda l: l.name)
def test_decoder_layer_m2048_sampled(cr, lin):
    _sampled(cr, "decoder_layer_m2048", lin)


@pytest.mark.parametrize("M", [1, 16, 128, 1024, 8192])
def test_gate_up_token_sweep_sampled(cr, M):
    w = workloads.WORKLOADS[f"gate_up_m{M}"]
    _sampled(cr, f"gate_up_m{M}", w.linears[0])


@pytest.mark.parametrize("lin", [l for l in workloads.WORKLOADS["w4a8_36_layers_m4096"].linears
                                 if l.name in ("k_proj", "gate_proj", "down_proj")],
                         ids=lambda l: l.name)
def test_w4a8_layer_m4096_sampled(cr, lin):
    _sampled(cr, "w4a8_36_layers_m4096", lin, weight_bits=4, layer=35)


def test_convrot_linear_object(cr):
    w = workloads.WORKLOADS["single_linear_m32"]
    x, W, _ = workloads.workload_inputs(w, w.linears[0])
    layer = cr.ConvRotLinear(W.cuda())
    Y = layer(x.cuda())
    yb, _ = _oracle_linear(x, W, None, 8)
    _assert_close(Y, yb, "ConvRotLinear")
    layer4 = cr.ConvRotLinear(W.cuda(), weight_bits=4)
    Y4 = layer4(x.cuda())
    yb4, _ = _oracle_linear(x, W, None, 4)
    _assert_close(Y4, yb4, "ConvRotLinear int4")
