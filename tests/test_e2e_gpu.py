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


def _check_calibration(x64, nw, W64, gpu_calib):
    """The GPU's SmoothQuant calibration against the oracle's, within the
    bounds of the calibration parity test (MOSS-Image card, "How it was made":
    alpha 0.5, folded as (1 + w) / s - 1); returns the oracle's (s, w') and
    the relative input perturbations the GPU's values add to each operand.

    Both sides derive the scale s and the folded norm weight w' on their own
    (fp32 on the GPU, float64 in the oracle).  Checked here:
      |s_gpu - s| <= 8u s,   |w'_gpu - w'| <= 10u |1 + w'| + 2u |w'|.
    s multiplies the weight's columns: a relative perturbation of at most 8u.
    The activation is multiplied by 1 + w'_gpu, whose relative distance from
    1 + w' is at most 10u + 2u |w'| / |1 + w'| (the fp32 rounding of w' is
    large against 1 + w' where w' is close to -1, i.e. where s is large).
    Both enter the code decisions through the error model's input term."""
    s_ref, f_ref = ref.smoothquant_scales(x64, nw.double().numpy(), 1e-6, W64, 0.5)
    sg, fg = (t.cpu().double().numpy() for t in gpu_calib)
    assert np.all(np.abs(sg - s_ref) <= 8 * _tol.U * s_ref), "SmoothQuant scale"
    m = np.abs(1.0 + f_ref)
    assert np.all(np.abs(fg - f_ref) <= 10 * _tol.U * m + 2 * _tol.U * np.abs(f_ref)), "folded norm weight"
    extra_x = 10 * _tol.U + 2 * _tol.U * float(np.max(np.abs(f_ref) / m))
    return s_ref, f_ref, extra_x, 8 * _tol.U


def _gpu_linear(cr, x, W, nw, weight_bits, group=256):
    """Every step on the GPU; returns Y, the codes the kernels chose and the
    GPU's calibration (scale, folded norm weight) or None."""
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
    Wc = Wq.cpu().numpy()
    if weight_bits == 4:
        Wc = ref.unpack_int4(Wc)
    calib = None if nw is None else (col, nwd)
    return Y, Xq.cpu().numpy(), (Wc, s_row.cpu().double().numpy()), calib


def _reference(x, W, nw, weight_bits, gpu_xq, gpu_wq, rows=None, cols=None, group=256,
               gpu_calib=None):
    """The oracle's output for the sampled rows/cols.

    Where the GPU chose the other code of a rounding tie (checked here to lie
    inside the fp32 tie window, and to be rare), both codes are correct; the
    reference then follows the GPU's choice so that the output comparison
    tests the part of the result that is unique."""
    x64, W64 = _f64(x), _f64(W)
    gpu_wq, gpu_srow = gpu_wq
    col = nwf = None
    extra_x = extra_w = 0.0
    if nw is not None:
        col, nwf, extra_x, extra_w = _check_calibration(x64, nw, W64, gpu_calib)
    if rows is not None:
        x64, gpu_xq = x64[rows], gpu_xq[rows]
    if cols is not None:
        W64, gpu_wq, gpu_srow = W64[cols], gpu_wq[cols], gpu_srow[cols]
    Xq, s_tok, v = ref.rotate_quant_act(x64, group, nwf, 1e-6)
    ratio, amax = _tol.row_error(v, group, nw is not None, extra_x)
    safe = np.where(s_tok > 0, s_tok, 1.0)[:, None]
    flips_x = _tol.check_codes(gpu_xq, Xq, v / safe, _tol.int8_code_window(ratio), "act codes")
    if weight_bits == 8:
        Wq, s_row, Wr = ref.quantize_weight(W64, group, col)
        s64 = np.max(np.abs(Wr), axis=1) / 127.0
        wr, _ = _tol.row_error(Wr, group, col is not None, extra_w)
        flips_w = _tol.check_codes(gpu_wq, Wq, Wr / np.where(s64 > 0, s64, 1.0)[:, None],
                                   _tol.int8_code_window(wr), "weight codes")
    else:
        o = ref.quantize_weight_w4(W64, group, col)
        Wq, s_row, Wr, s64 = o["codes"].astype(np.int64), o["s_row"], o["rotated"], o["s64"].copy()
        wr, _ = _tol.row_error(Wr, group, col is not None, extra_w)
        # every row's clip: the GPU's choice must be on the grid and within the
        # fp32 evaluation error of the float64 optimum (a neighbouring clip of
        # equal error is an equally correct result); the reference then takes
        # the oracle's codes at the GPU's clip and compares them code by code
        grid = ref.clip_grid(0.80, 1.00, 21)
        amax = np.max(np.abs(Wr), axis=1)
        s_row = s_row.astype(np.float64)
        flips_w = 0
        for n in range(Wr.shape[0]):
            if amax[n] == 0:
                assert gpu_srow[n] == 0 and not gpu_wq[n].any()
                continue
            s64[n], Wq[n] = _tol.check_w4_clip(Wr[n], gpu_srow[n], amax[n], o["err"][n], wr[n], grid)
            s_row[n] = np.float32(s64[n])
            flips_w += _tol.check_codes(gpu_wq[n:n + 1], Wq[n:n + 1], (Wr[n] / s64[n])[None, :],
                                        np.array([_tol.int4_code_window(wr[n])]), "int4 weight codes")
    Xa = np.where(gpu_xq != Xq, gpu_xq, Xq)
    Wa = np.where(gpu_wq != Wq, gpu_wq, Wq)
    yb, y, _ = ref.int8_linear(Xa, s_tok, Wa, s_row)
    return yb, flips_x + flips_w, Xq.size + Wq.size


def _assert_close(Y, y_ref, what):
    got = _f64(Y) if isinstance(Y, torch.Tensor) else Y
    tol = _tol.output_tol(y_ref)
    err = np.abs(got - y_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} outputs out of tolerance, worst "
                           f"{(err - tol).max():.3e}")


def _full(cr, x, W, nw, bits, group=256, what=""):
    Y, xq, wq, calib = _gpu_linear(cr, x, W, nw, bits, group)
    yb, flips, n = _reference(x, W, nw, bits, xq, wq, group=group, gpu_calib=calib)
    _assert_close(Y, yb, what)
    return flips, n


def test_single_linear_m32_all_outputs(cr):
    w = workloads.WORKLOADS["single_linear_m32"]
    x, W, nw = workloads.workload_inputs(w, w.linears[0])
    _full(cr, x, W, nw, 8, what="single linear")


def test_single_linear_group0_fallback(cr):
    w = workloads.WORKLOADS["single_linear_m32"]
    x, W, _ = workloads.workload_inputs(w, w.linears[0])
    _full(cr, x, W, None, 8, group=0, what="group 0")


def test_down_proj_m512_with_norm_all_outputs(cr):
    w = workloads.WORKLOADS["down_proj_m512"]
    x, W, nw = workloads.workload_inputs(w, w.linears[0])
    flips, n = _full(cr, x, W, nw, 8, what="down_proj with RMSNorm + SmoothQuant")
    assert flips <= 1e-4 * n


def _tile_sample(n, rng, count):
    """Indices into n rows or columns: `count` random ones, the first and the
    last, and one random index from every block of 128.  Every output tile
    the kernels use (128 x 16..128 in the swapped roles, 256 x 256 for CTA
    pairs, split or not) then holds at least one checked row and column."""
    pick = [rng.choice(n, min(count, n), replace=False), [0, n - 1]]
    pick += [[b + int(rng.integers(min(128, n - b)))] for b in range(0, n, 128)]
    return np.unique(np.concatenate(pick))


def _sampled(cr, wname, lin, M=None, weight_bits=8, layer=0, nrows=24, ncols=160):
    w = workloads.WORKLOADS[wname]
    x, W, nw = workloads.workload_inputs(w, lin, M=M, layer=layer)
    Y, xq, wq, calib = _gpu_linear(cr, x, W, nw, weight_bits)
    rng = np.random.default_rng(lin.N + lin.K + x.shape[0])
    rows = _tile_sample(x.shape[0], rng, nrows)
    cols = _tile_sample(lin.N, rng, ncols)
    yb, flips, n = _reference(x, W, nw, weight_bits, xq, wq, rows, cols, gpu_calib=calib)
    _assert_close(_f64(Y)[np.ix_(rows, cols)], yb, f"{wname}/{lin.name}")
    assert flips <= max(2, 1e-4 * n)


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
    for bits in (8, 4):
        layer = cr.ConvRotLinear(W.cuda(), weight_bits=bits)
        Y = layer(x.cuda())
        xq, _ = cr.convrot_rotate_quant_act(x.cuda())
        wq = layer.Wq.cpu().numpy()
        if bits == 4:
            wq = ref.unpack_int4(wq)
        yb, _, _ = _reference(x, W, None, bits, xq.cpu().numpy(),
                              (wq, layer.s_row.cpu().double().numpy()))
        _assert_close(Y, yb, f"ConvRotLinear int{bits}")


@pytest.mark.parametrize("K,N", [(1152, 4304), (4304, 1152)])
def test_group16_vision_linear_all_outputs(cr, K, N):
    # a vision-tower linear with 16-point ConvRot groups ("Qwen3-VL 8B - INT8
    # ConvRot", "Layer and group selection"): widths 1152 and 4304
    x = workloads.activations(64, K, outlier_count=K // 100, seed=K)
    W = workloads.weight(N, K, seed=N)
    _full(cr, x, W, None, 8, group=16, what=f"group-16 linear {K}->{N}")


@pytest.mark.parametrize("bits,group,K", [(8, 256, 4096), (4, 256, 1024), (8, 16, 1152)])
def test_checkpoint_round_trip_runs_the_same_layer(cr, tmp_path, bits, group, K):
    # a layer prepared on the GPU, written as a comfy_quant checkpoint, read
    # back and run: the stored codes and scales give the same output bits
    from w8a8_int8_quantized_rmsnorm_b200 import checkpoint as ck
    N = 512
    x = workloads.activations(48, K, outlier_count=K // 100, seed=5).cuda()
    lin = cr.ConvRotLinear(workloads.weight(N, K, seed=6).cuda(), weight_bits=bits, group=group)
    y0 = lin(x)
    p = str(tmp_path / "layer.safetensors")
    ck.save_quantized_layers(p, {"model.layers.3.mlp.down_proj": lin.to_checkpoint()})
    loaded = ck.load_quantized_layers(p)["model.layers.3.mlp.down_proj"]
    assert loaded["meta"]["convrot_groupsize"] == group
    lin2 = cr.ConvRotLinear.from_checkpoint(loaded)
    y1 = lin2(x)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


@pytest.mark.parametrize("sizes,K", [((4096, 1024, 1024), 4096), ((12288, 64), 4096), ((256, 48, 16), 512)])
def test_fused_projection_set_equals_separate_linears(cr, sizes, K):
    # one GEMM over concatenated rows gives each member's output bit for bit
    M = 96
    x = workloads.activations(M, K, outlier_count=K // 100, seed=7).cuda()
    nw = workloads.norm_weight(K).cuda()
    Ws = [workloads.weight(n, K, seed=10 + i).cuda() for i, n in enumerate(sizes)]
    fused = cr.ConvRotFusedLinear(Ws, norm_w=nw, x_calib=x)
    outs = fused(x)
    for W, y in zip(Ws, outs):
        lin = cr.ConvRotLinear(W, norm_w=fused.linear.norm_w, col_scale=fused.col_scale)
        assert torch.equal(lin(x), y)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0


@pytest.mark.parametrize("wname,sizes", [("attn_qkv_m2048", (4096, 1024, 1024)),
                                         ("gdn_in_proj_m2048", (12288, 64))])
def test_fused_projection_set_against_oracle(cr, wname, sizes):
    """A fused projection set (MOSS-Image card, file table, "Quantized" row:
    attention and gated-DeltaNet projections are quantised) against the
    oracle: one SmoothQuant calibration over the concatenated members'
    columns (they share the input and its norm), every member's rows
    quantised on their own, and each member's output the matching columns of
    the fused result."""
    w = workloads.WORKLOADS[wname]
    K = w.linears[0].K
    x = workloads.activations(w.M, K, outlier_count=w.n_outliers(K), outlier_scale=w.outlier_scale)
    nw = workloads.norm_weight(K)
    Ws = [workloads.weight(n, K, seed=10 + i) for i, n in enumerate(sizes)]
    xd = x.cuda()
    fused = cr.ConvRotFusedLinear([W.cuda() for W in Ws], norm_w=nw.cuda(), x_calib=xd)
    outs = fused(xd)
    assert [o.shape[1] for o in outs] == list(sizes)
    Y = torch.cat(outs, dim=1)
    xq, _ = cr.convrot_rotate_quant_act(xd, 256, fused.linear.norm_w, 1e-6)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    Wcat = torch.cat(Ws)
    # outputs on a tile-covering sample, against the oracle run on the
    # concatenated weight with one calibration over all members' columns
    # (checked against the GPU's shared calibration inside _reference)
    rng = np.random.default_rng(sum(sizes))
    rows = _tile_sample(w.M, rng, 24)
    cols = _tile_sample(sum(sizes), rng, 160)
    wq = (fused.linear.Wq.cpu().numpy(), fused.linear.s_row.cpu().double().numpy())
    yb, flips, n = _reference(x, Wcat, nw, 8, xq.cpu().numpy(), wq, rows, cols,
                              gpu_calib=(fused.col_scale, fused.linear.norm_w))
    _assert_close(_f64(Y)[np.ix_(rows, cols)], yb, f"{wname} fused set")
    assert flips <= max(2, 1e-4 * n)
