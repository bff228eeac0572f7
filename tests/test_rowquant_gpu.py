"""Parity of the row-quantisation kernels (activation rotate-quantise with the
fused RMSNorm, int8 and int4 weight preparation, SmoothQuant calibration)
against the CPU oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import workloads
from oracle import convrot_ref as ref
from tests import _tol

pytestmark = pytest.mark.gpu

cuda_ok = torch.cuda.is_available()


@pytest.fixture(scope="module")
def cr():
    if not cuda_ok:
        pytest.skip("needs a CUDA device")
    import w8a8_int8_quantized_rmsnorm_b200 as m
    m.lib()
    return m


def _f64(t):
    return t.detach().float().cpu().double().numpy()


def _check_act(cr, x_bf16, group, norm_w=None, eps=1e-6, max_flip_frac=None):
    x_dev = x_bf16.cuda()
    nw_dev = None if norm_w is None else norm_w.cuda()
    Xq, s_tok = cr.convrot_rotate_quant_act(x_dev, group, nw_dev, eps)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    q_ref, s_ref, v = ref.rotate_quant_act(_f64(x_bf16), group,
                                           None if norm_w is None else norm_w.double().numpy(), eps)
    ratio, amax = _tol.row_error(v, group, norm_w is not None)
    s_gpu = s_tok.cpu().double().numpy()
    tol = _tol.scale_rel_tol(ratio, norm_w is not None)
    zero = amax == 0
    assert np.all(s_gpu[zero] == 0)
    rel = np.abs(s_gpu - s_ref) / np.where(zero, 1.0, s_ref)
    assert np.all(rel <= tol), f"s_tok rel err {rel.max():.3e} > {tol[np.argmax(rel - tol)]:.3e}"
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(zero[:, None], 0.0, v / np.where(zero, 1.0, s_ref)[:, None])
    flips = _tol.check_codes(Xq.cpu().numpy(), q_ref, z, _tol.int8_code_window(ratio))
    if max_flip_frac is not None:
        assert flips <= max_flip_frac * q_ref.size
    return flips


@pytest.mark.parametrize("M", [1, 3, 33, 129])
@pytest.mark.parametrize("K", [256, 512, 768, 4096, 12288])
@pytest.mark.parametrize("norm", [False, True])
def test_act_rotate_quant_shapes(cr, M, K, norm):
    x = workloads.activations(M, K, outlier_count=max(1, K // 100), seed=M * 7 + K)
    nw = workloads.norm_weight(K) if norm else None
    _check_act(cr, x, 256, nw)


@pytest.mark.parametrize("K", [16, 48, 512, 1040, 4304])
def test_act_group0_plain_rowwise(cr, K):
    # widths the group does not divide fall back to plain row-wise int8
    x = workloads.activations(37, K, seed=K)
    _check_act(cr, x, 0)
    _check_act(cr, x, 0, workloads.norm_weight(K))


@pytest.mark.parametrize("M", [1, 37, 300])
@pytest.mark.parametrize("K", [16, 48, 1152, 4096, 4304])
@pytest.mark.parametrize("norm", [False, True])
def test_act_group16(cr, M, K, norm):
    # 16-point groups for widths 256 does not divide ("Qwen3-VL 8B - INT8
    # ConvRot", "Layer and group selection": vision widths 1152 and 4304)
    x = workloads.activations(M, K, outlier_count=max(1, K // 100), seed=M + K)
    _check_act(cr, x, 16, workloads.norm_weight(K) if norm else None)


@pytest.mark.parametrize("K", [16640, 32768, 131072])
def test_act_streaming_path_large_K(cr, K):
    # rows wider than one CTA team are processed in two passes
    x = workloads.activations(5, K, dist="student_t3", outlier_count=K // 100, seed=3)
    _check_act(cr, x, 256, workloads.norm_weight(K))
    _check_act(cr, x, 256)


def test_act_edge_rows(cr):
    K = 512
    x = torch.zeros(8, K)
    x[1] = 3.0                       # constant row -> one nonzero per group
    x[2, 300] = -2.5                 # one-hot -> a signed row of H
    x[3] = torch.linspace(-1, 1, K)  # smooth ramp
    x[4, ::2] = 1e-30                # tiny values (bf16 keeps the exponent range)
    x[5] = 3e30                      # huge constant
    x[6, 7] = 1.0
    x[6, 263] = 1.0
    x[7] = -x[3]
    xb = x.to(torch.bfloat16)
    _check_act(cr, xb, 256)
    _check_act(cr, xb, 256, workloads.norm_weight(K))
    _check_act(cr, xb, 0)


def test_act_exact_ties_round_half_even(cr):
    # group 0: values chosen so that v / s lands exactly on k + 1/2 with
    # absmax 127 (s = 1); round-half-even gives the even neighbour
    K = 16
    vals = [127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, -126.5, 100.5, 101.5, 0.0, 1.0, -1.0, 5.5, 6.5, 7.5]
    xb = torch.tensor([vals], dtype=torch.bfloat16)
    assert xb.float().tolist()[0] == vals
    Xq, s = cr.convrot_rotate_quant_act(xb.cuda(), 0)
    assert s.item() == 1.0
    assert Xq.cpu().tolist()[0] == [round(t) for t in vals]


def test_act_scale_invariance_with_norm(cr):
    x = workloads.activations(16, 1024, outlier_count=10)
    nw = workloads.norm_weight(1024).cuda()
    q1, s1 = cr.convrot_rotate_quant_act(x.cuda(), 256, nw, 0.0)
    q2, s2 = cr.convrot_rotate_quant_act((x.float() * 4.0).to(torch.bfloat16).cuda(), 256, nw, 0.0)
    assert torch.equal(q1, q2)
    assert torch.allclose(s1, s2, rtol=4e-7, atol=0)


@pytest.mark.parametrize("M,K,norm", [(5000, 1024, False), (2300, 2048, True), (1203, 4096, True),
                                      (601, 8192, False), (301, 16384, True), (901, 12288, False)])
def test_act_full_cta_plans(cr, M, K, norm):
    # M large enough that every CTA stages its full complement of rows: 32 warps
    # per CTA for teams of 1, 2, 4, 8 and 16 warps, 24 for the 12-warp team of
    # K = 12288; M is no multiple of the rows per stage, so the last unit is
    # ragged; every row checked
    x = workloads.activations(M, K, outlier_count=max(1, K // 100), seed=M + K)
    nw = workloads.norm_weight(K) if norm else None
    flips = _check_act(cr, x, 256, nw)
    assert flips <= 1e-4 * x.numel()


def test_act_full_size_down_proj(cr):
    # the down-proj workload at full size, every row checked
    w = workloads.WORKLOADS["down_proj_m512"]
    lin = w.linears[0]
    x, W, nw = workloads.workload_inputs(w, lin)
    flips = _check_act(cr, x, 256, nw)
    assert flips <= 1e-4 * x.numel()


def test_act_full_size_gate_up_sampled(cr):
    # M = 8192 x K = 4096 through the kernel at full size; sampled rows checked
    M, K = 8192, 4096
    x = workloads.activations(M, K, outlier_count=41)
    Xq, s_tok = cr.convrot_rotate_quant_act(x.cuda(), 256)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(M, 48, replace=False)
    rows = np.concatenate([rows, [0, M - 1]])
    q_ref, s_ref, v = ref.rotate_quant_act(_f64(x[rows]), 256)
    ratio, _ = _tol.row_error(v, 256, False)
    sg = s_tok.cpu().double().numpy()[rows]
    assert np.all(np.abs(sg - s_ref) <= _tol.scale_rel_tol(ratio, False) * s_ref)
    _tol.check_codes(Xq.cpu().numpy()[rows], q_ref, v / s_ref[:, None], _tol.int8_code_window(ratio))


# ---------------------------------------------------------------- weights
@pytest.mark.parametrize("N,K,group", [(8, 256, 256), (24, 512, 256), (136, 4096, 256), (40, 12288, 256),
                                       (16, 16640, 256), (24, 1152, 16), (40, 4304, 16), (8, 16640, 16)])
@pytest.mark.parametrize("colscale", [False, True])
def test_weight_int8(cr, N, K, group, colscale):
    W = workloads.weight(N, K, seed=N + K)
    cs = (torch.rand(K, generator=torch.Generator().manual_seed(5)) * 4 + 0.25) if colscale else None
    Wq, s_row = cr.convrot_quantize_weight(W.cuda(), group, None if cs is None else cs.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref32, Wr = ref.quantize_weight(_f64(W), group, None if cs is None else cs.double().numpy())
    s_ref = np.max(np.abs(Wr), axis=1) / 127.0
    ratio, _ = _tol.row_error(Wr, group, colscale)
    sg = s_row.cpu().double().numpy()
    assert np.all(np.abs(sg - s_ref) <= _tol.scale_rel_tol(ratio, False) * s_ref)
    _tol.check_codes(Wq.cpu().numpy(), q_ref, Wr / s_ref[:, None], _tol.int8_code_window(ratio))


def test_weight_int8_group0_and_zero_rows(cr):
    W = workloads.weight(16, 1040, seed=4).float()
    W[3] = 0
    Wb = W.to(torch.bfloat16)
    Wq, s_row = cr.convrot_quantize_weight(Wb.cuda(), 0)
    q_ref, _, Wr = ref.quantize_weight(_f64(Wb), 0)
    s_ref = np.max(np.abs(Wr), axis=1) / 127.0
    assert s_row[3].item() == 0 and not Wq[3].any()
    ratio, _ = _tol.row_error(Wr, 0, False)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s_ref[:, None] > 0, Wr / np.where(s_ref > 0, s_ref, 1)[:, None], 0)
    _tol.check_codes(Wq.cpu().numpy(), q_ref, z, _tol.int8_code_window(ratio))


def _w4_check(cr, W, group=256, cs=None, clip=(0.80, 1.00, 21)):
    Wq4, s_row = cr.convrot_quantize_weight_w4(W.cuda(), group, None if cs is None else cs.cuda(), *clip)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    out = ref.quantize_weight_w4(_f64(W), group, None if cs is None else cs.double().numpy(), *clip)
    Wr = out["rotated"]
    amax = np.max(np.abs(Wr), axis=1)
    grid = ref.clip_grid(*clip)
    sg = s_row.cpu().double().numpy()
    codes_gpu = ref.unpack_int4(Wq4.cpu().numpy()).astype(np.int64)
    ratio, _ = _tol.row_error(Wr, group, cs is not None)
    for n in range(W.shape[0]):
        if amax[n] == 0:
            assert sg[n] == 0 and not codes_gpu[n].any()
            continue
        s64, q = _tol.check_w4_clip(Wr[n], sg[n], amax[n], out["err"][n], ratio[n], grid)
        win4 = _tol.int4_code_window(ratio[n])
        _tol.check_codes(codes_gpu[n:n + 1], q[None, :], (Wr[n] / s64)[None, :], np.array([win4]),
                         "int4 codes")


@pytest.mark.parametrize("N,K", [(8, 256), (40, 512), (64, 4096), (16, 12288), (8, 16640)])
def test_weight_int4_clip_search(cr, N, K):
    _w4_check(cr, workloads.weight(N, K, seed=N * K))


@pytest.mark.parametrize("N,K", [(24, 1152), (8, 4320)])
def test_weight_int4_group16(cr, N, K):
    _w4_check(cr, workloads.weight(N, K, seed=N + 3 * K), group=16)


def test_weight_int4_group0_colscale_and_grid(cr):
    W = workloads.weight(24, 1056, seed=9)
    cs = torch.rand(1056, generator=torch.Generator().manual_seed(1)) + 0.5
    _w4_check(cr, W, 0, cs)
    _w4_check(cr, workloads.weight(16, 512, seed=2), 256, None, (1.0, 1.0, 1))
    _w4_check(cr, workloads.weight(16, 512, seed=3), 256, None, (0.5, 1.0, 51))


# ---------------------------------------------------------------- calibration
@pytest.mark.parametrize("M,K,N", [(64, 512, 32), (100, 4096, 40), (512, 12288, 64)])
def test_smoothquant_calibrate(cr, M, K, N):
    x = workloads.activations(M, K, dist="student_t3", outlier_count=max(1, K // 100),
                              outlier_scale=30.0)
    W = workloads.weight(N, K)
    nw = workloads.norm_weight(K)
    smooth, folded = cr.convrot_smoothquant_calibrate(x.cuda(), nw.cuda(), W.cuda(), 1e-6, 0.5)
    s_ref, f_ref = ref.smoothquant_scales(_f64(x), nw.double().numpy(), 1e-6, _f64(W), 0.5)
    sg = smooth.cpu().double().numpy()
    fg = folded.cpu().double().numpy()
    assert np.all(np.abs(sg - s_ref) <= 8 * _tol.U * s_ref)
    base = np.abs((1 + nw.double().numpy()) / s_ref)
    assert np.all(np.abs(fg - f_ref) <= 10 * _tol.U * base + 2 * _tol.U * np.abs(f_ref))
