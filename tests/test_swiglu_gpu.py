"""Parity of the MLP boundary with the oracle, through the C ABI: the gate/up
GEMM whose epilogue writes H = SiLU(gate) * up, the interleaved weight
layout, the fold of down_proj's SmoothQuant scales into up_proj's row scales,
and the whole block down(SiLU(gate(x)) * up(x)) stage by stage and end to end.

Each stage is compared on the inputs the GPU produced for it (the oracle takes
the GPU's codes and scales), so that a rounding tie decided the other way in
one stage does not show up as an error in the next; the end-to-end check runs
the oracle from x alone with the output tolerance of the linear."""
import numpy as np
import pytest
import torch

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


def _rand_i8(shape, seed, lo=-127, hi=128):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi, shape, generator=g, dtype=torch.int16).to(torch.int8)


def _rand_scales(n, seed, lo=1e-5, span=1e-3):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(n, generator=g, dtype=torch.float64) * span + lo).float()


def _acc_rows(X, W, rows, chunk=2048):
    """Exact int64 accumulators of the sampled token rows, in weight-row chunks."""
    Xs = X[rows].astype(np.float64)
    out = np.empty((len(rows), W.shape[0]), dtype=np.int64)
    for n0 in range(0, W.shape[0], chunk):
        out[:, n0:n0 + chunk] = (Xs @ W[n0:n0 + chunk].astype(np.float64).T).astype(np.int64)
    return out


def _h_ref_rows(X, st, Wgu, sgu, rows):
    """The oracle's H for the sampled rows (float64, then bf16), from exact sums."""
    acc = _acc_rows(X, Wgu, rows)
    y = ref.dequant(acc, st[rows], sgu)
    M, N2 = y.shape
    yv = y.reshape(M, N2 // 32, 2, 16)
    g = yv[:, :, 0, :].reshape(M, N2 // 2)
    u = yv[:, :, 1, :].reshape(M, N2 // 2)
    h = ref.silu(g) * u
    return ref.to_bf16(h), h


def _assert_bf16_step(got, hb, h64, what):
    # fp32 products and SiLU, one bf16 rounding: within one bf16 step of the
    # correctly rounded float64 value
    err = np.abs(got - hb)
    tol = _tol.bf16_ulp(h64) * 1.0001
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outputs off, worst {(err - tol).max():.3e}"


# ------------------------------------------------------------------ layout
@pytest.mark.parametrize("dtype,shape", [(torch.bfloat16, (48, 40)), (torch.int8, (64, 256)),
                                         (torch.float32, (1536,)), (torch.uint8, (32, 128))])
def test_interleave_gate_up_bit_exact(cr, dtype, shape):
    g = torch.Generator().manual_seed(5)
    if dtype.is_floating_point:
        A = torch.randn(shape, generator=g).to(dtype)
        B = torch.randn(shape, generator=g).to(dtype)
    else:
        A = torch.randint(0, 100, shape, generator=g).to(dtype)
        B = torch.randint(100, 200, shape, generator=g).to(dtype)
    out = cr.convrot_interleave_gate_up(A.cuda(), B.cuda()).cpu()
    want = ref.interleave_gate_up(A.view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy(),
                                  B.view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy())
    got = out.view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy()
    assert np.array_equal(got, want)


def test_interleave_rejects_partial_blocks(cr):
    A = torch.zeros(40, 16, dtype=torch.int8, device="cuda")
    with pytest.raises(cr.ConvRotError):
        cr.convrot_interleave_gate_up(A, A)


def test_fold_row_scales(cr):
    s = _rand_scales(4096, 7)
    sm = _rand_scales(4096, 8, lo=1e-2, span=30.0)
    got = cr.convrot_fold_row_scales(s.clone().cuda(), sm.cuda()).cpu().numpy()
    # one correctly rounded fp32 division of the fp32 inputs
    assert np.array_equal(got, s.numpy() / sm.numpy())
    np.testing.assert_allclose(got, ref.fold_smooth_into_rows(s.double().numpy(), sm.double().numpy()),
                               rtol=2.0 ** -24)


# ------------------------------------------------------------------ the GEMM
SHAPES = [
    # (M, I, K): swapped operand roles for M <= 128, CTA pairs above; I = 48
    # and 520 leave a partial 128- or 256-row weight tile; (100, 9600): 19200
    # weight rows, more 128-row decode tiles than SMs
    (1, 256, 512), (3, 48, 256), (16, 1024, 4096), (40, 528, 1040), (128, 2048, 4096),
    (100, 9600, 1040),
    (129, 272, 512), (256, 1024, 4096), (300, 1040, 1040), (512, 1536, 4096),
]


@pytest.mark.parametrize("M,I,K", SHAPES)
def test_int8_linear_swiglu(cr, M, I, K):
    X = _rand_i8((M, K), M + 3 * K)
    W = _rand_i8((2 * I, K), I + 5 * K)
    # scales that put g and u in the range where SiLU is neither linear nor
    # zero: a typical |acc| is 127^2 / 3 * sqrt(K)
    base = 1.0 / (127.0 ** 2 / 3.0 * K ** 0.5)
    st = _rand_scales(M, 1, lo=base, span=2 * base)
    sgu = _rand_scales(2 * I, 2, lo=0.5, span=3.0)
    H = cr.convrot_int8_linear_swiglu(X.cuda(), st.cuda(), W.cuda(), sgu.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    hb, h64, _ = ref.swiglu_linear(X.numpy(), st.double().numpy(), W.numpy(), sgu.double().numpy())
    assert np.abs(h64).max() > 1.0  # the activation's non-linear range is exercised
    _assert_bf16_step(_f64(H), hb, h64, f"swiglu {M}x{I}x{K}")


@pytest.mark.parametrize("M,I,K", [(1, 256, 512), (33, 528, 1056), (129, 272, 512), (512, 1536, 4096)])
def test_w4a8_linear_swiglu(cr, M, I, K):
    X = _rand_i8((M, K), 2 * M + K)
    codes = torch.randint(-8, 8, (2 * I, K), generator=torch.Generator().manual_seed(I + K))
    packed = torch.from_numpy(ref.pack_int4(codes.numpy()))
    st = _rand_scales(M, 3)
    sgu = _rand_scales(2 * I, 4, lo=1e-3, span=2e-2)
    H = cr.convrot_w4a8_linear_swiglu(X.cuda(), st.cuda(), packed.cuda(), sgu.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    hb, h64, _ = ref.swiglu_linear(X.numpy(), st.double().numpy(), ref.unpack_int4(packed.numpy()),
                                   sgu.double().numpy())
    _assert_bf16_step(_f64(H), hb, h64, f"w4a8 swiglu {M}x{I}x{K}")


# Shapes whose plan splits tiles by K: partial tiles meet in the workspace and
# the finalising unit applies the SwiGLU epilogue to the summed accumulators.
STREAM_K = [(16, 2048, 12288), (768, 3200, 12288)]


@pytest.mark.parametrize("M,I,K", STREAM_K)
def test_swiglu_stream_k_sampled_and_workspace_clean(cr, M, I, K):
    assert cr.convrot_swiglu_workspace_bytes(M, I, K, 8) > 0
    ws = cr.Workspace()
    X = _rand_i8((M, K), 17)
    W = _rand_i8((2 * I, K), 18)
    st = _rand_scales(M, 5)
    sgu = _rand_scales(2 * I, 6, lo=1e-4, span=2e-3)
    Xd, Wd, std, sgd = X.cuda(), W.cuda(), st.cuda(), sgu.cuda()
    rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 24)])
    hb, h64 = _h_ref_rows(X.numpy(), st.double().numpy(), W.numpy(), sgu.double().numpy(), rows)
    first = None
    for _ in range(2):
        H = cr.convrot_int8_linear_swiglu(Xd, std, Wd, sgd, workspace=ws)
        torch.cuda.synchronize()
        got = _f64(H)
        _assert_bf16_step(got[rows], hb, h64, f"stream-K swiglu {M}x{I}x{K}")
        if first is None:
            first = got
        else:
            assert np.array_equal(first, got)  # integer sums: the same bits every call
    assert int(ws.buf.count_nonzero().item()) == 0


def test_swiglu_full_size_gate_up_sampled(cr):
    # the gate/up projection of the decoder layer's MLP at the bench size
    M, I, K = 2048, 12288, 4096
    X = _rand_i8((M, K), 21)
    W = _rand_i8((2 * I, K), 22)
    st = _rand_scales(M, 7)
    sgu = _rand_scales(2 * I, 8, lo=1e-4, span=1e-3)
    H = cr.convrot_int8_linear_swiglu(X.cuda(), st.cuda(), W.cuda(), sgu.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    rows = np.unique(np.r_[0, 255, 256, M - 1, np.random.default_rng(3).integers(0, M, 12)])
    hb, h64 = _h_ref_rows(X.numpy(), st.double().numpy(), W.numpy(), sgu.double().numpy(), rows)
    _assert_bf16_step(_f64(H)[rows], hb, h64, "full-size swiglu")


def test_swiglu_edge_cases(cr):
    # M = 0 does nothing; I not a multiple of 16 and an odd row count are rejected
    X = torch.zeros(0, 256, dtype=torch.int8, device="cuda")
    W = torch.zeros(64, 256, dtype=torch.int8, device="cuda")
    s = torch.ones(64, device="cuda")
    H = cr.convrot_int8_linear_swiglu(X, s[:0], W, s)
    assert H.shape == (0, 32)
    with pytest.raises(cr.ConvRotError):
        cr.convrot_int8_linear_swiglu(torch.zeros(4, 256, dtype=torch.int8, device="cuda"), s[:4],
                                      W[:40], s[:40])
    # all-zero up rows give exactly zero, whatever the gate
    M, I, K = 20, 64, 256
    Xr = _rand_i8((M, K), 9).cuda()
    Wr = _rand_i8((2 * I, K), 10)
    sg = _rand_scales(2 * I, 11).cuda()
    Wr.view(I // 16, 2, 16, K)[:, 1] = 0
    Hz = cr.convrot_int8_linear_swiglu(Xr, _rand_scales(M, 12).cuda(), Wr.cuda(), sg)
    assert int(Hz.count_nonzero().item()) == 0


# ------------------------------------------------------------------ the MLP block
def _mlp_inputs(M, Hd, I, seed=0):
    import workloads
    x = workloads.activations(M, Hd, outlier_count=max(1, Hd // 100), seed=seed)
    nw = workloads.norm_weight(Hd)
    Wg = workloads.weight(I, Hd, seed=1)
    Wu = workloads.weight(I, Hd, seed=2)
    Wd = workloads.weight(Hd, I, seed=3)
    return x, nw, Wg, Wu, Wd


def test_mlp_block_stages_and_end_to_end(cr):
    M, Hd, I = 96, 512, 1024
    eps = 1e-6
    x, nw, Wg, Wu, Wd = _mlp_inputs(M, Hd, I)
    xd, Wgd, Wud, Wdd = x.cuda(), Wg.cuda(), Wu.cuda(), Wd.cuda()
    # ---- GPU, every step through the C ABI
    col, nwf = cr.convrot_smoothquant_calibrate(xd, nw.cuda(), torch.cat([Wgd, Wud]), eps, 0.5)
    Wq_g, s_g = cr.convrot_quantize_weight(Wgd, 256, col)
    Wq_u, s_u = cr.convrot_quantize_weight(Wud, 256, col)
    Wq_gu = cr.convrot_interleave_gate_up(Wq_g, Wq_u)
    Xq, s_tok = cr.convrot_rotate_quant_act(xd, 256, nwf, eps)
    h0 = cr.convrot_int8_linear_swiglu(Xq, s_tok, Wq_gu, cr.convrot_interleave_gate_up(s_g, s_u))
    smooth_d, _ = cr.convrot_smoothquant_calibrate(h0, None, Wdd, eps, 0.5)
    s_u_f = cr.convrot_fold_row_scales(s_u.clone(), smooth_d)
    s_gu = cr.convrot_interleave_gate_up(s_g, s_u_f)
    h = cr.convrot_int8_linear_swiglu(Xq, s_tok, Wq_gu, s_gu)
    Hq, s_h = cr.convrot_rotate_quant_act(h, 256, None, eps)
    Wq_d, s_d = cr.convrot_quantize_weight(Wdd, 256, smooth_d)
    y = cr.convrot_int8_linear(Hq, s_h, Wq_d, s_d)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0

    # ---- stage by stage on the GPU's own inputs
    sd_ref = ref.smoothquant_scales_of(_f64(h0), _f64(Wd))
    np.testing.assert_allclose(_f64(smooth_d), sd_ref, rtol=16 * _tol.U)
    hb, h64, _ = ref.swiglu_linear(Xq.cpu().numpy(), _f64(s_tok), Wq_gu.cpu().numpy(), _f64(s_gu))
    _assert_bf16_step(_f64(h), hb, h64, "MLP H")
    q_ref, s_ref, v = ref.rotate_quant_act(_f64(h), 256)
    ratio, _ = _tol.row_error(v, 256, False)
    assert np.all(np.abs(_f64(s_h) - s_ref) <= _tol.scale_rel_tol(ratio, False) * s_ref)
    _tol.check_codes(Hq.cpu().numpy(), q_ref, v / np.where(s_ref > 0, s_ref, 1)[:, None],
                     _tol.int8_code_window(ratio), "down_proj input codes")
    yb, y64, _ = ref.int8_linear(Hq.cpu().numpy(), _f64(s_h), Wq_d.cpu().numpy(), _f64(s_d))
    _assert_bf16_step(_f64(y), yb, y64, "MLP output")

    # ---- end to end: the oracle from x alone.  Where a rounding decision of
    # the GPU (an int8 code at a tie, a bf16 value of H one step off) is one of
    # the correct results, checked here, the oracle continues from the GPU's
    # choice so that the comparison tests what is unique.
    x64, nw64 = _f64(x), nw.double().numpy()
    sc, wf = ref.smoothquant_scales(x64, nw64, eps, np.concatenate([_f64(Wg), _f64(Wu)]), 0.5)
    extra = 16 * _tol.U  # the two sides' calibrated scales differ by fp32 rounding

    def adopt_w(gpu_q, W64, cs):
        q, s_r, Wr = ref.quantize_weight(W64, 256, cs)
        s64 = np.max(np.abs(Wr), axis=1) / 127.0
        r, _ = _tol.row_error(Wr, 256, cs is not None, extra)
        _tol.check_codes(gpu_q, q, Wr / np.where(s64 > 0, s64, 1.0)[:, None], _tol.int8_code_window(r),
                         "weight codes")
        return np.where(gpu_q != q, gpu_q, q), s_r.astype(np.float64)

    def adopt_act(gpu_q, a64, nwv, pre):
        q, s_r, v = ref.rotate_quant_act(a64, 256, nwv, eps)
        r, _ = _tol.row_error(v, 256, pre, extra)
        _tol.check_codes(gpu_q, q, v / np.where(s_r > 0, s_r, 1.0)[:, None], _tol.int8_code_window(r),
                         "activation codes")
        return np.where(gpu_q != q, gpu_q, q), s_r

    def adopt_h(gpu_h, hb, h64, rel):
        err = np.abs(gpu_h - hb)
        assert np.all(err <= _tol.bf16_ulp(h64) * 1.0001 + rel * np.abs(h64)), "H beyond one bf16 step"
        return gpu_h

    qg, sg = adopt_w(Wq_g.cpu().numpy(), _f64(Wg), sc)
    qu, su = adopt_w(Wq_u.cpu().numpy(), _f64(Wu), sc)
    qgu = ref.interleave_gate_up(qg, qu)
    Xq_r, st_r = adopt_act(Xq.cpu().numpy(), x64, wf, True)
    hb0, h064, _ = ref.swiglu_linear(Xq_r, st_r, qgu, ref.interleave_gate_up(sg, su))
    h0_r = adopt_h(_f64(h0), hb0, h064, 8 * _tol.U)
    sd_r = ref.smoothquant_scales_of(h0_r, _f64(Wd))
    hb1, h164, _ = ref.swiglu_linear(Xq_r, st_r, qgu,
                                     ref.interleave_gate_up(sg, ref.fold_smooth_into_rows(su, sd_r)))
    h_r = adopt_h(_f64(h), hb1, h164, 8 * _tol.U + extra)
    Hq_r, sh_r = adopt_act(Hq.cpu().numpy(), h_r, None, False)
    qd, sdr = adopt_w(Wq_d.cpu().numpy(), _f64(Wd), sd_r)
    y_r, _, _ = ref.int8_linear(Hq_r, sh_r, qd, sdr)
    err = np.abs(_f64(y) - y_r)
    tol = _tol.output_tol(y_r)
    assert not (err > tol).any(), f"{(err > tol).sum()} MLP outputs off, worst {(err - tol).max():.3e}"


def test_convrot_mlp_class_matches_the_abi_steps(cr):
    M, Hd, I = 64, 512, 1024
    x, nw, Wg, Wu, Wd = _mlp_inputs(M, Hd, I, seed=4)
    mlp = cr.ConvRotMLP(Wg.cuda(), Wu.cuda(), Wd.cuda(), norm_w=nw.cuda(), x_calib=x.cuda())
    y = mlp(x.cuda())
    torch.cuda.synchronize()
    assert y.shape == (M, Hd) and torch.isfinite(y.float()).all()
    # the same block through the oracle's float path (no quantisation) is
    # close: W8A8 with rotation keeps the relative error small
    x64 = _f64(x)
    a = ref.rmsnorm(x64, nw.double().numpy(), 1e-6)
    h = ref.silu(a @ _f64(Wg).T) * (a @ _f64(Wu).T)
    y_f = h @ _f64(Wd).T
    rel = np.linalg.norm(_f64(y) - y_f) / np.linalg.norm(y_f)
    assert rel < 0.05, rel


def test_w4a8_swiglu_stream_k_and_max_k(cr):
    # int4 weights through the split-tile schedule, and the longest K the ABI takes
    for (M, I, K) in [(768, 3200, 12288), (3, 16, 131072)]:
        X = _rand_i8((M, K), M + 1)
        codes = torch.randint(-8, 8, (2 * I, K), generator=torch.Generator().manual_seed(K))
        packed = torch.from_numpy(ref.pack_int4(codes.numpy()))
        st = _rand_scales(M, 13)
        sgu = _rand_scales(2 * I, 14, lo=1e-3, span=2e-2)
        H = cr.convrot_w4a8_linear_swiglu(X.cuda(), st.cuda(), packed.cuda(), sgu.cuda())
        torch.cuda.synchronize()
        assert cr.convrot_device_status() == 0
        rows = np.unique(np.r_[0, M - 1, np.random.default_rng(K).integers(0, M, 8)])
        hb, h64 = _h_ref_rows(X.numpy(), st.double().numpy(), ref.unpack_int4(packed.numpy()),
                              sgu.double().numpy(), rows)
        _assert_bf16_step(_f64(H)[rows], hb, h64, f"w4a8 swiglu {M}x{I}x{K}")
