"""Parity of the weight-only path with the oracle, through the C ABI: the
rotated bf16 activations, the bf16 tensor-core GEMM over int8 weight codes
(expanded in shared memory) with its fp32 accumulators, the bf16 output, and
the whole layer against the float product."""
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


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _i8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int16).to(torch.int8)


@pytest.mark.parametrize("M,K,group,norm", [(1, 256, 256, False), (37, 4096, 256, True), (5, 12288, 256, True),
                                            (64, 1152, 16, True), (9, 4304, 16, False), (33, 1040, 0, True),
                                            (3, 16640, 256, True)])
def test_rotate_act_bf16(cr, M, K, group, norm):
    x = workloads.activations(M, K, outlier_count=max(1, K // 100), seed=K + M)
    nw = workloads.norm_weight(K) if norm else None
    Xr = cr.convrot_rotate_act_bf16(x.cuda(), group, None if nw is None else nw.cuda(), 1e-6)
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    v = ref.rotate_act(_f64(x), group, None if nw is None else nw.double().numpy(), 1e-6)
    got = _f64(Xr)
    # fp32 transform and scale (error below 12u of the group's 2-norm), one bf16 rounding
    if group:
        gn = np.sqrt(np.sum(v.reshape(M, K // group, group) ** 2, axis=2))
        e32 = np.repeat(gn, group, axis=1) * 12 * _tol.U
    else:
        e32 = np.abs(v) * 6 * _tol.U
    err = np.abs(got - ref.to_bf16(v))
    assert np.all(err <= _tol.bf16_ulp(v) * 1.0001 + 2 * e32), f"worst {np.max(err - _tol.bf16_ulp(v)):.3e}"


# (16, 20480, 4096) and (100, 20480, 4096) split the K range of some tiles over
# two CTAs (stream-K with fp32 partial sums); the others run whole tiles
SHAPES = [(1, 256, 256), (16, 1024, 4096), (40, 520, 1040), (128, 4096, 4096), (129, 264, 512),
          (512, 4096, 4096), (1000, 1032, 2080), (16, 20480, 1024), (16, 20480, 4096),
          (100, 20480, 4096)]


def _operands(M, N, K):
    Xr = _bf16((M, K), M + K)
    Wq = _i8((N, K), N + K)
    s = (torch.rand(N, generator=torch.Generator().manual_seed(N)) * 1e-2 + 1e-3).float()
    return Xr, Wq, s


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_weight_only_accumulators(cr, M, N, K):
    Xr, Wq, _ = _operands(M, N, K)
    acc = cr.convrot_weight_only_gemm_f32(Xr.cuda(), Wq.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    X64, W64 = _f64(Xr), Wq.numpy().astype(np.float64)
    want = X64 @ W64.T
    mag = np.abs(X64) @ np.abs(W64).T
    err = np.abs(acc.cpu().double().numpy() - want)
    # products of bf16 and int8 are exact in fp32; only the fp32 sums round
    bound = 4 * np.sqrt(K) * _tol.U * mag + 1e-30
    assert np.all(err <= bound), f"worst relative to the bound {np.max(err / bound):.2f}"


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_weight_only_linear_bf16(cr, M, N, K):
    Xr, Wq, s = _operands(M, N, K)
    Y = cr.convrot_weight_only_linear(Xr.cuda(), Wq.cuda(), s.cuda())
    torch.cuda.synchronize()
    yb, y64 = ref.weight_only_linear(_f64(Xr), Wq.numpy(), s.double().numpy())
    mag = (np.abs(_f64(Xr)) @ np.abs(Wq.numpy().astype(np.float64)).T) * s.double().numpy()[None, :]
    err = np.abs(_f64(Y) - yb)
    assert np.all(err <= _tol.bf16_ulp(y64) * 1.0001 + 8 * np.sqrt(K) * _tol.U * mag)


@pytest.mark.parametrize("M,K,N,group", [(1, 4096, 1024, 256), (64, 4096, 4096, 256), (300, 12288, 1024, 256),
                                         (48, 1152, 4304, 16)])
def test_weight_only_layer_end_to_end(cr, M, K, N, group):
    x = workloads.activations(M, K, outlier_count=max(1, K // 100), seed=M)
    nw = workloads.norm_weight(K)
    W = workloads.weight(N, K, seed=N)
    lin = cr.ConvRotLinear(W.cuda(), group=group, norm_w=nw.cuda())
    Y = lin.forward_weight_only(x.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    # the oracle from x with the GPU's weight codes and scales (the weight
    # preparation's own parity is tested elsewhere)
    v = ref.rotate_act(_f64(x), group, nw.double().numpy(), 1e-6)
    yb, y64 = ref.weight_only_linear(ref.to_bf16(v), lin.Wq.cpu().numpy(), _f64(lin.s_row))
    tol = _tol.output_tol(y64)
    err = np.abs(_f64(Y) - y64)
    assert np.all(err <= tol), f"{np.sum(err > tol)} outputs off"
    # and the layer approximates the float product (weight rounding only)
    y_f = ref.rmsnorm(_f64(x), nw.double().numpy(), 1e-6) @ _f64(W).T
    assert np.linalg.norm(_f64(Y) - y_f) / np.linalg.norm(y_f) < 0.02


@pytest.mark.parametrize("M,N,K", [(17, 136, 256), (65, 264, 512), (2, 16, 131072)])
def test_weight_only_ragged_token_tiles_and_max_k(cr, M, N, K):
    # partial token tiles of every width the swapped roles use, and the longest K
    Xr, Wq, s = _operands(M, N, K)
    Y = cr.convrot_weight_only_linear(Xr.cuda(), Wq.cuda(), s.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    yb, y64 = ref.weight_only_linear(_f64(Xr), Wq.numpy(), s.double().numpy())
    mag = (np.abs(_f64(Xr)) @ np.abs(Wq.numpy().astype(np.float64)).T) * s.double().numpy()[None, :]
    assert np.all(np.abs(_f64(Y) - yb) <= _tol.bf16_ulp(y64) * 1.0001 + 8 * np.sqrt(K) * _tol.U * mag)


def test_weight_only_edge_cases(cr):
    # M = 0 is a no-op; mismatched K and a K that is not a multiple of 16 are rejected
    Wq = torch.zeros(16, 256, dtype=torch.int8, device="cuda")
    s = torch.ones(16, device="cuda")
    Y = cr.convrot_weight_only_linear(torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda"), Wq, s)
    assert Y.shape == (0, 16)
    with pytest.raises(ValueError):
        cr.convrot_weight_only_linear(torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda"), Wq, s)
    with pytest.raises(cr.ConvRotError):
        cr.convrot_weight_only_linear(torch.zeros(4, 40, dtype=torch.bfloat16, device="cuda"),
                                      torch.zeros(16, 40, dtype=torch.int8, device="cuda"), s)
    # an all-zero weight row gives exact zeros
    Xr, Wq2, s2 = _operands(9, 32, 512)
    Wq2[5] = 0
    Y2 = cr.convrot_weight_only_linear(Xr.cuda(), Wq2.cuda(), s2.cuda())
    assert not Y2[:, 5].any()


@pytest.mark.parametrize("M,N,K", [(16, 20480, 4096), (100, 20480, 4096)])
def test_weight_only_split_tiles_deterministic(cr, M, N, K):
    """Split tiles have at most two fp32 parts, so repeated calls agree bit for
    bit whatever the order the parts arrive in; the workspace is zero again."""
    Xr, Wq, s = _operands(M, N, K)
    assert cr.convrot_weight_only_workspace_bytes(M, N, K) > 0
    ws = cr.Workspace()
    Xd, Wd, sd = Xr.cuda(), Wq.cuda(), s.cuda()
    ys = [cr.convrot_weight_only_linear(Xd, Wd, sd, workspace=ws) for _ in range(6)]
    acc = [cr.convrot_weight_only_gemm_f32(Xd, Wd, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    for a in acc[1:]:
        assert torch.equal(a, acc[0])
    assert int(ws.buf.count_nonzero()) == 0
