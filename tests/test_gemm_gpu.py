"""Parity of the tcgen05 W8A8 / W4A8 GEMM kernels with the oracle, through the
C ABI: int32 accumulators bit-exact, bf16 outputs within one bf16 rounding of
the float64 dequantisation, over shapes that exercise both operand roles,
ragged tails in M, N and K, data-parallel and stream-K schedules."""
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


def _rand_i8(shape, seed, lo=-128, hi=128):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi, shape, generator=g, dtype=torch.int16).to(torch.int8)


def _rand_scales(n, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(n, generator=g, dtype=torch.float64) * 1e-3 + 1e-5).float()


SHAPES = [
    # (M, N, K): operand roles swap at M <= 128; above it CTA pairs take
    # 256 x 256 tiles, a single wave of at most one tile per four-CTA cluster
    # splits K over two pairs, larger grids split by stream-K (520 x 3000: one
    # partial wave of 36 pair tiles; 2200 x 2248: a full wave of 74 and a tail
    # of 7; both ragged in M, N and K).  Decode shapes with more 128-row weight
    # tiles than SMs (100 x 19000: ragged; 128 x 24576: the gate/up decode
    # GEMM, all outputs)
    (1, 256, 512), (3, 136, 512), (16, 1024, 4096), (17, 264, 1040), (40, 512, 256),
    (64, 128, 768), (100, 2056, 144), (128, 520, 4096), (100, 19000, 1040), (128, 24576, 4096),
    (129, 264, 512), (256, 512, 4096), (300, 1032, 1040), (512, 4096, 12288),
    (1024, 1024, 4096), (2048, 1536, 16), (777, 8, 32),
    (1280, 2560, 1088), (520, 3000, 1040), (2200, 2248, 4000),
    # the decode GEMMs at full size (stream-K over 192 weight tiles, split tiles
    # summed at L2), every output
    (1, 24576, 4096), (16, 24576, 4096),
    # long K: the pair kernel rasterises in groups of as many 256-row activation
    # tiles as fit ~40 MB (here 5 of the 9, the second group partial)
    (2100, 1040, 32768),
    (2048, 4096, 1024),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_int8_gemm_s32_bit_exact(cr, M, N, K):
    X = _rand_i8((M, K), M * 31 + K)
    W = _rand_i8((N, K), N * 17 + K)
    acc = cr.convrot_int8_gemm_s32(X.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    want = ref.int_matmul(X.numpy(), W.numpy())
    got = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, want), f"{np.count_nonzero(got != want)} mismatches"


def test_int8_gemm_s32_bit_exact_gate_up_m8192(cr):
    """Every int32 accumulator of the largest single-GPU W8A8 shape (fused
    gate+up, 8192 tokens x 24576 rows x K 4096: the bench's default
    workload, in the launch configuration it times) against the oracle's
    exact integer matmul, in blocks of 1024 tokens."""
    M, N, K = 8192, 24576, 4096
    X = _rand_i8((M, K), 8192 + K, -127, 128)
    W = _rand_i8((N, K), N + K, -127, 128)
    acc = cr.convrot_int8_gemm_s32(X.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    got = acc.cpu().numpy()
    del acc
    Xn, Wn = X.numpy(), W.numpy()
    for m0 in range(0, M, 1024):
        want = ref.int_matmul(Xn[m0:m0 + 1024], Wn)
        bad = np.count_nonzero(got[m0:m0 + 1024].astype(np.int64) != want)
        assert bad == 0, f"tokens {m0}..{m0 + 1023}: {bad} mismatches"


def test_int8_gemm_s32_extreme_operands(cr):
    M, N, K = 130, 264, 12288
    X = torch.full((M, K), 127, dtype=torch.int8)
    X[1::2] = -127
    W = torch.full((N, K), -127, dtype=torch.int8)
    W[::3, ::2] = 127
    acc = cr.convrot_int8_gemm_s32(X.cuda(), W.cuda()).cpu().numpy()
    assert np.array_equal(acc.astype(np.int64), ref.int_matmul(X.numpy(), W.numpy()))
    assert acc[0, 1] == -127 * 127 * K


@pytest.mark.parametrize("M,N,K", SHAPES[:-1])
def test_int8_linear_bf16(cr, M, N, K):
    X = _rand_i8((M, K), M + 5 * K, -127, 128)
    W = _rand_i8((N, K), N + 3 * K, -127, 128)
    st = _rand_scales(M, 1)
    sr = _rand_scales(N, 2)
    Y = cr.convrot_int8_linear(X.cuda(), st.cuda(), W.cuda(), sr.cuda())
    torch.cuda.synchronize()
    yb, y64, _ = ref.int8_linear(X.numpy(), st.double().numpy(), W.numpy(), sr.double().numpy())
    got = Y.float().cpu().double().numpy()
    # fp32 product then one bf16 rounding: at most one bf16 step from the
    # correctly rounded float64 value
    assert np.all(np.abs(got - yb) <= _tol.bf16_ulp(y64) * 1.0001)


PACK_SHAPES = [(1, 256, 512), (16, 1024, 4096), (33, 264, 1056), (128, 520, 4096),
               (129, 264, 512), (512, 4096, 12288), (1000, 1032, 2080), (2100, 1040, 32768),
               (4096, 4096, 4096)]


def _rand_w4(N, K, seed):
    codes = torch.randint(-8, 8, (N, K), generator=torch.Generator().manual_seed(seed))
    packed = ref.pack_int4(codes.numpy())
    return codes.numpy().astype(np.int8), torch.from_numpy(packed)


@pytest.mark.parametrize("M,N,K", PACK_SHAPES)
def test_w4a8_gemm_s32_bit_exact(cr, M, N, K):
    X = _rand_i8((M, K), 7 * M + K)
    codes, packed = _rand_w4(N, K, N + K)
    acc = cr.convrot_w4a8_gemm_s32(X.cuda(), packed.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_device_status() == 0
    want = ref.int_matmul(X.numpy(), ref.unpack_int4(packed.numpy()))
    assert np.array_equal(codes, ref.unpack_int4(packed.numpy()))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), want)


@pytest.mark.parametrize("M,N,K", PACK_SHAPES)
def test_w4a8_linear_bf16(cr, M, N, K):
    X = _rand_i8((M, K), M + K, -127, 128)
    _, packed = _rand_w4(N, K, 3 * N + K)
    st = _rand_scales(M, 3)
    sr = _rand_scales(N, 4)
    Y = cr.convrot_w4a8_linear(X.cuda(), st.cuda(), packed.cuda(), sr.cuda())
    torch.cuda.synchronize()
    yb, y64, _ = ref.w4a8_linear(X.numpy(), st.double().numpy(), packed.numpy(), sr.double().numpy())
    got = Y.float().cpu().double().numpy()
    assert np.all(np.abs(got - yb) <= _tol.bf16_ulp(y64) * 1.0001)


# Shapes whose plan splits tiles by K (stream-K), so partial tiles meet in the
# workspace: a 16-token swap-kernel GEMM, and 75 pair tiles on 74 CTA pairs
# with long K.
STREAM_K_SHAPES = [(16, 4096, 12288), (768, 6400, 12288)]


@pytest.mark.parametrize("M,N,K", STREAM_K_SHAPES)
def test_workspace_reuse_and_determinism(cr, M, N, K):
    # reusing the workspace for further calls only gives the right answer if
    # every call restores the tile counters and accumulators to zero
    assert cr.convrot_linear_workspace_bytes(M, N, K, 8) > 0
    ws = cr.Workspace()
    X = _rand_i8((M, K), 11)
    W = _rand_i8((N, K), 12)
    want = ref.int_matmul(X.numpy(), W.numpy())
    Xd, Wd = X.cuda(), W.cuda()
    for _ in range(3):
        acc = cr.convrot_int8_gemm_s32(Xd, Wd, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), want)
    # counters and accumulators are back at zero
    assert int(ws.buf.count_nonzero().item()) == 0


def test_workspace_shared_across_shapes(cr):
    # one buffer, calls of different shapes and operand roles in a row
    ws = cr.Workspace()
    for (M, N, K) in [(16, 4096, 12288), (1, 24576, 4096), (129, 264, 512), (2048, 1024, 4096),
                      (512, 4096, 12288), (16, 1024, 4096), (768, 4096, 8192), (16, 4096, 12288)]:
        X = _rand_i8((M, K), M + N)
        W = _rand_i8((N, K), N + K)
        acc = cr.convrot_int8_gemm_s32(X.cuda(), W.cuda(), workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref.int_matmul(X.numpy(), W.numpy()))


def test_workspace_too_small_is_rejected(cr):
    M, N, K = STREAM_K_SHAPES[0]
    assert cr.convrot_linear_workspace_bytes(M, N, K, 8) > 0
    X = torch.zeros(M, K, dtype=torch.int8, device="cuda")
    W = torch.zeros(N, K, dtype=torch.int8, device="cuda")
    s = torch.ones(max(M, N), device="cuda")
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    import ctypes
    lib = cr.lib()
    st = lib.convrot_int8_linear(ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                 ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(s.data_ptr()),
                                 M, N, K, ctypes.c_void_p(Y.data_ptr()), None, 0, None)
    assert st == 7
