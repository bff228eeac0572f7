"""The allocation-free W8A8 linear (convrot_int8_linear_noalloc) against the
regular entry point (convrot_int8_linear with a caller workspace) and the
oracle.

The allocation-free entry point exists for callers that cannot allocate
device memory where they run the layer; it uses a fixed 24 MiB array inside
the library as the GEMM's split-tile workspace.  Both entry points run the
same kernels and schedule, so their outputs must agree within the output
tolerance the other tests use (in fact bit for bit), and both must be within
one bf16 step of the oracle's correctly rounded float64 result.  Two calls in
a row check that the shared array is left fit for the next call.  This file
is collected last so that, run after the other tests, it also sees a library
that has already served other shapes.
"""
import ctypes

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


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int16).to(torch.int8)
    W = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int16).to(torch.int8)
    st = (torch.rand(M, generator=g, dtype=torch.float64) * 1e-3 + 1e-5).float()
    sr = (torch.rand(N, generator=g, dtype=torch.float64) * 1e-3 + 1e-5).float()
    return X.cuda(), st.cuda(), W.cuda(), sr.cuda()


def _noalloc_c_abi(cr, X, st, W, sr):
    """Calls the C entry point directly through ctypes."""
    M, K = X.shape
    N = W.shape[0]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = cr.lib().convrot_int8_linear_noalloc(
        ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(st.data_ptr()),
        ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(sr.data_ptr()), M, N, K,
        ctypes.c_void_p(Y.data_ptr()), stream)
    return status, Y


@pytest.mark.parametrize("M,N,K", [(1, 24576, 4096), (16, 4096, 12288), (100, 1032, 1040),
                                   (128, 4096, 4096), (2048, 4096, 4096)])
def test_noalloc_matches_workspace_entry_point_twice(cr, M, N, K):
    need = cr.convrot_linear_workspace_bytes(M, N, K, 8)
    X, st, W, sr = _operands(M, N, K, M + N + K)
    want = cr.convrot_int8_linear(X, st, W, sr, workspace=cr.Workspace())
    torch.cuda.synchronize()
    expect = want.float().cpu().double().numpy()
    tol = _tol.output_tol(expect)
    # the oracle on the same int8 operands and scales: one bf16 rounding of
    # the exact float64 dequantisation
    yb, y64, _ = ref.int8_linear(X.cpu().numpy(), st.cpu().double().numpy(), W.cpu().numpy(),
                                 sr.cpu().double().numpy())
    ulp = _tol.bf16_ulp(y64) * 1.0001
    for _ in range(2):
        status, Y = _noalloc_c_abi(cr, X, st, W, sr)
        torch.cuda.synchronize()
        if need > 24 << 20:
            assert status == 7  # CONVROT_ERR_WORKSPACE: shape too large for the fixed array
            continue
        assert status == 0
        got = Y.float().cpu().double().numpy()
        assert np.all(np.abs(got - expect) <= tol)
        assert np.array_equal(got, expect)
        assert np.all(np.abs(got - yb) <= ulp)
    assert cr.convrot_device_status() == 0


def test_noalloc_rejects_bad_arguments(cr):
    A = ctypes.c_void_p(0x10000)
    lib = cr.lib()
    assert lib.convrot_int8_linear_noalloc(None, A, A, A, 4, 16, 512, A, None) == 1
    assert lib.convrot_int8_linear_noalloc(A, A, A, A, 4, 12, 512, A, None) == 2
    assert lib.convrot_int8_linear_noalloc(A, A, A, A, 0, 16, 512, A, None) == 0
