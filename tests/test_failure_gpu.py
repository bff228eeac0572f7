"""Failure path of the bounded waits, exercised without a fault.

Every mbarrier wait in the kernels gives up after a bounded number of cycles,
records the wait site in the device error word and lets the kernel return, so
that a broken pipeline ends with an error status instead of a hung GPU.  The
self-test kernel makes one such wait run out on purpose (nothing arrives on its
barrier, and its limit is short); the status must say so, the word must clear
on read, and the context must stay usable for ordinary calls.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import convrot_ref as ref

pytestmark = pytest.mark.gpu

ERR_DEVICE_TIMEOUT = 6
SITE_SELFTEST = 15


@pytest.fixture(scope="module")
def cr():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_quantized_rmsnorm_b200 as m
    m.lib()
    return m


def _status(lib):
    detail = ctypes.c_uint32(0)
    st = lib.convrot_device_status(None, ctypes.byref(detail))
    return st, detail.value


def test_timeout_is_reported_and_cleared(cr):
    lib = cr.lib()
    torch.cuda.synchronize()
    assert _status(lib) == (0, 0)
    assert lib.convrot_selftest_wait_timeout(2_000_000, None) == 0
    st, detail = _status(lib)
    assert st == ERR_DEVICE_TIMEOUT
    assert detail & 1
    assert (detail >> 8) & 0xFF == SITE_SELFTEST
    assert _status(lib) == (0, 0)  # read and cleared


def test_context_survives_a_timeout(cr):
    lib = cr.lib()
    for _ in range(2):
        assert lib.convrot_selftest_wait_timeout(1000, None) == 0
    assert _status(lib)[0] == ERR_DEVICE_TIMEOUT
    g = torch.Generator().manual_seed(5)
    X = torch.randint(-127, 128, (200, 1024), generator=g, dtype=torch.int16).to(torch.int8)
    W = torch.randint(-127, 128, (264, 1024), generator=g, dtype=torch.int16).to(torch.int8)
    acc = cr.convrot_int8_gemm_s32(X.cuda(), W.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref.int_matmul(X.numpy(), W.numpy()))
    assert _status(lib) == (0, 0)
