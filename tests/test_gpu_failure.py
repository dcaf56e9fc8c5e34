"""Failure detection on the GPU without a fault: a bounded wait that nothing completes expires,
the kernel records its code and returns, the host reads the code, and the context stays usable."""
import ctypes as C

import numpy as np
import pytest

import oracle
from sparse_compensated_vq_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_compensated_vq_b200 import vqlin
    return vqlin


def test_expired_wait_is_reported_and_cleared(vq):
    import torch
    assert vq.device_error() == 0
    s = torch.cuda.current_stream().cuda_stream
    assert vq.vqlin_selftest_wait_timeout(2000, C.c_void_p(s)) == 0     # 2 ms limit
    assert vq.device_error() == 7
    assert vq.device_error() == 0                                        # read clears it


def test_context_usable_after_expired_wait(vq):
    import torch
    s = torch.cuda.current_stream().cuda_stream
    assert vq.vqlin_selftest_wait_timeout(1000, C.c_void_p(s)) == 0
    assert vq.device_error() == 7
    L, xb = G.workload("qproj")
    m = vq.VQLinear(L)
    x = G.torch_x(xb[:1], "f16")
    y = m.gemv_ws(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(y), oracle.gemv_f64(L, synth.bits_to_f64(xb[:1], "f16")), "f32", "after expired wait")


def test_selftest_rejects_bad_limits(vq):
    assert vq.vqlin_selftest_wait_timeout(0, None) == 1
    assert vq.vqlin_selftest_wait_timeout(2_000_000, None) == 1
