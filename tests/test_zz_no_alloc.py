"""vqlin_gemv_noalloc against vqlin_gemv_ws (needs a B200).

Some callers cannot allocate device memory once they are running (their pool
owns the GPU's memory, or cudaMalloc's implicit synchronisation is not
allowed), so they cannot hand vqlin_gemv_ws a scratch buffer.
vqlin_gemv_noalloc uses a scratch array built into the library instead.  This
file is named to be collected last, and its test works in a fresh process as
well as after the other GPU tests.
"""
import ctypes as C

import numpy as np
import pytest

from sparse_compensated_vq_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _layer():
    # wide enough (n_in = 6144 -> 12 slabs of 64 sub-vectors) that the decode kernel
    # splits its columns and really accumulates in the scratch array
    rng = np.random.default_rng(4242)
    L = synth.random_layer(rng, 520, 6144, 8, 256, 8, col_scale=True, outlier_frac=0.01, outlier_scale=0.1)
    return L, rng


def test_noalloc_matches_workspace_variant_twice_in_a_row():
    import torch
    from sparse_compensated_vq_b200 import vqlin
    assert torch.cuda.is_available()
    L, rng = _layer()
    m = vqlin.VQLinear(L)
    stream = torch.cuda.current_stream().cuda_stream
    for call, batch in enumerate((3, 3)):
        xb = synth.activations(rng, batch, L.n_in, "f16")
        x = G.torch_x(xb, "f16")
        y_ref = torch.empty((batch, L.n_out), dtype=torch.float16, device="cuda")
        ws = torch.empty(int(vqlin.vqlin_gemv_workspace_size(m.handle, batch)), dtype=torch.uint8, device="cuda")
        vqlin.check(vqlin.vqlin_gemv_ws(m.handle, x.data_ptr(), vqlin.VQLIN_F16, batch, y_ref.data_ptr(),
                                        vqlin.VQLIN_F16, ws.data_ptr(), ws.numel(), stream), "gemv_ws")
        y = torch.full((batch, L.n_out), float("nan"), dtype=torch.float16, device="cuda")
        vqlin.check(vqlin.vqlin_gemv_noalloc(m.handle, x.data_ptr(), vqlin.VQLIN_F16, batch, y.data_ptr(),
                                             vqlin.VQLIN_F16, stream), "gemv_noalloc")
        torch.cuda.synchronize()
        G.assert_close(G.to_f64(y), G.to_f64(y_ref), "f16", "no-alloc call %d" % call)


@pytest.mark.parametrize("batch", [1, 4])
def test_noalloc_headline_layer_against_the_oracle(batch):
    """The 4096x4096 layer with a 65536-entry codebook: the built-in scratch holds its
    codebook-stationary partial sums, so the call runs the same two kernels as
    vqlin_gemv_ws (not the scratch-free fallback) and matches the CPU oracle."""
    import torch
    import oracle
    from sparse_compensated_vq_b200 import vqlin
    L, xb = synth.qproj(4)
    m = vqlin.VQLinear(L)
    stream = torch.cuda.current_stream().cuda_stream
    x = G.torch_x(xb[:batch], "f16")
    y = torch.full((batch, L.n_out), float("nan"), dtype=torch.float32, device="cuda")
    for call in range(2):
        n0 = vqlin.vqlin_kernel_launches()
        vqlin.check(vqlin.vqlin_gemv_noalloc(m.handle, x.data_ptr(), vqlin.VQLIN_F16, batch, y.data_ptr(),
                                             vqlin.VQLIN_F32, stream), "gemv_noalloc")
        assert vqlin.vqlin_kernel_launches() - n0 == 2      # codebook-stationary grid + finalize
        torch.cuda.synchronize()
        assert vqlin.device_error() == 0
        ref = oracle.gemv_f64(L, synth.bits_to_f64(xb[:batch], "f16"))
        G.assert_close(G.to_f64(y), ref, "f32", "no-alloc qproj B=%d call %d" % (batch, call))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    from sparse_compensated_vq_b200 import vqlin
    rng = np.random.default_rng(7)
    L = synth.random_layer(rng, 131073, 64, 8, 16, 4, row_scale=False, nnz=0)   # 16 * 131073 > 2097152
    m = vqlin.VQLinear(L)
    x = torch.zeros((16, 64), dtype=torch.float16, device="cuda")
    y = torch.zeros((16, 131073), dtype=torch.float16, device="cuda")
    st = vqlin.vqlin_gemv_noalloc(m.handle, x.data_ptr(), vqlin.VQLIN_F16, 16, y.data_ptr(), vqlin.VQLIN_F16, None)
    assert st == vqlin.VQLIN_ERR_UNSUPPORTED
    assert b"scratch" in vqlin.vqlin_last_error()
    torch.cuda.synchronize()
