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


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    from sparse_compensated_vq_b200 import vqlin
    rng = np.random.default_rng(7)
    L = synth.random_layer(rng, 17000, 64, 8, 16, 4, row_scale=False, nnz=0)   # 16 * 17000 > 262144
    m = vqlin.VQLinear(L)
    x = torch.zeros((16, 64), dtype=torch.float16, device="cuda")
    y = torch.zeros((16, 17000), dtype=torch.float16, device="cuda")
    st = vqlin.vqlin_gemv_noalloc(m.handle, x.data_ptr(), vqlin.VQLIN_F16, 16, y.data_ptr(), vqlin.VQLIN_F16, None)
    assert st == vqlin.VQLIN_ERR_UNSUPPORTED
    assert b"scratch" in vqlin.vqlin_last_error()
    torch.cuda.synchronize()
