"""Nearest-centroid assignment on the GPU vs the oracle: bit-exact indices (both sides take the
decision in the same binary32 arithmetic), every vector length, residual stage, ragged sizes,
ties, a 65536-entry codebook, and argument errors."""
import ctypes as C

import numpy as np
import pytest

import oracle
from sparse_compensated_vq_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_compensated_vq_b200 import vqlin
    return vqlin


def run_assign(vq, V, C1, C2=None):
    import torch
    n, d = V.shape
    dv = torch.from_numpy(V.astype(np.int16)).cuda()
    dc1 = torch.from_numpy(C1.astype(np.int16)).cuda()
    dc2 = torch.from_numpy(C2.astype(np.int16)).cuda() if C2 is not None else None
    i1 = torch.zeros(max(n, 1), dtype=torch.int32, device="cuda")
    i2 = torch.zeros(max(n, 1), dtype=torch.int32, device="cuda")
    st = vq.vqlin_assign(dv.data_ptr(), n, d, dc1.data_ptr(), C1.shape[0], dc2.data_ptr() if dc2 is not None else None,
                         C2.shape[0] if C2 is not None else 0, i1.data_ptr(), i2.data_ptr(),
                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, vq.vqlin_last_error()
    torch.cuda.synchronize()
    a = i1.cpu().numpy().view(np.uint32)[:n]
    b = i2.cpu().numpy().view(np.uint32)[:n] if C2 is not None else None
    return a, b


@pytest.mark.parametrize("d", [4, 6, 8, 12])
@pytest.mark.parametrize("n", [1, 255, 1000])
def test_assign_matches_oracle(vq, d, n):
    rng = np.random.default_rng(700 + 10 * d + n)
    C1 = synth.f16_bits(rng.normal(0, 1, (300, d)))
    C2 = synth.f16_bits(rng.normal(0, 0.2, (50, d)))
    V = synth.f16_bits(rng.normal(0, 1, (n, d)))
    g1, g2 = run_assign(vq, V, C1, C2)
    o1, o2 = oracle.assign_f32(V, C1, C2)
    assert (g1 == o1).all() and (g2 == o2).all()
    g1s, _ = run_assign(vq, V, C1)
    assert (g1s == o1).all()


def test_assign_ties_and_exact_hits(vq):
    rng = np.random.default_rng(71)
    d = 8
    base = synth.f16_bits(rng.normal(0, 1, (40, d)))
    C = np.concatenate([base, base, base[::-1]]).astype(np.uint16)   # every entry three times
    V = base[rng.integers(0, 40, 500)]
    g, _ = run_assign(vq, V, C)
    o, _ = oracle.assign_f32(V, C)
    assert (g == o).all() and (g < 40).all()


def test_assign_large_codebook_across_tiles(vq):
    rng = np.random.default_rng(72)
    d, k = 8, 65536
    C1 = synth.f16_bits(rng.normal(0, 0.02, (k, d)))
    V = synth.f16_bits(rng.normal(0, 0.02, (700, d)))
    g, _ = run_assign(vq, V, C1)
    o, _ = oracle.assign_f32(V, C1)
    assert (g == o).all()


def test_assign_argument_errors(vq):
    p = C.c_void_p(16)
    assert vq.vqlin_assign(p, 4, 5, p, 4, None, 0, p, None, None) == 2          # d unsupported
    assert vq.vqlin_assign(p, 4, 8, p, 0, None, 0, p, None, None) == 1          # k1 < 1
    assert vq.vqlin_assign(p, 4, 8, p, 4, None, 3, p, p, None) == 1             # k2 > 0 without C2
    assert vq.vqlin_assign(None, 0, 8, None, 4, None, 0, None, None, None) == 0  # n = 0: nothing to do


def test_assign_full_encode_workload_sampled(vq):
    """The bench's encode workload at full size (all 2,097,152 sub-vectors of a 4096x4096 weight,
    K = 4096), checked against the oracle on 2048 sampled sub-vectors."""
    rng = synth.rng_for(6)
    d, k = 8, 4096
    C1 = synth.f16_bits(rng.normal(0.0, 0.02, (k, d)))
    V = synth.f16_bits(rng.normal(0.0, 0.02, (4096 * 4096 // d, d)))
    g, _ = run_assign(vq, V, C1)
    pick = np.random.default_rng(5).choice(V.shape[0], 2048, replace=False)
    o, _ = oracle.assign_f32(V[pick], C1)
    assert (g[pick] == o).all()
