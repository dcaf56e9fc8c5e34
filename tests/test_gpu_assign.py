"""Nearest-centroid assignment on the GPU against the exact oracle.

The pages define the assignment as the plain Euclidean argmin (VPTQ page, "Step 3"; the
residual stage quantises v - C1[i1], "Residual Vector Quantization").  The kernel takes the
decision in binary32, so near ties several indices are correct to that precision.  Each GPU
index is therefore checked for validity against exact distances from the oracle:

  first stage   D(g) (1 - eps) <= D(o) (1 + eps),    eps = (d + 3) 2^-24,

where o is the exact argmin (the kernel's distance to centroid i is within eps D(i) of the
exact one: d rounded subtractions and d fused multiply-adds or d products and d sums);

  residual      D2(g2) <= D2(o2) + B(g2) + B(o2),  B(j) = eps (D2(j) + A(j)) + A(j),

with o2 the exact argmin for the residual v - C1[g1] of the kernel's own first choice, and
A(j) = sum_t 2 |r_t - c_jt| |r_t| u + r_t^2 u^2 (u = 2^-24) the effect of rounding r = v - C1[g1]
to binary32.  Where the exact minimum is unique beyond that slack, validity forces equality.
Exact hits (distance 0) are exact in binary32 too, so there the lowest index is required."""
import ctypes as C
from fractions import Fraction

import numpy as np
import pytest

import oracle
from sparse_compensated_vq_b200 import synth
from tests import exact

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


U = Fraction(1, 2 ** 24)


def _units(bits):
    return [exact.f16_frac(int(b)) for b in bits]


def check_valid(V, C1, g1, C2=None, g2=None):
    """Assert the GPU's indices are nearest centroids up to binary32 rounding; returns the
    fraction of sub-vectors where they equal the exact argmin."""
    n, d = V.shape
    eps = (d + 3) * U
    o1, _ = oracle.assign_exact(V, C1)
    same = 0
    for s in range(n):
        dg = oracle.sqdist_exact(V[s], C1[g1[s]])
        do = oracle.sqdist_exact(V[s], C1[o1[s]])
        assert dg * (1 - eps) <= do * (1 + eps), "stage 1, sub-vector %d: %d vs exact %d" % (s, g1[s], o1[s])
        same += int(g1[s] == o1[s])
    if C2 is not None:
        o2 = oracle.residual_assign_exact(V, C1, g1, C2)
        for s in range(n):
            r = [a - b for a, b in zip(_units(V[s]), _units(C1[g1[s]]))]

            def bound(j):
                c = _units(C2[j])
                A = sum(2 * abs(rt - ct) * abs(rt) * U + rt * rt * U * U for rt, ct in zip(r, c))
                D = Fraction(oracle.sqdist_exact(V[s], C2[j], base=C1[g1[s]]), 2 ** 48)
                return D, eps * (D + A) + A

            Dg, Bg = bound(int(g2[s]))
            Do, Bo = bound(int(o2[s]))
            assert Dg <= Do + Bg + Bo, "residual stage, sub-vector %d: %d vs exact %d" % (s, g2[s], o2[s])
            same += int(g2[s] == o2[s])
        return same / (2 * n)
    return same / n


@pytest.mark.parametrize("d", [4, 6, 8, 12])
@pytest.mark.parametrize("n", [1, 255, 1000])
def test_assign_valid_nearest_centroids(vq, d, n):
    rng = np.random.default_rng(700 + 10 * d + n)
    C1 = synth.f16_bits(rng.normal(0, 1, (300, d)))
    C2 = synth.f16_bits(rng.normal(0, 0.2, (50, d)))
    V = synth.f16_bits(rng.normal(0, 1, (n, d)))
    g1, g2 = run_assign(vq, V, C1, C2)
    agree = check_valid(V, C1, g1, C2, g2)
    assert agree > 0.98
    g1s, _ = run_assign(vq, V, C1)
    assert (g1s == g1).all()                  # the first stage does not depend on the second


def test_assign_ties_and_exact_hits(vq):
    rng = np.random.default_rng(71)
    d = 8
    base = synth.f16_bits(rng.normal(0, 1, (40, d)))
    C = np.concatenate([base, base, base[::-1]]).astype(np.uint16)   # every entry three times
    V = base[rng.integers(0, 40, 500)]
    g, _ = run_assign(vq, V, C)
    o, _ = oracle.assign_exact(V, C)
    assert (g == o).all() and (g < 40).all()


def test_assign_large_codebook_across_tiles(vq):
    rng = np.random.default_rng(72)
    d, k = 8, 65536
    C1 = synth.f16_bits(rng.normal(0, 0.02, (k, d)))
    V = synth.f16_bits(rng.normal(0, 0.02, (700, d)))
    g, _ = run_assign(vq, V, C1)
    assert check_valid(V, C1, g) > 0.95


def test_assign_argument_errors(vq):
    p = C.c_void_p(16)
    assert vq.vqlin_assign(p, 4, 5, p, 4, None, 0, p, None, None) == 2          # d unsupported
    assert vq.vqlin_assign(p, 4, 8, p, 0, None, 0, p, None, None) == 1          # k1 < 1
    assert vq.vqlin_assign(p, 4, 8, p, 4, None, 3, p, p, None) == 1             # k2 > 0 without C2
    assert vq.vqlin_assign(None, 0, 8, None, 4, None, 0, None, None, None) == 0  # n = 0: nothing to do


def test_assign_full_encode_workload_sampled(vq):
    """The bench's encode workload at full size (all 2,097,152 sub-vectors of a 4096x4096 weight,
    K = 4096), checked for validity against the exact oracle on 2048 sampled sub-vectors."""
    rng = synth.rng_for(6)
    d, k = 8, 4096
    C1 = synth.f16_bits(rng.normal(0.0, 0.02, (k, d)))
    V = synth.f16_bits(rng.normal(0.0, 0.02, (4096 * 4096 // d, d)))
    g, _ = run_assign(vq, V, C1)
    pick = np.random.default_rng(5).choice(V.shape[0], 2048, replace=False)
    assert check_valid(V[pick], C1, g[pick]) > 0.95
