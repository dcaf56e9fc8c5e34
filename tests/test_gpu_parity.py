"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Bit-exact: field unpacking and dequantisation.  Within the tolerance of
gpu_util.assert_close: GEMV (batch 1..16) and the prefill GEMM.  Full-size
workloads are checked on every output of the GEMV and on sampled rows of the
GEMM; small random layers span several tiles and ragged tails; special cases
reduce to closed forms; invalid inputs must return an error status.
"""
import json
import os

import numpy as np
import pytest

import oracle
from sparse_compensated_vq_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def vq():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from sparse_compensated_vq_b200 import vqlin
    return vqlin


def small_layers():
    """Random layers covering every format feature; sizes span several CTAs and ragged tails."""
    specs = [
        dict(n_out=37, n_in=100, d=4, k1=16, bits1=4),
        dict(n_out=130, n_in=264, d=8, k1=256, bits1=8, col_scale=True, nnz=300),
        dict(n_out=64, n_in=200, d=8, k1=4096, bits1=12, k2=4096, bits2=12, nnz=150, n_ocols=9, ko=256, bits_o=8),
        dict(n_out=33, n_in=75, d=4, k1=100, bits1=7, k2=30, bits2=5, col_scale=True, nnz=60, n_ocols=6, ko=50, bits_o=6),
        dict(n_out=17, n_in=512, d=8, k1=65536, bits1=16, col_scale=True, nnz=100),
        dict(n_out=50, n_in=64, d=8, k1=8192, bits1=13, nnz=0, n_ocols=5, ko=8192, bits_o=13),
        dict(n_out=9, n_in=40, d=8, k1=65536, bits1=16, k2=65536, bits2=16, nnz=20),
        dict(n_out=300, n_in=24, d=4, k1=3, bits1=2, row_scale=False, nnz=100),
        # VPTQ's other vector lengths (CUDA-core decode path)
        dict(n_out=45, n_in=130, d=6, k1=256, bits1=8, col_scale=True, nnz=80),
        dict(n_out=70, n_in=300, d=12, k1=4096, bits1=12, k2=256, bits2=8, nnz=90, n_ocols=10, ko=64, bits_o=6),
        dict(n_out=19, n_in=96, d=6, k1=1, bits1=1, nnz=5),
        dict(n_out=40, n_in=192, d=12, k1=512, bits1=9, col_scale=True, nnz=30),
        # residual codebook + outlier block with n_in % 8 == 0, so the prefill GEMM covers both
        dict(n_out=96, n_in=208, d=4, k1=100, bits1=7, k2=30, bits2=5, col_scale=True, nnz=60, n_ocols=6, ko=50, bits_o=6),
        # VSR blocks (SCVQ), codebook groups (VPTQ group_num), symmetric codebooks (SCVQ)
        dict(n_out=130, n_in=264, d=8, k1=256, bits1=8, col_scale=True, nnz=200, vsr_blocks=260),            # 13
        dict(n_out=70, n_in=520, d=8, k1=256, bits1=8, n_groups=3, col_scale=True, nnz=90),                  # 14
        dict(n_out=40, n_in=512, d=8, k1=65536, bits1=16, cb_symmetry=1, col_scale=True, nnz=50, vsr_blocks=30),  # 15
        dict(n_out=50, n_in=133, d=4, k1=64, bits1=6, k2=16, bits2=4, n_groups=2, cb_symmetry=1, n_ocols=7,
             ko=32, bits_o=5, nnz=40, vsr_blocks=25),                                                         # 16
        dict(n_out=45, n_in=300, d=12, k1=128, bits1=7, cb_symmetry=1, nnz=30, vsr_blocks=20),              # 17
        dict(n_out=64, n_in=200, d=8, k1=4096, bits1=12, k2=256, bits2=8, n_groups=2, nnz=40, vsr_blocks=16,
             n_ocols=9, ko=64, bits_o=6),                                                                     # 18
        dict(n_out=33, n_in=96, d=8, k1=1024, bits1=10, n_groups=12, cb_symmetry=1, nnz=10),                 # 19 one position per group
    ]
    out = []
    for t, kw in enumerate(specs):
        kw = dict(kw)
        rng = np.random.default_rng(500 + t)
        nnz = kw.pop("nnz", 10)
        out.append(synth.random_layer(rng, cb_std=0.3, res_std=0.05, nnz=nnz, outlier_scale=1.0, **kw))
    return out


SMALL = small_layers()


def full_layer(name):
    if name == "tiny":
        return G.workload("tiny")[0]
    if name in ("qproj", "downproj", "prefill") or name.startswith("vlen"):
        return G.workload(name)[0]
    idx = int(name.split(":")[1])
    return G.workload("smollm")[0][idx]


FULL = ["tiny", "qproj", "downproj"] + ["smollm:%d" % i for i in range(7)] + ["vlen6", "vlen12"]


# ------------------------------------------------------------------ unpack
@pytest.mark.parametrize("t", range(len(SMALL)))
def test_unpack_small_bit_exact(vq, t):
    L = SMALL[t]
    m = vq.VQLinear(L)
    got = m.unpack_indices(0).cpu().numpy().view(np.uint32)
    assert (got == oracle.unpack(L.codes, L.n_sub, L.bits1 + L.bits2)).all()
    assert (got == L.fields).all()
    if L.n_ocols:
        got_o = m.unpack_indices(1).cpu().numpy().view(np.uint32)
        assert (got_o == oracle.unpack(L.codes_o, L.n_sub_o, L.bits_o)).all()


@pytest.mark.parametrize("name", ["qproj", "downproj", "smollm:6"])
def test_unpack_full_bit_exact(vq, name):
    L = full_layer(name)
    m = vq.VQLinear(L)
    got = m.unpack_indices(0).cpu().numpy().view(np.uint32)
    assert (got == oracle.unpack(L.codes, L.n_sub, L.bits1 + L.bits2)).all()


# ------------------------------------------------------------------ dequant
@pytest.mark.parametrize("t", range(len(SMALL)))
def test_dequant_small_bit_exact(vq, t):
    L = SMALL[t]
    W = vq.VQLinear(L).dequant().cpu().numpy().view(np.uint16)
    assert (W == oracle.dequant_exact(L)).all()


@pytest.mark.parametrize("name", FULL)
def test_dequant_full_bit_exact(vq, name):
    L = full_layer(name)
    W = vq.VQLinear(L).dequant().cpu().numpy().view(np.uint16)
    ref = oracle.dequant_exact(L)
    bad = np.argwhere(W != ref)
    assert bad.size == 0, "first mismatches %s: got %s want %s" % (bad[:5].tolist(), W[tuple(bad[0])], ref[tuple(bad[0])])


def test_dequant_with_leading_dimension(vq):
    import torch
    L = SMALL[1]
    ldw = L.n_in + 24
    buf = torch.full((L.n_out, ldw), 12345, dtype=torch.int16, device="cuda")
    vq.VQLinear(L).dequant(out=buf.view(torch.float16))
    got = buf.cpu().numpy().view(np.uint16)
    assert (got[:, :L.n_in] == oracle.dequant_exact(L)).all()
    assert (got[:, L.n_in:] == 12345).all()


def test_dequant_rounding_vectors(vq):
    """Each golden rounding case as a one-entry-codebook layer: every element hits it."""
    g = json.load(open(os.path.join(GOLDEN, "f16_rounding.json")))
    for c in g["cases"]:
        hx = lambda s: None if s is None else int(s, 16)
        d = 4
        c2 = hx(c["c2"])
        L = synth.LayerData(
            n_out=2, n_in=8, d=d, k1=1, bits1=1, codes=synth.pack_fields(np.zeros((2, 2), np.uint32), 1),
            codebook1=np.full((1, d), hx(c["c1"]), np.uint16),
            k2=1 if c2 is not None else 0, bits2=1 if c2 is not None else 0,
            codebook2=np.full((1, d), c2, np.uint16) if c2 is not None else None,
            row_scale=np.full(2, hx(c["r"]), np.uint16) if c["r"] else None,
            col_scale=np.full(8, hx(c["c"]), np.uint16) if c["c"] else None)
        if c2 is not None:
            L.codes = synth.pack_fields(np.zeros((2, 2), np.uint32), 2)
        W = vq.VQLinear(L).dequant().cpu().numpy().view(np.uint16)
        assert (W == hx(c["expect"])).all(), c["note"]


def test_outlier_positions_exact_on_gpu(vq):
    L = full_layer("qproj")
    W = vq.VQLinear(L).dequant().cpu().numpy().view(np.uint16)
    rows = np.repeat(np.arange(L.n_out), np.diff(L.row_ptr))
    assert (W[rows, L.col_idx] == L.values).all()


# ------------------------------------------------------------------ gemv
def run_gemv(vq, L, xbits, xdt, ydt, m=None):
    import torch
    m = m or vq.VQLinear(L)
    x = G.torch_x(xbits, xdt)
    y = m.gemv(x, out_dtype=G.torch_dtype(ydt))
    torch.cuda.synchronize()
    return G.to_f64(y)


@pytest.mark.parametrize("t", range(len(SMALL)))
@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_gemv_small(vq, t, batch):
    L = SMALL[t]
    rng = np.random.default_rng(900 + t * 17 + batch)
    xb = synth.activations(rng, batch, L.n_in, "f16")
    y = run_gemv(vq, L, xb, "f16", "f32")
    G.assert_close(y, oracle.gemv_f64(L, synth.bits_to_f64(xb, "f16")), "f32", "small %d B=%d" % (t, batch))


@pytest.mark.parametrize("xdt,ydt", [("f16", "f16"), ("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32"), ("f32", "f16")])
def test_gemv_dtypes(vq, xdt, ydt):
    L = SMALL[2]
    rng = np.random.default_rng(77)
    xb = synth.activations(rng, 5, L.n_in, xdt)
    y = run_gemv(vq, L, xb, xdt, ydt)
    G.assert_close(y, oracle.gemv_f64(L, synth.bits_to_f64(xb, xdt)), ydt, "dtypes")


@pytest.mark.parametrize("name,batch", [(n, b) for n in FULL for b in (1, 16)] + [("downproj", 4)])
def test_gemv_full(vq, name, batch):
    L = full_layer(name)
    if name.startswith("smollm"):
        xb = G.workload("smollm")[1][int(name.split(":")[1])]
        xdt = "bf16"
        batch = min(batch, 8)
    else:
        xb = G.workload(name)[1]
        xdt = "f16"
    xb = xb[:batch]
    y = run_gemv(vq, L, xb, xdt, "f32")
    G.assert_close(y, oracle.gemv_f64(L, synth.bits_to_f64(xb, xdt)), "f32", "%s B=%d" % (name, batch))


def test_gemv_every_batch_size(vq):
    L = SMALL[3]
    m = vq.VQLinear(L)
    rng = np.random.default_rng(5)
    xb = synth.activations(rng, 16, L.n_in, "f16")
    ref = oracle.gemv_f64(L, synth.bits_to_f64(xb, "f16"))
    for b in range(1, 17):
        G.assert_close(run_gemv(vq, L, xb[:b], "f16", "f32", m), ref[:b], "f32", "B=%d" % b)


# ------------------------------------------------------------------ special cases (closed forms)
def test_gemv_single_entry_codebook_and_ragged_tail(vq):
    rng = np.random.default_rng(21)
    n_out, n_in, d = 45, 1001, 8
    n_sub = -(-n_in // d)
    c0 = synth.f16_bits(rng.normal(0, 1, (1, d)))
    L = synth.LayerData(n_out=n_out, n_in=n_in, d=d, k1=1, bits1=1,
                        codes=synth.pack_fields(np.zeros((n_out, n_sub), np.uint32), 1), codebook1=c0,
                        row_scale=synth.f16_bits(rng.uniform(0.5, 1.5, n_out)))
    xb = synth.activations(rng, 2, n_in, "f16")
    x = synth.bits_to_f64(xb, "f16")
    r = L.row_scale.view(np.float16).astype(np.float64)
    cv = np.tile(c0.view(np.float16).astype(np.float64)[0], n_sub)[:n_in]
    ref = (x @ cv)[:, None] * r[None, :]
    G.assert_close(run_gemv(vq, L, xb, "f16", "f32"), ref, "f32", "K=1")


def test_gemv_one_hot_codebook(vq):
    rng = np.random.default_rng(22)
    d, k, n_out, n_in = 8, 256, 70, 512
    cb = np.zeros((k, d)); cb[np.arange(k), np.arange(k) % d] = 1.0
    fields = rng.integers(0, k, size=(n_out, n_in // d)).astype(np.uint32)
    L = synth.LayerData(n_out=n_out, n_in=n_in, d=d, k1=k, bits1=8, codes=synth.pack_fields(fields, 8),
                        codebook1=synth.f16_bits(cb))
    xb = synth.activations(rng, 1, n_in, "f16")
    x = synth.bits_to_f64(xb, "f16")[0]
    cols = np.arange(n_in // d)[None, :] * d + (fields % d)
    ref = x[cols].sum(axis=1)[None, :]
    G.assert_close(run_gemv(vq, L, xb, "f16", "f32"), ref, "f32", "one-hot")


def test_gemv_fully_dense_sparse_set(vq):
    rng = np.random.default_rng(23)
    n_out, n_in = 40, 96
    V = rng.normal(0, 1, (n_out, n_in)).astype(np.float16)
    L = synth.random_layer(rng, n_out, n_in, 8, 256, 8, col_scale=True, nnz=0)
    L.row_ptr = (np.arange(n_out + 1) * n_in).astype(np.int32)
    L.col_idx = np.tile(np.arange(n_in), n_out).astype(np.int32)
    L.values = V.reshape(-1).view(np.uint16)
    xb = synth.activations(rng, 4, n_in, "f16")
    ref = synth.bits_to_f64(xb, "f16") @ V.astype(np.float64).T
    G.assert_close(run_gemv(vq, L, xb, "f16", "f32"), ref, "f32", "dense CSR")
    W = vq.VQLinear(L).dequant().cpu().numpy()
    assert (W.view(np.uint16) == V.view(np.uint16)).all()


def test_gemv_all_columns_in_outlier_block(vq):
    rng = np.random.default_rng(24)
    L = synth.random_layer(rng, 20, 48, 8, 16, 4, n_ocols=48, ko=64, bits_o=6, col_scale=True, nnz=30)
    xb = synth.activations(rng, 2, 48, "f16")
    G.assert_close(run_gemv(vq, L, xb, "f16", "f32"), oracle.gemv_f64(L, synth.bits_to_f64(xb, "f16")), "f32", "all-outlier")
    assert (vq.VQLinear(L).dequant().cpu().numpy().view(np.uint16) == oracle.dequant_exact(L)).all()


# ------------------------------------------------------------------ gemm
def run_gemm(vq, L, Xbits, xdt, ydt):
    import torch
    m = vq.VQLinear(L)
    X = G.torch_x(Xbits, xdt)
    Y = m.gemm(X, out_dtype=G.torch_dtype(ydt))
    torch.cuda.synchronize()
    assert vq.device_error() == 0, "a GEMM pipeline wait expired"
    return G.to_f64(Y)


@pytest.mark.parametrize("t", [0, 1, 2, 4, 10, 11, 12, 13, 14, 15, 18, 19])
@pytest.mark.parametrize("M", [1, 77, 256])
def test_gemm_small(vq, t, M):
    L = SMALL[t]
    if L.n_in % 8:
        pytest.skip("gemm needs n_in % 8 == 0")
    rng = np.random.default_rng(40 + M + t)
    Xb = synth.activations(rng, M, L.n_in, "bf16")
    Y = run_gemm(vq, L, Xb, "bf16", "f32")
    G.assert_close(Y, oracle.gemv_f64(L, synth.bits_to_f64(Xb, "bf16")), "f32", "gemm small")


@pytest.mark.parametrize("M", [1, 300, 513, 1100, 1600, 2100])
def test_gemm_fused_ragged_tiles(vq, M):
    """The fused prefill (weight tiles dequantised in shared memory): 300 weight rows (three
    128-row tiles, the last ragged), 200 columns (three whole K-blocks and a partial one), row and
    column scales and CSR replacements; M covers one and two activation halves and one to five
    512-row groups, so clusters of 2 and 4 CTAs sharing each weight tile, with CTAs past the last
    activation row (1 and 300: one group in a cluster of 2; 1100: 3 groups in a cluster of 4;
    2100: 5 groups in 2 clusters of 4)."""
    import torch
    rng = np.random.default_rng(4300 + M)
    L = synth.random_layer(rng, 300, 200, 8, 256, 8, col_scale=True, cb_std=0.3, nnz=700, outlier_scale=1.0)
    Xb = synth.activations(rng, M, L.n_in, "f16")
    m = vq.VQLinear(L)
    n0 = vq.vqlin_kernel_launches()
    Y = m.gemm(G.torch_x(Xb, "f16"), out_dtype=torch.float32)
    assert vq.vqlin_kernel_launches() - n0 == 1          # one fused kernel, no dequant pass
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(Y), oracle.gemv_f64(L, synth.bits_to_f64(Xb, "f16")), "f32", "fused gemm M=%d" % M)


@pytest.mark.parametrize("t", [13, 14, 15, 19])
@pytest.mark.parametrize("M", [1100, 2100])
def test_gemm_fused_cluster_formats(vq, t, M):
    """VSR blocks, codebook groups and the symmetric codebook through the fused prefill when
    2 and 4 CTAs share each weight tile (each dequantises a part of the tile's rows)."""
    import torch
    L = SMALL[t]
    rng = np.random.default_rng(4400 + M + t)
    Xb = synth.activations(rng, M, L.n_in, "f16")
    m = vq.VQLinear(L)
    n0 = vq.vqlin_kernel_launches()
    Y = m.gemm(G.torch_x(Xb, "f16"), out_dtype=torch.float32)
    assert vq.vqlin_kernel_launches() - n0 == 1
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(Y), oracle.gemv_f64(L, synth.bits_to_f64(Xb, "f16")), "f32", "fused gemm t=%d M=%d" % (t, M))


@pytest.mark.parametrize("M", [300, 1100])
@pytest.mark.parametrize("ydt", ["f16", "bf16"])
def test_gemm_fused_16bit_outputs(vq, M, ydt):
    """16-bit outputs of the fused prefill are staged through shared memory and written as row
    segments of Y; n_out = 300 (not a multiple of 8) takes the element-wise tail of that write,
    M = 1100 leaves CTAs past the last activation row."""
    import torch
    rng = np.random.default_rng(4500 + M)
    L = synth.random_layer(rng, 300, 200, 8, 256, 8, col_scale=True, cb_std=0.3, nnz=700, outlier_scale=1.0)
    Xb = synth.activations(rng, M, L.n_in, "f16")
    m = vq.VQLinear(L)
    Y = m.gemm(G.torch_x(Xb, "f16"), out_dtype=G.torch_dtype(ydt))
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(Y), oracle.gemv_f64(L, synth.bits_to_f64(Xb, "f16")), ydt, "fused gemm %s M=%d" % (ydt, M))


@pytest.mark.parametrize("M", [600, 2100])
def test_gemm_fused_dense_sparse_part(vq, M):
    """Rows with many CSR entries in one 64-column block (more than the sparse warp's four
    prefetched ones) and many VSR blocks, through the fused prefill: 25% of the elements are CSR
    entries and a third of the remaining sub-vectors VSR blocks."""
    import torch
    rng = np.random.default_rng(4600 + M)
    n_out, n_in = 140, 264
    L = synth.random_layer(rng, n_out, n_in, 8, 256, 8, col_scale=True, cb_std=0.3,
                           nnz=n_out * n_in // 4, outlier_scale=1.0, vsr_blocks=n_out * (n_in // 8) // 8)
    Xb = synth.activations(rng, M, L.n_in, "f16")
    m = vq.VQLinear(L)
    n0 = vq.vqlin_kernel_launches()
    Y = m.gemm(G.torch_x(Xb, "f16"), out_dtype=torch.float32)
    assert vq.vqlin_kernel_launches() - n0 == 1
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(Y), oracle.gemv_f64(L, synth.bits_to_f64(Xb, "f16")), "f32", "fused gemm dense sparse M=%d" % M)


def test_gemm_fused_more_ctas_than_sms(vq):
    """A fused prefill whose grid (11 weight tiles x 16 activation groups = 176 CTAs in clusters
    of 4) does not fit on the GPU at once, so clusters run in more than one wave."""
    import torch
    rng = np.random.default_rng(4700)
    L = synth.random_layer(rng, 1300, 136, 8, 256, 8, col_scale=True, cb_std=0.3, nnz=900, outlier_scale=1.0)
    M = 8192
    Xb = synth.activations(rng, M, L.n_in, "f16")
    m = vq.VQLinear(L)
    Y = m.gemm(G.torch_x(Xb, "f16"), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    rows = np.sort(rng.choice(M, 256, replace=False))
    G.assert_close(G.to_f64(Y)[rows], oracle.gemv_f64(L, synth.bits_to_f64(Xb[rows], "f16")), "f32", "fused gemm 176 CTAs")


def test_gemm_prefill_sampled_rows(vq):
    L, Xb = G.workload("prefill")
    Y = run_gemm(vq, L, Xb, "bf16", "bf16")
    rng = np.random.default_rng(99)
    rows = np.sort(rng.choice(Xb.shape[0], 48, replace=False))
    ref = oracle.gemv_f64(L, synth.bits_to_f64(Xb[rows], "bf16"))
    G.assert_close(Y[rows], ref, "bf16", "prefill sampled")


# ------------------------------------------------------------------ invalid input -> status, never a fault
def test_invalid_data_is_rejected(vq):
    rng = np.random.default_rng(31)
    L = synth.random_layer(rng, 8, 32, 8, 5, 3, nnz=0)
    L.codes = synth.pack_fields(np.full((8, 4), 6, np.uint32), 3)      # index 6 >= k1 = 5
    with pytest.raises(vq.VQLinError) as e:
        vq.VQLinear(L)
    assert e.value.status == vq.VQLIN_ERR_INVALID_DATA
    L = synth.random_layer(rng, 8, 32, 8, 8, 3, nnz=5)
    L.col_idx = L.col_idx.copy(); L.col_idx[:] = 40                    # column out of range
    with pytest.raises(vq.VQLinError) as e:
        vq.VQLinear(L)
    assert e.value.status == vq.VQLIN_ERR_INVALID_DATA
    L = synth.random_layer(rng, 8, 32, 8, 8, 3, nnz=0)
    L.codebook1 = L.codebook1.copy(); L.codebook1[3, 2] = 0x7E00         # NaN
    with pytest.raises(vq.VQLinError) as e:
        vq.VQLinear(L)
    assert e.value.status == vq.VQLIN_ERR_INVALID_DATA


def test_call_errors_are_statuses(vq):
    import torch
    L = SMALL[1]
    m = vq.VQLinear(L)
    x = torch.zeros((17, L.n_in), dtype=torch.float16, device="cuda")
    y = torch.zeros((17, L.n_out), dtype=torch.float32, device="cuda")
    assert vq.vqlin_gemv(m.handle, x.data_ptr(), vq.VQLIN_F16, 17, y.data_ptr(), vq.VQLIN_F32, None) == vq.VQLIN_ERR_UNSUPPORTED
    assert vq.vqlin_gemv(m.handle, x.data_ptr() + 2, vq.VQLIN_F16, 1, y.data_ptr(), vq.VQLIN_F32, None) == vq.VQLIN_ERR_INVALID_ARG
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    assert vq.vqlin_gemm(m.handle, x.data_ptr(), vq.VQLIN_F16, 4, y.data_ptr(), vq.VQLIN_F32, ws.data_ptr(), 16, None) == vq.VQLIN_ERR_WORKSPACE
    torch.cuda.synchronize()


def test_device_pointers_create(vq):
    """create() also accepts device arrays (src_on_host = 0)."""
    import torch
    L = SMALL[2]
    dev = synth.LayerData(**{k: (torch.from_numpy(np.ascontiguousarray(v)).cuda() if isinstance(v, np.ndarray) and k not in ("fields", "fields_o") else v)
                             for k, v in L.__dict__.items()})
    W = vq.VQLinear(dev).dequant().cpu().numpy().view(np.uint16)
    assert (W == oracle.dequant_exact(L)).all()


# ------------------------------------------------------------------ gemv with a caller workspace (split columns)
@pytest.mark.parametrize("name,batch,ydt", [("downproj", 1, "f16"), ("downproj", 4, "f16"), ("downproj", 16, "bf16"),
                                            ("smollm:6", 8, "f16"), ("qproj", 4, "f16"), ("smollm:0", 1, "f32")])
def test_gemv_ws_full(vq, name, batch, ydt):
    import torch
    L = full_layer(name)
    if name.startswith("smollm"):
        xb = G.workload("smollm")[1][int(name.split(":")[1])][:batch]
        xdt = "bf16"
    else:
        xb = G.workload(name)[1][:batch]
        xdt = "f16"
    m = vq.VQLinear(L)
    x = G.torch_x(xb, xdt)
    ws = torch.full((m_ws := int(vq.vqlin_gemv_workspace_size(m.handle, batch)),), 0x7F, dtype=torch.uint8, device="cuda")
    y = m.gemv_ws(x, workspace=ws, out_dtype=G.torch_dtype(ydt))
    y2 = m.gemv(x, out_dtype=G.torch_dtype(ydt))
    torch.cuda.synchronize()
    ref = oracle.gemv_f64(L, synth.bits_to_f64(xb, xdt))
    G.assert_close(G.to_f64(y), ref, ydt, "gemv_ws %s B=%d" % (name, batch))
    G.assert_close(G.to_f64(y2), ref, ydt, "gemv %s B=%d" % (name, batch))
    assert m_ws >= batch * L.n_out * 4


def test_gemv_ws_errors(vq):
    import torch
    L = SMALL[1]
    m = vq.VQLinear(L)
    x = torch.zeros((2, L.n_in), dtype=torch.float16, device="cuda")
    y = torch.zeros((2, L.n_out), dtype=torch.float16, device="cuda")
    need = int(vq.vqlin_gemv_workspace_size(m.handle, 2))
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    assert vq.vqlin_gemv_ws(m.handle, x.data_ptr(), vq.VQLIN_F16, 2, y.data_ptr(), vq.VQLIN_F16, ws.data_ptr(), need - 1, None) == vq.VQLIN_ERR_WORKSPACE
    assert vq.vqlin_gemv_ws(m.handle, x.data_ptr(), vq.VQLIN_F16, 2, y.data_ptr(), vq.VQLIN_F16, ws.data_ptr() + 16, need, None) == vq.VQLIN_ERR_WORKSPACE
    assert vq.vqlin_gemv_ws(m.handle, x.data_ptr(), vq.VQLIN_F16, 2, y.data_ptr(), vq.VQLIN_F16, ws.data_ptr(), need, None) == vq.VQLIN_OK
    torch.cuda.synchronize()


# ------------------------------------------------------------------ codebook-stationary path (large K, caller workspace)
def cs_layers():
    rng = np.random.default_rng(8080)
    out = [
        synth.random_layer(rng, 300, 1024, 8, 65536, 16, col_scale=True, nnz=500, name="cs_h1"),
        synth.random_layer(rng, 2100, 520, 8, 20000, 15, nnz=300, n_ocols=8, ko=64, bits_o=6, name="cs_h2_oddk"),
    ]
    # skewed: every index in the first slice -> one block's entry stream is far larger than its buffer
    n_out, n_in = 2048, 2048
    fields = rng.integers(0, 600, size=(n_out, n_in // 8)).astype(np.uint32)
    L = synth.random_layer(rng, n_out, n_in, 8, 65536, 16, col_scale=True, nnz=200, name="cs_skewed")
    L.codes = synth.pack_fields(fields, 16)
    L.fields = fields
    out.append(L)
    # symmetric K = 65536 codebook (16384 stored entries) with VSR blocks, and 4 groups of a
    # K = 4096 codebook (a 16384-entry virtual codebook): both take the codebook-stationary layout
    out.append(synth.random_layer(rng, 600, 1024, 8, 65536, 16, cb_symmetry=1, col_scale=True, nnz=300,
                                  vsr_blocks=500, name="cs_sym_vsr"))
    out.append(synth.random_layer(rng, 2100, 768, 8, 4096, 12, n_groups=4, nnz=400, vsr_blocks=300,
                                  name="cs_groups"))
    return out


CS = cs_layers()


@pytest.mark.parametrize("t", range(len(CS)))
@pytest.mark.parametrize("batch", [1, 2, 3, 4])
def test_gemv_codebook_stationary(vq, t, batch):
    import torch
    L = CS[t]
    rng = np.random.default_rng(60 + 10 * t + batch)
    xb = synth.activations(rng, batch, L.n_in, "f16")
    m = vq.VQLinear(L)
    x = G.torch_x(xb, "f16")
    y = m.gemv_ws(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert vq.device_error() == 0
    G.assert_close(G.to_f64(y), oracle.gemv_f64(L, synth.bits_to_f64(xb, "f16")), "f32", "%s B=%d" % (L.name, batch))


def test_gemv_codebook_stationary_full_qproj(vq):
    import torch
    L, xb = G.workload("qproj")
    m = vq.VQLinear(L)
    for batch in (1, 4):
        x = G.torch_x(xb[:batch], "f16")
        y = m.gemv_ws(x, out_dtype=torch.float16)
        torch.cuda.synchronize()
        G.assert_close(G.to_f64(y), oracle.gemv_f64(L, synth.bits_to_f64(xb[:batch], "f16")), "f16", "qproj cs B=%d" % batch)


def test_kernel_launch_counter(vq):
    """Every call enqueues at least one of the library's kernels and the counter sees each one."""
    import torch
    L, xb = G.workload("qproj")
    m = vq.VQLinear(L)
    x = G.torch_x(xb[:1], "f16")
    n0 = vq.vqlin_kernel_launches()
    m.gemv_ws(x, out_dtype=torch.float16)
    n1 = vq.vqlin_kernel_launches()
    assert n1 - n0 == 2          # codebook-stationary slice kernel + finalize
    s = SMALL[0]
    ms = vq.VQLinear(s)
    n0 = vq.vqlin_kernel_launches()
    ms.gemv(G.torch_x(synth.activations(np.random.default_rng(1), 2, s.n_in, "f16"), "f16"))
    ms.dequant()
    torch.cuda.synchronize()
    assert vq.vqlin_kernel_launches() - n0 >= 2


def test_codebook_stationary_is_deterministic(vq):
    """The fixed-point row sums do not depend on the order of the atomics: repeated calls agree bit for bit."""
    import torch
    L, xb = G.workload("qproj")
    m = vq.VQLinear(L)
    x = G.torch_x(xb[:4], "f16")
    ys = [m.gemv_ws(x, out_dtype=torch.float32).cpu().numpy().view(np.uint32) for _ in range(3)]
    assert (ys[0] == ys[1]).all() and (ys[0] == ys[2]).all()


# ------------------------------------------------------------------ bit accounting of a created layer
def test_library_info_matches_the_vptq_worked_example(vq):
    """The library's own accounting for a 4096x4096 layer with V = 8 and k = 256 (VPTQ page,
    "Compression ratio calculation", the example taken from its section 2.2): ratio 15.97 and
    about 1.002 bits per weight, as printed there."""
    g = json.load(open(os.path.join(GOLDEN, "vptq_compression_example.json")))
    rng = np.random.default_rng(4096)
    L = synth.random_layer(rng, 4096, 4096, g["V"], g["k"], 8, row_scale=False, nnz=0)
    info = vq.VQLinear(L).info()
    assert round(info["vptq_compression_ratio"], g["ratio_printed_decimals"]) == g["ratio_printed"]
    assert round(info["vptq_bits_per_weight"], g["bits_printed_decimals"]) == g["bits_printed"]
    assert abs(16.0 / info["vptq_compression_ratio"] - info["vptq_bits_per_weight"]) < 1e-12
    assert info["index_bytes"] == 4096 * 512 and info["codebook_bytes"] == 2 * 8 * 256
