"""Pins of the CPU oracle against facts fixed outside it (CPU only).

- the worked compression example the VPTQ page prints;
- a hand-worked 2x8 layer (golden file);
- hand-derived IEEE fp16 rounding vectors, including the double-rounding trap;
- hand-derived packed-field byte strings;
- exact rational brute force (tests/exact.py) on small random layers covering
  residual codebooks, outlier columns, row/column scales and the sparse set;
- closed forms: one-hot codebook, K = 1, a 100%-dense sparse set, exact
  power-of-two data, the outlier invariant, RVQ's k1*k2 reconstructions;
- library routines: numpy's fp16 cast and widening for every bit pattern.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from sparse_compensated_vq_b200 import synth
from tests import exact

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def hx(s):
    return None if s is None else int(s, 16)


# ---------------------------------------------------------------- accounting
def test_vptq_compression_worked_example():
    g = load("vptq_compression_example.json")
    ratio = oracle.vptq_compression_ratio(g["n_elems"], g["V"], g["k"])
    assert round(ratio, g["ratio_printed_decimals"]) == g["ratio_printed"]
    assert round(16.0 / ratio, g["bits_printed_decimals"]) == g["bits_printed"]
    # exact value of the printed formula: 16*M / (V*k*16 + M*8/V) with M = 2^24
    assert ratio == pytest.approx(16 * 2**24 / (8 * 256 * 16 + 2**24), rel=1e-15)


def test_compression_ratio_ceil_log2():
    # k not a power of two takes ceil(log2 k) index bits
    r = oracle.vptq_compression_ratio(4096 * 4096, 6, 4000)
    assert r == pytest.approx(16 * 4096 * 4096 / (6 * 4000 * 16 + 4096 * 4096 * 12 / 6))


# ---------------------------------------------------------------- fp16 pins
def test_f16_widening_matches_numpy_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(b) for b in bits[::7]])
    r = ref[::7]
    same = (got == r) | (np.isnan(got) & np.isnan(r))
    assert same.all()


def test_bf16_widening_matches_numpy():
    bits = np.arange(0, 65536, 5, dtype=np.uint32).astype(np.uint16)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = np.array([oracle.bf16_to_f64(b) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_round_f16_matches_numpy_on_doubles():
    # a double is rounded once by numpy's cast: must equal the oracle's integer rounding
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-5, 2000), rng.normal(0, 3e4, 2000),
                           np.ldexp(rng.integers(1, 4096, 500).astype(np.float64), rng.integers(-40, 8, 500)),
                           np.array([65519.99, 65520.0, 65504.0, 2.0**-25, 3 * 2.0**-26, 2.0**-24])])
    for v in vals:
        m, e = np.frexp(abs(v))
        mant = int(m * 2.0**53)
        got = oracle.round_f16(1 if v < 0 else 0, mant, int(e) - 53)
        assert got == int(np.float16(v).view(np.uint16)), v


def test_round_f16_matches_rational_rounding():
    rng = np.random.default_rng(8)
    for _ in range(2000):
        mant = int(rng.integers(1, 2**62)) * int(rng.integers(1, 2**11))
        e = int(rng.integers(-110, -40))
        assert oracle.round_f16(0, mant, e) == exact.rne_f16(Fraction(mant) * Fraction(2) ** e)


def test_rounding_vectors_golden():
    g = load("f16_rounding.json")
    for c in g["cases"]:
        got = oracle.body_f16(hx(c["c1"]), hx(c["c2"]), hx(c["r"]), hx(c["c"]))
        assert got == hx(c["expect"]), c["note"]
        if "fp32_chain" in c:
            # the trap is real: a float32 chain lands on the other neighbour
            v = np.float32(exact.f16_float(hx(c["c1"])))
            for k in ("c2",):
                if c[k]:
                    v = np.float32(v + np.float32(exact.f16_float(hx(c[k]))))
            for k in ("r", "c"):
                if c[k]:
                    v = np.float32(v * np.float32(exact.f16_float(hx(c[k]))))
            assert int(np.float16(v).view(np.uint16)) == hx(c["fp32_chain"])


# ---------------------------------------------------------------- packing
def test_packed_field_bytes_golden():
    g = load("packed_fields.json")
    for c in g["cases"]:
        w = c["w"]
        fields = [hx(f) for f in c["fields"]]
        want = bytes.fromhex(c["bytes"].replace(" ", ""))
        row = np.frombuffer(want, dtype=np.uint8)[None, :]
        got = oracle.unpack(row, len(fields), w)[0].tolist()
        assert got == fields
        packed = synth.pack_fields(np.array([fields], dtype=np.uint32), w)
        assert packed.tobytes() == want
        if "i1" in c:
            f = got[0]
            assert f & ((1 << c["bits1"]) - 1) == hx(c["i1"]) and f >> c["bits1"] == hx(c["i2"])


@pytest.mark.parametrize("w", [1, 3, 4, 7, 8, 9, 12, 13, 16, 17, 24, 31, 32])
def test_unpack_matches_bigint_reading(w):
    rng = np.random.default_rng(w)
    n_fields = 37
    stride = synth.packed_row_bytes(n_fields, w) + 5
    codes = rng.integers(0, 256, size=(4, stride), dtype=np.uint8)
    got = oracle.unpack(codes, n_fields, w)
    for i in range(4):
        for s in range(n_fields):
            assert got[i, s] == exact.field(codes[i].tobytes(), s, w)
    # and the generator's serialiser round-trips through it
    fields = (rng.integers(0, 2**w, size=(3, n_fields), dtype=np.uint64)).astype(np.uint32)
    assert (oracle.unpack(synth.pack_fields(fields, w), n_fields, w) == fields).all()


# ---------------------------------------------------------------- hand-worked layer
def _layer_from_golden(g):
    cb = synth.f16_bits(np.array(g["codebook"], dtype=np.float64))
    fields = np.array(g["indices"], dtype=np.uint32)
    codes = synth.pack_fields(fields, g["bits"])
    vals = synth.f16_bits(np.array(g["csr"]["values"]))
    return synth.LayerData(
        n_out=len(g["indices"]), n_in=len(g["x"]), d=g["d"], k1=g["k"], bits1=g["bits"], codes=codes,
        codebook1=cb, row_scale=synth.f16_bits(g["row_scale"]), col_scale=synth.f16_bits(g["col_scale"]),
        row_ptr=np.array(g["csr"]["row_ptr"], np.int32), col_idx=np.array(g["csr"]["col_idx"], np.int32),
        values=vals)


def test_hand_worked_2x8():
    g = load("hand_2x8.json")
    L = _layer_from_golden(g)
    W = oracle.dequant_f64(L)
    assert W.tolist() == g["W"]
    Wb = oracle.dequant_exact(L)
    assert (Wb == synth.f16_bits(np.array(g["W"]))).all()
    y = oracle.gemv_f64(L, np.array([g["x"]], dtype=np.float64))
    assert y[0].tolist() == g["y"]


# ---------------------------------------------------------------- brute force
CASES = [
    dict(n_out=5, n_in=16, d=4, k1=16, bits1=4),
    dict(n_out=3, n_in=10, d=4, k1=5, bits1=3, row_scale=True, col_scale=True),            # ragged tail
    dict(n_out=4, n_in=24, d=8, k1=256, bits1=8, col_scale=True, nnz=9),
    dict(n_out=6, n_in=20, d=4, k1=12, bits1=4, k2=7, bits2=3, col_scale=True, nnz=7),      # residual
    dict(n_out=4, n_in=19, d=4, k1=16, bits1=4, n_ocols=5, ko=9, bits_o=4, col_scale=True, nnz=6),  # outlier block
    dict(n_out=3, n_in=26, d=8, k1=4096, bits1=12, k2=4096, bits2=12, n_ocols=3, ko=256, bits_o=8, nnz=10),
    dict(n_out=2, n_in=12, d=4, k1=65536, bits1=16, col_scale=True, row_scale=False, nnz=0),
    # VPTQ's other vector lengths
    dict(n_out=4, n_in=17, d=6, k1=9, bits1=4, col_scale=True, nnz=5),                      # d = 6, ragged tail
    dict(n_out=3, n_in=30, d=6, k1=16, bits1=4, k2=5, bits2=3, n_ocols=7, ko=3, bits_o=2, nnz=4),
    dict(n_out=3, n_in=29, d=12, k1=32, bits1=5, col_scale=True, nnz=6),                    # d = 12, ragged tail
    dict(n_out=2, n_in=40, d=12, k1=256, bits1=8, k2=16, bits2=4, n_ocols=13, ko=7, bits_o=3, col_scale=True, nnz=5),
    # codebook groups (VPTQ group_num), symmetric codebooks (SCVQ), VSR blocks (SCVQ)
    dict(n_out=4, n_in=40, d=4, k1=16, bits1=4, n_groups=3, col_scale=True, nnz=4),         # 10 positions, 3 groups
    dict(n_out=3, n_in=44, d=4, k1=8, bits1=3, k2=4, bits2=2, n_groups=4, n_ocols=4, ko=5, bits_o=3, nnz=3),
    dict(n_out=5, n_in=24, d=8, k1=64, bits1=6, cb_symmetry=1, col_scale=True, nnz=6),
    dict(n_out=4, n_in=30, d=6, k1=32, bits1=5, cb_symmetry=1, n_groups=2, k2=3, bits2=2, nnz=3),
    dict(n_out=6, n_in=27, d=4, k1=16, bits1=4, col_scale=True, nnz=8, vsr_blocks=9),      # ragged tail block possible
    dict(n_out=5, n_in=34, d=8, k1=64, bits1=6, cb_symmetry=1, n_groups=2, n_ocols=5, ko=6, bits_o=3, nnz=6,
         vsr_blocks=6),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_dequant_matches_rational_brute_force(case):
    kw = dict(CASES[case])
    rng = np.random.default_rng(100 + case)
    kw.setdefault("row_scale", True)
    nnz = kw.pop("nnz", 3)
    L = synth.random_layer(rng, cb_std=0.5, res_std=0.05, nnz=nnz, outlier_scale=2.0, **kw)
    Wq, Wbits = exact.exact_layer(L)
    got = oracle.dequant_exact(L)
    assert got.tolist() == Wbits
    W64 = oracle.dequant_f64(L)
    for i in range(L.n_out):
        for j in range(L.n_in):
            ref = float(Wq[i][j])
            assert W64[i, j] == pytest.approx(ref, rel=2.0**-52, abs=0.0)
    x = rng.standard_normal((3, L.n_in)).astype(np.float16).astype(np.float64)
    y = oracle.gemv_f64(L, x)
    yq = exact.exact_matvec(Wq, x)
    for b in range(3):
        scale = sum(abs(float(Wq[i][j]) * x[b, j]) for i in range(L.n_out) for j in range(L.n_in))
        for i in range(L.n_out):
            assert abs(y[b, i] - float(yq[b][i])) <= 4 * L.n_in * 2.0**-53 * scale


# ---------------------------------------------------------------- groups, symmetric codebooks, VSR
def test_identical_group_codebooks_reduce_to_one_codebook():
    """n_groups copies of the same codebook decode like the single codebook (VPTQ's group
    partitioning with nothing to specialise)."""
    rng = np.random.default_rng(120)
    L1 = synth.random_layer(rng, 7, 80, 8, 32, 5, col_scale=True, nnz=9)
    for G in (2, 3, 10):
        LG = synth.LayerData(**{k: v for k, v in L1.__dict__.items()})
        LG.n_groups = G
        LG.codebook1 = np.tile(L1.codebook1, (G, 1))
        assert (oracle.dequant_exact(LG) == oracle.dequant_exact(L1)).all()


def test_group_boundaries_follow_the_position_ranges():
    """Group g owns positions [g * ceil(n_sub / G), ...): with one-hot codebooks whose group g
    entry is the value g + 1 everywhere, every decoded weight names its group."""
    n_out, d, G, k1 = 3, 4, 3, 2
    n_sub = 7                                         # groups of 3, 3, 1 positions
    cb = np.concatenate([np.full((k1, d), g + 1.0) for g in range(G)])
    L = synth.LayerData(n_out=n_out, n_in=n_sub * d, d=d, k1=k1, bits1=1,
                        codes=synth.pack_fields(np.zeros((n_out, n_sub), np.uint32), 1),
                        codebook1=synth.f16_bits(cb), n_groups=G)
    W = oracle.dequant_f64(L)
    want = np.repeat(np.array([1, 1, 1, 2, 2, 2, 3], float), d)
    assert (W == want[None, :]).all()


def test_symmetric_codebook_equals_its_expansion():
    """A symmetric codebook decodes like the plain codebook of its k1 entries, built here with
    numpy negation: pattern 0 +, 1 all -, 2 odd elements -, 3 even elements -."""
    rng = np.random.default_rng(121)
    for d, G in ((4, 1), (8, 2), (12, 1)):
        L = synth.random_layer(rng, 6, 6 * d + 3, d, 16, 4, cb_symmetry=1, n_groups=G, col_scale=True, nnz=5)
        base = L.codebook1.view(np.float16).astype(np.float64).reshape(G, 4, d)
        sign = np.ones((4, d))
        sign[1] = -1
        sign[2, 1::2] = -1
        sign[3, 0::2] = -1
        full = (sign[None, :, None, :] * base[:, None, :, :]).reshape(G * 16, d)
        P = synth.LayerData(**{k: v for k, v in L.__dict__.items()})
        P.cb_symmetry = 0
        P.codebook1 = synth.f16_bits(full)
        assert (oracle.dequant_exact(L) == oracle.dequant_exact(P)).all()


def _vsr_as_csr(L):
    """The same layer with every VSR block written as d CSR entries (main columns, REPLACE)."""
    main = np.array([j for j in range(L.n_in) if j not in set(L.ocols.tolist())])
    rows, cols, vals = [], [], []
    for i in range(L.n_out):
        if L.nnz:
            for e in range(L.row_ptr[i], L.row_ptr[i + 1]):
                rows.append(i); cols.append(int(L.col_idx[e])); vals.append(int(L.values[e]))
        for b in range(L.vsr_row_ptr[i], L.vsr_row_ptr[i + 1]):
            for t in range(L.d):
                q = int(L.vsr_pos[b]) * L.d + t
                if q < main.size:
                    rows.append(i); cols.append(int(main[q])); vals.append(int(L.vsr_values[b, t]))
    rp, ci, v = synth.csr_from_positions(L.n_out, np.array(rows), np.array(cols), np.array(vals, np.uint16))
    C = synth.LayerData(**{k: v for k, v in L.__dict__.items()})
    C.row_ptr, C.col_idx, C.values = rp, ci, v
    C.vsr_row_ptr = C.vsr_pos = C.vsr_values = None
    return C


def test_vsr_blocks_equal_their_csr_entries():
    rng = np.random.default_rng(122)
    for kw in (dict(d=8, n_ocols=0), dict(d=4, n_ocols=5), dict(d=12, n_ocols=3)):
        L = synth.random_layer(rng, 9, 101, kw["d"], 64, 6, n_ocols=kw["n_ocols"], ko=8, bits_o=3,
                               col_scale=True, nnz=25, vsr_blocks=14)
        assert L.vsr_nblocks == 14
        C = _vsr_as_csr(L)
        assert (oracle.dequant_exact(L) == oracle.dequant_exact(C)).all()
        x = rng.standard_normal((2, L.n_in))
        assert np.array_equal(oracle.gemv_f64(L, x), oracle.gemv_f64(C, x))


def test_vsr_full_rows_are_dense_rows():
    rng = np.random.default_rng(123)
    d, n_in = 8, 40
    L = synth.random_layer(rng, 3, n_in, d, 16, 4, col_scale=True, nnz=0)
    V = rng.normal(0, 1, (3, n_in)).astype(np.float16)
    L.vsr_row_ptr = (np.arange(4) * (n_in // d)).astype(np.int32)
    L.vsr_pos = np.tile(np.arange(n_in // d), 3).astype(np.int32)
    L.vsr_values = V.reshape(-1, d).view(np.uint16)
    assert (oracle.dequant_exact(L) == V.view(np.uint16)).all()


def test_malformed_vsr_is_reported():
    rng = np.random.default_rng(124)
    L = synth.random_layer(rng, 4, 32, 8, 16, 4, nnz=0, vsr_blocks=3)
    bad = synth.LayerData(**{k: v for k, v in L.__dict__.items()})
    bad.vsr_pos = L.vsr_pos.copy(); bad.vsr_pos[0] = 4                      # position >= n_sub
    with pytest.raises(oracle.OracleError):
        oracle.dequant_exact(bad)
    row = int(np.nonzero(np.diff(L.vsr_row_ptr))[0][0])
    s0 = int(L.vsr_pos[L.vsr_row_ptr[row]])
    over = synth.LayerData(**{k: v for k, v in L.__dict__.items()})
    over.row_ptr = np.zeros(5, np.int32); over.row_ptr[row + 1:] = 1
    over.col_idx = np.array([s0 * 8 + 3], np.int32); over.values = synth.f16_bits([1.0])   # inside a block
    with pytest.raises(oracle.OracleError):
        oracle.dequant_exact(over)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(3)
    L = synth.random_layer(rng, 9, 40, 8, 64, 6, col_scale=True, nnz=12, n_ocols=4, ko=16, bits_o=4)
    x = rng.standard_normal((2, 40))
    full = oracle.gemv_f64(L, x)
    rows = [7, 0, 3]
    assert (oracle.gemv_f64(L, x, rows=rows) == full[:, rows]).all()
    assert (oracle.dequant_f64(L, rows=rows) == oracle.dequant_f64(L)[rows]).all()


# ---------------------------------------------------------------- invariants / closed forms
def test_outlier_positions_reproduce_stored_values_exactly():
    rng = np.random.default_rng(11)
    L = synth.random_layer(rng, 64, 96, 8, 256, 8, col_scale=True, nnz=300, outlier_scale=5.0,
                           n_ocols=7, ko=32, bits_o=5)
    W = oracle.dequant_exact(L)
    for i in range(L.n_out):
        for e in range(L.row_ptr[i], L.row_ptr[i + 1]):
            assert W[i, L.col_idx[e]] == L.values[e]
    W64 = oracle.dequant_f64(L)
    for i in range(L.n_out):
        for e in range(L.row_ptr[i], L.row_ptr[i + 1]):
            assert W64[i, L.col_idx[e]] == float(L.values[e:e + 1].view(np.float16)[0])


def test_rvq_decodes_all_k1_times_k2_pairs():
    # VPTQ page, "Residual Vector Quantization": k1*k2 distinct reconstructions C[i1] + Cres[i2]
    d, k1, k2 = 4, 4, 4
    c1 = synth.f16_bits(np.array([[1, 2, 3, 4], [-1, 0.5, 0, 2], [8, -8, 4, -4], [0.25, 0.5, 0.75, 1]]))
    c2 = synth.f16_bits(np.array([[0.125, 0, 0, 0], [0, 0.0625, 0, 0], [0, 0, 0.03125, 0], [0, 0, 0, 0.015625]]))
    pairs = [(a, b) for a in range(k1) for b in range(k2)]
    fields = np.array([[a | (b << 2) for a, b in pairs]], dtype=np.uint32)
    L = synth.LayerData(n_out=1, n_in=d * len(pairs), d=d, k1=k1, bits1=2, k2=k2, bits2=2,
                        codes=synth.pack_fields(fields, 4), codebook1=c1, codebook2=c2)
    W = oracle.dequant_f64(L)[0].reshape(len(pairs), d)
    f = lambda h: h.view(np.float16).astype(np.float64)
    for t, (a, b) in enumerate(pairs):
        assert (W[t] == f(c1[a]) + f(c2[b])).all()
    assert len({tuple(r) for r in W}) == k1 * k2
    # a residual codebook of +0 reduces to the single-stage decode
    L0 = synth.LayerData(n_out=1, n_in=L.n_in, d=d, k1=k1, bits1=2, k2=k2, bits2=2, codes=L.codes,
                         codebook1=c1, codebook2=np.zeros_like(c2))
    single = synth.LayerData(n_out=1, n_in=d * len(pairs), d=d, k1=k1, bits1=4,
                             codes=synth.pack_fields(fields & 3, 4), codebook1=c1)
    assert (oracle.dequant_exact(L0) == oracle.dequant_exact(single)).all()


@pytest.mark.parametrize("d", [4, 6, 8, 12])
def test_one_hot_codebook_gather_sum(d):
    # C[k] = e_(k mod d): y_i = r_i * sum_s c_j x_j with j = s*d + (idx mod d)
    rng = np.random.default_rng(12 + d)
    k = 64
    cb = np.zeros((k, d)); cb[np.arange(k), np.arange(k) % d] = 1.0
    n_out, n_in = 7, 5 * d
    fields = rng.integers(0, k, size=(n_out, n_in // d)).astype(np.uint32)
    rs = synth.f16_bits(rng.uniform(0.5, 1.5, n_out)); cs = synth.f16_bits(rng.uniform(0.5, 1.5, n_in))
    L = synth.LayerData(n_out=n_out, n_in=n_in, d=d, k1=k, bits1=6, codes=synth.pack_fields(fields, 6),
                        codebook1=synth.f16_bits(cb), row_scale=rs, col_scale=cs)
    x = rng.standard_normal((2, n_in))
    y = oracle.gemv_f64(L, x)
    r = rs.view(np.float16).astype(np.float64); c = cs.view(np.float16).astype(np.float64)
    for b in range(2):
        for i in range(n_out):
            ref = 0.0
            for s in range(n_in // d):
                j = s * d + int(fields[i, s]) % d
                ref += r[i] * c[j] * x[b, j]
            assert y[b, i] == pytest.approx(ref, rel=1e-13)


def test_single_entry_codebook():
    rng = np.random.default_rng(13)
    d, n_out, n_in = 4, 5, 22
    c0 = synth.f16_bits(rng.normal(0, 1, (1, d)))
    n_sub = -(-n_in // d)
    L = synth.LayerData(n_out=n_out, n_in=n_in, d=d, k1=1, bits1=1,
                        codes=synth.pack_fields(np.zeros((n_out, n_sub), np.uint32), 1), codebook1=c0,
                        row_scale=synth.f16_bits(rng.uniform(0.5, 1.5, n_out)))
    x = rng.standard_normal((1, n_in))
    y = oracle.gemv_f64(L, x)[0]
    r = L.row_scale.view(np.float16).astype(np.float64)
    cvals = c0.view(np.float16).astype(np.float64)[0]
    for i in range(n_out):
        assert y[i] == pytest.approx(r[i] * sum(cvals[j % d] * x[0, j] for j in range(n_in)), rel=1e-13)


def test_fully_dense_sparse_set_is_a_plain_matvec():
    rng = np.random.default_rng(14)
    n_out, n_in = 6, 16
    V = rng.normal(0, 1, (n_out, n_in)).astype(np.float16)
    L = synth.random_layer(rng, n_out, n_in, 4, 16, 4, col_scale=True, nnz=0)
    L.row_ptr = (np.arange(n_out + 1) * n_in).astype(np.int32)
    L.col_idx = np.tile(np.arange(n_in), n_out).astype(np.int32)
    L.values = V.reshape(-1).view(np.uint16)
    x = rng.standard_normal((3, n_in))
    assert (oracle.dequant_exact(L) == V.view(np.uint16)).all()
    np.testing.assert_allclose(oracle.gemv_f64(L, x), x @ V.astype(np.float64).T, rtol=1e-14, atol=1e-14)


def test_power_of_two_data_is_exact():
    rng = np.random.default_rng(15)
    n_out, n_in, d = 6, 32, 8
    cb = synth.f16_bits(np.ldexp(rng.choice([-1.0, 1.0], (16, d)), rng.integers(-6, 3, (16, d))))
    fields = rng.integers(0, 16, size=(n_out, n_in // d)).astype(np.uint32)
    L = synth.LayerData(n_out=n_out, n_in=n_in, d=d, k1=16, bits1=4, codes=synth.pack_fields(fields, 4),
                        codebook1=cb, row_scale=synth.f16_bits(np.ldexp(1.0, rng.integers(-2, 3, n_out))),
                        col_scale=synth.f16_bits(np.ldexp(1.0, rng.integers(-2, 3, n_in))))
    x = np.ldexp(1.0, rng.integers(-3, 3, (1, n_in)))
    Wq, _ = exact.exact_layer(L)
    yq = exact.exact_matvec(Wq, x)
    assert oracle.gemv_f64(L, x)[0].tolist() == [float(v) for v in yq[0]]


# ---------------------------------------------------------------- invalid data
def test_index_out_of_range_is_reported():
    rng = np.random.default_rng(16)
    L = synth.random_layer(rng, 3, 8, 4, 5, 3, nnz=0)
    L.codes = synth.pack_fields(np.array([[0, 1], [2, 5], [4, 4]], np.uint32), 3)
    with pytest.raises(oracle.OracleError):
        oracle.dequant_exact(L)


def test_malformed_csr_is_reported():
    rng = np.random.default_rng(17)
    L = synth.random_layer(rng, 3, 8, 4, 8, 3, nnz=0)
    L.row_ptr = np.array([0, 2, 2, 3], np.int32)
    L.col_idx = np.array([5, 5, 1], np.int32)       # duplicate column in row 0
    L.values = synth.f16_bits([1.0, 2.0, 3.0])
    with pytest.raises(oracle.OracleError):
        oracle.dequant_exact(L)


# ---------------------------------------------------------------- nearest-centroid assignment
# VPTQ page, "Step 3": Q_V(v) = argmin_i ||v - C_i||^2; "Residual Vector Quantization":
# i2 = argmin_j ||(v - C1[i1]) - Cres_j||^2.  The oracle computes these exactly (integer units of
# 2^-24), ties to the lowest index.  The pins: an independent exact-rational brute force, the
# one-dimensional case against numpy's argmin on exact float64 differences, a case that float64
# squares cannot decide, exact hits and ties, scaling invariance, constructed residual pairs, and
# the oracle's own exact distances against the brute force.


def _exact_sqdist(v_bits, c_bits, base_bits=None):
    base = [0] * len(v_bits) if base_bits is None else [exact.f16_frac(int(b)) for b in base_bits]
    return sum(((exact.f16_frac(int(a)) - o - exact.f16_frac(int(b))) ** 2
                for a, o, b in zip(v_bits, base, c_bits)), Fraction(0))


def _brute_argmin(v_bits, C, base_bits=None):
    dist = [_exact_sqdist(v_bits, C[i], base_bits) for i in range(len(C))]
    return min(range(len(C)), key=lambda i: (dist[i], i))


@pytest.mark.parametrize("d", [4, 6, 8, 12])
def test_assign_is_the_exact_argmin(d):
    rng = np.random.default_rng(300 + d)
    k1, k2, n = 37, 11, 25
    C1 = synth.f16_bits(rng.normal(0, 1, (k1, d)))
    C2 = synth.f16_bits(rng.normal(0, 0.3, (k2, d)))
    V = synth.f16_bits(rng.normal(0, 1, (n, d)))
    i1, i2 = oracle.assign_exact(V, C1, C2)
    for s in range(n):
        a = _brute_argmin(V[s], C1)
        assert int(i1[s]) == a
        assert int(i2[s]) == _brute_argmin(V[s], C2, base_bits=C1[a])
    # the residual stage for a prescribed first choice
    forced = rng.integers(0, k1, n).astype(np.uint32)
    r2 = oracle.residual_assign_exact(V, C1, forced, C2)
    for s in range(n):
        assert int(r2[s]) == _brute_argmin(V[s], C2, base_bits=C1[forced[s]])


def test_sqdist_is_exact():
    rng = np.random.default_rng(310)
    for d in (1, 4, 8, 12):
        v, c, b = (synth.f16_bits(rng.normal(0, 100, d)) for _ in range(3))
        assert Fraction(oracle.sqdist_exact(v, c), 2 ** 48) == _exact_sqdist(v, c)
        assert Fraction(oracle.sqdist_exact(v, c, b), 2 ** 48) == _exact_sqdist(v, c, b)
    # the extremes of the format: largest finite values of opposite sign, smallest subnormal
    v = np.array([0x7BFF, 0x0001, 0x8001], np.uint16)
    c = np.array([0xFBFF, 0x8001, 0x0001], np.uint16)
    assert Fraction(oracle.sqdist_exact(v, c), 2 ** 48) == _exact_sqdist(v, c)


def test_assign_one_dimension_is_the_nearest_value():
    """d = 1: the nearest scalar; fp16 differences are exact in float64, so numpy's argmin of
    |v - c| (first index on ties) is the exact answer."""
    rng = np.random.default_rng(311)
    C = synth.f16_bits(rng.normal(0, 1, (200, 1)))
    V = synth.f16_bits(rng.normal(0, 1.2, (500, 1)))
    i1, _ = oracle.assign_exact(V, C)
    cv = C[:, 0].view(np.float16).astype(np.float64)
    vv = V[:, 0].view(np.float16).astype(np.float64)
    assert (i1 == np.argmin(np.abs(vv[:, None] - cv[None, :]), axis=1)).all()


def test_assign_decides_where_double_precision_squares_tie():
    """||(0,0) - (1024, 2^-24)||^2 = 2^20 + 2^-48 rounds to 2^20 in float64, a tie with (1024, 0);
    exactly, (1024, 0) is closer."""
    V = synth.f16_bits(np.array([[0.0, 0.0]]))
    C = synth.f16_bits(np.array([[1024.0, 2.0 ** -24], [1024.0, 0.0]]))
    f = C.view(np.float16).astype(np.float64)
    assert (f ** 2).sum(axis=1)[0] == (f ** 2).sum(axis=1)[1]
    assert oracle.assign_exact(V, C)[0].tolist() == [1]


def test_assign_exact_hits_and_ties_take_the_lowest_index():
    rng = np.random.default_rng(41)
    d = 8
    base = synth.f16_bits(rng.normal(0, 1, (10, d)))
    C = np.concatenate([base, base[[3, 7]], base]).astype(np.uint16)   # duplicates at 10, 11 and 12..21
    V = base[[3, 7, 0, 9]]
    i1, _ = oracle.assign_exact(V, C)
    assert i1.tolist() == [3, 7, 0, 9]
    # equidistant centroids: v halfway (exactly) between two candidates
    C2 = synth.f16_bits(np.array([[0, 0, 0, 0], [2, 0, 0, 0], [1, 0, 0, 1.5], [1, 0, 0, -1.5]]))
    V2 = synth.f16_bits(np.array([[1, 0, 0, 0]]))
    assert oracle.assign_exact(V2, C2)[0].tolist() == [0]
    C3 = C2[[1, 0, 2, 3]]                      # the same tie with the candidates swapped
    assert oracle.assign_exact(V2, C3)[0].tolist() == [0]


def test_assign_invariant_under_power_of_two_scaling():
    rng = np.random.default_rng(312)
    d = 8
    Cf = rng.normal(0, 1, (64, d)).astype(np.float16).astype(np.float64)
    Vf = rng.normal(0, 1, (300, d)).astype(np.float16).astype(np.float64)
    a, _ = oracle.assign_exact(synth.f16_bits(Vf), synth.f16_bits(Cf))
    b, _ = oracle.assign_exact(synth.f16_bits(Vf * 4.0), synth.f16_bits(Cf * 4.0))
    assert (a == b).all()


def test_residual_stage_recovers_constructed_pairs():
    # C1 entries far apart (multiples of 8), residual entries small (multiples of 1/4, |.| <= 1):
    # every v = C1[a] + C2[b] is exact in fp16 and its two-stage argmin is (a, b)
    rng = np.random.default_rng(42)
    d, k1, k2 = 6, 12, 9
    C1 = synth.f16_bits(8.0 * rng.integers(-6, 7, (k1, d)))
    C1 = np.unique(C1, axis=0)[:k1]
    k1 = len(C1)
    C2 = synth.f16_bits(0.25 * rng.integers(-4, 5, (k2, d)))
    C2 = np.unique(C2, axis=0)
    k2 = len(C2)
    pairs = [(a, b) for a in range(k1) for b in range(k2)]
    f = lambda h: h.view(np.float16).astype(np.float64)
    V = synth.f16_bits(np.array([f(C1[a]) + f(C2[b]) for a, b in pairs]))
    i1, i2 = oracle.assign_exact(V, C1, C2)
    assert list(zip(i1.tolist(), i2.tolist())) == pairs


def test_assign_rejects_non_finite_input():
    C = synth.f16_bits(np.ones((2, 4)))
    V = np.array([[0x7C00, 0, 0, 0]], dtype=np.uint16)     # +inf
    with pytest.raises(oracle.OracleError):
        oracle.assign_exact(V, C)
