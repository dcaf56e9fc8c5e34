"""Exact rational brute force for tiny layers, used to pin the oracle.

Written independently of oracle.c: fp16 values are widened through numpy,
products and sums are Python Fractions, indices are read from a Python big
integer, and the final rounding to fp16 is done on Fractions.  Signs of zero
results come from numpy's IEEE double arithmetic.
"""
from fractions import Fraction

import numpy as np


def f16_frac(bits: int) -> Fraction:
    return Fraction(float(np.array([bits], dtype=np.uint16).view(np.float16)[0]))


def f16_float(bits: int) -> float:
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


def rne_f16(q: Fraction, negative_zero: bool = False) -> int:
    """Nearest fp16 (ties to even, overflow to inf) of an exact rational."""
    sign = 1 if (q < 0 or (q == 0 and negative_zero)) else 0
    a = abs(q)
    if a == 0:
        return sign << 15
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -14)
    n = a / Fraction(2) ** (e - 10)
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    if fl == 0:
        return sign << 15
    if fl >= 2048:
        fl //= 2
        e += 1
    if e == -14 and fl < 1024:
        return (sign << 15) | fl
    ef = e + 15
    if ef >= 31:
        return (sign << 15) | 0x7C00
    return (sign << 15) | (ef << 10) | (fl - 1024)


def field(row_bytes: bytes, s: int, w: int) -> int:
    return (int.from_bytes(row_bytes, "little") >> (s * w)) & ((1 << w) - 1)


def exact_layer(L):
    """Exact weights of a LayerData: (W as Fractions [n_out][n_in], fp16 bits [n_out][n_in])."""
    n_out, n_in, d = L.n_out, L.n_in, L.d
    ocols = [int(j) for j in L.ocols]
    out_rank = {j: p for p, j in enumerate(ocols)}
    main = [j for j in range(n_in) if j not in out_rank]
    main_rank = {j: q for q, j in enumerate(main)}
    w = L.bits1 + L.bits2
    csr = {}
    if L.nnz:
        for i in range(n_out):
            for e in range(int(L.row_ptr[i]), int(L.row_ptr[i + 1])):
                csr[(i, int(L.col_idx[e]))] = int(L.values[e])
    # VSR blocks: whole main-column sub-vectors, every element replaced
    n_sub = -(-len(main) // d)
    if getattr(L, "vsr_pos", None) is not None:
        for i in range(n_out):
            for b in range(int(L.vsr_row_ptr[i]), int(L.vsr_row_ptr[i + 1])):
                s = int(L.vsr_pos[b])
                for t in range(d):
                    if s * d + t < len(main):
                        j = main[s * d + t]
                        assert (i, j) not in csr
                        csr[(i, j)] = int(L.vsr_values[b, t])
    groups = max(1, int(getattr(L, "n_groups", 1) or 1))
    gsize = -(-n_sub // groups) if n_sub else 1
    sym = int(getattr(L, "cb_symmetry", 0) or 0)

    def main_value(g, i1, t):
        """Element t of entry i1 of group g's main codebook (symmetric: base entry times a sign pattern)."""
        if not sym:
            return int(L.codebook1[g * L.k1 + i1, t])
        k1s = L.k1 // 4
        pattern, base = divmod(i1, k1s)
        v = int(L.codebook1[g * k1s + base, t])
        negate = pattern == 1 or (pattern == 2 and t % 2 == 1) or (pattern == 3 and t % 2 == 0)
        return v ^ 0x8000 if negate else v

    W = [[None] * n_in for _ in range(n_out)]
    B = [[0] * n_in for _ in range(n_out)]
    for i in range(n_out):
        row = L.codes[i].tobytes()
        row_o = L.codes_o[i].tobytes() if L.n_ocols else b""
        for j in range(n_in):
            if (i, j) in csr:
                v = csr[(i, j)]
                W[i][j] = f16_frac(v)
                B[i][j] = v
                continue
            if j in out_rank:
                p = out_rank[j]
                io = field(row_o, p // d, L.bits_o)
                assert io < L.ko
                terms = [int(L.codebook_o[io, p % d])]
            else:
                q = main_rank[j]
                f = field(row, q // d, w)
                i1, i2 = f & ((1 << L.bits1) - 1), f >> L.bits1
                assert i1 < L.k1
                g = (q // d) // gsize
                terms = [main_value(g, i1, q % d)]
                if L.k2:
                    assert i2 < L.k2
                    terms.append(int(L.codebook2[g * L.k2 + i2, q % d]))
            val = sum((f16_frac(t) for t in terms), Fraction(0))
            fl = np.float64(f16_float(terms[0]))
            for t in terms[1:]:
                fl = fl + np.float64(f16_float(t))
            for sc in ((L.row_scale[i] if L.row_scale is not None else None),
                       (L.col_scale[j] if L.col_scale is not None else None)):
                if sc is not None:
                    val *= f16_frac(int(sc))
                    fl = fl * np.float64(f16_float(int(sc)))
            W[i][j] = val
            B[i][j] = rne_f16(val, negative_zero=bool(np.signbit(fl)))
    return W, B


def exact_matvec(W, x_rows):
    """y[m][i] = sum_j W[i][j] * x[m][j] exactly (x as floats, converted exactly)."""
    out = []
    for x in x_rows:
        xf = [Fraction(float(v)) for v in x]
        out.append([sum((wij * xj for wij, xj in zip(Wi, xf)), Fraction(0)) for Wi in W])
    return out
