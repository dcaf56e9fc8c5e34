"""Seeded synthetic layers and activations.

Inputs only: random draws, their conversion to fp16/bf16 bit patterns, and
the serialisation of index fields into the packed byte format of the layer
description (fields of w bits, least significant bit first, per row).  Nothing
here dequantises or multiplies; both the CUDA path and the CPU oracle take
their inputs from here.

Workloads (shapes and distributions of the VQ-for-LLM pages: LLaMA-2-7B and
SmolLM2-1.7B layers at 2-4 bits per weight; seeds PCG64(20260000 + n)):

  0 tiny      256x256, d=4, K=256 u8 codes, row scales, 1% uniform outliers
  1 qproj     4096x4096, d=8, K=65536 u16 codes (2 bits/weight), row+col scales,
              1% uniform outliers
  2 downproj  4096x11008, d=8, residual VQ 12+12 bits (K=4096 each), 110 outlier
              columns with a K=256 u8 codebook, row scales, 0.5% uniform outliers
  3 smollm    the seven linears of a SmolLM2-1.7B decoder layer, d=8, K=256,
              2% outliers placed with column probability ~ |z|^4, z ~ N(0,1)
  4 prefill   X 2048x4096 bf16 times the qproj-shaped weight
  5 vlen      4096x4096 at vector length d in {4, 6, 8, 12} with a K=4096 fp16 codebook
              (12-bit codes: 3, 2, 1.5, 1 bits/weight), row+col scales, 1% uniform
              outliers: VPTQ's vector-length trend (one seed per d)
  7 qproj_sym the qproj shape with a symmetric codebook: 16384 stored entries addressed as
              65536 (SCVQ's quarter-size codebook)
  8 smollm_vsr the seven SmolLM2-1.7B linears with their 2% salient weights stored as whole
              sub-vectors (VSR blocks, 2% of the sub-vectors, position probability ~ |z|^4)
              instead of scattered CSR entries
  9 qproj_groups the qproj shape with its 512 positions split into 4 groups of 65536-entry
              codebooks (VPTQ's group_num)
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

SEED_BASE = 20260000


# ---------------------------------------------------------------------------
# bit patterns
# ---------------------------------------------------------------------------
def f16_bits(a) -> np.ndarray:
    """numpy float -> IEEE fp16 bit patterns (numpy's round-to-nearest-even cast)."""
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def bf16_bits(a) -> np.ndarray:
    """float32 values -> bfloat16 bit patterns, round to nearest even (finite inputs)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bits_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """fp16/bf16/f32 storage -> float64 (exact widening)."""
    if dtype == "f16":
        return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.asarray(bits, dtype=np.float32).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# packed index format
# ---------------------------------------------------------------------------
def packed_row_bytes(n_fields: int, w: int) -> int:
    return (n_fields * w + 7) // 8


def pack_fields(fields: np.ndarray, w: int, stride: Optional[int] = None) -> np.ndarray:
    """Serialise uint32 fields [n_rows, n_fields] of width w into [n_rows, stride] bytes.

    Field s of a row occupies bits [s*w, s*w+w) of the row's byte string, least
    significant bit first; bytes past the last field are zero.
    """
    fields = np.ascontiguousarray(fields, dtype=np.uint32)
    n_rows, n_fields = fields.shape
    need = packed_row_bytes(n_fields, w)
    stride = need if stride is None else stride
    assert stride >= need
    out = np.zeros((n_rows, stride), dtype=np.uint8)
    step = max(1, (1 << 24) // max(1, n_fields * w))
    shifts = np.arange(w, dtype=np.uint32)
    for r0 in range(0, n_rows, step):
        f = fields[r0:r0 + step]
        bits = ((f[:, :, None] >> shifts) & 1).astype(np.uint8).reshape(f.shape[0], n_fields * w)
        packed = np.packbits(bits, axis=1, bitorder="little")
        out[r0:r0 + step, :packed.shape[1]] = packed
    return out


# ---------------------------------------------------------------------------
# layer description (numpy, host)
# ---------------------------------------------------------------------------
@dataclass
class LayerData:
    n_out: int
    n_in: int
    d: int
    k1: int
    bits1: int
    codes: np.ndarray                    # uint8 [n_out, stride]
    codebook1: np.ndarray                # uint16 fp16 [k1, d]
    k2: int = 0
    bits2: int = 0
    codebook2: Optional[np.ndarray] = None
    row_scale: Optional[np.ndarray] = None
    col_scale: Optional[np.ndarray] = None
    ocols: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int32))
    ko: int = 0
    bits_o: int = 0
    codebook_o: Optional[np.ndarray] = None
    codes_o: Optional[np.ndarray] = None
    row_ptr: Optional[np.ndarray] = None  # int32 [n_out+1]
    col_idx: Optional[np.ndarray] = None  # int32 [nnz]
    values: Optional[np.ndarray] = None   # uint16 fp16 [nnz]
    # VSR blocks: whole main-column sub-vectors replaced (block-row format)
    vsr_row_ptr: Optional[np.ndarray] = None  # int32 [n_out+1]
    vsr_pos: Optional[np.ndarray] = None      # int32 [nblocks]
    vsr_values: Optional[np.ndarray] = None   # uint16 fp16 [nblocks, d]
    n_groups: int = 1                         # codebook groups over the sub-vector positions
    cb_symmetry: int = 0                      # 1: codebook1 stores k1/4 base entries (sign patterns)
    name: str = ""
    # the decoded fields the generator drew (for tests of the packer only)
    fields: Optional[np.ndarray] = None
    fields_o: Optional[np.ndarray] = None

    @property
    def n_ocols(self) -> int:
        return int(self.ocols.size)

    @property
    def n_sub(self) -> int:
        return -(-(self.n_in - self.n_ocols) // self.d)

    @property
    def n_sub_o(self) -> int:
        return -(-self.n_ocols // self.d)

    @property
    def nnz(self) -> int:
        return 0 if self.col_idx is None else int(self.col_idx.size)

    @property
    def vsr_nblocks(self) -> int:
        return 0 if self.vsr_pos is None else int(self.vsr_pos.size)

    def abi_bytes(self) -> dict:
        """Bytes of the stored layer in the description's own format (rows unpadded)."""
        w = self.bits1 + self.bits2
        idx = self.n_out * packed_row_bytes(self.n_sub, w)
        if self.n_ocols:
            idx += self.n_out * packed_row_bytes(self.n_sub_o, self.bits_o)
        g = max(1, self.n_groups)
        k1s = self.k1 // 4 if self.cb_symmetry else self.k1
        cb = 2 * self.d * (g * (k1s + self.k2) + (self.ko if self.n_ocols else 0))
        sc = (2 * self.n_out if self.row_scale is not None else 0) + (2 * self.n_in if self.col_scale is not None else 0)
        sp = self.nnz * 6 + (4 * (self.n_out + 1) if self.nnz else 0)
        vs = self.vsr_nblocks * (4 + 2 * self.d) + (4 * (self.n_out + 1) if self.vsr_nblocks else 0)
        oc = 4 * self.n_ocols
        return {"index": idx, "codebook": cb, "scale": sc, "sparse": sp, "vsr": vs, "ocols": oc,
                "total": idx + cb + sc + sp + vs + oc}


def csr_from_positions(n_out: int, rows: np.ndarray, cols: np.ndarray, vals: np.ndarray):
    order = np.lexsort((cols, rows))
    rows, cols, vals = rows[order], cols[order], vals[order]
    row_ptr = np.zeros(n_out + 1, dtype=np.int64)
    np.cumsum(np.bincount(rows, minlength=n_out), out=row_ptr[1:])
    return row_ptr.astype(np.int32), cols.astype(np.int32), vals


def uniform_positions(rng, n_out: int, n_in: int, nnz: int):
    lin = rng.choice(n_out * n_in, size=nnz, replace=False)
    return (lin // n_in).astype(np.int64), (lin % n_in).astype(np.int64)


def hessian_positions(rng, n_out: int, n_in: int, nnz: int):
    """Column j receives outliers with probability ~ |z_j|^4 (z ~ N(0,1)); columns
    that would exceed n_out entries are capped and the excess redrawn among the
    others; rows within a column are uniform without replacement."""
    z = rng.standard_normal(n_in)
    p = np.abs(z) ** 4
    p /= p.sum()
    counts = rng.multinomial(nnz, p)
    for _ in range(100):
        over = counts > n_out
        if not over.any():
            break
        excess = int((counts[over] - n_out).sum())
        counts[over] = n_out
        free = counts < n_out
        q = np.where(free, p, 0.0)
        q /= q.sum()
        counts += rng.multinomial(excess, q)
    rows, cols = [], []
    for j in np.nonzero(counts)[0]:
        r = rng.choice(n_out, size=int(counts[j]), replace=False)
        rows.append(r)
        cols.append(np.full(r.size, j))
    return np.concatenate(rows).astype(np.int64), np.concatenate(cols).astype(np.int64)


def vsr_positions(rng, n_out: int, n_sub: int, nblocks: int, positions: str = "uniform"):
    """(row, sub-vector) pairs of whole-sub-vector blocks: uniform over the grid, or with the
    sub-vector position drawn with probability ~ |z_s|^4 (z ~ N(0,1)) and the rows uniform
    without replacement within a position (salient input features, as for the Hessian-style
    element outliers)."""
    if positions == "uniform":
        lin = rng.choice(n_out * n_sub, size=nblocks, replace=False)
        return (lin // n_sub).astype(np.int64), (lin % n_sub).astype(np.int64)
    return hessian_positions(rng, n_out, n_sub, nblocks)


def random_layer(rng, n_out, n_in, d, k1, bits1, *, k2=0, bits2=0, cb_std=0.02, res_std=0.005,
                 row_scale=True, col_scale=False, n_ocols=0, ko=256, bits_o=8,
                 outlier_frac=0.01, outlier_scale=0.1, positions="uniform", nnz=None,
                 stride=None, name="", n_groups=1, cb_symmetry=0, vsr_frac=0.0, vsr_blocks=None,
                 vsr_positions_kind="uniform") -> LayerData:
    """One layer with the given shape; every draw comes from `rng` in a fixed order.

    n_groups > 1 or cb_symmetry = 1 change the codebook draws (n_groups codebooks back to back;
    k1/4 base entries each); VSR blocks (vsr_frac of the main sub-vectors, or vsr_blocks of them)
    are drawn after everything else, and CSR entries that fall inside a block are dropped."""
    g = max(1, n_groups)
    k1s = k1 // 4 if cb_symmetry else k1
    assert not cb_symmetry or k1 % 4 == 0
    cb1 = f16_bits(rng.normal(0.0, cb_std, size=(g * k1s, d)))
    cb2 = f16_bits(rng.normal(0.0, res_std, size=(g * k2, d))) if k2 else None
    ocols = np.sort(rng.choice(n_in, size=n_ocols, replace=False)).astype(np.int32) if n_ocols else np.zeros(0, np.int32)
    n_sub = -(-(n_in - n_ocols) // d)
    i1 = rng.integers(0, k1, size=(n_out, n_sub), dtype=np.int64)
    fields = i1.astype(np.uint32)
    if k2:
        i2 = rng.integers(0, k2, size=(n_out, n_sub), dtype=np.int64)
        fields = (i1 | (i2 << bits1)).astype(np.uint32)
    codes = pack_fields(fields, bits1 + bits2, stride)
    cbo = codes_o = fields_o = None
    if n_ocols:
        cbo = f16_bits(rng.normal(0.0, cb_std, size=(ko, d)))
        n_sub_o = -(-n_ocols // d)
        fields_o = rng.integers(0, ko, size=(n_out, n_sub_o), dtype=np.int64).astype(np.uint32)
        codes_o = pack_fields(fields_o, bits_o)
    rs = f16_bits(rng.uniform(0.5, 1.5, size=n_out)) if row_scale else None
    cs = f16_bits(rng.uniform(0.5, 1.5, size=n_in)) if col_scale else None
    if nnz is None:
        nnz = int(round(outlier_frac * n_out * n_in))
    if nnz:
        if positions == "uniform":
            rows, cols = uniform_positions(rng, n_out, n_in, nnz)
        else:
            rows, cols = hessian_positions(rng, n_out, n_in, nnz)
        vals = f16_bits(rng.standard_t(3, size=nnz) * outlier_scale)
        row_ptr, col_idx, values = csr_from_positions(n_out, rows, cols, vals)
    else:
        row_ptr = col_idx = values = None
    vsr_rp = vsr_pos = vsr_vals = None
    nb = vsr_blocks if vsr_blocks is not None else int(round(vsr_frac * n_out * n_sub))
    if nb:
        vr, vs = vsr_positions(rng, n_out, n_sub, nb, vsr_positions_kind)
        vv = f16_bits(rng.standard_t(3, size=(nb, d)) * outlier_scale)
        order = np.lexsort((vs, vr))
        vr, vs, vv = vr[order], vs[order], vv[order]
        vsr_rp = np.zeros(n_out + 1, dtype=np.int64)
        np.cumsum(np.bincount(vr, minlength=n_out), out=vsr_rp[1:])
        vsr_rp, vsr_pos, vsr_vals = vsr_rp.astype(np.int32), vs.astype(np.int32), vv
        if row_ptr is not None:
            # keep the element CSR disjoint from the blocks (main columns only carry blocks)
            is_out = np.zeros(n_in, bool)
            is_out[ocols] = True
            qrank = np.cumsum(~is_out) - 1
            blocked = set(zip(vr.tolist(), vs.tolist()))
            rows_e = np.repeat(np.arange(n_out), np.diff(row_ptr))
            keep = np.array([is_out[j] or (int(i), int(qrank[j]) // d) not in blocked
                             for i, j in zip(rows_e, col_idx)], dtype=bool)
            row_ptr, col_idx, values = csr_from_positions(n_out, rows_e[keep], col_idx[keep].astype(np.int64),
                                                          values[keep])
    return LayerData(n_out=n_out, n_in=n_in, d=d, k1=k1, bits1=bits1, codes=codes, codebook1=cb1,
                     k2=k2, bits2=bits2, codebook2=cb2, row_scale=rs, col_scale=cs, ocols=ocols,
                     ko=ko if n_ocols else 0, bits_o=bits_o if n_ocols else 0, codebook_o=cbo,
                     codes_o=codes_o, row_ptr=row_ptr, col_idx=col_idx, values=values, name=name,
                     fields=fields, fields_o=fields_o, vsr_row_ptr=vsr_rp, vsr_pos=vsr_pos, vsr_values=vsr_vals,
                     n_groups=g, cb_symmetry=cb_symmetry)


def activations(rng, batch: int, n_in: int, dtype: str = "f16") -> np.ndarray:
    """x ~ N(0,1) as fp16/bf16 bit patterns or float32 [batch, n_in]."""
    x = rng.standard_normal((batch, n_in)).astype(np.float32)
    if dtype == "f16":
        return f16_bits(x)
    if dtype == "bf16":
        return bf16_bits(x)
    return x


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------
def rng_for(config_no: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(SEED_BASE + config_no))


def tiny():
    rng = rng_for(0)
    L = random_layer(rng, 256, 256, 4, 256, 8, cb_std=0.02, row_scale=True, col_scale=False,
                     outlier_frac=0.01, outlier_scale=0.2, name="tiny_256x256_d4_k256")
    return L, activations(rng, 1, 256, "f16")


def qproj(batch: int = 1):
    rng = rng_for(1)
    L = random_layer(rng, 4096, 4096, 8, 65536, 16, cb_std=0.02, row_scale=True, col_scale=True,
                     outlier_frac=0.01, outlier_scale=0.1, name="llama2_7b_qproj_4096x4096_d8_k65536")
    return L, activations(rng, batch, 4096, "f16")


def downproj(batch: int = 1):
    rng = rng_for(2)
    L = random_layer(rng, 4096, 11008, 8, 4096, 12, k2=4096, bits2=12, cb_std=0.02, res_std=0.005,
                     row_scale=True, col_scale=False, n_ocols=110, ko=256, bits_o=8,
                     outlier_frac=0.005, outlier_scale=0.1, name="llama2_7b_downproj_4096x11008_rvq12x12_ocol110")
    return L, activations(rng, batch, 11008, "f16")


SMOLLM_SHAPES = [("q_proj", 2048, 2048), ("k_proj", 2048, 2048), ("v_proj", 2048, 2048),
                 ("o_proj", 2048, 2048), ("gate_proj", 8192, 2048), ("up_proj", 8192, 2048),
                 ("down_proj", 2048, 8192)]


def smollm(batch: int = 1):
    rng = rng_for(3)
    layers, xs = [], []
    for name, n_out, n_in in SMOLLM_SHAPES:
        L = random_layer(rng, n_out, n_in, 8, 256, 8, cb_std=0.02, row_scale=True, col_scale=False,
                         outlier_frac=0.02, outlier_scale=0.1, positions="hessian",
                         name="smollm2_1.7b_" + name)
        layers.append(L)
    for name, n_out, n_in in SMOLLM_SHAPES:
        xs.append(activations(rng, batch, n_in, "bf16"))
    return layers, xs


def prefill(m: int = 2048):
    rng = rng_for(4)
    L = random_layer(rng, 4096, 4096, 8, 65536, 16, cb_std=0.02, row_scale=True, col_scale=True,
                     outlier_frac=0.01, outlier_scale=0.1, name="prefill_qproj_4096x4096_d8_k65536")
    return L, activations(rng, m, 4096, "bf16")


def vlen(d: int, batch: int = 1):
    rng = rng_for(5 * 100 + d)
    L = random_layer(rng, 4096, 4096, d, 4096, 12, cb_std=0.02, row_scale=True, col_scale=True,
                     outlier_frac=0.01, outlier_scale=0.1, name="vlen_4096x4096_d%d_k4096" % d)
    return L, activations(rng, batch, 4096, "f16")


def qproj_sym(batch: int = 1):
    rng = rng_for(7)
    L = random_layer(rng, 4096, 4096, 8, 65536, 16, cb_std=0.02, row_scale=True, col_scale=True,
                     outlier_frac=0.01, outlier_scale=0.1, cb_symmetry=1,
                     name="llama2_7b_qproj_4096x4096_d8_k65536_symmetric")
    return L, activations(rng, batch, 4096, "f16")


def smollm_vsr(batch: int = 1):
    rng = rng_for(8)
    layers, xs = [], []
    for name, n_out, n_in in SMOLLM_SHAPES:
        L = random_layer(rng, n_out, n_in, 8, 256, 8, cb_std=0.02, row_scale=True, col_scale=False,
                         nnz=0, outlier_scale=0.1, vsr_frac=0.02, vsr_positions_kind="hessian",
                         name="smollm2_1.7b_" + name + "_vsr")
        layers.append(L)
    for name, n_out, n_in in SMOLLM_SHAPES:
        xs.append(activations(rng, batch, n_in, "bf16"))
    return layers, xs


def qproj_groups(batch: int = 1, groups: int = 4):
    rng = rng_for(9)
    L = random_layer(rng, 4096, 4096, 8, 65536, 16, cb_std=0.02, row_scale=True, col_scale=True,
                     outlier_frac=0.01, outlier_scale=0.1, n_groups=groups,
                     name="llama2_7b_qproj_4096x4096_d8_k65536_groups%d" % groups)
    return L, activations(rng, batch, 4096, "f16")
