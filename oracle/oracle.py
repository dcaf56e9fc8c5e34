"""ctypes front end of oracle.c (test infrastructure only).

The layer argument is any object with the attributes of a layer description
(n_out, n_in, d, k1, bits1, k2, bits2, codes, codebook1, codebook2,
row_scale, col_scale, ocols, ko, bits_o, codebook_o, codes_o, row_ptr,
col_idx, values) holding numpy arrays; fp16 data is passed as uint16 bit
patterns.  Every numeric step runs in oracle.c; this file only marshals.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_ERRORS = {1: "index out of range", 2: "non-finite value", 3: "malformed CSR", 4: "out of memory"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, no fused multiply-add)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=gnu99", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(C.Structure):
    _fields_ = [
        ("n_out", C.c_int32), ("n_in", C.c_int32), ("d", C.c_int32),
        ("k1", C.c_int32), ("bits1", C.c_int32), ("k2", C.c_int32), ("bits2", C.c_int32),
        ("codes", C.c_void_p), ("stride", C.c_int64),
        ("cb1", C.c_void_p), ("cb2", C.c_void_p),
        ("rs", C.c_void_p), ("cs", C.c_void_p),
        ("n_ocols", C.c_int32), ("ocols", C.c_void_p),
        ("ko", C.c_int32), ("bits_o", C.c_int32), ("cbo", C.c_void_p), ("codes_o", C.c_void_p),
        ("stride_o", C.c_int64),
        ("nnz", C.c_int64), ("row_ptr", C.c_void_p), ("col_idx", C.c_void_p), ("values", C.c_void_p),
        ("vsr_nb", C.c_int64), ("vsr_row_ptr", C.c_void_p), ("vsr_pos", C.c_void_p), ("vsr_values", C.c_void_p),
        ("n_groups", C.c_int32), ("cb_symmetry", C.c_int32),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # VQ_ORACLE_LIB points the pins at another build of oracle.c (the
            # mutation test plants mistakes in a copy to show the pins catch them)
            lib = C.CDLL(os.environ.get("VQ_ORACLE_LIB") or build())
            P = C.c_void_p
            lib.oracle_f16_to_f64.restype = C.c_double
            lib.oracle_f16_to_f64.argtypes = [C.c_uint16]
            lib.oracle_bf16_to_f64.restype = C.c_double
            lib.oracle_bf16_to_f64.argtypes = [C.c_uint16]
            lib.oracle_round_f16_parts.restype = C.c_uint16
            lib.oracle_round_f16_parts.argtypes = [C.c_int, C.c_uint64, C.c_uint64, C.c_int]
            lib.oracle_body_f16.restype = C.c_int
            lib.oracle_body_f16.argtypes = [C.c_uint16, P, P, P, P]
            lib.oracle_unpack.restype = None
            lib.oracle_unpack.argtypes = [P, C.c_int64, C.c_int32, C.c_int32, C.c_int, P]
            lib.oracle_dequant_exact.restype = C.c_int
            lib.oracle_dequant_exact.argtypes = [C.POINTER(_Layer), P, C.c_int64]
            lib.oracle_dequant_f64_rows.restype = C.c_int
            lib.oracle_dequant_f64_rows.argtypes = [C.POINTER(_Layer), P, C.c_int32, P]
            lib.oracle_gemv_f64_rows.restype = C.c_int
            lib.oracle_gemv_f64_rows.argtypes = [C.POINTER(_Layer), P, C.c_int32, P, C.c_int64, P]
            lib.oracle_vptq_compression_ratio.restype = C.c_double
            lib.oracle_vptq_compression_ratio.argtypes = [C.c_int64, C.c_int32, C.c_int64]
            lib.oracle_assign_exact.restype = C.c_int
            lib.oracle_assign_exact.argtypes = [P, C.c_int64, C.c_int32, P, C.c_int32, P, C.c_int32, P, P]
            lib.oracle_residual_assign_exact.restype = C.c_int
            lib.oracle_residual_assign_exact.argtypes = [P, C.c_int64, C.c_int32, P, C.c_int32, P, P, C.c_int32, P]
            lib.oracle_sqdist_exact.restype = C.c_int
            lib.oracle_sqdist_exact.argtypes = [P, P, P, C.c_int32, C.POINTER(C.c_uint64), C.POINTER(C.c_uint64)]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dtype)


def _marshal(layer):
    """Build the C struct; returns (struct, keep-alive list)."""
    keep = []

    def arr(name, dtype):
        a = getattr(layer, name, None)
        a = _c(a, dtype)
        keep.append(a)
        return a

    codes = arr("codes", np.uint8)
    cb1 = arr("codebook1", np.uint16)
    cb2 = arr("codebook2", np.uint16)
    rs = arr("row_scale", np.uint16)
    cs = arr("col_scale", np.uint16)
    ocols = arr("ocols", np.int32)
    cbo = arr("codebook_o", np.uint16)
    codes_o = arr("codes_o", np.uint8)
    row_ptr = arr("row_ptr", np.int32)
    col_idx = arr("col_idx", np.int32)
    values = arr("values", np.uint16)
    vsr_row_ptr = arr("vsr_row_ptr", np.int32)
    vsr_pos = arr("vsr_pos", np.int32)
    vsr_values = arr("vsr_values", np.uint16)
    n_ocols = 0 if ocols is None else int(ocols.size)
    nnz = 0 if col_idx is None else int(col_idx.size)
    nvsr = 0 if vsr_pos is None else int(vsr_pos.size)
    L = _Layer(
        n_out=layer.n_out, n_in=layer.n_in, d=layer.d,
        k1=layer.k1, bits1=layer.bits1, k2=getattr(layer, "k2", 0) or 0, bits2=getattr(layer, "bits2", 0) or 0,
        codes=_ptr(codes), stride=codes.shape[1] if codes.ndim == 2 else codes.size // layer.n_out,
        cb1=_ptr(cb1), cb2=_ptr(cb2), rs=_ptr(rs), cs=_ptr(cs),
        n_ocols=n_ocols, ocols=_ptr(ocols),
        ko=getattr(layer, "ko", 0) or 0, bits_o=getattr(layer, "bits_o", 0) or 0,
        cbo=_ptr(cbo), codes_o=_ptr(codes_o),
        stride_o=0 if codes_o is None else (codes_o.shape[1] if codes_o.ndim == 2 else codes_o.size // layer.n_out),
        nnz=nnz, row_ptr=_ptr(row_ptr) if nnz else None, col_idx=_ptr(col_idx) if nnz else None,
        values=_ptr(values) if nnz else None,
        vsr_nb=nvsr, vsr_row_ptr=_ptr(vsr_row_ptr) if nvsr else None, vsr_pos=_ptr(vsr_pos) if nvsr else None,
        vsr_values=_ptr(vsr_values) if nvsr else None,
        n_groups=int(getattr(layer, "n_groups", 1) or 1), cb_symmetry=int(getattr(layer, "cb_symmetry", 0) or 0),
    )
    return L, keep


def _check(rc):
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, "error %d" % rc))


def f16_to_f64(h: int) -> float:
    return _load().oracle_f16_to_f64(int(h))


def bf16_to_f64(h: int) -> float:
    return _load().oracle_bf16_to_f64(int(h))


def round_f16(sign: int, mant: int, exp2: int) -> int:
    """fp16 bits of (-1)^sign * mant * 2^exp2 rounded to nearest, ties to even."""
    assert 0 <= mant < (1 << 128)
    return int(_load().oracle_round_f16_parts(int(sign), mant >> 64, mant & ((1 << 64) - 1), int(exp2)))


def body_f16(c1: int, c2: int | None = None, r: int | None = None, c: int | None = None) -> int:
    """fp16 bits of r*c*(c1 + c2) rounded once from the exact value (absent terms omitted)."""
    lib = _load()
    boxes = [None if v is None else C.c_uint16(v) for v in (c2, r, c)]
    out = C.c_uint16(0)
    ptrs = [None if b is None else C.addressof(b) for b in boxes]
    _check(lib.oracle_body_f16(int(c1), ptrs[0], ptrs[1], ptrs[2], C.addressof(out)))
    return int(out.value)


def unpack(codes: np.ndarray, n_fields: int, w: int) -> np.ndarray:
    """Fields of width w of every row of a [n_rows, stride] byte matrix -> uint32 [n_rows, n_fields]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n_rows, stride = codes.shape
    out = np.zeros((n_rows, n_fields), dtype=np.uint32)
    _load().oracle_unpack(_ptr(codes), stride, n_rows, n_fields, int(w), _ptr(out))
    return out


def dequant_exact(layer) -> np.ndarray:
    """fp16 bit patterns [n_out, n_in] of the dequantised weight (bit-exact definition)."""
    L, keep = _marshal(layer)
    W = np.zeros((layer.n_out, layer.n_in), dtype=np.uint16)
    _check(_load().oracle_dequant_exact(C.byref(L), _ptr(W), layer.n_in))
    return W


def _rows(layer, rows):
    if rows is None:
        return np.arange(layer.n_out, dtype=np.int32)
    return np.ascontiguousarray(rows, dtype=np.int32)


def dequant_f64(layer, rows=None) -> np.ndarray:
    """Double-precision weights of the given rows (all rows by default) -> [n_rows, n_in]."""
    L, keep = _marshal(layer)
    r = _rows(layer, rows)
    W = np.zeros((r.size, layer.n_in), dtype=np.float64)
    _check(_load().oracle_dequant_f64_rows(C.byref(L), _ptr(r), r.size, _ptr(W)))
    return W


def gemv_f64(layer, x: np.ndarray, rows=None) -> np.ndarray:
    """y[m, t] = sum_j W[rows[t], j] * x[m, j] in double; x is float64 [m, n_in]."""
    L, keep = _marshal(layer)
    r = _rows(layer, rows)
    x = np.ascontiguousarray(np.atleast_2d(x), dtype=np.float64)
    assert x.shape[1] == layer.n_in
    Y = np.zeros((x.shape[0], r.size), dtype=np.float64)
    _check(_load().oracle_gemv_f64_rows(C.byref(L), _ptr(r), r.size, _ptr(x), x.shape[0], _ptr(Y)))
    return Y


def vptq_compression_ratio(n_elems: int, V: int, k: int) -> float:
    return float(_load().oracle_vptq_compression_ratio(int(n_elems), int(V), int(k)))


def assign_exact(V: np.ndarray, C1: np.ndarray, C2: np.ndarray | None = None):
    """Exact nearest-centroid indices of fp16 sub-vectors V [n, d] (uint16 bits) in C1 [k1, d]
    and, with a residual codebook C2 [k2, d], of v - C1[i1] in C2 (oracle.c:
    oracle_assign_exact; ties keep the lowest index).  Returns (idx1, idx2) as uint32 arrays;
    idx2 is None without C2."""
    lib = _load()
    V = _c(V, np.uint16)
    C1 = _c(C1, np.uint16)
    n, d = V.shape
    k1 = C1.shape[0]
    assert C1.shape[1] == d
    i1 = np.zeros(n, np.uint32)
    i2 = None
    k2 = 0
    c2p = None
    if C2 is not None:
        C2 = _c(C2, np.uint16)
        assert C2.shape[1] == d
        k2 = C2.shape[0]
        i2 = np.zeros(n, np.uint32)
        c2p = _ptr(C2)
    _check(lib.oracle_assign_exact(_ptr(V), C.c_int64(n), C.c_int32(d), _ptr(C1), C.c_int32(k1), c2p, C.c_int32(k2),
                                   _ptr(i1), _ptr(i2) if i2 is not None else None))
    return i1, i2


def residual_assign_exact(V: np.ndarray, C1: np.ndarray, idx1: np.ndarray, C2: np.ndarray) -> np.ndarray:
    """Exact residual-stage indices for a given first-stage choice: argmin_j ||(V[s] -
    C1[idx1[s]]) - C2_j||^2 (oracle.c: oracle_residual_assign_exact)."""
    lib = _load()
    V = _c(V, np.uint16)
    C1 = _c(C1, np.uint16)
    C2 = _c(C2, np.uint16)
    idx1 = _c(idx1, np.uint32)
    n, d = V.shape
    i2 = np.zeros(n, np.uint32)
    _check(lib.oracle_residual_assign_exact(_ptr(V), C.c_int64(n), C.c_int32(d), _ptr(C1), C.c_int32(C1.shape[0]),
                                            _ptr(idx1), _ptr(C2), C.c_int32(C2.shape[0]), _ptr(i2)))
    return i2


def sqdist_exact(v: np.ndarray, c: np.ndarray, base: np.ndarray | None = None) -> int:
    """Exact ||v - base - c||^2 of fp16 vectors (uint16 bits, base optional) as an integer count
    of 2^-48 (oracle.c: oracle_sqdist_exact)."""
    lib = _load()
    v = _c(v, np.uint16)
    c = _c(c, np.uint16)
    b = _c(base, np.uint16)
    hi, lo = C.c_uint64(0), C.c_uint64(0)
    _check(lib.oracle_sqdist_exact(_ptr(v), _ptr(b), _ptr(c), C.c_int32(v.size), C.byref(hi), C.byref(lo)))
    return (int(hi.value) << 64) | int(lo.value)
