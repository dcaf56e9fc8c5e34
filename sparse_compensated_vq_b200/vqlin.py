"""ctypes binding of libvqlin.so (include/vqlin.h).

Argument marshalling only: every step of create/dequant/gemv/gemm runs in the
compiled library.  Device memory and streams come from PyTorch.  Importing this
module loads libvqlin.so and raises ImportError if it has not been built
(``python -m sparse_compensated_vq_b200.build``); there is no fallback.

Every function that include/vqlin.h declares is exposed here under its own name
(the list is ``EXPORTS``) with ctypes argument types; these are the C entry points
themselves.  :class:`VQLinear` wraps the layer calls for torch tensors.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvqlin.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libvqlin.so is not built: run `python -m sparse_compensated_vq_b200.build` (no CPU fallback)")

_lib = C.CDLL(LIB_PATH)

VQLIN_OK, VQLIN_ERR_INVALID_ARG, VQLIN_ERR_UNSUPPORTED, VQLIN_ERR_INVALID_DATA, VQLIN_ERR_OOM, \
    VQLIN_ERR_CUDA, VQLIN_ERR_WORKSPACE = range(7)
VQLIN_F32, VQLIN_F16, VQLIN_BF16 = 0, 1, 2
MAX_BATCH = 16


class vqlin_desc(C.Structure):
    _fields_ = [
        ("n_out", C.c_int32), ("n_in", C.c_int32), ("d", C.c_int32), ("src_on_host", C.c_int32),
        ("k1", C.c_int32), ("bits1", C.c_int32), ("k2", C.c_int32), ("bits2", C.c_int32),
        ("codes", C.c_void_p), ("row_stride_bytes", C.c_int64),
        ("codebook1", C.c_void_p), ("codebook2", C.c_void_p),
        ("row_scale", C.c_void_p), ("col_scale", C.c_void_p),
        ("n_ocols", C.c_int32), ("ocols", C.c_void_p),
        ("ko", C.c_int32), ("bits_o", C.c_int32), ("codebook_o", C.c_void_p), ("codes_o", C.c_void_p),
        ("o_row_stride_bytes", C.c_int64),
        ("nnz", C.c_int64), ("row_ptr", C.c_void_p), ("col_idx", C.c_void_p), ("values", C.c_void_p),
        ("vsr_nblocks", C.c_int64), ("vsr_row_ptr", C.c_void_p), ("vsr_pos", C.c_void_p),
        ("vsr_values", C.c_void_p),
        ("n_groups", C.c_int32), ("cb_symmetry", C.c_int32),
    ]


class vqlin_info(C.Structure):
    _fields_ = [
        ("n_out", C.c_int32), ("n_in", C.c_int32), ("d", C.c_int32), ("n_sub", C.c_int32),
        ("n_sub_o", C.c_int32), ("n_ocols", C.c_int32),
        ("nnz", C.c_int64), ("index_bytes", C.c_int64), ("codebook_bytes", C.c_int64),
        ("scale_bytes", C.c_int64), ("sparse_bytes", C.c_int64),
        ("vptq_compression_ratio", C.c_double), ("vptq_bits_per_weight", C.c_double),
        ("total_bits_per_weight", C.c_double), ("vsr_bytes", C.c_int64),
    ]


_P = C.c_void_p
_H = C.c_void_p          # vqlin_handle*
_S = C.c_int             # vqlin_status


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


vqlin_create = _sig("vqlin_create", _S, [C.POINTER(vqlin_desc), _P, C.POINTER(_H)])
vqlin_destroy = _sig("vqlin_destroy", _S, [_H])
vqlin_get_info = _sig("vqlin_get_info", _S, [_H, C.POINTER(vqlin_info)])
vqlin_dequant = _sig("vqlin_dequant", _S, [_H, _P, C.c_int64, _P])
vqlin_gemv = _sig("vqlin_gemv", _S, [_H, _P, C.c_int, C.c_int32, _P, C.c_int, _P])
vqlin_gemv_ws = _sig("vqlin_gemv_ws", _S, [_H, _P, C.c_int, C.c_int32, _P, C.c_int, _P, C.c_size_t, _P])
vqlin_gemv_workspace_size = _sig("vqlin_gemv_workspace_size", C.c_size_t, [_H, C.c_int32])
vqlin_gemv_noalloc = _sig("vqlin_gemv_noalloc", _S, [_H, _P, C.c_int, C.c_int32, _P, C.c_int, _P])
vqlin_gemm = _sig("vqlin_gemm", _S, [_H, _P, C.c_int, C.c_int64, _P, C.c_int, _P, C.c_size_t, _P])
vqlin_gemm_workspace_size = _sig("vqlin_gemm_workspace_size", C.c_size_t, [_H, C.c_int64])
vqlin_unpack_indices = _sig("vqlin_unpack_indices", _S, [_H, C.c_int32, _P, _P])
vqlin_status_string = _sig("vqlin_status_string", C.c_char_p, [_S])
vqlin_last_error = _sig("vqlin_last_error", C.c_char_p, [])
vqlin_abi_version = _sig("vqlin_abi_version", C.c_int32, [])
vqlin_device_error = _sig("vqlin_device_error", _S, [C.POINTER(C.c_int32)])
vqlin_kernel_launches = _sig("vqlin_kernel_launches", C.c_uint64, [])
vqlin_selftest_wait_timeout = _sig("vqlin_selftest_wait_timeout", _S, [C.c_int32, C.c_void_p])
vqlin_assign = _sig("vqlin_assign", _S, [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_int32, C.c_void_p,
                                              C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p])

EXPORTS = ["vqlin_create", "vqlin_destroy", "vqlin_get_info", "vqlin_dequant", "vqlin_gemv", "vqlin_gemm",
           "vqlin_gemm_workspace_size", "vqlin_unpack_indices", "vqlin_status_string", "vqlin_last_error",
           "vqlin_abi_version", "vqlin_device_error", "vqlin_gemv_ws", "vqlin_gemv_workspace_size", "vqlin_gemv_noalloc",
           "vqlin_kernel_launches", "vqlin_selftest_wait_timeout", "vqlin_assign"]


def device_error() -> int:
    """Synchronise and return (and clear) the code of a kernel that gave up a bounded wait."""
    c = C.c_int32(0)
    check(vqlin_device_error(C.byref(c)), "vqlin_device_error")
    return int(c.value)


class VQLinError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        msg = "%s: %s (%s)" % (where, vqlin_status_string(status).decode(), vqlin_last_error().decode())
        super().__init__(msg)


def check(status, where=""):
    if status != VQLIN_OK:
        raise VQLinError(status, where)


_DT = {"f32": VQLIN_F32, "f16": VQLIN_F16, "bf16": VQLIN_BF16}


def dtype_code(t) -> int:
    """torch dtype or 'f32'/'f16'/'bf16' -> vqlin_dtype."""
    if isinstance(t, str):
        return _DT[t]
    import torch
    return {torch.float32: VQLIN_F32, torch.float16: VQLIN_F16, torch.bfloat16: VQLIN_BF16}[t]


def _stream(stream):
    if stream is not None:
        return C.c_void_p(int(stream))
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(a):
    """Pointer of a numpy array or torch tensor (None -> NULL)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def make_desc(layer, keep: list) -> vqlin_desc:
    """vqlin_desc for an object with LayerData's attributes (numpy -> host, torch cuda -> device)."""
    def arr(name, dtype):
        a = getattr(layer, name, None)
        if a is None:
            return None
        if isinstance(a, np.ndarray):
            a = np.ascontiguousarray(a, dtype=dtype)
        keep.append(a)
        return a

    codes = arr("codes", np.uint8)
    on_host = isinstance(codes, np.ndarray)
    ocols = arr("ocols", np.int32)
    n_ocols = 0 if ocols is None else int(ocols.size if on_host else ocols.numel())
    codes_o = arr("codes_o", np.uint8)
    col_idx = arr("col_idx", np.int32)
    nnz = 0 if col_idx is None else int(col_idx.size if on_host else col_idx.numel())
    D = vqlin_desc()
    D.n_out, D.n_in, D.d, D.src_on_host = layer.n_out, layer.n_in, layer.d, 1 if on_host else 0
    D.k1, D.bits1 = layer.k1, layer.bits1
    D.k2, D.bits2 = getattr(layer, "k2", 0) or 0, getattr(layer, "bits2", 0) or 0
    D.codes, D.row_stride_bytes = _ptr(codes), int(codes.shape[1])
    D.codebook1, D.codebook2 = _ptr(arr("codebook1", np.uint16)), _ptr(arr("codebook2", np.uint16))
    D.row_scale, D.col_scale = _ptr(arr("row_scale", np.uint16)), _ptr(arr("col_scale", np.uint16))
    D.n_ocols, D.ocols = n_ocols, _ptr(ocols) if n_ocols else None
    if n_ocols:
        D.ko, D.bits_o = layer.ko, layer.bits_o
        D.codebook_o, D.codes_o = _ptr(arr("codebook_o", np.uint16)), _ptr(codes_o)
        D.o_row_stride_bytes = int(codes_o.shape[1])
    D.nnz = nnz
    if nnz:
        D.row_ptr, D.col_idx, D.values = _ptr(arr("row_ptr", np.int32)), _ptr(col_idx), _ptr(arr("values", np.uint16))
    vsr_pos = arr("vsr_pos", np.int32)
    nb = 0 if vsr_pos is None else int(vsr_pos.size if on_host else vsr_pos.numel())
    D.vsr_nblocks = nb
    if nb:
        D.vsr_row_ptr, D.vsr_pos = _ptr(arr("vsr_row_ptr", np.int32)), _ptr(vsr_pos)
        D.vsr_values = _ptr(arr("vsr_values", np.uint16))
    D.n_groups = int(getattr(layer, "n_groups", 1) or 1)
    D.cb_symmetry = int(getattr(layer, "cb_symmetry", 0) or 0)
    return D


class VQLinear:
    """A created layer.  Tensors passed in must be CUDA tensors on the handle's device."""

    def __init__(self, layer, stream=None):
        keep = []
        D = make_desc(layer, keep)
        h = _H()
        check(vqlin_create(C.byref(D), _stream(stream), C.byref(h)), "vqlin_create")
        self._h = h
        self.n_out, self.n_in, self.d = layer.n_out, layer.n_in, layer.d

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            vqlin_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self) -> dict:
        I = vqlin_info()
        check(vqlin_get_info(self._h, C.byref(I)), "vqlin_get_info")
        return {k: getattr(I, k) for k, _ in vqlin_info._fields_}

    def dequant(self, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty((self.n_out, self.n_in), dtype=torch.float16, device="cuda")
        check(vqlin_dequant(self._h, out.data_ptr(), out.stride(0), _stream(stream)), "vqlin_dequant")
        return out

    def gemv(self, x, out=None, out_dtype=None, stream=None):
        import torch
        x2 = x if x.dim() == 2 else x.view(1, -1)
        assert x2.is_contiguous() and x2.shape[1] == self.n_in
        if out is None:
            out = torch.empty((x2.shape[0], self.n_out), dtype=out_dtype or torch.float32, device=x.device)
        check(vqlin_gemv(self._h, x2.data_ptr(), dtype_code(x2.dtype), x2.shape[0], out.data_ptr(),
                         dtype_code(out.dtype), _stream(stream)), "vqlin_gemv")
        return out

    def gemv_ws(self, x, workspace=None, out=None, out_dtype=None, stream=None):
        import torch
        x2 = x if x.dim() == 2 else x.view(1, -1)
        assert x2.is_contiguous() and x2.shape[1] == self.n_in
        B = x2.shape[0]
        if out is None:
            out = torch.empty((B, self.n_out), dtype=out_dtype or torch.float32, device=x.device)
        if workspace is None:
            workspace = torch.empty(int(vqlin_gemv_workspace_size(self._h, B)), dtype=torch.uint8, device=x.device)
        check(vqlin_gemv_ws(self._h, x2.data_ptr(), dtype_code(x2.dtype), B, out.data_ptr(), dtype_code(out.dtype),
                            workspace.data_ptr(), workspace.numel(), _stream(stream)), "vqlin_gemv_ws")
        return out

    def workspace_size(self, m: int) -> int:
        return int(vqlin_gemm_workspace_size(self._h, m))

    def gemm(self, X, out=None, out_dtype=None, workspace=None, stream=None):
        import torch
        assert X.is_contiguous() and X.dim() == 2 and X.shape[1] == self.n_in
        m = X.shape[0]
        if out is None:
            out = torch.empty((m, self.n_out), dtype=out_dtype or torch.bfloat16, device=X.device)
        if workspace is None:
            workspace = torch.empty(self.workspace_size(m), dtype=torch.uint8, device=X.device)
        check(vqlin_gemm(self._h, X.data_ptr(), dtype_code(X.dtype), m, out.data_ptr(), dtype_code(out.dtype),
                         workspace.data_ptr(), workspace.numel(), _stream(stream)), "vqlin_gemm")
        return out

    def unpack_indices(self, which: int = 0, stream=None):
        import torch
        I = self.info()
        n = I["n_sub_o"] if which else I["n_sub"]
        out = torch.zeros((self.n_out, n), dtype=torch.int32, device="cuda")
        check(vqlin_unpack_indices(self._h, which, out.data_ptr(), _stream(stream)), "vqlin_unpack_indices")
        return out
