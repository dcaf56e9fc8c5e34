"""Helpers for the GPU parity tests (tolerance, tensor conversion, cached workloads)."""
import functools

import numpy as np

from sparse_compensated_vq_b200 import synth

# max|y - y_ref| <= REL * rms(y_ref) + ABS for fp32 outputs accumulated in fp32;
# an fp16/bf16 output adds one ulp of |y_ref| in that dtype (its own rounding).
REL, ABS = 2e-3, 1e-4


def ulp(y_ref: np.ndarray, dtype: str) -> np.ndarray:
    a = np.abs(y_ref)
    if dtype == "f32":
        return np.zeros_like(a)
    mant = 10 if dtype == "f16" else 7
    e = np.floor(np.log2(np.maximum(a, 1e-30)))
    e = np.maximum(e, -14 if dtype == "f16" else -126)
    return np.ldexp(1.0, (e - mant).astype(np.int64))


def assert_close(y: np.ndarray, y_ref: np.ndarray, out_dtype: str = "f32", what: str = ""):
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.isfinite(y).all(), what + ": non-finite output"
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    bound = REL * rms + ABS + ulp(y_ref, out_dtype)
    err = np.abs(y - y_ref)
    worst = int(np.argmax(err - bound)) if err.size else 0
    assert (err <= bound).all(), "%s: max excess at %d: |%g - %g| = %g > %g (rms %g)" % (
        what, worst, y.flat[worst], y_ref.flat[worst], err.flat[worst], bound.flat[worst], rms)


def torch_x(bits: np.ndarray, dtype: str):
    import torch
    if dtype == "f16":
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.float16))
    elif dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.float32))
    return t.cuda()


def torch_dtype(dtype: str):
    import torch
    return {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dtype]


def to_f64(t) -> np.ndarray:
    import torch
    return t.to(torch.float64).cpu().numpy()


@functools.lru_cache(maxsize=None)
def workload(name: str):
    if name == "tiny":
        return synth.tiny()
    if name == "qproj":
        return synth.qproj(16)
    if name == "downproj":
        return synth.downproj(16)
    if name == "smollm":
        return synth.smollm(8)
    if name == "prefill":
        return synth.prefill(2048)
    if name.startswith("vlen"):
        return synth.vlen(int(name[4:]), 16)
    raise KeyError(name)
