#!/usr/bin/env python3
"""Benchmark of the VQ + sparse linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vqlin|reference]
                    [--config qproj|tiny|downproj|smollm|prefill] [--batch B]

Default workload: the LLaMA-2-7B q_proj-shaped layer (4096x4096, d=8,
K=65536 fp16 codebook = 2 bits/weight, row and column scales, 1% CSR outliers),
batch-1 decode GEMV, fp16 x and y.  One step = one pass of the hot path
(one vqlin_gemv call; for `smollm` the seven linears of a decoder layer back to
back; for `prefill` one vqlin_gemm call).

Timing: W untimed eager steps, then the K steps are captured in one CUDA graph
(replayed once untimed to upload it) and replayed once between CUDA events on
the launching stream, with a barrier and a device synchronisation on both
sides; the maximum over ranks is reported.  Weights rotate through enough
independent copies to exceed 3x the L2 size, so every step streams its weights
from HBM.  SM clocks and throttle reasons are sampled through NVML during the
timed region.  `e2e` repeats the K steps through the same C-ABI calls with the
step's input copied from pinned host memory and its output read back to pinned
host memory every step: each step is one CUDA graph [copy x in, call(s), copy y
out] replayed and waited for on the host (stream synchronised).

One JSON line is printed by rank 0.  Under torchrun (N > 1) every rank runs an
independent replica (the layer shards by rows with no exchange; here each rank
runs the whole layer): scaling is weak and value sums the ranks' bytes over the
slowest rank's time.

--impl reference times the CPU oracle on the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_compensated_vq_b200 import synth  # noqa: E402

METRIC = "VQ+sparse GEMV us/call & HBM GB/s (% of B200 peak), 4096x4096 2-bit, batch 1"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# --------------------------------------------------------------------------- workloads
class Workload:
    def __init__(self, name, layers, xs, calls, kind, desc):
        self.name, self.layers, self.xs, self.calls, self.kind, self.desc = name, layers, xs, calls, kind, desc

    def weight_bytes(self):
        return sum(L.abi_bytes()["total"] for L in self.layers)

    def io_bytes(self):
        b = 0
        for (li, B) in self.calls:
            L = self.layers[li]
            xb = self.xs[li]
            b += xb[:B].nbytes + B * L.n_out * 2        # x in its dtype, y fp16/bf16
        return b

    def bytes_per_step(self):
        return self.weight_bytes() + self.io_bytes()

    def flops_per_step(self):
        return sum(2.0 * self.layers[li].n_out * self.layers[li].n_in * B for li, B in self.calls)


def make_workload(name: str, batch: int) -> Workload:
    if name == "qproj":
        L, xb = synth.qproj(batch)
        return Workload("llama2_7b_qproj_4096x4096_d8_k65536_2bit_b%d" % batch, [L], [xb], [(0, batch)], "gemv",
                        "4096x4096, d=8, K=65536 fp16 codebook (16-bit codes, 2 bits/weight), fp16 row+col scales, "
                        "1%% CSR outliers, fp16 x/y, batch %d" % batch)
    if name == "tiny":
        L, xb = synth.tiny()
        return Workload("tiny_256x256_d4_k256_b1", [L], [xb], [(0, 1)], "gemv", "256x256, d=4, K=256, 1% CSR")
    if name == "downproj":
        L, xb = synth.downproj(batch)
        return Workload("llama2_7b_downproj_4096x11008_rvq12x12_b%d" % batch, [L], [xb], [(0, batch)], "gemv",
                        "4096x11008, d=8, residual VQ 12+12 bits, 110 outlier columns (K=256), 0.5%% CSR, batch %d" % batch)
    if name == "smollm":
        Ls, xs = synth.smollm(batch)
        return Workload("smollm2_1.7b_layer_7linears_d8_k256_b%d" % batch, Ls, xs, [(i, batch) for i in range(7)],
                        "gemv", "7 linears of a SmolLM2-1.7B layer, d=8, K=256, 2%% Hessian-style outliers, bf16 x, batch %d" % batch)
    if name == "prefill":
        L, Xb = synth.prefill(2048)
        return Workload("prefill_2048x4096x4096_d8_k65536", [L], [Xb], [(0, 2048)], "gemm",
                        "X 2048x4096 bf16 times the q_proj-shaped VQ weight, bf16 Y")
    if name == "qproj_sym":
        L, xb = synth.qproj_sym(batch)
        return Workload("llama2_7b_qproj_4096x4096_d8_k65536_symmetric_b%d" % batch, [L], [xb], [(0, batch)], "gemv",
                        "4096x4096, d=8, symmetric codebook: 16384 stored fp16 entries addressed as 65536 "
                        "(16-bit codes), fp16 row+col scales, 1%% CSR outliers, fp16 x/y, batch %d" % batch)
    if name == "qproj_groups":
        L, xb = synth.qproj_groups(batch)
        return Workload("llama2_7b_qproj_4096x4096_d8_k65536_groups4_b%d" % batch, [L], [xb], [(0, batch)], "gemv",
                        "4096x4096, d=8, 4 codebook groups of 65536 fp16 entries (16-bit codes), fp16 row+col "
                        "scales, 1%% CSR outliers, fp16 x/y, batch %d" % batch)
    if name == "smollm_vsr":
        Ls, xs = synth.smollm_vsr(batch)
        return Workload("smollm2_1.7b_layer_7linears_d8_k256_vsr_b%d" % batch, Ls, xs, [(i, batch) for i in range(7)],
                        "gemv", "7 linears of a SmolLM2-1.7B layer, d=8, K=256, 2%% of the sub-vectors as VSR blocks "
                        "(position probability ~ |z|^4), bf16 x, batch %d" % batch)
    if name.startswith("vlen"):
        d = int(name[4:])
        L, xb = synth.vlen(d, batch)
        return Workload("vlen_4096x4096_d%d_k4096_b%d" % (d, batch), [L], [xb], [(0, batch)], "gemv",
                        "4096x4096, d=%d, K=4096 fp16 codebook (12-bit codes, %.3g bits/weight), fp16 row+col "
                        "scales, 1%% CSR outliers, fp16 x/y, batch %d" % (d, 12.0 / d, batch))
    raise SystemExit("unknown config " + name)


# --------------------------------------------------------------------------- helpers
def max_over_ranks(value: float, dist) -> float:
    """The largest `value` over all ranks (a device time: the job is as slow as its slowest rank).
    Every rank must call it at the same point.  NCCL reduces a CUDA tensor, gloo a CPU one."""
    if dist is None:
        return value
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_compensated_vq_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per launch from a committed ncu capture, if the kernels have not changed since."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(workload_name)
        if e and e.get("source_hash") == kernel_source_hash():
            return e.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index):
        self.samples, self.reasons, self.err = [], 0, None
        self.stop_flag = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report, do not fail the bench
            self.nv, self.err, self.max_mhz = None, str(e), None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception as e:
            self.err = str(e)

    def _run(self):
        while not self.stop_flag.is_set():
            self._sample()
            time.sleep(0.001)

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self.stop_flag.set()
            self.t.join()
            self._sample()

    def report(self):
        if not self.nv:
            return {"error": self.err}
        names = [n for b, n in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": names}


# --------------------------------------------------------------------------- our arm
def run_vqlin(args, rank, world, dist):
    import torch
    from sparse_compensated_vq_b200 import vqlin

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    wl = make_workload(args.config, args.batch)
    wbytes = wl.weight_bytes()
    n_copies = int(min(64, max(1, math.ceil(3 * L2_BYTES / wbytes))))
    if args.copies:
        n_copies = args.copies          # 1 = the same weights every step (warm L2), for diagnosis only
    copies = [[vqlin.VQLinear(L) for L in wl.layers] for _ in range(n_copies)]
    xdt = "bf16" if wl.name.startswith(("smollm", "prefill")) else "f16"
    tdt = torch.bfloat16 if xdt == "bf16" else torch.float16

    def dev_x(xb, B):
        a = np.ascontiguousarray(xb[:B])
        t = torch.from_numpy(a.view(np.int16)).cuda()
        return t.view(tdt)

    xs = [dev_x(wl.xs[li], B) for li, B in wl.calls]
    ys = [torch.empty((B, wl.layers[li].n_out), dtype=tdt, device="cuda") for li, B in wl.calls]
    if wl.kind == "gemm":
        ws = torch.empty(copies[0][0].workspace_size(wl.calls[0][1]), dtype=torch.uint8, device="cuda")
    else:   # gemv scratch for column-split accumulation (one buffer reused by every call of the step)
        need = max(int(vqlin.vqlin_gemv_workspace_size(copies[0][li].handle, B)) for li, B in wl.calls)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step(i, s_handle):
        c = copies[i % n_copies]
        for k, (li, B) in enumerate(wl.calls):
            h = c[li].handle
            if wl.kind == "gemv":
                st = vqlin.vqlin_gemv_ws(h, xs[k].data_ptr(), vqlin.dtype_code(tdt), B, ys[k].data_ptr(),
                                         vqlin.dtype_code(tdt), ws.data_ptr(), ws.numel(), s_handle)
            else:
                st = vqlin.vqlin_gemm(h, xs[k].data_ptr(), vqlin.dtype_code(tdt), B, ys[k].data_ptr(),
                                      vqlin.dtype_code(tdt), ws.data_ptr(), ws.numel(), s_handle)
            if st != 0:
                raise vqlin.VQLinError(st, "bench step")

    s_ptr = stream.cuda_stream
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, s_ptr)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = vqlin.vqlin_kernel_launches()    # the library counts every kernel it enqueues
    with torch.cuda.graph(g, stream=stream):
        cap = torch.cuda.current_stream().cuda_stream
        for i in range(args.steps):
            step(i, cap)
    timed_launches = vqlin.vqlin_kernel_launches() - n0
    g.replay()                      # upload (untimed)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    ms_max = ms
    if dist:
        ms_max = max_over_ranks(ms, dist)
    del g

    # ---- spread: the same calls as 20 windows of steps/20 calls, timed window by window
    n_win = 20
    per_win = max(1, args.steps // n_win)
    gw = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw, stream=stream):
        cap = torch.cuda.current_stream().cuda_stream
        for i in range(per_win):
            step(i, cap)
    gw.replay()
    torch.cuda.synchronize()
    wev = [torch.cuda.Event(enable_timing=True) for _ in range(n_win + 1)]
    with torch.cuda.stream(stream):
        wev[0].record(stream)
        for w_i in range(n_win):
            gw.replay()
            wev[w_i + 1].record(stream)
    torch.cuda.synchronize()
    win_us = sorted(wev[w_i].elapsed_time(wev[w_i + 1]) * 1e3 / (per_win * len(wl.calls)) for w_i in range(n_win))
    del gw
    spread = {"windows": n_win, "calls_per_window": per_win * len(wl.calls),
              "p10_us_per_call": round(win_us[int(0.1 * (n_win - 1))], 3),
              "p50_us_per_call": round(win_us[(n_win - 1) // 2], 3),
              "p90_us_per_call": round(win_us[int(0.9 * (n_win - 1))], 3)}

    # ---- end to end: host buffers, copies inside the timed region, result read each step
    x_host = [torch.from_numpy(np.ascontiguousarray(wl.xs[li][:B]).view(np.int16)).pin_memory() for li, B in wl.calls]
    y_host = [torch.empty((B, wl.layers[li].n_out), dtype=torch.int16).pin_memory() for li, B in wl.calls]
    n_e2e = args.steps
    # one CUDA graph per weight copy holding a whole step as a user runs it: the host->device
    # copy of x from pinned memory, the C-ABI call(s), the device->host copy of y; every timed
    # step replays one and waits for y on the host
    n_g = min(n_copies, n_e2e)
    e2e_graphs = []
    for gi in range(n_g):
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=stream):
            cap = torch.cuda.current_stream().cuda_stream
            for k in range(len(wl.calls)):
                xs[k].view(torch.int16).copy_(x_host[k], non_blocking=True)
            step(gi, cap)
            for k in range(len(wl.calls)):
                y_host[k].copy_(ys[k].view(torch.int16), non_blocking=True)
        e2e_graphs.append(ge)
    for ge in e2e_graphs:
        ge.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for i in range(n_e2e):
            e2e_graphs[i % n_g].replay()
            stream.synchronize()
        f1.record(stream)
    torch.cuda.synchronize()
    del e2e_graphs
    e2e_ms = f0.elapsed_time(f1)
    if dist:
        e2e_ms = max_over_ranks(e2e_ms, dist)
    h2d = sum(x.numel() * 2 for x in x_host)
    d2h = sum(y.numel() * 2 for y in y_host)

    hbm_peak, bf16_peak, bf16_sust, peak_src = load_peaks()
    bytes_step = wl.bytes_per_step()
    flops_step = wl.flops_per_step()
    sec_step = ms_max / 1e3 / args.steps
    value = world * bytes_step / sec_step / 1e9                   # GB/s, whole job
    per_launch_s = ms / 1e3 / args.steps
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "us_per_call": round(sec_step * 1e6 / len(wl.calls), 3),
        "config": {"workload": wl.name, "describe": wl.desc, "bytes_per_step": bytes_step,
                   "flops_per_step": flops_step, "weight_copies": n_copies,
                   "l2": "weights rotate through %d independent copies (%.0f MB > 3x L2)" % (n_copies, n_copies * wbytes / 1e6),
                   "parallelism": "replicas x%d" % world},
        "gpu_launches": int(timed_launches),
        "spread": spread,
    }
    if wl.kind == "gemv":
        achieved = bytes_step / per_launch_s / 1e9
        line["roofline"] = {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm_peak, "unit": "GB/s",
                            "frac": round(achieved / hbm_peak, 4), "peak_source": peak_src,
                            "traffic": recorded_traffic(wl.name),
                            "kernel": "vqlin gemv (fused dequant + sparse + GEMV), whole step of %d kernel launch(es)"
                                      % (timed_launches // args.steps)}
    else:
        achieved = flops_step / per_launch_s / 1e12
        line["roofline"] = {"bound": "tensor", "achieved": round(achieved, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                            "frac": round(achieved / bf16_peak, 4), "peak_source": peak_src + " bf16 (fp16 same rate)",
                            "traffic": recorded_traffic(wl.name), "kernel": "vqlin gemm step (bf16->fp16 activation convert + GEMM with weight tiles dequantised in shared memory)"}
    line["e2e"] = {"value": round(world * bytes_step * n_e2e / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                   "us_per_step": round(e2e_ms * 1e3 / n_e2e, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    line["clocks"] = sampler.report()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    for c in copies:
        for m in c:
            m.close()
    return line


# --------------------------------------------------------------------------- oracle on host cores
def oracle_step_fn(wl: Workload, rows_per_layer):
    import oracle
    xs = [synth.bits_to_f64(wl.xs[li][:B], "bf16" if wl.name.startswith(("smollm", "prefill")) else "f16")
          for li, B in wl.calls]
    if wl.kind == "gemm":
        xs = [x[:16] for x in xs]          # 16 of the 2048 tokens

    def fn():
        for k, (li, B) in enumerate(wl.calls):
            oracle.gemv_f64(wl.layers[li], xs[k], rows=np.arange(rows_per_layer[li], dtype=np.int32))
    return fn


def sample_fraction(wl, rows_per_layer):
    f = sum(rows_per_layer[li] / wl.layers[li].n_out for li, _ in wl.calls) / len(wl.calls)
    if wl.kind == "gemm":
        f *= 16 / 2048
    return f


def cpu_baseline(wl: Workload, budget_s=10.0):
    """The oracle timed on the host: one core, then every core (a spawn pool, each worker running
    the unchanged oracle on a disjoint range of output rows of every call)."""
    rows = [L.n_out for L in wl.layers]
    fn = oracle_step_fn(wl, rows)
    t0 = time.perf_counter()
    fn()
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / 2 / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    per = (time.perf_counter() - t0) / reps
    frac = sample_fraction(wl, rows)
    single = frac * wl.bytes_per_step() / per / 1e9
    out = {"value": round(single, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": "%d full passes of the oracle (%s) on one host core, %.2f s each; GEMM: 16 of 2048 tokens" % (
               reps, "dequantise to double + dense matvec", per)}
    try:
        import multiprocessing as mp
        from oracle import rows_pool
        n = max(1, min(os.cpu_count() or 1, 128))
        if n == 1:
            return out
        xs = [synth.bits_to_f64(wl.xs[li][:B], "bf16" if wl.name.startswith(("smollm", "prefill")) else "f16")
              for li, B in wl.calls]
        if wl.kind == "gemm":
            xs = [x[:16] for x in xs]
        tasks = []
        for k, (li, _) in enumerate(wl.calls):
            n_out = wl.layers[li].n_out
            step_rows = max(1, -(-n_out // (4 * n)))           # about four chunks per worker
            tasks += [(k, li, lo, min(n_out, lo + step_rows)) for lo in range(0, n_out, step_rows)]
        with mp.get_context("spawn").Pool(n, initializer=rows_pool.init, initargs=(wl.layers, xs)) as pool:
            pool.map(rows_pool.run, tasks)                      # warm: every worker has loaded the oracle
            t0 = time.perf_counter()
            passes = 0
            while True:
                pool.map(rows_pool.run, tasks)
                passes += 1
                if time.perf_counter() - t0 > budget_s / 2:
                    break
            per_all = (time.perf_counter() - t0) / passes
        allc = frac * wl.bytes_per_step() / per_all / 1e9
        out = {"value": round(allc, 4), "unit": "GB/s", "cores": n, "kind": "oracle",
               "sample": "%d full passes of the oracle (dequantise to double + dense matvec), rows split over %d "
                         "host cores (spawn pool, %d row ranges), %.3f s each; GEMM: 16 of 2048 tokens" % (
                             passes, n, len(tasks), per_all),
               "single_core": {"value": round(single, 4), "seconds_per_pass": round(per, 3)}}
    except Exception as exc:                                    # keep the one-core number
        out["all_cores_error"] = str(exc)[:200]
    return out


def run_reference(args, rank, world):
    wl = make_workload(args.config, args.batch)
    rows = [max(1, L.n_out // 64) for L in wl.layers]          # 1/64 of every layer per step
    fn = oracle_step_fn(wl, rows)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    el = time.perf_counter() - t0
    frac = sample_fraction(wl, rows)
    sec_step = el / args.steps
    value = frac * wl.bytes_per_step() / sec_step / 1e9
    sample = "each step: oracle on the first 1/64 of the rows of every layer (%s), one host core" % wl.name
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec_step * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "describe": wl.desc, "parallelism": "rank 0 only"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- main
def run_encode(args, rank, world, dist):
    """Nearest-centroid assignment of every sub-vector of a 4096x4096 fp16 weight (d = 8, about
    2.1 M sub-vectors) against a K = 4096 codebook (VPTQ's Q_V).  Same timing protocol as the
    decode bench; the roofline is the CUDA-core ALU: 2d + 1 binary32 lane operations (d
    subtractions, d fused multiply-adds, one comparison) per (sub-vector, centroid) against
    148 SMs x 128 FP32 lanes x the sampled SM clock."""
    import torch
    from sparse_compensated_vq_b200 import vqlin

    dev = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(dev)
    d, k, n_out, n_in = 8, 4096, 4096, 4096
    rng = synth.rng_for(6)
    C1 = synth.f16_bits(rng.normal(0.0, 0.02, (k, d)))
    V = synth.f16_bits(rng.normal(0.0, 0.02, (n_out * n_in // d, d)))
    n = V.shape[0]
    dv = torch.from_numpy(V.view(np.int16)).cuda()
    dc = torch.from_numpy(C1.view(np.int16)).cuda()
    idx = torch.empty(n, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()

    def step(s_ptr):
        st = vqlin.vqlin_assign(dv.data_ptr(), n, d, dc.data_ptr(), k, None, 0, idx.data_ptr(), None, s_ptr)
        if st != 0:
            raise vqlin.VQLinError(st, "assign")

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(stream.cuda_stream)
    torch.cuda.synchronize()
    steps = min(args.steps, 50)                   # a step is ~6 ms of ALU work
    g = torch.cuda.CUDAGraph()
    n0 = vqlin.vqlin_kernel_launches()
    with torch.cuda.graph(g, stream=stream):
        cap = torch.cuda.current_stream().cuda_stream
        for _ in range(steps):
            step(cap)
    launches = vqlin.vqlin_kernel_launches() - n0
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    if dist:
        ms = max_over_ranks(ms, dist)
    del g
    sec = ms / 1e3 / steps
    ops = float(n) * k * (2 * d + 1)
    clk = sampler.report()
    mhz = clk.get("sm_mhz") or 1965.0
    peak = 148 * 128 * mhz * 1e6 / 1e9             # Gop/s of binary32 add/sub/mul lanes
    return {"metric": "nearest-centroid assignment, sub-vectors per second", "value": round(world * n / sec / 1e6, 2),
            "unit": "M sub-vectors/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(ms / steps, 6), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": "encode_4096x4096_d8_k4096",
                       "describe": "assign the %d sub-vectors (d=8) of a 4096x4096 fp16 weight to a K=4096 fp16 codebook" % n,
                       "l2": "inputs 33.6 MB in HBM; the codebook tile is re-read from L2 by every block",
                       "parallelism": "replicas x%d" % world},
            "gpu_launches": int(launches),
            "roofline": {"bound": "alu", "achieved": round(ops / sec / 1e9, 1), "peak": round(peak, 1), "unit": "Gop/s",
                         "frac": round(ops / sec / 1e9 / peak, 4), "peak_source": "derived: 148 SMs x 128 FP32 lanes x SM clock",
                         "traffic": None},
            "clocks": clk}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="vqlin", choices=["vqlin", "reference"])
    ap.add_argument("--config", default="qproj",
                    choices=["qproj", "tiny", "downproj", "smollm", "prefill", "vlen4", "vlen6", "vlen8", "vlen12",
                             "qproj_sym", "qproj_groups", "smollm_vsr",
                             "encode"])
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=0, help="override the number of rotating weight copies")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as td
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = td
    line = run_encode(args, rank, world, dist) if args.config == "encode" else run_vqlin(args, rank, world, dist)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
