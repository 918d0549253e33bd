#!/usr/bin/env python
"""Benchmark: GPTQ quantization of one linear layer on B200.

One step = the whole hot path on one layer, inputs resident in HBM:
  H = 0;  H += 2 X X^T            (gptq_hessian_accumulate, tcgen05 SYRK)
  dead / act-order / damping / U  (gptq_cholesky_inverse)
  column sweep + lazy updates     (gptq_quantize_layer)
  int4 packing                    (gptq_pack_int4)
  dequantization to bf16          (gptq_dequant)
The default workload is the Llama-7B q_proj shape: W 4096x4096 bf16, X 4096
features x 262144 tokens bf16 (128 x 2048) with 8 outlier channels x20,
4-bit, group 128, act-order.  value = weights quantized per second over the
whole job (all ranks).  Under torchrun each rank quantizes its own replica
(the layer does not shard; no collective on the data path).

`--impl reference` times the fp64 CPU oracle instead, on a bounded sample of
the same workload per step (see cpu_sample()).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

SYRK_REV = "syrk-pair-v3-ordered-red"   # the SYRK kernel the committed traffic figure belongs to
METRIC = "weights quantized/sec (GPTQ 4-bit g128) + Hessian TFLOP/s, % of roofline, 1×B200"
UNIT = "weights/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="q_proj_7b")
    p.add_argument("--tokens", type=int, default=0,
                   help="override the workload's calibration token count (profiling runs)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-next", action="store_true",
                   help="skip the measurements of the consumer-side kernels")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the short runs of the other large workloads")
    p.add_argument("--no-lookahead", action="store_true",
                   help="run the factorisation and the sweep on one stream")
    p.add_argument("--only", choices=["dequant_matvec", "hadamard", "pipeline", "stack"], default=None,
                   help="run one consumer-side measurement alone and print its JSON "
                        "(for profiling; not the benchmark line)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def describe(wl) -> str:
    s = (f"{wl.name}: W {wl.rows}x{wl.n} {str(wl.w_dtype).split('.')[-1]}, X {wl.n}x{wl.ntok} "
         f"{str(wl.x_dtype).split('.')[-1]}")
    if wl.outliers:
        s += f" ({wl.outliers} outlier channels x{wl.outlier_gain:g})"
    g = "per-row" if wl.group_size <= 0 else f"g{wl.group_size}"
    s += f", {wl.bits}-bit {g}{' act-order' if wl.actorder else ''}, damp {wl.percdamp:g}, block {wl.block}"
    return s


# ----------------------------------------------------------------- clocks
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    Reads NVML from a background thread every ``period_s`` (read-only
    queries); if NVML is unavailable, falls back to ``nvidia-smi -lms 200``.
    Nothing here changes a GPU setting."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, uuid: str | None = None, period_s: float = 0.01):
        self.gpu = gpu_index
        self.uuid = uuid
        self.period = period_s
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []          # (sm_mhz, sm_max_mhz, set of reason names)
        self._stop = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, smax, {k for k, v in bits.items() if r & v}))
            except Exception:
                break
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self._stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def _read_smi(self):
        if not self.path or not os.path.exists(self.path):
            return
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, smax = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                reasons = {nm for nm, v in zip(REASON_NAMES, parts[5:9]) if v.lower() == "active"}
                self.samples.append((sm, smax, reasons))
        os.unlink(self.path)

    def summary(self):
        self._read_smi()
        if not self.samples:
            return None
        reasons = set()
        for _, _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(x[0] for x in self.samples),
                "sm_max_mhz": max(x[1] for x in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ----------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of ``x`` over all ranks (a device time: the job ends
    when its slowest rank does)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job units per second: every rank processes ``units_per_rank``
    per step (weak scaling), timed as the slowest rank's ``ms``."""
    return world * units_per_rank * steps / (ms / 1e3)


# ----------------------------------------------------------------- oracle sample
def cpu_sample(wl, W, X, tok_sample: int, row_sample: int):
    """Time the fp64 oracle on a bounded sample of the workload and scale it
    to the whole layer: H on `tok_sample` tokens (cost linear in tokens), U
    in full, sweep + packing on `row_sample` rows (rows are independent once
    U is known).  Returns (weights/s, description, seconds spent)."""
    import numpy as np
    from oracle import gptq_oracle as O

    t_all = time.perf_counter()
    # a sample never larger than the workload (nor than the inputs drawn for it)
    tok_sample = min(tok_sample, wl.ntok, X.shape[1])
    row_sample = min(row_sample, wl.rows, W.shape[0])
    Xs = X[:, :tok_sample].float().cpu().numpy()
    Ws = W[:row_sample].float().cpu().numpy().astype(np.float64)
    t0 = time.perf_counter()
    Hs = O.hessian(Xs)
    t_h = (time.perf_counter() - t0) * (wl.ntok / tok_sample)
    Hfull = Hs * (wl.ntok / tok_sample)          # a stand-in of the right scale for U
    t0 = time.perf_counter()
    prep = O.prepare(Hfull, Ws, wl.percdamp, wl.actorder)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    t_u = time.perf_counter() - t0
    t0 = time.perf_counter()
    res = O.sweep(prep["Wp"], U, wl.bits, wl.group_size)
    codes = np.empty_like(res["codes"])
    codes[:, prep["perm"]] = res["codes"]
    if wl.bits == 4:
        packed = O.pack_int4(codes)
    else:
        packed = O.pack_int3(codes)
    O.dequant(packed, wl.bits, wl.n, res["scales"], res["zeros"], wl.group_size)
    t_s = (time.perf_counter() - t0) * (wl.rows / row_sample)
    total = t_h + t_u + t_s
    desc = (f"fp64 NumPy oracle: H on {tok_sample} of {wl.ntok} tokens (time x{wl.ntok / tok_sample:g}), "
            f"U in full (n={wl.n}), unblocked sweep + pack + dequant on {row_sample} of {wl.rows} rows "
            f"(time x{wl.rows / row_sample:g}); extrapolated layer time {total:.1f} s")
    return wl.rows * wl.n / total, desc, time.perf_counter() - t_all


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    return host_cores()


# ----------------------------------------------------------------- dequant x activation
def measure_dequant_matvec(G, dev, packed, bits, n, scales, zeros, group_size, g_idx, batch=1,
                           iters=20, label="", perm=None):
    """Device time of gptq_dequant_matvec on `batch` bf16 activation vectors,
    L2 flushed before every launch by reading 256 MiB (a read leaves clean
    lines; a write would leave dirty ones whose write-back the timed call
    pays); bytes = everything the call must read or write once."""
    import torch
    x = torch.randn(batch, n, device=dev).to(torch.bfloat16)
    y = torch.empty(batch, packed.shape[0], dtype=torch.float32, device=dev)
    flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
    ts = []
    for i in range(iters + 3):
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        G.gptq_dequant_matvec(packed, bits, n, scales, zeros, x, group_size, g_idx, perm=perm,
                              out=y)
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b))
    t = statistics.median(ts) / 1e3
    nbytes = sum(int(v.numel() * v.element_size()) for v in (packed, scales, zeros, x, y)
                 if v is not None) + (int(g_idx.numel() * 4) if g_idx is not None else 0) \
        + (int(perm.numel() * 4) if perm is not None else 0)
    pk = peaks()
    gbs = nbytes / t / 1e9
    mma = (bits in (3, 4) and x.dtype == torch.bfloat16 and g_idx is None and n % 32 == 0
           and (group_size <= 0 or (group_size >= 32 and group_size & (group_size - 1) == 0)))
    return {"shape": label, "order": "sweep (perm)" if perm is not None else
            ("original (g_idx)" if g_idx is not None else "original"),
            "kernel": "tensor-core (mma.sync)" if mma else (
                "row-per-lane fp32 pipe (g_idx)"
                if g_idx is not None and n % (32 if bits == 4 else 128) == 0 else "fp32 pipe"),
            "batch": batch, "bits": bits, "us": round(t * 1e6, 2),
            "bytes": nbytes, "gbs": round(gbs, 1), "peak_gbs": pk["hbm_gbs"],
            "frac": round(gbs / pk["hbm_gbs"], 4), "l2": "flushed (256 MiB read) before each launch"}


def _codes_70b(dev):
    """Random int4 codes and rulers of the 70B down-proj shape (8192 x 28672,
    g128) and a random act-order permutation with its g_idx."""
    import torch
    r7, n7 = 8192, 28672
    gen = torch.Generator(device=dev)
    gen.manual_seed(77)
    pk7 = torch.randint(-2 ** 31, 2 ** 31 - 1, (r7, n7 // 8), generator=gen, device=dev,
                        dtype=torch.int64).to(torch.int32)
    sc7 = torch.rand(r7, n7 // 128, generator=gen, device=dev) * 0.01 + 1e-4
    z7 = torch.randint(0, 16, (r7, n7 // 128), generator=gen, device=dev,
                       dtype=torch.int64).to(torch.uint8)
    pm7 = torch.randperm(n7, generator=gen, device=dev).to(torch.int32)
    gi7 = torch.empty_like(pm7)
    gi7[pm7.long()] = (torch.arange(n7, device=dev, dtype=torch.int32) // 128)
    return pk7, sc7, z7, pm7, gi7


def measure_dequant_70b(G, dev):
    """The fused dequant x activation on the 70B down-proj shape: codes in
    original order with g_idx (row-per-lane FP32-pipe kernel) and in sweep order with perm
    (tensor-core kernel), 1 and 8 activation vectors."""
    pk7, sc7, z7, pm7, gi7 = _codes_70b(dev)
    n7 = 28672
    label7 = "8192x28672 (70B down-proj shape)"
    out = []
    for b in (1, 8):
        out.append(measure_dequant_matvec(G, dev, pk7, 4, n7, sc7, z7, 128, gi7, batch=b,
                                          label=label7))
        out.append(measure_dequant_matvec(G, dev, pk7, 4, n7, sc7, z7, 128, None, batch=b,
                                          label=label7, perm=pm7))
    # 3-bit codes of the same shape (the first 3/4 of the int4 words' bits as
    # int3 words, zero points reduced to 3 bits), sweep order, 1 vector
    pk3 = pk7.view(-1)[: 8192 * 28672 * 3 // 32].view(8192, -1)
    z3 = z7 & 7
    out.append(measure_dequant_matvec(G, dev, pk3, 3, n7, sc7, z3, 128, None, batch=1,
                                      label=label7, perm=pm7))
    return out


def stream_read_gbs(dev):
    """A plain streaming read of the 70B shape's code bytes with the same L2
    flush: what one pass over 117 MB reaches on this part."""
    import torch
    pk7 = _codes_70b(dev)[0]
    flush = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
    ts = []
    for i in range(13):
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        pk7.view(torch.float32).sum()
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b))
    return round(pk7.numel() * 4 / (statistics.median(ts) / 1e3) / 1e9, 1)


def measure_hadamard(G, dev, iters=10):
    """Device time of the random-sign Hadamard rotation (blocks of 1024) of
    the 70B down-proj workload's operands, in place: X 28672 x 16384 tokens
    and W 8192 x 28672, both bf16 (each larger than L2, so no flush);
    bytes = one read and one write of every element."""
    import torch
    out = []
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    s = (torch.randint(0, 2, (28672,), generator=gen, device=dev) * 2 - 1).float()
    for what, shape in (("X (cols)", (28672, 16384)), ("W (rows)", (8192, 28672))):
        A = torch.randn(*shape, generator=gen, device=dev).to(torch.bfloat16)
        fn = G.gptq_hadamard_cols if what.startswith("X") else G.gptq_hadamard_rows
        ts = []
        for i in range(iters + 3):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn(A, s, 1024, out=A)
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b))
        t = statistics.median(ts) / 1e3
        nbytes = 2 * A.numel() * 2
        pk = peaks()
        line = {"operand": f"{what} {shape[0]}x{shape[1]} bf16, in place", "us": round(t * 1e6, 1),
                "bytes": nbytes, "gbs": round(nbytes / t / 1e9, 1), "peak_gbs": pk["hbm_gbs"],
                "frac": round(nbytes / t / 1e9 / pk["hbm_gbs"], 4)}
        if what.startswith("W"):
            # the same rotation as fp32 matrix products (28 blocks), for context
            H = torch.ones(1, 1, device=dev)
            while H.shape[0] < 1024:
                H = torch.cat([torch.cat([H, H], 1), torch.cat([H, -H], 1)], 0)
            H = H / 32
            Wf = A.float()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for k in range(28):
                sl = slice(1024 * k, 1024 * (k + 1))
                A[:, sl] = ((Wf[:, sl] * s[None, sl]) @ H.T).to(torch.bfloat16)
            b.record()
            torch.cuda.synchronize()
            line["fp32_matmul_us"] = round(a.elapsed_time(b) * 1e3, 1)
            del Wf, H
        out.append(line)
        del A
    return out


def measure_pipeline(G, dev, reps=3):
    """One 7B-shaped decoder block (q, k, v, o, gate, up, down; 4-bit g128,
    65536 tokens per linear, synthetic bf16 inputs resident on the device)
    quantized linear after linear on one stream, and with the Hessian of
    linear l + 1 overlapping the rest of linear l.  weights/s over the block."""
    import torch
    import workloads
    shapes = [(r, n) for _, r, n in workloads.STACK_7B_LINEARS]
    ntok = 65536
    gen = torch.Generator(device=dev)
    gen.manual_seed(4000)
    Ws = [(torch.randn(r, n, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
          for r, n in shapes]
    Xs = [torch.randn(n, ntok, generator=gen, device=dev).to(torch.bfloat16) for _, n in shapes]
    pipe = G.LayerPipeline(shapes, ntok, bits=4, group_size=128, device=dev)
    nw = sum(r * n for r, n in shapes)
    res = {"block": "7B decoder block: q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008",
           "tokens_per_linear": ntok, "weights": nw}
    for mode, ov in (("one_stream", False), ("overlapped", True)):
        ts = []
        for i in range(reps + 1):
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            pipe.run(Ws, Xs, overlap=ov)
            b.record()
            torch.cuda.synchronize()
            if i >= 1:
                ts.append(a.elapsed_time(b))
        pipe.check_info()
        t = statistics.median(ts)
        res[mode] = {"ms": round(t, 3), "weights_per_s": round(nw / (t / 1e3), 1)}
    res["speedup"] = round(res["one_stream"]["ms"] / res["overlapped"]["ms"], 3)
    del pipe, Ws, Xs
    return res


def measure_stack(G, dev, blocks=32):
    """The 7B-shaped decoder stack: 32 blocks x 7 linears (q, k, v, o
    4096x4096; gate, up 11008x4096; down 4096x11008), bf16 N(0, 0.02^2)
    weights, one seeded X of 65536 tokens N(0,1) per linear, 4-bit g128,
    quantized linear after linear on one stream.  Each block's inputs are
    drawn on the device before its timed run (drawing is not timed); the
    stack's time is the sum of the 32 blocks' CUDA-event times.  Block 0 runs
    once untimed first (warm-up)."""
    import torch
    import workloads
    shapes = [(r, n) for _, r, n in workloads.STACK_7B_LINEARS]
    ntok = 65536
    pipe = G.LayerPipeline(shapes, ntok, bits=4, group_size=128, device=dev)

    def inputs(b):
        wls = [workloads.stack_7b_workload(b, l, ntok) for l in range(len(shapes))]
        return ([workloads.make_weights(wl, dev) for wl in wls],
                [workloads.make_calibration(wl, dev) for wl in wls])

    Ws, Xs = inputs(0)
    pipe.run(Ws, Xs)
    torch.cuda.synchronize()
    ts = []
    for b in range(blocks):
        del Ws, Xs
        Ws, Xs = inputs(b)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        a.record()
        pipe.run(Ws, Xs)
        e.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(e))
    pipe.check_info()
    del Ws, Xs, pipe
    torch.cuda.empty_cache()
    nw = blocks * sum(r * n for r, n in shapes)
    flops = blocks * sum(float(n) * (n + 1) * ntok for _, n in shapes)
    total = sum(ts)
    return {"workload": "stack_7b: %d blocks x 7 linears (q,k,v,o 4096x4096; gate,up "
                        "11008x4096; down 4096x11008) bf16, X 65536 tokens per linear, "
                        "4-bit g128, one stream" % blocks,
            "linears": blocks * len(shapes), "weights": nw, "ms_total": round(total, 2),
            "weights_per_s": nw / (total / 1e3),
            "block_ms": {"min": round(min(ts), 3), "median": round(statistics.median(ts), 3),
                         "max": round(max(ts), 3)},
            "hessian_flops_total": flops,
            "note": "sum of per-block CUDA-event times; inputs drawn between blocks, untimed"}


# ----------------------------------------------------------------- per-stage rooflines
def fp32_accurate_peak(pk) -> float:
    """TFLOP/s of fp32-accurate products on the tensor cores: the measured
    bf16 dense rate halved (TF32 runs at half the bf16 rate) and divided by
    the three TF32 products of the hi/lo split."""
    return pk["bf16_tflops"] / 2.0 / 3.0


def stage_rooflines(wl, stage_ms: dict, pk) -> dict:
    """Roofline of every stage after the Hessian, from its CUDA-event time.

    S3 (Cholesky + triangular inverse): n^3/3 + n^3/3 flops against the
    fp32-accurate tensor peak.  S5-S6 (sweep + lazy updates): rows n^2 flops
    against the same peak, and its bytes (W read as stored, the upper half of
    U, the packed codes and the rulers) against HBM; the bound is the larger
    of the two times.  S7 (pack) and S8 (dequant): bytes against HBM."""
    rows, n, b = wl.rows, wl.n, wl.bits
    G = 1 if wl.group_size <= 0 else -(-n // wl.group_size)
    wbytes = 2 if str(wl.w_dtype).endswith("bfloat16") else 4
    pf = fp32_accurate_peak(pk) * 1e12
    hbm = pk["hbm_gbs"] * 1e9
    out = {"fp32_accurate_peak_tflops": round(pf / 1e12, 1),
           "fp32_accurate_peak_source": f"{pk['_source']} bf16 burst / 2 (TF32) / 3 (products)"}
    f3 = 2.0 * n ** 3 / 3.0
    t3 = stage_ms["cholesky_inverse"] / 1e3
    out["cholesky_inverse"] = {"bound": "tensor", "algorithmic_flops": f3,
                               "achieved_tflops": round(f3 / t3 / 1e12, 2),
                               "frac": round((f3 / pf) / t3, 4), "ms": round(t3 * 1e3, 4)}
    f56 = float(rows) * n * n
    b56 = rows * n * wbytes + 2.0 * n * n + rows * n * b / 8.0 + rows * G * 5.0
    t56 = stage_ms["sweep"] / 1e3
    tf, tb = f56 / pf, b56 / hbm
    out["sweep"] = {"bound": "tensor" if tf >= tb else "hbm", "algorithmic_flops": f56,
                    "algorithmic_bytes": b56, "achieved_tflops": round(f56 / t56 / 1e12, 2),
                    "achieved_gbs": round(b56 / t56 / 1e9, 1),
                    "frac": round(max(tf, tb) / t56, 4), "ms": round(t56 * 1e3, 4)}
    b7 = rows * n * (1 + b / 8.0)
    t7 = stage_ms["pack"] / 1e3
    out["pack"] = {"bound": "hbm", "algorithmic_bytes": b7, "achieved_gbs": round(b7 / t7 / 1e9, 1),
                   "frac": round((b7 / hbm) / t7, 4), "ms": round(t7 * 1e3, 4)}
    b8 = rows * n * (b / 8.0 + 2) + rows * G * 5.0
    t8 = stage_ms["dequant"] / 1e3
    out["dequant"] = {"bound": "hbm", "algorithmic_bytes": b8,
                      "achieved_gbs": round(b8 / t8 / 1e9, 1),
                      "frac": round((b8 / hbm) / t8, 4), "ms": round(t8 * 1e3, 4)}
    return out


def measure_layer(G, wl, dev, steps, warmup, stream, lookahead=True, clock=None, world=1,
                  barrier=None):
    """The timed loop of one workload: `warmup` untimed steps, then `steps`
    steps bracketed by CUDA events on `stream`, per-stage events inside every
    step.  Returns (LayerQuantizer, W, X, dict of timings)."""
    import torch
    import workloads
    W, X = workloads.make_inputs(wl, device=dev)
    lq = G.LayerQuantizer(wl.rows, wl.n, wl.ntok, wl.bits, wl.group_size, wl.percdamp,
                          wl.actorder, x_dtype=X.dtype, w_dtype=W.dtype,
                          out_dtype=torch.bfloat16, device=dev, lookahead=lookahead)
    for _ in range(warmup):
        lq.run(W, X, stream=stream)
    torch.cuda.synchronize()
    lq.check_info()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    launches0 = G.gptq_launch_count()
    import contextlib
    with (clock if clock is not None else contextlib.nullcontext()):
        t0.record(stream)
        for k in range(steps):
            lq.run(W, X, stream=stream, events=evs[k])
        t1.record(stream)
        torch.cuda.synchronize()
    if barrier:
        barrier()
    lq.check_info()
    launches = G.gptq_launch_count() - launches0
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    names = list(G.LayerQuantizer.STAGES)
    stage = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
             for i, nm in enumerate(names)}
    return lq, W, X, {"ms": ms, "stage_ms": stage, "launches": launches}


def extra_workload(G, name, dev, stream, steps=3, warmup=2):
    """A short driver-observed run of another large workload: weights/s,
    Hessian TFLOP/s against the measured bf16 peak, per-stage times and
    rooflines."""
    import torch
    import workloads
    wl = workloads.WORKLOADS[name]
    torch.cuda.empty_cache()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clk = ClockSampler(dev.index or 0, uuid)
    lq, W, X, t = measure_layer(G, wl, dev, steps, warmup, stream, clock=clk)
    pk = peaks()
    flops = float(wl.n) * (wl.n + 1) * wl.ntok
    th = t["stage_ms"]["hessian"] / 1e3
    res = {"workload": describe(wl), "steps": steps, "warmup": warmup,
           "ms_per_step": round(t["ms"] / steps, 3),
           "weights_per_s": wl.rows * wl.n * steps / (t["ms"] / 1e3),
           "hessian_tflops": round(flops / th / 1e12, 1),
           "hessian_frac_of_bf16_peak": round(flops / th / 1e12 / pk["bf16_tflops"], 4),
           "stage_ms": {k: round(v, 4) for k, v in t["stage_ms"].items()},
           "roofline_stages": stage_rooflines(wl, t["stage_ms"], pk),
           "gpu_launches": t["launches"], "clocks": clk.summary()}
    del lq, W, X
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import post_weight_quantization_25_b200 as G
    import workloads

    torch.cuda.set_device(local_rank)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        wl = dataclasses.replace(wl, ntok=args.tokens)
    dev = torch.device("cuda", local_rank)
    rows, n, N = wl.rows, wl.n, wl.ntok
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    clk = ClockSampler(local_rank, uuid)
    lq, W, X, t = measure_layer(G, wl, dev, args.steps, args.warmup, stream,
                                lookahead=not args.no_lookahead, clock=clk, world=world,
                                barrier=barrier)
    ms, stage, launches = t["ms"], t["stage_ms"], t["launches"]
    x_gb = X.numel() * X.element_size() / 1e9
    ms_step = ms / args.steps
    value = job_throughput(world, rows * n, args.steps, ms)
    flops = float(n) * (n + 1) * N
    t_h = stage["hessian"] / 1e3
    pk = peaks()
    achieved = flops / t_h / 1e12
    traffic = None
    tf_path = os.path.join(ROOT, "profiles", "syrk_traffic.json")
    if os.path.exists(tf_path):
        with open(tf_path) as f:
            tj = json.load(f)
        if tj.get("workload") == wl.name and tj.get("kernel_rev") == SYRK_REV:
            traffic = tj.get("bytes_per_launch")
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4), "traffic": traffic,
            "kernel": "syrk_bf16_pair_kernel (+ mirror) in gptq_hessian_accumulate",
            "peak_source": f"{pk['_source']} bf16 burst", "algorithmic_flops": flops,
            "frac_of_sustained_peak": round(
                achieved / pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]),
                4)}
    roof_stages = stage_rooflines(wl, stage, pk)

    # the consumer of the packed codes (fused dequant x activation), outside
    # the timed step: on this layer's own output, and on the 70B down-proj
    # shape (8192 x 28672, 4-bit g128, act-order g_idx) with random codes
    nxt = None
    if rank == 0 and not args.no_next and wl.bits in (3, 4):
        import torch
        torch.cuda.synchronize()
        mv = [measure_dequant_matvec(G, dev, lq.packed, wl.bits, n, lq.scales, lq.zeros,
                                     wl.group_size, lq.g_idx, label=f"{rows}x{n} (this layer)")]
        if wl.actorder:
            sw = G.gptq_gather_columns_u8(lq.codes, lq.perm)
            pk_sw = (G.gptq_pack_int4 if wl.bits == 4 else G.gptq_pack_int3)(sw)
            mv.append(measure_dequant_matvec(G, dev, pk_sw, wl.bits, n, lq.scales, lq.zeros,
                                             wl.group_size, None, perm=lq.perm,
                                             label=f"{rows}x{n} (this layer)"))
            del sw, pk_sw
        mv += measure_dequant_70b(G, dev)
        nxt = {"dequant_matvec": mv, "stream_read_117MB_gbs": stream_read_gbs(dev),
               "stream_read_note": "torch fp32 sum over 8192x28672 int4 codes' bytes "
                                   "(a plain read pass), same L2 flush",
               "hadamard_rotation": measure_hadamard(G, dev),
               "layer_pipeline": measure_pipeline(G, dev)}

    # end to end through the same C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        # the calibration set as it arrives from the host: batches of 16
        # sequences (32768 tokens), each a contiguous pinned n x 32768 tensor;
        # run_streamed copies them in on a copy stream while H accumulates
        nbatch = max(1, N // 32768)
        bt = ((N + nbatch - 1) // nbatch + 7) // 8 * 8   # rows 16-byte aligned
        Xh = [torch.empty(n, min(bt, N - a), dtype=X.dtype).pin_memory()
              for a in range(0, N, bt)]
        for i, xb in enumerate(Xh):
            xb.copy_(X[:, i * bt: i * bt + xb.shape[1]])
        Wh = torch.empty_like(W, device="cpu").pin_memory()
        Wh.copy_(W)
        outs = [lq.packed, lq.scales, lq.zeros, lq.g_idx]
        outs_h = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]

        def e2e_step():
            lq.run_streamed(Wh, Xh, stream=stream)
            for t, th in zip(outs, outs_h):
                th.copy_(t, non_blocking=True)

        for _ in range(max(1, min(args.warmup, 2))):
            e2e_step()
        barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(a.elapsed_time(b), world, dev)
        h2d = X.numel() * X.element_size() + W.numel() * W.element_size()
        d2h = sum(t.numel() * t.element_size() for t in outs)
        e2e = {"value": job_throughput(world, rows * n, args.steps, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / args.steps,
               "mode": f"LayerQuantizer.run_streamed: W and {len(Xh)} pinned host batches of "
                       f"{bt} tokens copied in on a copy stream, overlapping the batch-by-batch "
                       f"Hessian; packed codes, scales, zeros, g_idx copied out"}
        del Xh, Wh

    # short driver-observed runs of the other large workloads (3-bit 7B
    # down-proj; the rotated 70B down-proj), after this layer's buffers are freed
    extra = None
    if rank == 0 and world == 1 and not args.no_extra and args.workload == "q_proj_7b" \
            and not args.tokens:
        Wc, Xc = W.cpu(), X[:, :8192].cpu()  # what the CPU baseline below reads
        del lq, W, X
        torch.cuda.empty_cache()
        extra = {name: extra_workload(G, name, dev, stream)
                 for name in ("down_proj_7b", "down_proj_70b")}
        extra["stack_7b"] = measure_stack(G, dev)
        W, X = Wc, Xc

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, _ = cpu_sample(wl, W, X, **CPU_SAMPLE)
        cpu = {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 in / f32", "data": "synthetic",
            "config": {"workload": describe(wl), "rows": rows, "n": n, "tokens": N,
                       "bits": wl.bits, "group_size": wl.group_size, "actorder": wl.actorder,
                       "l2": "inputs larger than L2 (X is %.2f GB)" % x_gb,
                       "parallelism": f"{world} independent replicas"},
            "hessian_tflops": achieved,
            "stage_ms": {k: round(v, 4) for k, v in stage.items()},
            "roofline": roof,
            "roofline_stages": roof_stages,
            "extra_workloads": extra,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "lookahead": not args.no_lookahead,
            "next": nxt,
        }
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- reference arm
CPU_SAMPLE = {"tok_sample": 4096, "row_sample": 64}   # both CPU legs time this sample


def run_reference(args, rank, world):
    """The fp64 oracle on the host cores, one bounded sample of the workload
    per step (cpu_sample); value = the layer's weights over the layer time
    extrapolated from the sample, ms_per_step = the measured time of one
    sample (what the driver's clock sees)."""
    if rank != 0:
        return
    import workloads

    wl = workloads.WORKLOADS[args.workload]
    W = workloads.make_weights(wl, "cpu", rows=CPU_SAMPLE["row_sample"])
    X = workloads.make_calibration(wl, "cpu", ntok=CPU_SAMPLE["tok_sample"])
    layer_s, wall_s = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        v, desc, spent = cpu_sample(wl, W, X, **CPU_SAMPLE)
        if i >= args.warmup:
            layer_s.append(wl.rows * wl.n / v)
            wall_s.append(spent)
    t_layer = statistics.mean(layer_s)
    value = wl.rows * wl.n / t_layer
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(wall_s) * 1e3,
            "extrapolated_layer_s": t_layer,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(wl), "rows": wl.rows, "n": wl.n,
                       "tokens": wl.ntok, "bits": wl.bits, "group_size": wl.group_size,
                       "actorder": wl.actorder, "parallelism": "rank 0 only"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.only:
        import torch
        import post_weight_quantization_25_b200 as G
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        if rank == 0:
            fn = {"dequant_matvec": measure_dequant_70b, "hadamard": measure_hadamard,
                  "pipeline": measure_pipeline, "stack": measure_stack}[args.only]
            print(json.dumps({"only": args.only, "result": fn(G, dev)}), flush=True)
        return
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
