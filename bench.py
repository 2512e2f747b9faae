#!/usr/bin/env python
"""Benchmark of the weight-quantised GEMM at FLUX DiT linear shapes on B200.

One step = one qgemm over the headline workload (FLUX double-stream image
QKV projection: X bf16 [4096, 3072] times a 4-bit group-64 W [9216, 3072]
plus a bf16 bias), inputs resident in HBM. Prints ONE JSON line on stdout
(rank 0): the headline, a few KB. The detailed sections (every workload
linear, the path crossover, the fused epilogues, the policy sweep) go to
stderr as JSON lines of their own, and to --report FILE when given.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--report FILE]

Multi-GPU (torchrun, one process per GPU): the GEMM runs as independent
replicas, one per rank, with no collective on the data path ("scaling":
"weak"); the time is the max over ranks.

Timing: CUDA events on the launching stream, after warm-up, with a barrier
and synchronize on both sides. Inputs rotate over enough copies that the
working set of consecutive steps exceeds the 126 MB L2. The per-shape sweep
(every workload, both paths) times a CUDA graph of back-to-back launches.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HEADLINE_CID, HEADLINE_LIN = 1, 0
L2_BYTES = 126 * 1024 * 1024
METRIC = "qgemm TFLOP/s (GB/s at small M) and % of roofline at FLUX DiT linear shapes"


# ----------------------------------------------------------------------------
# peaks
# ----------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json)"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback (earlier measurement on this pool)"}


def alg_bytes(lin, M=None):
    """Bytes the method must move: packed W + scales (+ biases) + X + out (+ bias)."""
    from weight_quantised_gemm_b200 import qgemm_pack_sizes
    M = lin.M if M is None else M
    p, s, b = qgemm_pack_sizes(lin.N, lin.K, lin.bits, lin.group)
    return p + s + b + M * lin.K * 2 + M * lin.N * 2 + (lin.N * 2 if lin.bias else 0)


def kernel_source_hash():
    """Hash of the headline kernel's device code (comments and whitespace
    removed, host launcher excluded), so that a comment or launcher edit does
    not void the committed ncu counters."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_quantised_gemm_b200", "csrc")
    for f in ("large_m.cu", "dequant.cuh", "epilogue.cuh", "ptx.cuh"):
        src = open(os.path.join(csrc, f)).read()
        if f == "large_m.cu":  # the device code only: the launcher below its host-side marker does not count
            src = src.split("// host side")[0]
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the headline kernel from the committed ncu
    summary, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "large_m_qkv_4096x9216x3072_counters.json")
    if not os.path.exists(p):
        return None, "no ncu summary committed"
    d = json.load(open(p))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None, "kernel changed since the ncu capture"
    return int(d["dram_bytes_read"]) + int(d["dram_bytes_write"]), "ncu capture " + d.get("when", "")


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds
    while the bench runs (NVML, read-only; nvidia-smi as a fallback). The
    report covers the samples taken between mark_begin() and mark_end(), the
    timed region."""
    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.sw_power_cap,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.hw_power_brake_slowdown")

    def __init__(self, device_id: str, period_s: float = 0.001):
        self.dev = device_id
        self.period = period_s
        self.samples = []  # (t, sm_mhz, power_w, [reason names])
        self.sm_max = None
        self.source = None
        self.t_begin = self.t_end = None
        self._stop = threading.Event()
        self.thread = None
        self.proc = None
        self._read = None  # one NVML sample -> (t, sm_mhz, power_w, reasons), or None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.dev.startswith("GPU-") or self.dev.startswith("MIG-"):
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.dev)
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.dev))

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.sm_max = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.source = "nvml"

            def read_one():
                t = time.monotonic()
                try:
                    clk = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                except Exception:  # a failed read only loses that sample
                    return None
                try:
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                except Exception:
                    pw = None
                try:
                    bits = get_reasons(h)
                except Exception:
                    bits = 0
                return (t, clk, pw, [n for n, b in self.REASONS if bits & b])
            self._read = read_one

            def loop():
                while not self._stop.is_set():
                    r = read_one()
                    if r is not None:
                        self.samples.append(r)
                    self._stop.wait(self.period)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.source = "nvidia-smi"

        def read():
            for line in self.proc.stdout:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != 8:
                    continue
                try:
                    clk, mx, pw = float(parts[0]), float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                self.sm_max = mx
                names = [n for (n, _), v in zip(self.REASONS, parts[3:]) if v.lower().startswith("active")]
                self.samples.append((time.monotonic(), clk, pw, names))
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def sample_now(self):
        """One sample from the calling thread (NVML only): called while the
        timed launches are queued on the GPU, so that even a timed region
        shorter than the sampling period holds at least one sample."""
        if self._read is not None:
            r = self._read()
            if r is not None:
                self.samples.append(r)

    def mark_begin(self):
        self.t_begin = time.monotonic()

    def mark_end(self):
        self.t_end = time.monotonic()

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        rows = list(self.samples)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0, "source": self.source}
        lo = self.t_begin if self.t_begin is not None else rows[0][0]
        hi = self.t_end if self.t_end is not None else rows[-1][0]
        timed = [r for r in rows if lo <= r[0] <= hi]
        reasons = sorted({n for r in timed for n in r[3]})
        return {"sm_mhz": statistics.median(r[1] for r in timed) if timed else None, "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(rows), "samples_in_timed_region": len(timed),
                "sm_mhz_min_in_timed_region": min((r[1] for r in timed), default=None),
                "power_w_max": max((r[2] for r in rows if r[2] is not None), default=None),
                "period_ms": self.period * 1e3, "source": self.source}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def smi_device_id(local_rank: int) -> str:
    """nvidia-smi's id for this process's GPU (CUDA_VISIBLE_DEVICES may list indices or UUIDs)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (every rank gets it). NCCL reduces a CUDA
    tensor, gloo a CPU one."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def replica_throughput(flops_per_step: float, steps: int, elapsed_s: float, world: int) -> dict:
    """Whole-job throughput of `world` independent replicas, each running
    `steps` steps: the slowest rank's time (max over ranks) sets the job time."""
    t = max_over_ranks(elapsed_s, world)
    return {"elapsed_s": t, "tflops": world * flops_per_step * steps / t / 1e12,
            "ms_per_step": t / steps * 1e3}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def make_device_inputs(lin, cid, li, copies, M=None):
    """Packed weights, X, bias and out buffers, `copies` independent sets."""
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    X, W, bias = WL.make_inputs(lin, cid, li, M=M)
    pw = wq.qgemm_pack(W, lin.bits)
    M = X.shape[0]
    sets = []
    for _ in range(copies):
        dw = pw.to_device("cuda")
        Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
        bd = None if bias is None else torch.from_numpy(bias.view(np.int16)).cuda().view(torch.bfloat16)
        out = torch.empty((M, lin.N), dtype=torch.bfloat16, device="cuda")
        sets.append((Xd, dw, bd, out))
    return sets, (X, W, bias, pw)


def copies_for(nbytes: int, minimum: int) -> int:
    return max(minimum, -(-3 * L2_BYTES // max(nbytes, 1)))


def time_graph(fn_list, reps: int = 5):
    """Per-launch device time of a CUDA graph replaying fn_list (back-to-back launches)."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for fn in fn_list[:3]:
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for fn in fn_list:
            fn()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3 / len(fn_list))
    del g
    return statistics.median(times)


def sweep(peaks):
    """Every workload linear: time, TFLOP/s, GB/s and roofline fraction (small-M
    rows also with launch overlap and beside the streaming floor of the same
    launch), and config 4's cosine against dense bf16."""
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    res = []
    P = peaks["bf16_tflops"] * 1e12
    BW = peaks["hbm_gbs"] * 1e9

    def one(cid, li, lin, M, path, launches):
        ab = alg_bytes(lin, M)
        ncopy = copies_for(ab, 3 if M > 16 else 32)
        sets, host = make_device_inputs(lin, cid, li, ncopy, M=M)
        fns = [(lambda s=s: wq.qgemm(s[0], s[1], bias=s[2], out=s[3], path=path)) for s in sets]
        reps_list = (fns * (-(-launches // len(fns))))[:max(launches, len(fns))]
        t = time_graph(reps_list)
        wq.check_device_status()
        flops = 2 * M * lin.N * lin.K
        t_roof = max(flops / P, ab / BW)
        entry = {"workload": cid, "linear": lin.name, "M": M, "N": lin.N, "K": lin.K, "bits": lin.bits,
                 "path": "small" if path == wq.QGEMM_PATH_SMALL_M else "large" if path == wq.QGEMM_PATH_LARGE_M
                 else ("small" if wq.qgemm_select_path(M, lin.N, lin.K, lin.bits) == 1 else "large"),
                 "us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 1), "gbs": round(ab / t / 1e9, 1),
                 "bound": "tensor" if flops / P >= ab / BW else "hbm",
                 "roofline_us": round(t_roof * 1e6, 2), "frac_of_roofline": round(t_roof / t, 3),
                 "copies": ncopy}
        if entry["path"] == "small":
            def rep(fl):
                return (fl * (-(-launches // len(fl))))[:max(launches, len(fl))]
            # the same launches with QGEMM_FLAG_OVERLAP_PREVIOUS: each GEMV's weight
            # stream may start while the previous one in the stream finishes
            fo = [(lambda s=s: wq.qgemm(s[0], s[1], bias=s[2], out=s[3], path=path, overlap_previous=True))
                  for s in sets]
            to = time_graph(rep(fo))
            # the streaming floor: the same kernel, grid, clusters and ring moving
            # the same weight bytes with no arithmetic (qgemm_debug_stream)
            tf = time_graph(rep([(lambda s=s: wq.qgemm_debug_stream(s[0], s[1])) for s in sets]))
            tfo = time_graph(rep([(lambda s=s: wq.qgemm_debug_stream(s[0], s[1], overlap_previous=True))
                                  for s in sets]))
            wq.check_device_status()
            entry["us_overlap_previous"] = round(to * 1e6, 2)
            entry["frac_of_roofline_overlap_previous"] = round(t_roof / to, 3)
            entry["us_stream_floor"] = round(tf * 1e6, 2)
            entry["us_stream_floor_overlap_previous"] = round(tfo * 1e6, 2)
            entry["kernel_over_floor"] = round(t / tf, 3)
            entry["kernel_over_floor_overlap_previous"] = round(to / tfo, 3)
        return entry, sets, host

    for cid in range(len(WL.WORKLOADS)):
        wl = WL.workload(cid)
        for li, lin in enumerate(wl.linears):
            entry, sets, host = one(cid, li, lin, lin.M, wq.QGEMM_PATH_AUTO, 100 if lin.M <= 16 else 20)
            if lin.M > 16 and cid in (1, 2, 4):
                # context: dense bf16 torch.matmul (cuBLAS) at the same shape, same graph timing
                Xd0 = sets[0][0]
                Wb = torch.from_numpy(host[1]).cuda().to(torch.bfloat16)
                ob = torch.empty((lin.M, lin.N), dtype=torch.bfloat16, device="cuda")
                td = time_graph([lambda: torch.matmul(Xd0, Wb.T, out=ob)] * 10)
                entry["dense_bf16_torch_us"] = round(td * 1e6, 2)
                entry["dense_bf16_torch_tflops"] = round(2 * lin.M * lin.N * lin.K / td / 1e12, 1)
                del Wb, ob
            if cid == 4:
                Xd, dw, bd, out = sets[0]
                X, W, bias, pw = host
                Wb = torch.from_numpy(W).cuda().to(torch.bfloat16)
                yq = wq.qgemm(Xd, dw, bias=bd).double()
                yd = (Xd @ Wb.T).double()
                entry["cosine_vs_dense_bf16"] = float(torch.nn.functional.cosine_similarity(
                    yq.flatten(), yd.flatten(), dim=0))
                entry["packed_bytes_over_dense_bf16"] = round(pw.nbytes / (lin.N * lin.K * 2), 4)
                entry["packed_bytes_over_dense_fp32"] = round(pw.nbytes / (lin.N * lin.K * 4), 4)
                entry["_yq"], entry["_yd"] = yq.flatten().cpu(), yd.flatten().cpu()
                del Wb
            res.append(entry)
            del sets
            torch.cuda.empty_cache()
    # config 4 as a whole block
    blk = [e for e in res if e["workload"] == 4]
    yq = torch.cat([e.pop("_yq") for e in blk])
    yd = torch.cat([e.pop("_yd") for e in blk])
    block = {"cosine_vs_dense_bf16_all_five": float(torch.nn.functional.cosine_similarity(yq, yd, dim=0)),
             "us_total": round(sum(e["us"] for e in blk), 1)}
    wl4 = WL.workload(4)
    packed = sum(wq.qgemm_pack_sizes(l.N, l.K, l.bits, l.group)[0] + 2 * wq.qgemm_pack_sizes(l.N, l.K, l.bits,
                                                                                             l.group)[1]
                 for l in wl4.linears)
    dense = sum(l.N * l.K for l in wl4.linears)
    block["packed_over_dense_bf16"] = round(packed / (2 * dense), 4)
    block["packed_over_dense_fp32"] = round(packed / (4 * dense), 4)
    block["tflops"] = round(sum(2 * l.M * l.N * l.K for l in wl4.linears) / (block["us_total"] * 1e-6) / 1e12, 1)
    torch.cuda.empty_cache()
    return res, block


def grouped_sweep(peaks):
    """The mixed FLUX block's five linears at decode M: one grouped call per
    format (4-bit QKV and MLP up; 8-bit modulation, out projection and MLP
    down), as consecutive overlapped launches (the default) and as one
    persistent launch, against one plain call per linear, CUDA-graph timing
    over rotating weight copies, GB/s against the summed algorithmic bytes."""
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    BW = peaks["hbm_gbs"] * 1e9
    wl = WL.workload(4)
    rows = []
    for M in (1, 16):
        for bits in (4, 8):
            lins = [(li, l) for li, l in enumerate(wl.linears) if l.bits == bits]
            ab = sum(alg_bytes(l, M) for _, l in lins)
            ncopy = max(4, -(-3 * L2_BYTES // ab))
            host = []
            for li, l in lins:
                X, W, _ = WL.make_inputs(l, 4, li, M=M)
                host.append((l, X, wq.qgemm_pack(W, bits)))
            sets = [[(torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16), pw.to_device("cuda"), None,
                      torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda")) for l, X, pw in host]
                    for _ in range(ncopy)]

            def grouped(probs, ov):
                return lambda: wq.qgemm_grouped([(x, d, b) for x, d, b, _ in probs], outs=[o for *_, o in probs],
                                                overlap_previous=ov)

            def grouped_one_launch(probs, ov):
                return lambda: wq.qgemm_grouped([(x, d, b) for x, d, b, _ in probs], outs=[o for *_, o in probs],
                                                overlap_previous=ov, one_launch=True)

            def separate(probs, ov):
                return lambda: [wq.qgemm(x, d, bias=b, out=o, overlap_previous=ov) for x, d, b, o in probs]
            n = max(ncopy, 24)
            res = {"M": M, "bits": bits, "linears": [l.name for _, l in lins], "alg_bytes": ab, "copies": ncopy}
            for name, mk in (("grouped", grouped), ("grouped_one_launch", grouped_one_launch), ("separate", separate)):
                for ov in (False, True):
                    t = time_graph([mk(sets[i % ncopy], ov) for i in range(n)])
                    key = name + ("_overlap_previous" if ov else "")
                    res[f"us_{key}"] = round(t * 1e6, 2)
                    res[f"gbs_{key}"] = round(ab / t / 1e9, 1)
                    res[f"frac_of_hbm_roofline_{key}"] = round(ab / BW / t, 3)
            wq.check_device_status()
            rows.append(res)
            del sets
            torch.cuda.empty_cache()
    return rows


CROSSOVER_SHAPES = ((12288, 3072), (9216, 3072), (18432, 3072), (3072, 3072), (3072, 12288))
CROSSOVER_M = (1, 2, 4, 8, 12, 16, 24, 32, 48, 64)


def crossover_sweep():
    """Both kernel paths at M = 1..64 on every (N, K) of the FLUX workloads in
    every format (CUDA-graph timing over rotating weight copies): the
    measurements the path table is read from."""
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    rows = []
    for N, K in CROSSOVER_SHAPES:
        for bits in (1, 2, 4, 8):
            dist = {1: "binary", 2: "ternary"}.get(bits, "normal")
            W = WL.make_w(9, bits, N, K, dist, wq.GROUP_OF_BITS[bits])
            pw = wq.qgemm_pack(W, bits)
            wbytes = pw.nbytes
            ncopy = max(8, -(-3 * L2_BYTES // wbytes))
            dws = [pw.to_device("cuda") for _ in range(ncopy)]
            for M in CROSSOVER_M:
                X = WL.make_x(9, bits, M, K, "normal")
                Xd = torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16)
                out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                entry = {"N": N, "K": K, "bits": bits, "M": M}
                for name, path in (("small", wq.QGEMM_PATH_SMALL_M), ("large", wq.QGEMM_PATH_LARGE_M)):
                    if name == "small" and M > 64:
                        continue
                    fns = [(lambda d=d: wq.qgemm(Xd, d, out=out, path=path)) for d in dws]
                    launches = max(len(fns), 64 if M <= 32 else 16)
                    t = time_graph((fns * (-(-launches // len(fns))))[:launches])
                    entry[f"us_{name}"] = round(t * 1e6, 2)
                wq.check_device_status()
                entry["faster"] = "small" if entry.get("us_small", float("inf")) < entry["us_large"] else "large"
                entry["table"] = "small" if wq.qgemm_select_path(M, N, K, bits) == 1 else "large"
                rows.append(entry)
                del Xd, out
            del dws
            torch.cuda.empty_cache()
    return rows


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    peaks = load_peaks()
    lin = WL.workload(HEADLINE_CID).linears[HEADLINE_LIN]
    ab = alg_bytes(lin)
    ncopy = copies_for(ab, 3)
    sets, host = make_device_inputs(lin, HEADLINE_CID, HEADLINE_LIN, ncopy)
    flops = 2 * lin.M * lin.N * lin.K
    stream = torch.cuda.current_stream()

    def step(i):
        Xd, dw, bd, out = sets[i % ncopy]
        wq.qgemm(Xd, dw, bias=bd, out=out, stream=stream)

    clocks = ClockSampler(smi_device_id(local_rank))
    clocks.start()
    for i in range(args.warmup):
        step(i)
    barrier(world)
    st = wq.qgemm_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    clocks.mark_begin()
    t0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t1.record(stream)
    clocks.sample_now()  # the queued launches are running now
    barrier(world)
    clocks.mark_end()
    clk = clocks.stop()
    st = wq.qgemm_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")
    elapsed = t0.elapsed_time(t1) * 1e-3
    kernel_t = statistics.fmean(a.elapsed_time(b) for a, b in ev) * 1e-3
    job = replica_throughput(flops, args.steps, elapsed, world)
    elapsed_max = job["elapsed_s"]
    kernel_max = max_over_ranks(kernel_t, world)

    # end to end through the public API with host buffers: pinned X in, out back
    X, W, bias, pw = host
    e2e = run_e2e(sets, X, lin, args, world)

    result = None
    if rank == 0:
        result = assemble_ours(args, world, lin, ncopy, job, kernel_max, e2e, clk, peaks)
    return result, peaks, sets[0][3]


def assemble_ours(args, world, lin, ncopy, job, kernel_s, e2e, clk, peaks) -> dict:
    """The headline result of our arm from its measurements: `job` from
    replica_throughput, `kernel_s` the mean per-launch event time (max over
    ranks), `e2e` from run_e2e, `clk` from ClockSampler.stop()."""
    flops = 2 * lin.M * lin.N * lin.K
    ab = alg_bytes(lin)
    achieved = flops / kernel_s / 1e12
    traffic, traffic_src = profiled_traffic()
    roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": traffic,
            "peak_source": peaks["source"] + ", burst bf16 (kernel timed on its own)",
            "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
            "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": ab,
            "traffic_source": traffic_src, "kernel": f"large_m_kernel<{lin.bits}>"}
    elapsed = job["elapsed_s"]
    return {
        "metric": METRIC, "value": round(job["tflops"], 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; W ~ N(0,0.02) RTN 4-bit g64, X ~ N(0,1), bias ~ N(0,0.01))",
        "config": {"workload": "FLUX double-stream image QKV projection: X bf16 [4096,3072] x W 4-bit "
                               "group-64 [9216,3072] + bias bf16 [9216] -> bf16 [4096,9216]",
                   "M": lin.M, "N": lin.N, "K": lin.K, "bits": lin.bits, "group": lin.group,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs rotate over {ncopy} copies ({ncopy * ab / 1e6:.0f} MB > 126 MB L2)"},
        "gbs": round(ab * args.steps * world / elapsed / 1e9, 1),
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": {k: clk.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "clocks_detail": clk,
        "impl": "ours",
    }


def run_case(args):
    """One workload linear, launched back to back with a CUDA event pair per
    launch (the form a profiler captures). --case 3:tern_m1:M=16"""
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    parts = args.case.split(":")
    cid = int(parts[0])
    names = [l.name for l in WL.workload(cid).linears]
    li = names.index(parts[1]) if len(parts) > 1 else 0
    lin = WL.workload(cid).linears[li]
    M = int(parts[2].split("=")[1]) if len(parts) > 2 else lin.M
    ab = alg_bytes(lin, M)
    ncopy = copies_for(ab, 3 if M > 16 else 32)
    sets, _ = make_device_inputs(lin, cid, li, ncopy, M=M)
    for i in range(args.warmup):
        Xd, dw, bd, out = sets[i % ncopy]
        wq.qgemm(Xd, dw, bias=bd, out=out)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        Xd, dw, bd, out = sets[i % ncopy]
        ev[i][0].record()
        wq.qgemm(Xd, dw, bias=bd, out=out)
        ev[i][1].record()
    torch.cuda.synchronize()
    wq.check_device_status()
    t = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e-3
    fns = [(lambda s=s: wq.qgemm(s[0], s[1], bias=s[2], out=s[3])) for s in sets]
    launches = max(len(fns), 100 if M <= 16 else 20)
    tg = time_graph((fns * (-(-launches // len(fns))))[:launches])
    wq.check_device_status()
    flops = 2 * M * lin.N * lin.K
    return {"case": args.case, "M": M, "N": lin.N, "K": lin.K, "bits": lin.bits,
            "path": "small" if wq.qgemm_select_path(M, lin.N, lin.K, lin.bits) == 1 else "large",
            "us_per_launch_events": round(t * 1e6, 2), "us_graph": round(tg * 1e6, 2),
            "tflops_graph": round(flops / tg / 1e12, 1), "gbs_graph": round(ab / tg / 1e9, 1), "copies": ncopy,
            "env": {k: os.environ[k] for k in ("QGEMM_PATH", "QGEMM_LARGE_PAIR") if k in os.environ},
            "note": "per-launch events include host launch gaps for short kernels; the graph timing does not"}


def run_grouped_case(args):
    """The mixed FLUX block's linears of one format at decode M as one
    persistent grouped launch (QGEMM_FLAG_GROUPED_ONE_LAUNCH), back to back
    with a CUDA event pair per launch (the form a profiler captures).
    --grouped BITS:M, e.g. 8:1"""
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    bits, M = (int(v) for v in args.grouped.split(":"))
    wl = WL.workload(4)
    lins = [(li, l) for li, l in enumerate(wl.linears) if l.bits == bits]
    if not lins:
        raise SystemExit(f"the mixed block has no {bits}-bit linear")
    ab = sum(alg_bytes(l, M) for _, l in lins)
    ncopy = max(4, -(-3 * L2_BYTES // ab))
    host = []
    for li, l in lins:
        X, W, _ = WL.make_inputs(l, 4, li, M=M)
        host.append((l, X, wq.qgemm_pack(W, bits)))
    sets = [[(torch.from_numpy(X.view(np.int16)).cuda().view(torch.bfloat16), pw.to_device("cuda"), None)
             for l, X, pw in host] for _ in range(ncopy)]
    outs = [torch.empty((M, l.N), dtype=torch.bfloat16, device="cuda") for l, _, _ in host]
    for i in range(args.warmup):
        wq.qgemm_grouped(sets[i % ncopy], outs=outs, one_launch=True)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        ev[i][0].record()
        wq.qgemm_grouped(sets[i % ncopy], outs=outs, one_launch=True)
        ev[i][1].record()
    torch.cuda.synchronize()
    wq.check_device_status()
    t = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e-3
    tg = time_graph([(lambda s=s: wq.qgemm_grouped(s, outs=outs, one_launch=True)) for s in sets] * max(1, 24 // ncopy))
    wq.check_device_status()
    return {"grouped": args.grouped, "linears": [l.name for l, _, _ in host], "alg_bytes": ab, "copies": ncopy,
            "us_per_launch_events": round(t * 1e6, 2), "us_graph": round(tg * 1e6, 2),
            "gbs_graph": round(ab / tg / 1e9, 1)}


def run_e2e(sets, X_host_bits, lin, args, world):
    """Pipelined host->device->host: per step, copy X in from pinned memory,
    qgemm, copy out back to pinned memory, on three streams (PCIe in, compute,
    PCIe out) with double buffers."""
    import numpy as np
    import torch

    import weight_quantised_gemm_b200 as wq
    M = lin.M
    xh = [torch.from_numpy(X_host_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory() for _ in range(2)]
    oh = [torch.empty((M, lin.N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [sets[i % len(sets)][0] for i in range(2)]
    od = [sets[i % len(sets)][3] for i in range(2)]
    dw, bd = sets[0][1], sets[0][2]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_o = [torch.cuda.Event() for _ in range(2)]
    steps = max(10, min(args.steps, 100))

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[b])
                xd[b].copy_(xh[b], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_c):
                s_c.wait_event(ev_in[b])
                if i >= 2:
                    s_c.wait_event(ev_o[b])
                wq.qgemm(xd[b], dw, bias=bd, out=od[b], stream=s_c)
                ev_c[b].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[b])
                oh[b].copy_(od[b], non_blocking=True)
                ev_o[b].record(s_out)

    run(4)
    barrier(world)
    t0 = time.perf_counter()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(steps)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    barrier(world)
    dt = e0.elapsed_time(e1) * 1e-3
    wall = time.perf_counter() - t0
    dt = max_over_ranks(dt, world)
    flops = 2 * M * lin.N * lin.K
    return {"value": round(world * flops * steps / dt / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": M * lin.K * 2, "d2h_bytes_per_step": M * lin.N * 2,
            "steps": steps, "ms_per_step": round(dt / steps * 1e3, 4), "wall_s": round(wall, 3),
            "how": "pinned host X -> device, qgemm, device out -> pinned host; copies and compute on three "
                   "streams with double buffers; weights resident on the device"}


# ----------------------------------------------------------------------------
# CPU baseline: the oracle as it stands
# ----------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's guess."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_oracle_sample(target_s: float, lin=None, cid=HEADLINE_CID, li=HEADLINE_LIN, runs: int = 3):
    """Times the oracle (dequantisation of the whole W + fp64 matmul) on a
    bounded sample of the workload's rows, `runs` times, and extrapolates the
    median run to the full M: returns (TFLOP/s, seconds spent, description,
    sample rows, per-run TFLOP/s)."""
    import numpy as np

    import oracle as O
    import workloads as WL
    lin = WL.workload(cid).linears[li] if lin is None else lin
    X, W, bias = WL.make_inputs(lin, cid, li)
    p, s, b = O.pack_ref(W, lin.bits, lin.group)

    def one(rows):
        t0 = time.perf_counter()
        Wq = O.wq_exact(p, s, b, lin.bits, lin.group, lin.K)
        t_deq = time.perf_counter() - t0
        t1 = time.perf_counter()
        out = O.bf16_bits_to_f64(X[:rows]) @ Wq.T
        if bias is not None:
            out += O.bf16_bits_to_f64(bias)[None, :]
        return t_deq, time.perf_counter() - t1

    # the sample: grow the rows until one run takes its share of the budget or covers M
    rows, spent = 16, 0.0
    while True:
        t_deq, t_mm = one(rows)
        spent += t_deq + t_mm
        if t_deq + t_mm >= target_s / (2 * runs) or rows >= lin.M:
            break
        rows = min(lin.M, rows * 4)
    flops = 2 * lin.M * lin.N * lin.K
    per_run = []
    for _ in range(runs):
        t_deq, t_mm = one(rows)
        spent += t_deq + t_mm
        per_run.append(flops / (t_deq + t_mm * lin.M / rows) / 1e12)
    med = statistics.median(per_run)
    desc = (f"oracle (numpy fp64): dequantisation of the full W [{lin.N},{lin.K}] + matmul of X rows "
            f"0..{rows - 1} of {lin.M}, extrapolated to all {lin.M} rows; median of {runs} runs")
    return med, spent, desc, rows, per_run


def cpu_baseline(target_s: float) -> dict:
    """The main arm's cpu_baseline: the oracle on the host cores, median of
    three runs of a bounded sample of the headline workload."""
    v, spent, desc, rows, per_run = cpu_oracle_sample(target_s)
    return {"value": round(v, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle", "sample": desc,
            "cpu_model": cpu_model(), "runs_tflops": [round(x, 6) for x in per_run], "seconds": round(spent, 2)}


def fused_sweep():
    """The fused epilogues on the FLUX shapes they serve, against the unfused
    sequence (qgemm, then a torch elementwise kernel), both in CUDA graphs."""
    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    rows = []
    cases = [(2, 0, wq.QGEMM_EPI_GELU_TANH), (4, 2, wq.QGEMM_EPI_RESIDUAL_GATE), (4, 4, wq.QGEMM_EPI_RESIDUAL_GATE)]
    for cid, li, op in cases:
        lin = WL.workload(cid).linears[li]
        ab = alg_bytes(lin)
        ncopy = copies_for(ab, 3)
        sets, _ = make_device_inputs(lin, cid, li, ncopy)
        g = torch.Generator(device="cuda").manual_seed(0)
        res = [torch.randn((lin.M, lin.N), device="cuda", generator=g).to(torch.bfloat16) for _ in range(ncopy)]
        gate = torch.randn((lin.N,), device="cuda", generator=g).to(torch.bfloat16)

        def fused(i):
            Xd, dw, bd, out = sets[i]
            return lambda: wq.qgemm_fused(Xd, dw, op, bias=bd, residual=res[i], gate=gate, out=out)

        def unfused(i):
            Xd, dw, bd, out = sets[i]
            if op == wq.QGEMM_EPI_GELU_TANH:
                return lambda: torch.nn.functional.gelu(wq.qgemm(Xd, dw, bias=bd, out=out), approximate="tanh")
            return lambda: torch.addcmul(res[i], gate, wq.qgemm(Xd, dw, bias=bd, out=out))

        n = max(ncopy, 12)
        tf = time_graph([fused(i % ncopy) for i in range(n)])
        tu = time_graph([unfused(i % ncopy) for i in range(n)])
        wq.check_device_status()
        rows.append({"workload": cid, "linear": lin.name, "epilogue": {1: "gelu_tanh", 2: "residual_gate"}[op],
                     "M": lin.M, "N": lin.N, "K": lin.K, "bits": lin.bits, "fused_us": round(tf * 1e6, 2),
                     "unfused_us": round(tu * 1e6, 2), "saved_us": round((tu - tf) * 1e6, 2)})
        del sets, res
        torch.cuda.empty_cache()
    return rows


def policy_sweep():
    """Every assignment of 4 or 8 bits to the five linears of the mixed FLUX
    block (workload 4), on its synthetic weights: the block's cosine against
    dense bf16 (outputs concatenated) and its packed size, with the Pareto
    front marked. The pages' policy (8 bits for the linears whose output
    scales the residual stream, 4 for the rest) is one of the 32."""
    import itertools

    import torch

    import weight_quantised_gemm_b200 as wq
    import workloads as WL
    wl = WL.workload(4)
    yq, yd, sizes = {}, [], {}
    for li, lin in enumerate(wl.linears):
        X, W, bias = WL.make_inputs(lin, 4, li)
        Xd = torch.from_numpy(X.view("int16")).cuda().view(torch.bfloat16)
        bd = None if bias is None else torch.from_numpy(bias.view("int16")).cuda().view(torch.bfloat16)
        Wb = torch.from_numpy(W).cuda().to(torch.bfloat16)
        yd.append((Xd @ Wb.T).double().flatten() if bd is None else (Xd @ Wb.T + bd).double().flatten())
        del Wb
        for bits in (4, 8):
            dw = wq.qgemm_pack(W, bits).to_device()
            yq[(li, bits)] = wq.qgemm(Xd, dw, bias=bd).double().flatten()
            sizes[(li, bits)] = dw.nbytes
            del dw
        wq.check_device_status()
    dense_bytes = sum(2 * l.N * l.K for l in wl.linears)
    # the per-layer terms the policy module works from, reduced on the device
    terms = []
    for li, lin in enumerate(wl.linears):
        dl = yd[li]
        opts = {}
        for bits in (4, 8):
            e = yq[(li, bits)] - dl
            opts[bits] = (sizes[(li, bits)], float(e @ dl), float(e @ e))
        terms.append((lin.name, float(dl @ dl), opts))
    rows = []
    d = torch.cat(yd)
    for combo in itertools.product((4, 8), repeat=len(wl.linears)):
        q = torch.cat([yq[(li, b)] for li, b in enumerate(combo)])
        cos = float(torch.nn.functional.cosine_similarity(q, d, dim=0))
        size = sum(sizes[(li, b)] for li, b in enumerate(combo))
        rows.append({"bits": dict(zip([l.name for l in wl.linears], combo)), "cosine_vs_dense_bf16": cos,
                     "packed_over_dense_bf16": round(size / dense_bytes, 4),
                     "pages_policy": combo == tuple(l.bits for l in wl.linears)})
    for r in rows:  # Pareto: no other assignment is at least as small and strictly more accurate (or vice versa)
        r["pareto"] = not any((o["packed_over_dense_bf16"] <= r["packed_over_dense_bf16"] and
                               o["cosine_vs_dense_bf16"] > r["cosine_vs_dense_bf16"]) or
                              (o["packed_over_dense_bf16"] < r["packed_over_dense_bf16"] and
                               o["cosine_vs_dense_bf16"] >= r["cosine_vs_dense_bf16"]) for o in rows)
    rows.sort(key=lambda r: r["packed_over_dense_bf16"])
    del yq, yd
    torch.cuda.empty_cache()
    return {"assignments": rows, "policy_module": policy_module_report(terms, dense_bytes, rows)}


def policy_module_report(terms, dense_bytes, rows, min_cosine=0.999):
    """The policy module's answers from per-layer terms (name, ||d||^2,
    {bits: (bytes, <e, d>, ||e||^2)}), with its cosines checked against the
    directly computed ones of `rows` (every assignment, as policy_sweep
    reports them)."""
    import weight_quantised_gemm_b200.policy as P
    layers = [P.LayerStats(n, D, {b: P.Option(b, nb, a, e) for b, (nb, a, e) in o.items()}) for n, D, o in terms]
    front = P.frontier(layers)
    worst = max(abs(P.cosine(layers, r["bits"]) - r["cosine_vs_dense_bf16"]) for r in rows)
    best = P.cheapest(layers, min_cosine)
    return {"front": [{"bits": p.bits, "cosine_vs_dense_bf16": p.cosine,
                       "packed_over_dense_bf16": round(p.nbytes / dense_bytes, 4)} for p in front],
            "max_abs_cosine_difference_vs_direct": worst,
            f"cheapest_with_cosine_at_least_{min_cosine}": None if best is None else best.bits}


def headline_parity(out, rows: int = 64) -> dict:
    """Part of the CPU-baseline leg: the oracle on sampled rows of the
    headline workload (the first rows and rows spread over all M), against
    the output of the timed run (`out`, the bf16 [M, N] tensor it wrote),
    with the parity gate's two measures."""
    import numpy as np
    import torch

    import oracle as O
    import workloads as WL
    lin = WL.workload(HEADLINE_CID).linears[HEADLINE_LIN]
    X, W, bias = WL.make_inputs(lin, HEADLINE_CID, HEADLINE_LIN)
    p, s, b = O.pack_ref(W, lin.bits, lin.group)
    idx = np.unique(np.concatenate([np.arange(rows // 2), np.linspace(0, lin.M - 1, rows // 2).astype(np.int64)]))
    ref = O.qgemm_ref_rows(idx, X, p, s, b, lin.bits, lin.group, lin.K, bias)
    got = out[torch.as_tensor(idx, device=out.device)].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    y = O.bf16_bits_to_f64(got)
    return {"rows_checked": int(idx.size), "rel_frobenius": O.rel_frobenius(y, ref), "max_abs_rel": O.max_abs_rel(y, ref),
            "within_tolerance": bool(O.within_tolerance(y, ref)),
            "tolerance": {"rel_frobenius": O.REL_FROB_TOL, "max_abs_rel": O.MAX_ABS_TOL},
            "reference": "oracle (fp64, exact quantised weights)"}


def cpu_oracle_single_core():
    """The oracle on one host core for config 0 (tiny; median of 20 runs) and
    config 3 at M=1 (ternary decode; median of 3 runs): seconds per GEMM,
    dequantisation included."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    import workloads as WL
    out = {}
    with threadpool_limits(limits=1):
        for cid, li, runs in ((0, 0, 20), (3, 0, 3)):
            lin = WL.workload(cid).linears[li]
            X, W, bias = WL.make_inputs(lin, cid, li)
            p, s, b = O.pack_ref(W, lin.bits, lin.group)
            ts = []
            for _ in range(runs):
                t0 = time.perf_counter()
                O.qgemm_ref(X, p, s, b, lin.bits, lin.group, lin.K, bias)
                ts.append(time.perf_counter() - t0)
            t = statistics.median(ts)
            out[f"{cid}:{lin.name}"] = {"seconds": round(t, 4), "gflops": round(2 * lin.M * lin.N * lin.K / t / 1e9, 3),
                                        "runs": runs}
    return out


REFERENCE_SECONDS = 150.0   # the reference arm's whole run (warm-up and timed steps)


def run_reference(args, rank, world):
    """The base contract's reference arm, here the oracle on the host cores:
    each step is a bounded sample of the headline workload."""
    if rank != 0:
        return None
    import numpy as np

    import oracle as O
    import workloads as WL
    lin = WL.workload(HEADLINE_CID).linears[HEADLINE_LIN]
    X, W, bias = WL.make_inputs(lin, HEADLINE_CID, HEADLINE_LIN)
    p, s, b = O.pack_ref(W, lin.bits, lin.group)
    total_steps = args.steps + args.warmup
    budget = REFERENCE_SECONDS / max(total_steps, 1)   # seconds per step so the run ends within minutes

    def w_rows(n):
        # the first n rows of W: scales and biases are group-major [K / group, N]
        return O.wq_exact(p[:n], s[:, :n], None if b is None else b[:, :n], lin.bits, lin.group, lin.K)

    # a step: dequantise a block of W rows and multiply a block of X rows with it
    t0 = time.perf_counter()
    w_rows(256)
    t_deq_256 = time.perf_counter() - t0
    n_rows = int(max(64, min(lin.N, 256 * budget * 0.5 / max(t_deq_256, 1e-6))))
    n_rows -= n_rows % 16
    m_rows = 64

    def one_step():
        Wq = w_rows(n_rows)
        out = O.bf16_bits_to_f64(X[:m_rows]) @ Wq.T
        if bias is not None:
            out += O.bf16_bits_to_f64(bias[:n_rows])[None, :]
        return out

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    flops = 2 * m_rows * n_rows * lin.K
    value = flops * args.steps / dt / 1e12
    cores = blas_threads()
    sample = (f"per step: dequantise W rows 0..{n_rows - 1} of {lin.N} and multiply X rows 0..{m_rows - 1} of "
              f"{lin.M} with them in fp64 (oracle as it stands)")
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "FLUX double-stream image QKV projection: X bf16 [4096,3072] x W 4-bit "
                                   "group-64 [9216,3072] + bias bf16 [9216] -> bf16 [4096,9216]",
                       "M": lin.M, "N": lin.N, "K": lin.K, "bits": lin.bits, "group": lin.group},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------

def report_section(res: dict, key: str, fn):
    """Runs an optional part of the report after the headline measurement:
    a failure is recorded in the line (`errors`) instead of losing the
    measurement already taken. Returns fn()'s result, or None."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001 - any failure of an optional section
        res.setdefault("errors", {})[key] = f"{type(e).__name__}: {e}"[:500]
        return None


class Reporter:
    """The detailed report sections (per-workload sweep, path crossover, fused
    epilogues, policy sweep): one JSON line each on stderr, and the same lines
    appended to `path` when one is given. stdout carries only the headline."""

    def __init__(self, path=None):
        self.path = path
        if path:
            os.makedirs(os.path.dirname(os.path.abspath(path)), exist_ok=True)
            open(path, "w").close()

    def __call__(self, section: str, data) -> None:
        line = json.dumps({"report": section, "data": data})
        print(line, file=sys.stderr, flush=True)
        if self.path:
            with open(self.path, "a") as fh:
                fh.write(line + "\n")


HEADLINE_KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                 "scaling", "vs_baseline", "dtype", "data", "config", "gbs", "roofline", "e2e", "gpu_launches",
                 "clocks", "cpu_baseline", "parity", "peaks", "sweep_summary", "errors", "impl")
HEADLINE_MAX_BYTES = 6000


def sweep_summary(sweep_rows, block) -> dict:
    """A few numbers per workload linear for the headline line: microseconds
    per launch (CUDA graph) and the fraction of the shape's roofline; the
    full rows go to the report sections."""
    out = {}
    for e in sweep_rows or ():
        out[f"{e['workload']}:{e['linear']}"] = [e["us"], e["frac_of_roofline"]]
    if block:
        out["4:block"] = [block["us_total"], block.get("cosine_vs_dense_bf16_all_five")]
    return out


def headline_line(res: dict) -> str:
    """The one JSON line the bench prints on stdout: the contract's keys and
    the short summaries, never the detailed sections (those go to the
    Reporter). Long optional values are dropped, in reverse order of
    importance, until the line is within HEADLINE_MAX_BYTES."""
    line = {k: res[k] for k in HEADLINE_KEYS if k in res}
    for drop in ("sweep_summary", "errors", "parity", "peaks", "clocks_detail"):
        s = json.dumps(line)
        if len(s) <= HEADLINE_MAX_BYTES:
            return s
        line.pop(drop, None)
    return json.dumps(line)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-workload sweep")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--crossover", action="store_true",
                    help="also time both kernel paths at M = 1..64 on every workload shape and format")
    ap.add_argument("--report", default=None,
                    help="also write the detailed report sections (JSON lines) to this file")
    ap.add_argument("--grouped", default=None,
                    help="time the mixed block's linears of one format as one persistent grouped launch, BITS:M "
                         "(e.g. 8:1)")
    ap.add_argument("--case", default=None,
                    help="time one workload linear alone, e.g. 3:tern_m1:M=16 (workload:linear[:M=..])")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = dist_env()
    if world != args.gpus and "RANK" in os.environ:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    import torch
    torch.cuda.set_device(local_rank)
    if args.case:
        print(json.dumps(run_case(args)), flush=True)
        return 0
    if args.grouped:
        print(json.dumps(run_grouped_case(args)), flush=True)
        return 0
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res, peaks, headline_out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            report = Reporter(args.report)
            if not args.no_sweep and world == 1:
                out = report_section(res, "sweep", lambda: sweep(peaks))
                if out is not None:
                    rows, block = out
                    report("sweep", rows)
                    report("workload4_block", block)
                    res["sweep_summary"] = sweep_summary(rows, block)
                if args.crossover:
                    cross = report_section(res, "path_crossover", crossover_sweep)
                    if cross is not None:
                        report("path_crossover", cross)
                grp = report_section(res, "grouped", lambda: grouped_sweep(peaks))
                if grp is not None:
                    report("grouped", grp)
                    res.setdefault("sweep_summary", {}).update(
                        {f"grouped:{r['bits']}bit:M{r['M']}": [r["us_grouped"], r["frac_of_hbm_roofline_grouped"]]
                         for r in grp})
                fused = report_section(res, "fused_epilogues", fused_sweep)
                if fused is not None:
                    report("fused_epilogues", fused)
                pol = report_section(res, "policy_sweep", policy_sweep)
                if pol is not None:
                    report("policy_sweep", pol)
            if not args.no_cpu and world == 1:
                def cpu_legs():
                    res["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
                    report("cpu_oracle_single_core", cpu_oracle_single_core())
                    res["parity"] = headline_parity(headline_out)
                report_section(res, "cpu_baseline", cpu_legs)
            res["peaks"] = peaks
            report("clocks_detail", res.get("clocks_detail"))
            print(headline_line(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
