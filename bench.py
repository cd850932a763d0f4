#!/usr/bin/env python
"""Benchmark of the W4A16 decode path on a 70B-shaped model (synthetic weights).

Workload ("full70b"): 80 layers x {qkv 8192->10240, o 8192->8192, gate+up
8192->57344, down 28672->8192} = 68.45 G weights, bf16 ~ N(0, 0.02) drawn
on the GPU from fixed seeds, quantised to INT4 with groups of 128 (bf16 s and
z: 4.25 bits per weight, 36.4 GB), the bf16 weights then discarded.  A step is
one decode step: every one of the 320 linears at M = 1 (one bf16 activation
vector ~ N(0, 1) each), i.e. the whole packed model is streamed from HBM
once; the weights (36.4 GB) exceed L2 (126 MB) by ~290x, so no L2 flush is
needed between steps.

The line printed carries
  value      weight GB/s of the M = 1 decode step (algorithmic bytes: packed
             codes, scales, zero-points, activations and outputs) over the
             timed steps, CUDA events on the launch stream, max over ranks;
  m128       the same 320 linears at M = 128 (TFLOP/s, fraction of the bf16
             dense tensor peak);
  rows       each hot-path step measured in the same run: INT4 quantisation of
             the whole model, INT8 per-channel quantisation and the W8A16
             matmul at K = N = 8192, the W4A16 matmul per linear shape;
  e2e        the M = 1 step through the C ABI with the activations copied in
             from pinned host memory and the outputs read back every step;
  roofline   the dominant kernel (the W4A16 M = 1 matmul) against the
             measured HBM copy bandwidth;
  cpu_baseline  the CPU oracle on a bounded sample of the same workload.
`--impl reference` times the CPU oracle alone on the same metric.  Several
GPUs run independent replicas (weak scaling; no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import wq_inputs  # noqa: E402

METRIC = "W4A16 weight GB/s and % HBM peak at M=1; TFLOP/s and % tensor peak at M=128"
G = 128


M1_PROFILE = os.path.join(ROOT, "profiles", "gemv_w4a16_m1_full70b_layer.txt")
M1_SOURCES = [os.path.join(ROOT, "group_wise_weight_b200", "csrc", f)
              for f in ("wq_gemv_m1.cu", "wq_common.cuh", "wq_sm100.cuh")]


def kernel_source_hash(paths=None):
    import hashlib
    h = hashlib.sha256()
    for p in (M1_SOURCES if paths is None else paths):
        h.update(open(p, "rb").read())
    return h.hexdigest()


def m1_traffic_per_launch():
    """DRAM bytes (read + write) per launch of the M = 1 kernel, averaged over the four linear shapes of
    one layer, from the committed ncu summary -- or None when the kernel's sources have changed since
    those counters were taken (the summary records the hash of the sources it profiled)."""
    if not os.path.exists(M1_PROFILE):
        return None
    fields = {}
    for line in open(M1_PROFILE):
        if ":" in line and line.split(":", 1)[0].strip() in ("traffic_per_launch_bytes", "kernel_source_sha256"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return int(fields["traffic_per_launch_bytes"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; only scalars cross ranks)
# ---------------------------------------------------------------------------

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _scalar_device():
    """Where the scalars that cross ranks live: the GPU under NCCL, the host under gloo."""
    import torch.distributed as dist
    return torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")


def reduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=_scalar_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=_scalar_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(bytes_this_rank: float, ms_this_rank: float, world: int) -> float:
    """Whole-job GB/s of independent replicas: the bytes all ranks moved over the slowest rank's time."""
    return reduce_sum(bytes_this_rank, world) / (reduce_max(ms_this_rank, world) * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.index = vis.split(",")[local_rank] if vis else str(local_rank)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), float(p[3]), p[4], p[5], p[6], p[7], p[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        load = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        for r in load:
            for name, v in (("hw_slowdown", r[4]), ("hw_thermal_slowdown", r[5]),
                            ("sw_thermal_slowdown", r[6]), ("sw_power_cap", r[7])):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in load),
                "power_w_max": max(r[2] for r in load), "reasons": sorted(reasons), "samples": len(load)}


# ---------------------------------------------------------------------------
# the model
# ---------------------------------------------------------------------------

def workload_config(layers: int) -> dict:
    """The workload both arms report (the 70B-shaped decode step at M = 1)."""
    shapes = [(K, N) for _ in range(layers) for _, K, N in wq_inputs.FULL70B_LINEARS]
    return {"workload": f"full70b decode step: {layers} layers x (qkv 8192->10240, o 8192->8192, "
                        "gate+up 8192->57344, down 28672->8192), W4A16 g128 bf16 s/z, M=1",
            "layers": layers, "linears_per_step": len(shapes), "weights": sum(K * N for K, N in shapes),
            "bytes_per_step": sum(linear_bytes(1, N, K) for K, N in shapes)}


def linear_bytes(M, N, K, g=G):
    """Algorithmic bytes of one W4A16 call: packed codes, bf16 s and z, bf16 x and y."""
    return N * K // 2 + 2 * 2 * N * (K // g) + 2 * M * K + 2 * M * N


class Model:
    def __init__(self, layers: int, wq, device):
        self.wq = wq
        self.linears = []  # (name, K, N, q, s, z)
        quant_ms = 0.0
        quant_bytes = 0
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for layer in range(layers):
            # a layer's four bf16 weights (1.7 GB) are generated first, then quantised back to back, the way a
            # model is quantised: events around the layer's four calls
            ws, outs = [], []
            for j, (name, K, N) in enumerate(wq_inputs.FULL70B_LINEARS):
                ws.append(wq_inputs.llm_weight(N, K, wq_inputs.full70b_seed(layer, j), outlier_frac=0.0, device=device))
                outs.append((name, K, N, torch.empty((N, K // 2), dtype=torch.uint8, device=device),
                             torch.empty((N, K // G), dtype=torch.bfloat16, device=device),
                             torch.empty((N, K // G), dtype=torch.bfloat16, device=device)))
            ev0.record()
            for w, (name, K, N, q, s, z) in zip(ws, outs):
                wq.wq_quantize_int4(w, G, q, s, z)
            ev1.record()
            ev1.synchronize()
            quant_ms += ev0.elapsed_time(ev1)
            for name, K, N, q, s, z in outs:
                quant_bytes += N * K * 2 + N * K // 2 + 4 * N * (K // G)
                self.linears.append((name, K, N, q, s, z))
            del ws
        torch.cuda.empty_cache()
        self.quant_ms, self.quant_bytes = quant_ms, quant_bytes
        self.weights = sum(K * N for _, K, N, *_ in self.linears)
        # one workspace serves every call: calls run in order on one stream, each re-zeroes its tile counters,
        # and every kernel keeps those in the workspace's first 64 KB, below any partial sums
        need = max(wq.wq_gemm_workspace_bytes(M, N, K, G, 4) for M in (1, 128) for _, K, N, *_ in self.linears)
        self.ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=device)

    def buffers(self, M, device, seed=0):
        xs, ys = [], []
        for i, (name, K, N, *_) in enumerate(self.linears):
            xs.append(wq_inputs.plain_activations(M, K, seed + i, device=device))
            ys.append(torch.empty((M, N), dtype=torch.bfloat16, device=device))
        return xs, ys

    def step(self, xs, ys):
        f = self.wq.wq_gemm_w4a16
        for (name, K, N, q, s, z), x, y in zip(self.linears, xs, ys):
            f(x, q, s, z, G, y=y, workspace=self.ws)

    def step_bytes(self, M):
        return sum(linear_bytes(M, N, K) for _, K, N, *_ in self.linears)


def time_steps(fn, steps, warmup, world):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def graph_of(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the path once outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


# ---------------------------------------------------------------------------
# rows measured beside the step
# ---------------------------------------------------------------------------

def int8_rows(wq, device, copies=8, reps=5):
    """a2 + a6: INT8 per-channel quantise and W8A16 at K = N = 8192, rotating over copies (> 3x L2)."""
    K = N = 8192
    ws = [wq_inputs.block_outlier_weight(N, K, wq_inputs.SEEDS["gran"] + c, device=device) for c in range(copies)]
    qs = [torch.empty((N, K), dtype=torch.int8, device=device) for _ in range(copies)]
    ss = [torch.empty((N, 1), dtype=torch.bfloat16, device=device) for _ in range(copies)]
    x = wq_inputs.activations(1, K, 4, device=device)
    y = torch.empty((1, N), dtype=torch.bfloat16, device=device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for c in range(copies):
        wq.wq_quantize_int8(ws[c], None, qs[c], ss[c])
    torch.cuda.synchronize()
    e0.record()
    for r in range(reps):
        for c in range(copies):
            wq.wq_quantize_int8(ws[c], None, qs[c], ss[c])
    e1.record()
    e1.synchronize()
    qms = e0.elapsed_time(e1) / (reps * copies)
    del ws
    torch.cuda.empty_cache()
    wsp = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(1, N, K, K, 8)), dtype=torch.uint8, device=device)
    for c in range(copies):
        wq.wq_gemm_w8a16(x, qs[c], ss[c], None, y=y, workspace=wsp)
    torch.cuda.synchronize()
    e0.record()
    for r in range(reps * 4):
        for c in range(copies):
            wq.wq_gemm_w8a16(x, qs[c], ss[c], None, y=y, workspace=wsp)
    e1.record()
    e1.synchronize()
    gms = e0.elapsed_time(e1) / (reps * 4 * copies)
    qbytes = N * K * 2 + N * K + 2 * N
    gbytes = N * K + 2 * N + 2 * K + 2 * N
    return ({"us": qms * 1e3, "GB_s": qbytes / (qms * 1e-3) / 1e9, "shape": "K=N=8192 bf16->int8 per-channel"},
            {"us": gms * 1e3, "GB_s": gbytes / (gms * 1e-3) / 1e9, "shape": "K=N=8192 per-channel, M=1"})


def sym_int4_row(wq, device, copies=8, reps=5):
    """Symmetric INT4 quantisation (levels -7..7, g = 128) at K = N = 8192, rotating over copies (> 3x L2)."""
    K = N = 8192
    ws = [wq_inputs.llm_weight(N, K, wq_inputs.SEEDS["gran"] + 100 + c, device=device) for c in range(copies)]
    qs = [torch.empty((N, K // 2), dtype=torch.uint8, device=device) for _ in range(copies)]
    ss = [torch.empty((N, K // G), dtype=torch.bfloat16, device=device) for _ in range(copies)]
    zs = [torch.empty((N, K // G), dtype=torch.bfloat16, device=device) for _ in range(copies)]
    for c in range(copies):
        wq.wq_quantize_int4_sym(ws[c], G, qs[c], ss[c], zs[c])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for r in range(reps):
        for c in range(copies):
            wq.wq_quantize_int4_sym(ws[c], G, qs[c], ss[c], zs[c])
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / (reps * copies)
    del ws
    torch.cuda.empty_cache()
    nbytes = N * K * 2 + N * K // 2 + 4 * N * (K // G)
    return {"us": round(ms * 1e3, 2), "GB_s": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "shape": "K=N=8192 bf16->symmetric int4 g128 (zero-points 8)"}


def _time_rotating(calls, reps):
    """Average device time of one call: the calls (over rotating buffers, together larger than L2) captured
    in one CUDA graph, replayed reps times between events."""
    g = graph_of(lambda: [c() for c in calls])
    g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / (reps * len(calls))  # us


def _w4_copies(wq, N, K, g, copies, seed, device):
    out = []
    for c in range(copies):
        w = wq_inputs.llm_weight(N, K, seed + c, device=device)
        out.append(wq.wq_quantize_int4(w, g))
        del w
    torch.cuda.empty_cache()
    return out


def config_rows(wq, device, peaks, reps=10):
    """The named configurations other than the 70B step, each with its weights rotated past L2:
    decode up-projection at M = 1; the batch sweep M in {1, 8, 32, 128} on K = 8192, N = 28672 with the
    bf16 unquantised matmul (cuBLAS through torch) on the same shapes as the reference point; the
    granularity variants at K = N = 8192 (INT4 g32 at M = 1, 16; W8A16 per channel at M = 16)."""
    rows = {}
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    # config 2: K = 4096, N = 14336, M = 1, 13 copies of 31.2 MB (> 3 x L2)
    K, N = 4096, 14336
    cps = _w4_copies(wq, N, K, G, 13, 20_000, device)
    x = wq_inputs.activations(1, K, 2, device=device)
    y = torch.empty((1, N), dtype=torch.bfloat16, device=device)
    ws = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(1, N, K, G, 4)), dtype=torch.uint8, device=device)
    us = _time_rotating([lambda c=c: wq.wq_gemm_w4a16(x, *c, G, y=y, workspace=ws) for c in cps], reps)
    b = linear_bytes(1, N, K)
    rows["cfg2_decode_up_m1"] = {"us": round(us, 2), "GB_s": round(b / us / 1e3, 1),
                                 "frac_hbm": round(b / us / 1e3 / hbm, 3), "ideal_us": round(b / hbm / 1e3, 2),
                                 "shape": "K=4096 N=14336 M=1 W4A16 g128, 13 weight copies rotated"}
    # f1: the same shape through the column-scaled entry point (x / s fused into the M = 1 kernel's staging)
    sc = wq_inputs.channel_scales(K, 2).to(device)
    us_cs = _time_rotating([lambda c=c: wq.wq_gemm_w4a16_colscaled(x, sc, *c, G, y=y, workspace=ws) for c in cps], reps)
    rows["f1_colscaled_m1"] = {"us": round(us_cs, 2), "GB_s": round(b / us_cs / 1e3, 1),
                               "vs_plain": round(us_cs / us, 3),
                               "shape": "as cfg2, y = bf16(x / s) w_hat, s per input channel"}
    del cps
    torch.cuda.empty_cache()
    # config 3: K = 8192, N = 28672, 4 copies of 124.8 MB; bf16 reference: 1 copy of 470 MB
    K, N = 8192, 28672
    cps = _w4_copies(wq, N, K, G, 4, 30_000, device)
    wb = wq_inputs.llm_weight(N, K, 30_100, device=device)
    sweep = {}
    for M in (1, 8, 32, 128):
        x = wq_inputs.activations(M, K, 3, device=device)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(M, N, K, G, 4)), dtype=torch.uint8, device=device)
        us = _time_rotating([lambda c=c: wq.wq_gemm_w4a16(x, *c, G, y=y, workspace=ws) for c in cps], reps)
        yb = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        us_bf16 = _time_rotating([lambda: torch.matmul(x, wb.t(), out=yb)], reps)
        b4, bb = linear_bytes(M, N, K), N * K * 2 + 2 * M * K + 2 * M * N
        fl = 2.0 * M * N * K
        sweep[f"M{M}"] = {"w4_us": round(us, 2), "w4_GB_s": round(b4 / us / 1e3, 1), "w4_TF_s": round(fl / us / 1e6, 1),
                          "w4_frac": round(max(b4 / us / 1e3 / hbm, fl / us / 1e6 / tc), 3),
                          "bf16_us": round(us_bf16, 2), "bf16_TF_s": round(fl / us_bf16 / 1e6, 1),
                          "w4_speedup_vs_bf16": round(us_bf16 / us, 2)}
    rows["cfg3_batch_sweep"] = dict(sweep, shape="K=8192 N=28672 W4A16 g128 (4 copies rotated) vs bf16 "
                                                 "torch.matmul (cuBLAS, 470 MB weight)")
    del cps, wb
    torch.cuda.empty_cache()
    # config 4: INT4 g32 at M = 1, 16 (10 copies of 41.9 MB); W8A16 per channel at M = 16 (8 copies of 67 MB)
    K = N = 8192
    cps = []
    for c in range(10):
        w = wq_inputs.block_outlier_weight(N, K, 40_000 + c, device=device)
        cps.append(wq.wq_quantize_int4(w, 32))
        del w
    g32 = {}
    for M in (1, 16):
        x = wq_inputs.activations(M, K, 4, device=device)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(M, N, K, 32, 4)), dtype=torch.uint8, device=device)
        us = _time_rotating([lambda c=c: wq.wq_gemm_w4a16(x, *c, 32, y=y, workspace=ws) for c in cps], reps)
        b = linear_bytes(M, N, K, 32)
        g32[f"M{M}"] = {"us": round(us, 2), "GB_s": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / hbm, 3)}
    rows["cfg4_int4_g32"] = dict(g32, shape="K=N=8192 INT4 g32 (5.0 bits stored), 10 copies rotated")
    del cps
    torch.cuda.empty_cache()
    cps8 = []
    for c in range(8):
        w = wq_inputs.block_outlier_weight(N, K, 41_000 + c, device=device)
        cps8.append(wq.wq_quantize_int8(w, None))
        del w
    w8 = {}
    for M in (1, 16):
        x = wq_inputs.activations(M, K, 4, device=device)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        wsp = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(M, N, K, K, 8)), dtype=torch.uint8, device=device)
        us = _time_rotating([lambda c=c: wq.wq_gemm_w8a16(x, *c, None, y=y, workspace=wsp) for c in cps8], reps)
        b = N * K + 2 * N + 2 * M * K + 2 * M * N
        w8[f"M{M}"] = {"us": round(us, 2), "GB_s": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / hbm, 3)}
    rows["cfg4_w8a16_per_channel"] = dict(w8, shape="K=N=8192 INT8 per channel, 8 copies rotated")
    del cps8
    torch.cuda.empty_cache()
    return rows


def next_rows(wq, device, peaks, reps=5):
    """The NEXT rows on the 70B linear shapes at M = 128 (FP8 W8A8, NVFP4 W4A4: weights of one layer's four
    linears, each shape's copies rotated past L2) and the KV-cache read at the pages' geometry (batch 128,
    8,000-token contexts, 8 KV heads, 64 query heads, head_dim 128, one layer)."""
    rows = {}
    hbm = peaks["hbm_gbs"]
    M = 128
    fp8, nv = {}, {}
    tot_fp8 = tot_nv = 0.0
    for name, K, N in wq_inputs.FULL70B_LINEARS:
        copies = max(2, -(-400_000_000 // (N * K)))  # > 3 x L2 of FP8 weights
        x = wq_inputs.activations(M, K, 5, device=device)
        qx, sx = wq.wq_quantize_fp8_tensor(x)
        nx = wq.wq_quantize_nvfp4(x)
        c8, c4 = [], []
        for c in range(copies):
            w = wq_inputs.llm_weight(N, K, 50_000 + c, device=device)
            c8.append(wq.wq_quantize_fp8(w))
            c4.append(wq.wq_quantize_nvfp4(w))
            del w
        torch.cuda.empty_cache()
        y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws8 = torch.zeros(max(16, wq.wq_gemm_w8a8_fp8_workspace_bytes(M, N, K)), dtype=torch.uint8, device=device)
        ws4 = torch.zeros(max(16, wq.wq_gemm_nvfp4_workspace_bytes(M, N, K)), dtype=torch.uint8, device=device)
        us8 = _time_rotating([lambda c=c: wq.wq_gemm_w8a8_fp8(qx, sx, *c, y=y, workspace=ws8) for c in c8], reps)
        us4 = _time_rotating([lambda c=c: wq.wq_gemm_nvfp4(*nx, *c, y=y, workspace=ws4) for c in c4], reps)
        fl = 2.0 * M * N * K
        b8 = N * K + 4 * N + M * K + 2 * M * N
        b4 = N * K // 2 + N * K // 16 + M * K // 2 + M * K // 16 + 2 * M * N
        fp8[name] = {"us": round(us8, 2), "TF_s": round(fl / us8 / 1e6, 1), "GB_s": round(b8 / us8 / 1e3, 1),
                     "frac_hbm": round(b8 / us8 / 1e3 / hbm, 3)}
        nv[name] = {"us": round(us4, 2), "TF_s": round(fl / us4 / 1e6, 1), "GB_s": round(b4 / us4 / 1e3, 1),
                    "frac_hbm": round(b4 / us4 / 1e3 / hbm, 3)}
        tot_fp8 += us8
        tot_nv += us4
        del c8, c4
        torch.cuda.empty_cache()
    rows["f4_w8a8_fp8_m128"] = dict(fp8, step_ms_80_layers=round(80 * tot_fp8 / 1e3, 3),
                                    shape="E4M3 weights per channel, activations per tensor, M=128")
    rows["f2_nvfp4_m128"] = dict(nv, step_ms_80_layers=round(80 * tot_nv / 1e3, 3),
                                 shape="E2M1 + E4M3 block scales (16) + fp32 tensor scale, both operands, M=128")
    # KV-cache read: one layer at batch 128, 8,000 tokens, int4 (blocks of 128) and fp8
    g = wq_inputs.KV_70B
    B, T, H, Hq, D = g["B"], g["T"], g["H"], g["Hq"], g["D"]
    q = wq_inputs.queries(B, Hq, D, 6, device=device)
    lens = torch.full((B,), T, dtype=torch.int32, device=device)
    ws = torch.empty(wq.wq_decode_attention_workspace_bytes(B, T, H), dtype=torch.uint8, device=device)
    o = torch.empty((B, Hq, D), dtype=torch.float32, device=device)
    kv4 = []
    for j in range(2):
        c = wq_inputs.kv_cache(B, T, H, D, 60 + j, device=device)
        qq, s, z = wq.wq_quantize_int4(c.reshape(B * T * H, D), 128)
        kv4.append((qq.reshape(B, T, H, D // 2), s, z))
        del c
    torch.cuda.empty_cache()
    us = _time_rotating([lambda: wq.wq_decode_attention_int4(q, *kv4[0], *kv4[1], lens, o=o, workspace=ws)], reps)
    b = 2 * B * T * H * (D // 2 + 4) + B * Hq * D * (2 + 4)
    rows["f3_kv_int4_read"] = {"us": round(us, 1), "GB_s": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / hbm, 3),
                               "step_ms_80_layers": round(80 * us / 1e3, 2),
                               "shape": "decode attention, B=128 T=8000 H=8 Hq=64 D=128, int4 K and V (g=128)"}
    del kv4
    torch.cuda.empty_cache()
    kv8 = []
    for j in range(2):
        c = wq_inputs.kv_cache(B, T, H, D, 62 + j, device=device)
        qq, s = wq.wq_quantize_fp8_tensor(c.reshape(B * T * H, D))
        kv8.append((qq.reshape(B, T, H, D), s))
        del c
    torch.cuda.empty_cache()
    us = _time_rotating([lambda: wq.wq_decode_attention_fp8(q, *kv8[0], *kv8[1], lens, o=o, workspace=ws)], reps)
    b = 2 * B * T * H * D + B * Hq * D * (2 + 4)
    rows["f3_kv_fp8_read"] = {"us": round(us, 1), "GB_s": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / hbm, 3),
                              "step_ms_80_layers": round(80 * us / 1e3, 2),
                              "shape": "decode attention, B=128 T=8000 H=8 Hq=64 D=128, fp8 E4M3 K and V"}
    del kv8
    torch.cuda.empty_cache()
    return rows


def per_linear_us(model, xs, ys, reps=5):
    """Average device time of each linear shape at M = 1: the 80 calls of one shape replayed as a CUDA
    graph (as in the step), events around the replays."""
    out = {}
    for name, K, N in wq_inputs.FULL70B_LINEARS:
        idx = [i for i, l in enumerate(model.linears) if l[0] == name]

        def calls():
            for i in idx:
                _, K_, N_, q, s, z = model.linears[i]
                model.wq.wq_gemm_w4a16(xs[i], q, s, z, G, y=ys[i], workspace=model.ws)

        g = graph_of(calls)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        del g
        us = e0.elapsed_time(e1) * 1e3 / (reps * len(idx))
        out[name] = {"us": round(us, 2), "GB_s": round(linear_bytes(1, N, K) / (us * 1e-6) / 1e9, 1)}
    return out


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(budget_s: float, model=None, seed=0):
    """Time the CPU oracle's W4A16 path (unpack, dequantise, binary64 matmul) at M = 1 on
    row blocks of the 70B-shaped linears until about budget_s seconds of CPU work.
    Returns (GB/s of algorithmic bytes, cores used, sample description)."""
    import oracle
    oracle.set_threads(os.cpu_count() or 1)
    cores = oracle.max_threads()
    rows_per_block = 512
    done_bytes, done_s, blocks = 0, 0.0, 0
    li = 0
    while done_s < budget_s:
        name, K, N = wq_inputs.FULL70B_LINEARS[li % 4]
        li += 1
        r0 = (blocks * 997) % max(1, N - rows_per_block)
        if model is not None:
            _, K_, N_, q, s, z = [l for l in model.linears if l[0] == name][0]
            packed = q[r0:r0 + rows_per_block].cpu().numpy()
            sv = s[r0:r0 + rows_per_block].float().cpu().numpy()
            zv = z[r0:r0 + rows_per_block].float().cpu().numpy()
        else:
            w = wq_inputs.llm_weight(rows_per_block, K, 7000 + blocks, outlier_frac=0.0).float().numpy()
            codes, sv, zv = oracle.quantize_int4(w, G)
            packed = oracle.pack_int4(codes)
        x = wq_inputs.plain_activations(1, K, seed + blocks).double().numpy()
        t0 = time.perf_counter()
        codes = oracle.unpack_int4(packed, K)
        oracle.gemm_w4a16(x, codes, sv, zv, G)
        done_s += time.perf_counter() - t0
        done_bytes += linear_bytes(1, rows_per_block, K)
        blocks += 1
    desc = (f"{blocks} blocks of {rows_per_block} rows of the 70B-shaped linears at M=1 "
            f"({done_bytes / 1e9:.2f} GB of algorithmic bytes, {done_s:.1f} s)")
    return done_bytes / done_s / 1e9, cores, desc


def run_reference(args, world, rank):
    if rank != 0:
        return
    total_s, total_b = 0.0, 0.0
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        oracle_sample(per_step / 4, seed=100 + i)
    gbs = []
    for i in range(args.steps):
        v, cores, desc = oracle_sample(per_step, seed=i)
        gbs.append(v)
    value = statistics.mean(gbs)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_config(args.layers), sample="bounded CPU sample of the step per timed step"),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------

CASES = ("fp8", "nvfp4", "quant_int4", "kv_int4", "kv_fp8", "w8a16", "w8a16_m1", "w4a16_m128", "w4a16_m1",
         "w4a16_m8")


def run_case(name, wq, dev):
    """One small case of one kernel, run twice (a warm-up launch, then the one a profiler captures): the
    gate+up shape (K = 8192, N = 57,344) for the matmuls and the quantiser, 32 sequences of 8,000 tokens for
    the KV-cache read.  Prints one JSON line with the second launch's time."""
    M, N, K = 128, 57344, 8192
    calls = []
    if name in ("fp8", "nvfp4"):
        w = wq_inputs.llm_weight(N, K, 1, device=dev)
        x = wq_inputs.activations(M, K, 2, device=dev)
        if name == "fp8":
            qw, sw = wq.wq_quantize_fp8(w)
            qx, sx = wq.wq_quantize_fp8_tensor(x)
            calls.append(lambda: wq.wq_gemm_w8a8_fp8(qx, sx, qw, sw))
        else:
            nw, nx = wq.wq_quantize_nvfp4(w), wq.wq_quantize_nvfp4(x)
            calls.append(lambda: wq.wq_gemm_nvfp4(*nx, *nw))
        del w
    elif name == "quant_int4":
        w = wq_inputs.llm_weight(N, K, 3, device=dev)
        calls.append(lambda: wq.wq_quantize_int4(w, 128))
    elif name in ("kv_int4", "kv_fp8"):
        B, T, H, Hq, D = 32, 8000, 8, 64, 128
        q = wq_inputs.queries(B, Hq, D, 6, device=dev)
        lens = torch.full((B,), T, dtype=torch.int32, device=dev)
        kv = []
        for j in range(2):
            c = wq_inputs.kv_cache(B, T, H, D, 60 + j, device=dev)
            if name == "kv_int4":
                qq, s, z = wq.wq_quantize_int4(c.reshape(B * T * H, D), 128)
                kv.append((qq.reshape(B, T, H, D // 2), s, z))
            else:
                qq, s = wq.wq_quantize_fp8_tensor(c.reshape(B * T * H, D))
                kv.append((qq.reshape(B, T, H, D), s))
            del c
        fn = wq.wq_decode_attention_int4 if name == "kv_int4" else wq.wq_decode_attention_fp8
        calls.append(lambda: fn(q, *kv[0], *kv[1], lens))
    elif name in ("w8a16", "w8a16_m1"):
        w = wq_inputs.llm_weight(8192, 8192, 7, device=dev)
        q8, s8 = wq.wq_quantize_int8(w, None)
        del w
        x = wq_inputs.plain_activations(M if name == "w8a16" else 1, 8192, 8, device=dev)
        ws8 = torch.zeros(max(16, wq.wq_gemm_workspace_bytes(x.shape[0], 8192, 8192, 8192, 8)), dtype=torch.uint8,
                          device=dev)
        calls.append(lambda: wq.wq_gemm_w8a16(x, q8, s8, None, workspace=ws8))
    elif name in ("w4a16_m128", "w4a16_m1", "w4a16_m8"):
        w = wq_inputs.llm_weight(N, K, 9, outlier_frac=0.0, device=dev)
        q4, s4, z4 = wq.wq_quantize_int4(w, 128)
        del w
        x = wq_inputs.plain_activations({"w4a16_m128": M, "w4a16_m1": 1, "w4a16_m8": 8}[name], K, 10, device=dev)
        ws = torch.zeros(max(1, wq.wq_gemm_workspace_bytes(x.shape[0], N, K, 128, 4)), dtype=torch.uint8, device=dev)
        calls.append(lambda: wq.wq_gemm_w4a16(x, q4, s4, z4, 128, workspace=ws))
    else:
        raise SystemExit(f"unknown case {name}; one of {', '.join(CASES)}")
    for c in calls:
        c()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for c in calls:
        c()
    e1.record()
    e1.synchronize()
    if wq.wq_device_status() != wq.WQ_OK:
        raise SystemExit(f"case {name}: device status {wq.wq_device_status()}")
    print(json.dumps({"case": name, "us": round(e0.elapsed_time(e1) * 1e3, 2)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wq", "reference"], default="wq")
    ap.add_argument("--layers", type=int, default=wq_inputs.FULL70B_LAYERS)
    ap.add_argument("--m128-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-configuration and NEXT rows")
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one small case of one kernel twice (for a profiler capture) and exit")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_init()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import group_wise_weight_b200 as wq
    wq.lib()  # fails loudly if the CUDA library is missing
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.case:
        run_case(args.case, wq, device)
        return
    peaks = load_peaks()

    model = Model(args.layers, wq, device)
    weights_total = model.weights
    xs1, ys1 = model.buffers(1, device)
    bytes1 = model.step_bytes(1)
    launches_per_step = len(model.linears)

    step1 = (lambda: model.step(xs1, ys1))
    g1 = None if args.no_graph else graph_of(step1)
    run1 = (lambda: g1.replay()) if g1 is not None else step1

    with Clocks(local) as clk:
        ms1_rank = time_steps(run1, args.steps, args.warmup, world)
    clocks = clk.summary()
    ms1 = reduce_max(ms1_rank, world)
    t_step = ms1 / args.steps
    value = job_throughput(bytes1 * args.steps, ms1_rank, world)

    # the same step through the C ABI with host buffers: pinned H2D of every activation, D2H of every output
    x_host = torch.cat([x.reshape(-1) for x in xs1]).cpu().pin_memory()
    y_host = torch.empty(sum(y.numel() for y in ys1), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x_host, device=device)
    y_dev = torch.empty_like(y_host, device=device)
    xs_view, ys_view, o1, o2 = [], [], 0, 0
    for x, y in zip(xs1, ys1):
        xs_view.append(x_dev[o1:o1 + x.numel()].view_as(x))
        ys_view.append(y_dev[o2:o2 + y.numel()].view_as(y))
        o1 += x.numel()
        o2 += y.numel()

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        model.step(xs_view, ys_view)
        y_host.copy_(y_dev, non_blocking=True)

    ms_e2e_rank = time_steps(e2e_step, args.steps, args.warmup, world)
    ms_e2e = reduce_max(ms_e2e_rank, world)
    e2e_value = job_throughput(bytes1 * args.steps, ms_e2e_rank, world)

    lin = per_linear_us(model, xs1, ys1)

    # M = 128 over the same model
    m128_steps = args.m128_steps if args.m128_steps is not None else max(3, args.steps // 4)
    xs128, ys128 = model.buffers(128, device, seed=10_000)
    step128 = (lambda: model.step(xs128, ys128))
    g128 = None if args.no_graph else graph_of(step128)
    run128 = (lambda: g128.replay()) if g128 is not None else step128
    ms128 = reduce_max(time_steps(run128, m128_steps, 3, world), world)
    flops128 = 2.0 * 128 * weights_total
    tflops128 = reduce_sum(flops128 * m128_steps, world) / (ms128 * 1e-3) / 1e12
    del xs128, ys128, g128
    torch.cuda.empty_cache()

    q8_row, g8_row = int8_rows(wq, device)
    sym_row = sym_int4_row(wq, device)
    extra = {}
    if not args.no_rows:
        extra.update(config_rows(wq, device, peaks))
        extra.update(next_rows(wq, device, peaks))

    quant_gbs = model.quant_bytes / (model.quant_ms * 1e-3) / 1e9

    cpu = None
    if rank == 0 and world == 1:
        v, cores, desc = oracle_sample(args.cpu_seconds, model=model)
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}

    per_gpu_gbs = bytes1 / (t_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8 x s8 -> s32 per group (int4 codes x exact radix-128 digits of bf16 x), f32 across groups", "data": "synthetic",
        "config": {"workload": f"full70b decode step: {args.layers} layers x (qkv 8192->10240, o 8192->8192, "
                               "gate+up 8192->57344, down 28672->8192), W4A16 g128 bf16 s/z, M=1",
                   "layers": args.layers, "linears_per_step": launches_per_step, "weights": weights_total,
                   "bytes_per_step": bytes1, "cuda_graph": g1 is not None,
                   "l2": "inputs larger than L2 (%.1f GB of packed weights per step vs 126 MB L2)" % (bytes1 / 1e9),
                   "parallelism": f"replicas x{world}"},
        "pct_hbm_peak": round(100 * per_gpu_gbs / peaks["hbm_gbs"], 1),
        "m128": {"tflops": round(tflops128, 1), "ms_per_step": round(ms128 / m128_steps, 3),
                 "pct_bf16_peak": round(100 * tflops128 / world / peaks["bf16_tflops"], 1),
                 "peak_tflops": peaks["bf16_tflops"],
                 "peak_kind": "burst (the timed region is %d steps of ~%d ms)" % (m128_steps, round(ms128 / m128_steps)),
                 "pct_bf16_sustained_peak": round(100 * tflops128 / world / peaks["bf16_tflops_sustained"], 1),
                 "steps": m128_steps},
        "rows": {
            "a1_quantize_int4": {"GB_s": round(quant_gbs, 1), "ms_total": round(model.quant_ms, 2),
                                 "shape": "all 320 linears, bf16 -> int4 g128, each layer's four calls back to back"},
            "a2_quantize_int8": {k: (round(v, 2) if isinstance(v, float) else v) for k, v in q8_row.items()},
            "a4_w4a16_m1_per_linear": lin,
            "a5_w4a16_m128": {"tflops": round(tflops128 / world, 1)},
            "a6_w8a16_m1": {k: (round(v, 2) if isinstance(v, float) else v) for k, v in g8_row.items()},
            "f1_quantize_int4_sym": sym_row,
            **extra,
        },
        "roofline": {"bound": "hbm", "kernel": "gemv_w4a16_m1_kernel", "achieved": round(per_gpu_gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(per_gpu_gbs / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"], "traffic": m1_traffic_per_launch(),
                     "traffic_source": "profiles/gemv_w4a16_m1_full70b_layer.txt (ncu dram read + write per "
                                       "launch, mean of one layer's four linears)",
                     "bytes_per_launch_avg": bytes1 // launches_per_step},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": x_host.numel() * 2,
                "d2h_bytes_per_step": y_host.numel() * 2, "ms_per_step": round(ms_e2e / args.steps, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g1
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
