#!/usr/bin/env python
"""Benchmark of the weight-quantized matrix-vector product on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload chain8|layer|probe|quantize|quantize_fp|qvm|qmm|moe|fmt_probe]
                    [--format FMT] [--sets SET,...] [--no-shapes]

Prints ONE JSON line (rank 0).  Metric: qmv microseconds per call and achieved
HBM GB/s.  Workloads (synthetic, seeded inputs from synth/):

  chain8 (default)  affine 8-bit, group 64, bf16, M=1, K=2560, output sizes
                    N in {1, 4, 3, 5, 12, 17, 4096}; for each N a chain of 64
                    dependent calls in which call t reads the previous output
                    zero-padded (N < K) or truncated (N >= K) to K.  One step =
                    all seven chains = 448 calls.
  layer             7B-class decode layer, affine 4-bit g64 bf16: QKV 6144x4096,
                    O 4096x4096, gate+up 28672x4096, down 4096x14336, run once at
                    M=1 and once at M=8 (8 calls per step).
  probe             bandwidth probe, affine 4-bit g64 bf16, N=K=16384, M=1:
                    three back-to-back calls per step, each on its own weight copy.
  quantize          the affine quantizer (qmv_quantize_affine) on a bf16
                    16384 x 16384 matrix -> 4-bit g64 (one call per step; its
                    metric is the quantizer's microseconds per call).
  quantize_fp       the FP quantizer (qmv_quantize_fp) on a bf16 16384 x 16384
                    matrix -> NVFP4 (one call per step).
  moe               MoE decode (qmv_affine_gather): 16 tokens routed by device
                    ids to one of 64 experts of 1536 x 2048 each (one call per step).
  qmm               small-M qmm (qmv_qmm_affine): the layer's four projections
                    at M=32 (4 calls per step).
  qvm               x times W stored [K, N] (qmv_qvm_affine), affine 4-bit g64
                    bf16, N=K=16384, M=1, with the K-split workspace: three
                    back-to-back calls per step, each on its own weight copy.
  fmt_probe         the probe in one Track-1 block-scaled format (--format,
                    default mxfp4) through qmv_block_scaled, bf16, N=K=16384.

Timing: W untimed warm-up steps, then K steps.  A step is ONE CUDA graph
holding every call of the workload (dependent calls linked by programmatic
dependent launch), as a decode step would run; it is bracketed by CUDA events
on the launching stream.  L2 is flushed before every step, outside the events
(a 512 MB buffer is written, then a 256 MB buffer is read so that no dirty
line's write-back falls inside the timed region), and the weights rotate
through copies totalling more than twice the L2 so calls read from HBM.  The
timed region is bracketed by a barrier and a device synchronize; multi-GPU runs
are N independent replicas (the path has no exchange step) and report the max
over ranks.  nvidia-smi clocks are sampled (20 ms) from the graph warm-up through
the timed region.  The per-shape lines (and the roofline's dominant kernel)
come from a second pass that replays each shape's own graph alone, L2 flushed,
between a pair of CUDA events (one graph launch per shape included).

--impl reference times the fp64 CPU oracle (the only other implementation of
this operation there is) on a bounded sample of the same workload, on the host
cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
CHAIN_NS = [1, 4, 3, 5, 12, 17, 4096]
CHAIN_K, CHAIN_BITS, CHAIN_G, CHAIN_CALLS = 2560, 8, 64, 64
LAYER = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096), ("down", 4096, 14336)]
METRIC = "qmv µs/call and achieved HBM GB/s (% of B200 peak) per format/bits/shape"


def affine_bytes(M, N, K, bits, g, eb=2):
    """Algorithmic bytes of one call: packed W + scales + biases + x + y."""
    return N * K * bits // 8 + 2 * N * (K // g) * eb + M * K * eb + M * N * eb


# ------------------------------------------------------------------ peaks --
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "weight_quantized_matrix_b200", "csrc")
    for f in sorted(os.listdir(d)):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_key(workload, fmt, kernel_key):
    """The traffic.json key of one workload's dominant kernel: the same kernel
    key moves different bytes in different workloads (and formats)."""
    w = f"{workload}:{fmt}" if workload == "fmt_probe" else workload
    return f"{w} | {kernel_key}"


def traffic_for(key):
    """dram bytes per launch from the committed ncu summary, only while the
    kernel sources are unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
    except ValueError:
        return None
    e = d.get(key)
    if not e or e.get("src_sha") != source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(values, world, device):
    """Each value's maximum over all ranks (one all_reduce MAX); the values
    themselves at world 1.  The timed totals of every rank go through it, so
    a multi-GPU run reports the slowest replica."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi samples (20 ms period) taken while the GPU is under load: it
    is started before the warm-up replays and stopped after the timed steps,
    so the window covers the timed region with load on both sides."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r.split(", ") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        rows = [r for r in rows if len(r) >= 10]

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        pw = [num(r[4]) for r in rows if num(r[4]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[6:10]):
                if v.strip() == "Active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(pw) if pw else None,
                "window": "warm-up replays + timed steps (continuous load), 20 ms period"}


# -------------------------------------------------------------- workloads --
class Chain8:
    """The chained 8-bit qmv workload (one step = 7 chains x 64 calls)."""
    name = "chained affine 8-bit g64 bf16 qmv, M=1, K=2560, N in {1,4,3,5,12,17,4096}, 64 calls per N"

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        self.sets = []
        for N in CHAIN_NS:
            c = synth.affine_case(1, N, CHAIN_K, CHAIN_BITS, CHAIN_G, "bf16", seed=1000 + N)
            per = affine_bytes(1, N, CHAIN_K, CHAIN_BITS, CHAIN_G) - CHAIN_K * 2 - N * 2
            copies = int(min(CHAIN_CALLS, max(1, np.ceil(2 * L2_BYTES / per))))
            ws = []
            for i in range(copies):
                ws.append(tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                                for a in (c["w"], c["scales"], c["biases"])))
            Lb = max(N, CHAIN_K)
            x0_host = torch.zeros(Lb, dtype=torch.bfloat16).pin_memory()
            x0_host[:CHAIN_K] = torch.from_numpy(c["x"][0, 0].view(np.int16)).view(torch.bfloat16)
            x0 = x0_host.to(dev)
            bufs = [torch.zeros(Lb, dtype=torch.bfloat16, device=dev) for _ in range(2)]
            y_host = torch.empty(N, dtype=torch.bfloat16).pin_memory()
            self.sets.append(dict(N=N, ws=ws, x0=x0, x0_host=x0_host, bufs=bufs, y_host=y_host))
        self.calls_per_step = CHAIN_CALLS * len(CHAIN_NS)
        self.kernel_key = {}

    def groups(self):
        return [(f"N={s['N']}", s) for s in self.sets]

    def graph_variants(self, s):
        return 1          # the weight rotation is inside the chain

    def run_group(self, s, e2e=False, v=0):
        q, N = self.q, s["N"]
        if e2e:
            s["x0"].copy_(s["x0_host"], non_blocking=True)
        bufs, ws = s["bufs"], s["ws"]
        for t in range(CHAIN_CALLS):
            xin = s["x0"] if t == 0 else bufs[(t - 1) % 2]
            w, sc, bi = ws[t % len(ws)]
            q.qmv_affine(xin, w, sc, bi, bufs[t % 2], 1, N, CHAIN_K, CHAIN_BITS, CHAIN_G, "bf16")
        if e2e:
            s["y_host"].copy_(bufs[(CHAIN_CALLS - 1) % 2][:N], non_blocking=True)
        return CHAIN_CALLS

    def group_bytes(self, s):
        return affine_bytes(1, s["N"], CHAIN_K, CHAIN_BITS, CHAIN_G) * CHAIN_CALLS

    def group_plan(self, s):
        return self.q.qmv_describe_plan("affine", 1, s["N"], CHAIN_K, CHAIN_BITS, CHAIN_G, "bf16")

    def h2d_d2h(self):
        return (sum(CHAIN_K * 2 for _ in self.sets) + sum(max(s["N"], CHAIN_K) * 2 - CHAIN_K * 2 for s in self.sets),
                sum(s["N"] * 2 for s in self.sets))

    def config(self):
        return {"workload": self.name, "bits": 8, "group": 64, "dtype": "bf16", "M": 1, "K": CHAIN_K,
                "N": CHAIN_NS, "calls_per_N": CHAIN_CALLS, "calls_per_step": self.calls_per_step,
                "chain": "x_{t+1} = y_t zero-padded (N<K) / truncated (N>=K) to K",
                "l2": "flushed before every step (512 MB write + 256 MB read); weights rotate through copies > 2x L2"}


class Layer:
    """7B-class decode layer, 4-bit g64 bf16, the four projections at M=1 and M=8."""
    name = "7B-class decode layer, affine 4-bit g64 bf16, QKV/O/gate+up/down at M=1 and M=8"

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        self.sets = []
        for M in (1, 8):
            for name, N, K in LAYER:
                c = synth.affine_case(M, N, K, 4, 64, "bf16", seed=2000 + N + K + M)
                per = affine_bytes(M, N, K, 4, 64)
                copies = int(max(1, min(8, np.ceil(2 * L2_BYTES / per))))
                ws = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                            for a in (c["w"], c["scales"], c["biases"])) for _ in range(copies)]
                x_host = torch.from_numpy(c["x"][0].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
                x = x_host.to(dev)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
                self.sets.append(dict(name=name, M=M, N=N, K=K, ws=ws, x=x, x_host=x_host, y=y, y_host=y_host, it=0))
        self.calls_per_step = len(self.sets)

    def groups(self):
        return [(f"{s['name']} M={s['M']}", s) for s in self.sets]

    def graph_variants(self, s):
        return len(s["ws"])   # one graph per weight copy; step k replays copy k

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        w, sc, bi = s["ws"][v % len(s["ws"])]      # weight copy v: copies rotate across steps
        self.q.qmv_affine(s["x"], w, sc, bi, s["y"], s["M"], s["N"], s["K"], 4, 64, "bf16")
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return 1

    def group_bytes(self, s):
        return affine_bytes(s["M"], s["N"], s["K"], 4, 64)

    def group_plan(self, s):
        return self.q.qmv_describe_plan("affine", s["M"], s["N"], s["K"], 4, 64, "bf16")

    def h2d_d2h(self):
        return (sum(s["M"] * s["K"] * 2 for s in self.sets), sum(s["M"] * s["N"] * 2 for s in self.sets))

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "M": [1, 8],
                "shapes_NxK": [[n, k] for _, n, k in LAYER], "calls_per_step": self.calls_per_step,
                "l2": "flushed before every step (512 MB write + 256 MB read); weights rotate through copies > 2x L2"}


class Probe(Layer):
    """Sustained streaming: each step makes CALLS calls, one on each of CALLS
    distinct weight copies (151 MB each, more than L2), back to back."""
    name = "bandwidth probe, affine 4-bit g64 bf16, N=K=16384, M=1"
    CALLS = 3

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        c = synth.affine_case(1, 16384, 16384, 4, 64, "bf16", seed=3000)
        ws = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                    for a in (c["w"], c["scales"], c["biases"])) for _ in range(3)]
        x_host = torch.from_numpy(c["x"][0].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        self.sets = [dict(name="probe", M=1, N=16384, K=16384, ws=ws, x=x_host.to(dev), x_host=x_host,
                          y=torch.empty((1, 16384), dtype=torch.bfloat16, device=dev),
                          y_host=torch.empty((1, 16384), dtype=torch.bfloat16).pin_memory(), it=0)]
        self.calls_per_step = self.CALLS

    def graph_variants(self, s):
        return 1

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        for c in range(self.CALLS):
            w, sc, bi = s["ws"][c]
            self.q.qmv_affine(s["x"], w, sc, bi, s["y"], 1, s["N"], s["K"], 4, 64, "bf16")
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return self.CALLS

    def group_bytes(self, s):
        return affine_bytes(1, s["N"], s["K"], 4, 64) * self.CALLS

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "M": 1, "N": 16384, "K": 16384,
                "calls_per_step": self.CALLS,
                "l2": "flushed before every step (512 MB write + 256 MB read); each of the step's 3 calls reads "
                      "its own 151 MB weight copy"}


def bs_layout(q, fmt):
    """synth.bs_case layout arguments (element, bits, block, scale type,
    global) of a Track-1 format, from the library's qmv_format_info."""
    info = q.qmv_format_info(fmt)
    e = ("int" if fmt.startswith(("int", "mxint")) else "e5m2" if "e5m2" in fmt
         else "e2m1" if info["element_bits"] == 4 else "e4m3")
    sk = {1: "e4m3" if info["has_global"] else "e8m0", 2: "f16", 4: "f32"}[info["scale_bytes"]]
    return e, info["element_bits"], info["block"], sk, info["has_global"]


def bs_bytes(q, fmt, M, N, K, eb=2):
    """Algorithmic bytes of one Track-1 call: codes + block scales (+ the NVFP4
    global) + x + y."""
    info = q.qmv_format_info(fmt)
    return (N * K * info["element_bits"] // 8 + N * (K // info["block"]) * info["scale_bytes"]
            + (4 if info["has_global"] else 0) + M * K * eb + M * N * eb)


class FmtProbe(Probe):
    """The bandwidth probe in one Track-1 block-scaled format (--format): each
    step makes CALLS calls of qmv_block_scaled, one on each of CALLS distinct
    N = K = 16384 weight copies, M = 1, bf16 x and y."""
    FMT = "mxfp4"
    name = "bandwidth probe, mxfp4 bf16, N=K=16384, M=1"

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        self.fmt = fmt = self.FMT
        N = K = 16384
        lay = bs_layout(q, fmt)
        c = synth.bs_case(1, N, K, *lay, "bf16", seed=3200)
        ws = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                    for a in (c["w"], c["scales"])) for _ in range(self.CALLS)]
        self.g = torch.tensor([c["global"]], dtype=torch.float32, device=dev) if lay[4] else None
        x_host = torch.from_numpy(c["x"][0].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        self.sets = [dict(name=f"{fmt} probe", M=1, N=N, K=K, ws=ws, x=x_host.to(dev), x_host=x_host,
                          y=torch.empty((1, N), dtype=torch.bfloat16, device=dev),
                          y_host=torch.empty((1, N), dtype=torch.bfloat16).pin_memory(), it=0)]
        self.calls_per_step = self.CALLS

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        for c in range(self.CALLS):
            w, sc = s["ws"][c]
            self.q.qmv_block_scaled(s["x"], w, sc, self.g, s["y"], 1, s["N"], s["K"], self.fmt, "bf16")
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return self.CALLS

    def group_bytes(self, s):
        return bs_bytes(self.q, self.fmt, 1, s["N"], s["K"]) * self.CALLS

    def group_plan(self, s):
        return self.q.qmv_describe_plan(self.fmt, 1, s["N"], s["K"], dtype="bf16")

    def config(self):
        return {"workload": self.name, "format": self.fmt, "dtype": "bf16", "M": 1, "N": 16384, "K": 16384,
                "calls_per_step": self.CALLS,
                "l2": "flushed before every step (512 MB write + 256 MB read); each of the step's 3 calls reads "
                      "its own weight copy"}


class Quantize(Layer):
    """The affine quantizer on the bandwidth-probe matrix: bf16 w [16384,
    16384] -> 4-bit g64 codes, scales, biases; two weight copies (537 MB each,
    more than L2) alternate across steps."""
    name = "affine quantizer, bf16 16384 x 16384 -> 4-bit g64"

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        N = K = 16384
        g = torch.Generator(device="cpu").manual_seed(4000)
        w_host = (torch.randn((N, K), generator=g) * 0.05).to(torch.bfloat16).pin_memory()
        ws = [w_host.to(dev) for _ in range(2)]
        self.sets = [dict(name="quantize", M=1, N=N, K=K, ws=ws, w_host=w_host,
                          wq=torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                          sc=torch.empty((N, K // 64), dtype=torch.bfloat16, device=dev),
                          bi=torch.empty((N, K // 64), dtype=torch.bfloat16, device=dev),
                          sc_host=torch.empty((N, K // 64), dtype=torch.bfloat16).pin_memory(), it=0)]
        self.calls_per_step = 1

    def graph_variants(self, s):
        return len(s["ws"])

    def run_group(self, s, e2e=False, v=0):
        w = s["ws"][v % len(s["ws"])]
        if e2e:
            w.copy_(s["w_host"], non_blocking=True)
        self.q.qmv_quantize_affine(w, s["wq"], s["sc"], s["bi"], s["N"], s["K"], 4, 64, "bf16")
        if e2e:
            s["sc_host"].copy_(s["sc"], non_blocking=True)
        return 1

    def group_bytes(self, s):
        N, K = s["N"], s["K"]
        return N * K * 2 + N * K // 2 + 2 * N * (K // 64) * 2

    def group_plan(self, s):
        return "path=quantize chunk=64 maxm=0 rows_per_warp=0 bits=4 group=64 dtype=bf16"

    def h2d_d2h(self):
        s = self.sets[0]
        return s["N"] * s["K"] * 2, s["N"] * (s["K"] // 64) * 2

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "N": 16384, "K": 16384,
                "calls_per_step": 1, "bytes_per_call": "w read + codes, scales, biases written",
                "l2": "flushed before every step (512 MB write + 256 MB read); 2 weight copies alternate"}


class Qmm(Layer):
    """Small-M qmm: the 7B-class layer's four projections (4-bit g64 bf16) at
    M = 32 through qmv_qmm_affine (4 calls per step)."""
    name = "small-M qmm, 7B-class layer projections, affine 4-bit g64 bf16, M=32"
    M = 32

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        self.sets = []
        for name, N, K in LAYER:
            c = synth.affine_case(self.M, N, K, 4, 64, "bf16", seed=5000 + N + K)
            per = affine_bytes(self.M, N, K, 4, 64)
            copies = int(max(1, min(8, np.ceil(2 * L2_BYTES / per))))
            ws = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                        for a in (c["w"], c["scales"], c["biases"])) for _ in range(copies)]
            x_host = torch.from_numpy(c["x"][0].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
            self.sets.append(dict(name=name, M=self.M, N=N, K=K, ws=ws, x=x_host.to(dev), x_host=x_host,
                                  y=torch.empty((self.M, N), dtype=torch.bfloat16, device=dev),
                                  y_host=torch.empty((self.M, N), dtype=torch.bfloat16).pin_memory(), it=0))
        self.calls_per_step = len(self.sets)

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        w, sc, bi = s["ws"][v % len(s["ws"])]
        self.q.qmv_qmm_affine(s["x"], w, sc, bi, s["y"], s["M"], s["N"], s["K"], 4, 64, "bf16")
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return 1

    def group_plan(self, s):
        return self.q.qmv_describe_plan("affine", s["M"], s["N"], s["K"], 4, 64, "bf16")

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "M": self.M,
                "shapes_NxK": [[n, k] for _, n, k in LAYER], "calls_per_step": self.calls_per_step,
                "l2": "flushed before every step (512 MB write + 256 MB read); weights rotate through copies > 2x L2"}


class QuantizeFp(Quantize):
    """The block-scaled FP quantizer on the bandwidth-probe matrix: bf16 w
    [16384, 16384] -> NVFP4 (E2M1 codes, E4M3 scale per 16, FP32 global)."""
    name = "FP quantizer, bf16 16384 x 16384 -> NVFP4"

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        N = K = 16384
        g = torch.Generator(device="cpu").manual_seed(4100)
        w_host = (torch.randn((N, K), generator=g) * 0.05).to(torch.bfloat16).pin_memory()
        ws = [w_host.to(dev) for _ in range(2)]
        self.sets = [dict(name="quantize_fp", M=1, N=N, K=K, ws=ws, w_host=w_host,
                          wq=torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                          sc=torch.empty((N, K // 16), dtype=torch.uint8, device=dev),
                          gs=torch.tensor([0.05 * 4 / (6 * 448)], dtype=torch.float32, device=dev),
                          sc_host=torch.empty((N, K // 16), dtype=torch.uint8).pin_memory(), it=0)]
        self.calls_per_step = 1

    def run_group(self, s, e2e=False, v=0):
        w = s["ws"][v % len(s["ws"])]
        if e2e:
            w.copy_(s["w_host"], non_blocking=True)
        self.q.qmv_quantize_fp(w, s["wq"], s["sc"], s["gs"], s["N"], s["K"], "nvfp4", "bf16")
        if e2e:
            s["sc_host"].copy_(s["sc"], non_blocking=True)
        return 1

    def group_bytes(self, s):
        N, K = s["N"], s["K"]
        return N * K * 2 + N * K // 2 + N * (K // 16)

    def group_plan(self, s):
        return "path=quantize_fp chunk=16 maxm=0 rows_per_warp=0 mode=nvfp4 dtype=bf16"

    def h2d_d2h(self):
        s = self.sets[0]
        return s["N"] * s["K"] * 2, s["N"] * (s["K"] // 16)

    def config(self):
        return {"workload": self.name, "mode": "nvfp4", "dtype": "bf16", "N": 16384, "K": 16384,
                "calls_per_step": 1, "bytes_per_call": "w read + codes and scale bytes written",
                "l2": "flushed before every step (512 MB write + 256 MB read); 2 weight copies alternate"}


class Moe(Layer):
    """MoE decode: 16 tokens, each routed (device-side ids) to one of 64
    experts of 1536 x 2048, 4-bit g64 bf16, one qmv_affine_gather call per step.
    Algorithmic bytes: the distinct experts' weights once, plus x and y."""
    name = "MoE decode gather-qmv, 16 tokens over 64 experts of 1536x2048, affine 4-bit g64 bf16, M=1"
    T, E, N, K = 16, 64, 1536, 2048

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        T, E, N, K = self.T, self.E, self.N, self.K
        g = np.random.default_rng(6000)
        rb = K * 4 // 8
        w = torch.from_numpy(g.integers(0, 256, size=(E, N, rb), dtype=np.uint8)).to(dev)
        sc = torch.from_numpy(synth.to_storage(g.uniform(0.005, 0.02, size=(E, N, K // 64)), "bf16").view(np.int16)).view(torch.bfloat16).to(dev)
        bi = torch.from_numpy(synth.to_storage(g.normal(0.0, 0.01, size=(E, N, K // 64)), "bf16").view(np.int16)).view(torch.bfloat16).to(dev)
        ids = g.integers(0, E, size=T).astype(np.int32)
        self.distinct = len(set(ids.tolist()))
        x_host = torch.from_numpy(synth.to_storage(g.standard_normal((T, 1, K)), "bf16").view(np.int16)).view(torch.bfloat16).pin_memory()
        self.sets = [dict(name="moe", M=1, N=N, K=K, w=w, sc=sc, bi=bi, ids=torch.from_numpy(ids).to(dev),
                          x=x_host.to(dev), x_host=x_host, y=torch.empty((T, 1, N), dtype=torch.bfloat16, device=dev),
                          y_host=torch.empty((T, 1, N), dtype=torch.bfloat16).pin_memory(), it=0)]
        self.calls_per_step = 1

    def graph_variants(self, s):
        return 1

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        self.q.qmv_affine_gather(s["x"], s["w"], s["sc"], s["bi"], s["ids"], s["y"], 1, self.N, self.K, 4, 64, "bf16",
                                 self.T, self.E)
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return 1

    def group_bytes(self, s):
        N, K = self.N, self.K
        return self.distinct * (N * K // 2 + 2 * N * (K // 64) * 2) + self.T * (K + N) * 2

    def group_plan(self, s):
        return "path=gather chunk=32 maxm=1 rows_per_warp=0 kernel=CUDA-core row-tiled bits=4 group=64 dtype=bf16"

    def h2d_d2h(self):
        return self.T * self.K * 2, self.T * self.N * 2

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "M": 1, "N": self.N, "K": self.K,
                "tokens": self.T, "experts": self.E, "distinct_experts": self.distinct, "calls_per_step": 1,
                "l2": "flushed before every step (512 MB write + 256 MB read)"}


class Qvm(Layer):
    """qvm on the bandwidth-probe matrix stored [K, N]: x [1, 16384] times
    4-bit g64 W [16384, 16384], bf16, with the K-split workspace; each step
    makes CALLS calls, one on each of CALLS distinct weight copies (151 MB
    each, more than L2), back to back."""
    name = "qvm, affine 4-bit g64 bf16, W stored [K, N], N=K=16384, M=1"
    CALLS = 3

    def __init__(self, q, torch, dev):
        self.q, self.torch = q, torch
        N = K = 16384
        c = synth.qvm_case(1, N, K, 4, 64, "bf16", seed=3100)
        ws = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev)
                    for a in (c["w"], c["scales"], c["biases"])) for _ in range(self.CALLS)]
        x_host = torch.from_numpy(c["x"].view(np.int16).copy()).view(torch.bfloat16).pin_memory()
        self.sets = [dict(name="qvm", M=1, N=N, K=K, ws=ws, x=x_host.to(dev), x_host=x_host,
                          work=torch.zeros(q.qmv_qvm_workspace_bytes(1, N), dtype=torch.uint8, device=dev),
                          y=torch.empty((1, N), dtype=torch.bfloat16, device=dev),
                          y_host=torch.empty((1, N), dtype=torch.bfloat16).pin_memory(), it=0)]
        self.calls_per_step = self.CALLS

    def graph_variants(self, s):
        return 1

    def run_group(self, s, e2e=False, v=0):
        if e2e:
            s["x"].copy_(s["x_host"], non_blocking=True)
        for c in range(self.CALLS):
            w, sc, bi = s["ws"][c]
            self.q.qmv_qvm_affine(s["x"], w, sc, bi, s["y"], 1, s["N"], s["K"], 4, 64, "bf16", workspace=s["work"])
        if e2e:
            s["y_host"].copy_(s["y"], non_blocking=True)
        return self.CALLS

    def group_bytes(self, s):
        return affine_bytes(1, s["N"], s["K"], 4, 64) * self.CALLS

    def group_plan(self, s):
        return "path=qvm chunk=32 maxm=1 rows_per_warp=0 bits=4 group=64 dtype=bf16"

    def h2d_d2h(self):
        s = self.sets[0]
        return s["K"] * 2, s["N"] * 2

    def config(self):
        return {"workload": self.name, "bits": 4, "group": 64, "dtype": "bf16", "M": 1, "N": 16384, "K": 16384,
                "calls_per_step": self.CALLS,
                "l2": "flushed before every step (512 MB write + 256 MB read); each of the step's 3 calls reads "
                      "its own 151 MB weight copy"}


WORKLOADS = {"chain8": Chain8, "layer": Layer, "probe": Probe, "quantize": Quantize, "qvm": Qvm, "qmm": Qmm, "moe": Moe,
             "quantize_fp": QuantizeFp, "fmt_probe": FmtProbe}


# ------------------------------------------- per format / bits / shape --
DT_BYTES = {"f32": 4, "f16": 2, "bf16": 2}
FP_MODES = ("mxfp4", "nvfp4", "mxfp8")


def fp_bytes(M, N, K, mode, batch=1, eb=2):
    """Algorithmic bytes of one FP call: codes + block scales (+ the NVFP4
    global) + x + y, times the batch."""
    bits, blk = synth.FP_BITS[mode], synth.FP_BLOCK[mode]
    per = N * K * bits // 8 + N * (K // blk) + (4 if mode == "nvfp4" else 0) + M * K * eb + M * N * eb
    return per * batch


def _copies(torch, dev, arrays, n):
    """n device copies of the same host arrays (distinct addresses, so each
    call of a rotation reads its weights from HBM after an L2 flush)."""
    base = [torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)).to(dev) for a in arrays]
    return [tuple(b) for b in [base]] + [tuple(b.clone() for b in base) for _ in range(n - 1)]


def _rotation(wbytes, cap=64, least=1):
    return int(max(least, min(cap, np.ceil(2 * L2_BYTES / max(wbytes, 1)))))


SHAPE_SETS = ("c1", "probe", "layer", "fp_chain", "fp_probe", "formats", "sweep")


def alu_peak_tflops(torch, dev, sm_max_mhz):
    """FP32 CUDA-core roof of this GPU: SMs x 128 FP32 lanes x 2 flops (FMA) x
    the highest SM clock seen (B200: 148 x 128 x 2 x 1965 MHz = 74.4 TFLOP/s)."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = sm_max_mhz or 1965.0
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def alu_roof(flops, us, alu_peak):
    """The FP32-ALU roof fields of a per-shape line (M >= 4 only): the dot
    products' 2*M*N*K flops at the measured time, against alu_peak.  Context:
    the tensor-core kernels do not run the products on that pipe."""
    if not flops or not alu_peak:
        return {}
    tf = flops / (us * 1e-6) / 1e12
    return {"alu_tflops": round(tf, 2), "alu_frac": round(tf / alu_peak, 4)}


def shape_lines(q, torch, dev, stream, flush, flush_rd, peak, sets=None, alu_peak=None):
    """Throughput per format, bits and shape (the metric's breakdown), each
    line from ONE CUDA graph of R calls back to back on R weight copies that
    together exceed twice the L2 (or, for the chained FP shapes, 64 dependent
    calls), replayed after an L2 flush between a pair of events on the
    launching stream; us_per_call = median replay time / R.  Sets: c1 (the
    small 4-bit config), probe (16384^2 4-bit, M = 1 and 8), layer (the 7B
    projections, M = 1 and 8), fp_chain (MXFP4 / NVFP4 / MXFP8 chains of the
    pages' shapes), fp_probe (16384^2 in each FP format, M = 1), sweep
    (2/3/5/6-bit x group 32/64/128 x f32/f16/bf16 x M = 1, 4 at N = K = 4096)
    and formats (every Track-1 block-scaled format at N = K = 8192, M = 1
    bf16, through qmv_block_scaled).  Each line also carries the 5th / 95th
    percentile of its replays, and lines with M >= 4 the FP32-ALU roof: 2*M*N*K
    flops per call against alu_peak (TFLOP/s)."""
    lines = []
    sets = sets or SHAPE_SETS

    def timed(tag, label, R, launch, nbytes, plan, reps=7, flops=None):
        for r in range(R):                          # eager warm-up (kernel attributes)
            launch(r)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(R):
                launch(r)
        g.replay(); g.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps):
            flush.fill_(i & 0xFF)
            flush_rd.max()
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        per = np.array([a.elapsed_time(b) for a, b in ev]) * 1e3 / R      # us per call, each replay
        us = float(np.median(per))
        gbs = nbytes / (us * 1e-6) / 1e9
        line = {"set": tag, "shape": label, "us_per_call": round(us, 3), "us_p5": round(float(np.percentile(per, 5)), 3),
                "us_p95": round(float(np.percentile(per, 95)), 3), "GB_s": round(gbs, 1),
                "frac_of_hbm": round(gbs / peak, 4), "calls_per_graph": R, "plan": plan}
        line.update(alu_roof(flops, us, alu_peak))
        lines.append(line)
        del g

    def affine(tag, label, M, N, K, bits, G, dtype, least=1, cap=64):
        c = synth.affine_case(M, N, K, bits, G, dtype, seed=7000 + N + K + 13 * bits + G + M)
        wb = affine_bytes(M, N, K, bits, G, DT_BYTES[dtype]) - M * K * DT_BYTES[dtype] - M * N * DT_BYTES[dtype]
        R = _rotation(wb, cap, least)
        ws = _copies(torch, dev, (c["w"], c["scales"], c["biases"]), R)
        x = torch.from_numpy(c["x"][0].view(np.uint8).reshape(-1).copy()).to(dev)
        y = torch.empty(M * N * DT_BYTES[dtype], dtype=torch.uint8, device=dev)

        def launch(r):
            w, sc, bi = ws[r]
            q.qmv_affine(x, w, sc, bi, y, M, N, K, bits, G, dtype)
        timed(tag, label, R, launch, affine_bytes(M, N, K, bits, G, DT_BYTES[dtype]),
              q.qmv_describe_plan("affine", M, N, K, bits, G, dtype), flops=2 * M * N * K if M >= 4 else None)

    with torch.cuda.stream(stream):
        if "c1" in sets:
            affine("c1", "affine b4 g64 bf16 M=1 N=256 K=512", 1, 256, 512, 4, 64, "bf16")
        if "probe" in sets:
            for M in (1, 8):
                affine("probe", f"affine b4 g64 bf16 M={M} N=K=16384", M, 16384, 16384, 4, 64, "bf16", least=3)
        if "layer" in sets:
            for M in (1, 8):
                for name, N, K in LAYER:
                    affine("layer", f"{name} {N}x{K} b4 g64 bf16 M={M}", M, N, K, 4, 64, "bf16", least=3)
        if "fp_chain" in sets:
            for mode in FP_MODES:
                for (N, K, B) in ((5, 1024, 2), (12, 4096, 1)):
                    c = synth.fp_case(1, N, K, mode, "bf16", seed=7100 + N + K, batch=B)
                    ws = _copies(torch, dev, (c["w"], c["scales"]), CHAIN_CALLS)
                    gs = (torch.tensor(np.full(B, c["global"], dtype=np.float32), device=dev)
                          if mode == "nvfp4" else None)
                    bufs = [torch.zeros(B * K, dtype=torch.bfloat16, device=dev) for _ in range(2)]
                    x0 = torch.from_numpy(c["x"].view(np.int16).reshape(-1).copy()).view(torch.bfloat16).to(dev)

                    def launch(t, ws=ws, gs=gs, bufs=bufs, x0=x0, N=N, K=K, B=B, mode=mode):
                        xin = x0 if t == 0 else bufs[(t - 1) % 2]
                        w, sc = ws[t]
                        q.qmv_fp_batched(xin, w, sc, gs, bufs[t % 2], 1, N, K, mode, "bf16", B, True)
                    timed("fp_chain", f"{mode} chain N={N} K={K} batch={B}", CHAIN_CALLS, launch,
                          fp_bytes(1, N, K, mode, B), q.qmv_describe_plan(mode, 1, N, K, 0, 0, "bf16"))
        if "fp_probe" in sets:
            for mode in FP_MODES:
                N = K = 16384
                c = synth.fp_case(1, N, K, mode, "bf16", seed=7200)
                R = 3
                ws = _copies(torch, dev, (c["w"], c["scales"]), R)
                gs = torch.tensor([c["global"]], dtype=torch.float32, device=dev) if mode == "nvfp4" else None
                x = torch.from_numpy(c["x"][0].view(np.int16).reshape(-1).copy()).view(torch.bfloat16).to(dev)
                y = torch.empty(N, dtype=torch.bfloat16, device=dev)

                def launch(r, ws=ws, gs=gs, x=x, y=y, mode=mode):
                    w, sc = ws[r]
                    q.qmv_fp(x, w, sc, gs, y, 1, 16384, 16384, mode, "bf16")
                timed("fp_probe", f"{mode} M=1 N=K=16384", R, launch, fp_bytes(1, N, K, mode),
                      q.qmv_describe_plan(mode, 1, N, K, 0, 0, "bf16"))
        if "formats" in sets:
            for fmt in q.FORMATS:
                N = K = 8192
                lay = bs_layout(q, fmt)
                c = synth.bs_case(1, N, K, *lay, "bf16", seed=7300 + q.FORMATS[fmt])
                wb = bs_bytes(q, fmt, 0, N, K)                     # codes + scales (M = 0: no x, y)
                R = _rotation(wb, 64, 3)
                ws = _copies(torch, dev, (c["w"], c["scales"]), R)
                gs = torch.tensor([c["global"]], dtype=torch.float32, device=dev) if lay[4] else None
                x = torch.from_numpy(c["x"][0].view(np.int16).reshape(-1).copy()).view(torch.bfloat16).to(dev)
                y = torch.empty(N, dtype=torch.bfloat16, device=dev)

                def launch(r, ws=ws, gs=gs, x=x, y=y, fmt=fmt):
                    w, sc = ws[r]
                    q.qmv_block_scaled(x, w, sc, gs, y, 1, 8192, 8192, fmt, "bf16")
                timed("formats", f"{fmt} M=1 N=K=8192 bf16", R, launch, bs_bytes(q, fmt, 1, N, K),
                      q.qmv_describe_plan(fmt, 1, N, K, dtype="bf16"))
        if "sweep" in sets:
            for bits in (2, 3, 5, 6):
                for G in (32, 64, 128):
                    for dtype in ("f32", "f16", "bf16"):
                        for M in (1, 4):
                            affine("sweep", f"affine b{bits} g{G} {dtype} M={M} N=K=4096", M, 4096, 4096, bits, G,
                                   dtype)
    return lines


# ---------------------------------------------------------------- our arm --
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: a CUDA device is required for --impl ours")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    import weight_quantized_matrix_b200 as q   # fails loudly if libqmv.so is missing

    wl = WORKLOADS[args.workload](q, torch, dev)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    # after the write pass, a read pass over another buffer larger than the L2
    # evicts the dirty lines, so their write-back is not charged to the timed
    # kernels; the L2 then holds only unrelated clean lines
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    groups = wl.groups()
    W = max(3, args.warmup)

    with torch.cuda.stream(stream):
        # eager warm-up through the public API (also sets kernel attributes)
        for k in range(W):
            for _, s in groups:
                wl.run_group(s, v=k)
        torch.cuda.synchronize()
        # One CUDA graph per STEP (all groups, their dependent launches with
        # programmatic-dependent-launch edges), one per weight-copy variant,
        # as a decode step would run; and one graph per group for the
        # per-shape breakdown.
        nv = max(wl.graph_variants(s) for _, s in groups)
        step_graphs = []
        for v in range(nv):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _, s in groups:
                    wl.run_group(s, v=v)
            step_graphs.append(g)
        group_graphs = []
        for _, s in groups:
            gs = []
            for v in range(wl.graph_variants(s)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    wl.run_group(s, v=v)
                gs.append(g)
            group_graphs.append(gs)
        clk = ClockSampler(local_rank)
        clk.start()
        t_load = time.perf_counter()
        k = 0
        while k < W or time.perf_counter() - t_load < 0.3:     # warm-up replays, >= 0.3 s of load
            step_graphs[k % nv].replay()
            k += 1
            if k % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()

        def timed(e2e):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            for k in range(args.steps):
                flush.fill_(k & 0xFF)                   # L2 flush, outside the events
                flush_rd.max()
                ev[k][0].record(stream)
                if e2e:
                    for _, s in groups:
                        wl.run_group(s, e2e=True, v=k)  # public API, host copies included
                else:
                    step_graphs[k % nv].replay()
                ev[k][1].record(stream)
            torch.cuda.synchronize()
            wall = time.perf_counter() - t0
            clocks = clk.stop() if not e2e else None
            if world > 1:
                dist.barrier()
            return np.array([a.elapsed_time(b) for (a, b) in ev]), wall, clocks   # ms per step

        step_ms, wall, clocks = timed(False)
        step_ms_e2e, _, _ = timed(True)

        # per-shape breakdown (not the headline): each group's own graph, L2
        # flushed before every replay, timed alone between a pair of events
        # (so it also carries one graph launch per group)
        reps = max(8, nv)
        per_group = []
        for gi, (_, s) in enumerate(groups):
            gs = group_graphs[gi]
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for r in range(reps):
                flush.fill_(r & 0xFF)
                flush_rd.max()
                ev[r][0].record(stream)
                gs[r % len(gs)].replay()
                ev[r][1].record(stream)
            torch.cuda.synchronize()
            per_group.append(np.array([a.elapsed_time(b) for a, b in ev]))   # ms per group replay
        del step_graphs, group_graphs

    tot_ms, tot_ms_e2e = max_over_ranks([float(step_ms.sum()), float(step_ms_e2e.sum())], world, dev)
    calls = wl.calls_per_step * args.steps * world
    us_per_call = tot_ms * 1e3 / calls
    us_per_call_e2e = tot_ms_e2e * 1e3 / calls

    # per-shape results and the dominant kernel (largest share of device time)
    shapes, by_kernel = [], {}
    peak, peak_kind = peaks()
    alu_peak = alu_peak_tflops(torch, dev, (clocks or {}).get("sm_max_mhz"))
    for gi, (label, s) in enumerate(groups):
        ms = float(np.mean(per_group[gi]))
        n = wl.calls_per_step // len(groups)        # calls per group replay
        b = wl.group_bytes(s)
        plan = wl.group_plan(s)
        kern = " ".join(w for w in plan.split() if w.split("=")[0] in ("path", "chunk", "maxm", "rows_per_warp"))
        gbs = b / (ms * 1e-3) / 1e9
        line = {"set": args.workload, "shape": label, "us_per_call": round(ms * 1e3 / n, 3),
                "us_p5": round(float(np.percentile(per_group[gi], 5)) * 1e3 / n, 3),
                "us_p95": round(float(np.percentile(per_group[gi], 95)) * 1e3 / n, 3),
                "GB_s": round(gbs, 1), "frac_of_hbm": round(gbs / peak, 4), "plan": plan}
        if isinstance(s, dict) and s.get("M", 0) >= 4 and "N" in s and "K" in s:
            line.update(alu_roof(2 * s["M"] * s["N"] * s["K"] * n, ms * 1e3, alu_peak))
        shapes.append(line)
        k = by_kernel.setdefault(kern, {"ms": 0.0, "launches": 0, "bytes": 0})
        k["ms"] += ms; k["launches"] += n; k["bytes"] += b
    dom_plan, dom = max(by_kernel.items(), key=lambda kv: kv[1]["ms"])
    achieved = dom["bytes"] / (dom["ms"] * 1e-3) / 1e9
    traffic = traffic_for(traffic_key(args.workload, args.format, dom_plan))
    h2d, d2h = wl.h2d_d2h()
    out = {
        "metric": METRIC, "value": round(us_per_call, 4), "unit": "us/call", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(tot_ms / args.steps, 4),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in/out, fp32 accumulate",
        "data": "synthetic (seeded)", "config": dict(wl.config(), parallelism=f"replicas x{world}"),
        "e2e": {"value": round(us_per_call_e2e, 4), "unit": "us/call", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": wl.calls_per_step * args.steps,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind,
                     "kernel": dom_plan, "kernel_share": round(dom["ms"] / sum(v["ms"] for v in by_kernel.values()), 3),
                     "bytes_per_launch": dom["bytes"] // max(1, dom["launches"]),
                     "avg_launch_us": round(dom["ms"] * 1e3 / max(1, dom["launches"]), 3)},
        "spread": {"unit": "us/call", "over": f"{args.steps} timed steps, this rank",
                   "p5": round(float(np.percentile(step_ms, 5)) * 1e3 / wl.calls_per_step, 4),
                   "p50": round(float(np.percentile(step_ms, 50)) * 1e3 / wl.calls_per_step, 4),
                   "p95": round(float(np.percentile(step_ms, 95)) * 1e3 / wl.calls_per_step, 4)},
        "clocks": clocks, "shapes": shapes, "wall_s_timed": round(wall, 3),
    }
    if args.workload == "chain8" and not args.no_shapes:
        # the metric's breakdown per format / bits / shape; not part of `value`
        out["shapes"] += shape_lines(q, torch, dev, stream, flush, flush_rd, peak, args.sets, alu_peak)
    if rank == 0:
        out["cpu_baseline"] = (cpu_baseline(args.workload) if not args.no_cpu_baseline
                               else {"value": None, "unit": "us/call", "kind": "oracle",
                                     "sample": "skipped (--no-cpu-baseline)"})
        print(json.dumps(out), flush=True)


# ------------------------------------------------- oracle (CPU) baseline --
def _oracle_sample(workload, budget_s=12.0, threads=None):
    """Time the oracle, as it stands, on a bounded sample of the workload and
    scale to microseconds per call of the full workload."""
    import oracle
    threads = threads or os.cpu_count() or 1
    t_by = {}
    if workload == "quantize":
        return _oracle_quantize_sample(budget_s, threads)
    if workload == "qvm":
        return _oracle_qvm_sample(budget_s, threads)
    if workload == "quantize_fp":
        return _oracle_quantize_fp_sample(budget_s, threads)
    if workload == "fmt_probe":
        return _oracle_fmt_probe_sample(budget_s, threads)
    if workload == "chain8":
        spec = [(1, N, CHAIN_K, CHAIN_BITS, CHAIN_G, CHAIN_CALLS) for N in CHAIN_NS]
    elif workload == "layer":
        spec = [(M, N, K, 4, 64, 1) for M in (1, 8) for _, N, K in LAYER]
    elif workload == "qmm":
        spec = [(32, N, K, 4, 64, 1) for _, N, K in LAYER]
    elif workload == "moe":
        spec = [(1, 1536, 2048, 4, 64, 16)]
    else:
        spec = [(1, 16384, 16384, 4, 64, 1)]
    per_shape_budget = budget_s / len(spec)
    sample = []
    total_us = 0.0
    for (M, N, K, bits, g, calls) in spec:
        c = synth.affine_case(M, N, K, bits, g, "bf16", seed=7)
        args = (c["x"][0], c["w"][0], c["scales"][0], c["biases"][0], M, N, K, bits, g, "bf16")
        rows_all = list(range(N))
        # grow the row sample until the budget for this shape is used
        nrows = min(N, 64)
        t0 = time.perf_counter()
        oracle.qmv_affine(*args, rows=rows_all[:nrows], threads=threads)
        dt = time.perf_counter() - t0
        while nrows < N and dt < per_shape_budget / 4:
            nrows = min(N, nrows * 4)
            t0 = time.perf_counter()
            oracle.qmv_affine(*args, rows=rows_all[:nrows], threads=threads)
            dt = time.perf_counter() - t0
        us_call = dt * 1e6 * (N / nrows)
        total_us += us_call * calls
        sample.append(f"M={M} N={N} K={K}: {nrows}/{N} rows, {dt:.3f}s")
    ncalls = 1 if workload == "moe" else sum(s[-1] for s in spec)     # moe: one call = all its tokens
    return total_us / ncalls, threads, "; ".join(sample)


def _oracle_fmt_probe_sample(budget_s, threads):
    """The oracle's Track-1 qmv (oracle.qmv_block_scaled) on a growing row
    sample of the format probe's 16384 x 16384 matrix, scaled to one call."""
    import oracle
    fmt = FmtProbe.FMT
    N = K = 16384
    c = synth.bs_case(1, N, K, *oracle.TRACK1[fmt], "bf16", seed=3200)
    args = (c["x"][0], c["w"][0], c["scales"][0], c["global"], 1, N, K, fmt, "bf16")
    nrows = 16
    while True:
        t0 = time.perf_counter()
        oracle.qmv_block_scaled(*args, rows=range(nrows), threads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or nrows >= N:
            break
        nrows = min(N, nrows * 4)
    return dt * 1e6 * (N / nrows), threads, f"{fmt} N={N} K={K} bf16: {nrows}/{N} rows, {dt:.3f}s"


def _oracle_quantize_fp_sample(budget_s, threads):
    """The oracle FP quantizer (NVFP4) on a growing row sample of the 16384 x
    16384 bf16 matrix, scaled to one full call."""
    import oracle
    N = K = 16384
    rng = np.random.default_rng(9)
    w = rng.standard_normal((N, K), dtype=np.float32).astype(np.float32) * np.float32(0.05)
    wb = (w.view(np.uint32) >> 16).astype(np.uint16)
    nrows = 16
    while True:
        t0 = time.perf_counter()
        oracle.quantize_fp(np.ascontiguousarray(wb[:nrows]), nrows, K, "nvfp4", "bf16",
                           global_scale=np.float32(0.05 * 4 / (6 * 448)), threads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or nrows >= N:
            break
        nrows = min(N, nrows * 4)
    return dt * 1e6 * (N / nrows), threads, f"NVFP4 N={N} K={K} bf16: {nrows}/{N} rows, {dt:.3f}s"


def _oracle_qvm_sample(budget_s, threads):
    """The oracle qvm on a growing column sample of the 16384 x 16384 4-bit
    matrix, scaled to one full call."""
    import oracle
    N = K = 16384
    c = synth.qvm_case(1, N, K, 4, 64, "bf16", seed=3100)
    args = (c["x"], c["w"], c["scales"], c["biases"], 1, N, K, 4, 64, "bf16")
    ncols = 16
    while True:
        t0 = time.perf_counter()
        oracle.qvm_affine(*args, cols=range(ncols), threads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or ncols >= N:
            break
        ncols = min(N, ncols * 4)
    return dt * 1e6 * (N / ncols), threads, f"qvm N={N} K={K} 4-bit g64 bf16: {ncols}/{N} columns, {dt:.3f}s"


def _oracle_quantize_sample(budget_s, threads):
    """The oracle quantizer on a growing row sample of the 16384 x 16384 bf16
    matrix, scaled to one full call."""
    import oracle
    N = K = 16384
    rng = np.random.default_rng(9)
    w = rng.standard_normal((N, K), dtype=np.float32).astype(np.float32) * np.float32(0.05)
    wb = (w.view(np.uint32) >> 16).astype(np.uint16)                 # bf16 bit patterns (truncated sample data)
    nrows = 16
    while True:
        t0 = time.perf_counter()
        oracle.quantize_affine(np.ascontiguousarray(wb[:nrows]), nrows, K, 4, 64, "bf16", threads=threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or nrows >= N:
            break
        nrows = min(N, nrows * 4)
    return dt * 1e6 * (N / nrows), threads, f"N={N} K={K} 4-bit g64 bf16: {nrows}/{N} rows, {dt:.3f}s"


def cpu_baseline(workload):
    v, cores, sample = _oracle_sample(workload, budget_s=12.0)
    v1, _, sample1 = _oracle_sample(workload, budget_s=4.0, threads=1)
    return {"value": round(v, 2), "unit": "us/call", "cores": cores, "kind": "oracle",
            "sample": "fp64 C oracle over row samples of every shape, scaled to full calls: " + sample,
            "value_1thread": round(v1, 2), "sample_1thread": sample1}


def run_reference(args, rank, world):
    """The oracle on the host cores, rank 0 only.  Each step is one bounded
    sample of the workload; the per-step budget keeps the whole run near a
    minute whatever --steps is."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    budget = max(0.2, min(6.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        _oracle_sample(args.workload, budget_s=budget)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, cores, sample = _oracle_sample(args.workload, budget_s=budget)
        vals.append(v)
    v = float(np.mean(vals))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": "us/call", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic (seeded)",
        "config": {"workload": wl.name},
        "ms_per_step": round((time.perf_counter() - t0) * 1e3 / max(1, args.steps), 2),
        "cpu_baseline": {"value": round(v, 2), "unit": "us/call", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 2), "unit": "us/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="chain8")
    ap.add_argument("--no-shapes", action="store_true",
                    help="chain8 only: skip the per format / bits / shape lines")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the oracle on the host cores (profiling runs)")
    ap.add_argument("--format", default="mxfp4",
                    help="fmt_probe: the Track-1 format (a qmv_block_scaled name, e.g. mxfp4, nvfp8, int4)")
    ap.add_argument("--sets", type=lambda v: tuple(v.split(",")), default=None,
                    help="chain8: comma-separated subset of the shape sets " + ",".join(SHAPE_SETS))
    args = ap.parse_args()
    FmtProbe.FMT = args.format
    FmtProbe.name = f"bandwidth probe, {args.format} bf16, N=K=16384, M=1"
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
