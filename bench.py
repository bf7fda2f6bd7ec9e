#!/usr/bin/env python
"""Throughput of the group-wise affine quantized products on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nvq|reference]

One step is one pass of the hot path over one batch of the headline workload:
a 4-bit, group-64 decode product y = x . w^T with x [1, 4096] bf16 and
W [14336, 4096] (Llama-8B MLP shape) on each of the weight copies the batch
holds (as many copies as it takes to touch more than 3x the L2 cache before a
copy is read again: 13 on B200), i.e. one nv_qmm call per copy. The JSON line
reports HBM GB/s of algorithmic bytes (codes + scales + biases + x + y); the
other workloads (8-bit and transposed decode, few rows, prefill, mixture of
experts with 4-bit and with bf16 weights, dequantization to bf16) are
measured in the same run, with the same step definition, and reported under
"also".

Timing: W untimed warm-up steps, then K timed steps captured in CUDA graphs and
bracketed by a barrier and torch.cuda.synchronize(); device time from CUDA
events on the launching stream; max over ranks. Within a step the calls rotate
over the weight copies, so the set touched between two uses of a copy exceeds
the L2 cache.
Multi-GPU runs are independent replicas (the product does not shard here):
value = bytes processed by all ranks / max time. After timing, each workload's
own output is checked against plain torch arithmetic on the GPU
(`output_check` in the JSON line).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from group_wise_affine_dequant_b200 import workloads as W  # noqa: E402

METRIC = "4-bit g64 qmm: decode HBM GB/s (% of 8 TB/s); prefill TFLOP/s; gather_qmm tok/s"
HBM_NOMINAL_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def qbytes(N, K, bits, gs, sbytes=2):
    """Bytes of a quantized [N, K] matrix: codes + scales + biases."""
    return N * K * bits // 8 + 2 * (N * K // gs) * sbytes


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(v: float, ws: int, device) -> float:
    """The largest of every rank's value (every rank gets it): the job's time
    is its slowest replica's. A collective on `device` (cuda for NCCL, cpu
    for gloo); a plain return on one rank."""
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_rate(ws: int, units_per_step: float, steps: int, ms_max: float) -> float:
    """Whole-job rate of N independent replicas: the units all ranks processed
    divided by the slowest rank's time (per second)."""
    return ws * units_per_step * steps / (ms_max / 1e3)


# ------------------------------------------------------------ output checks
# Each timed workload's own output is checked after timing against plain torch
# arithmetic on the GPU (codes unpacked with shifts and masks, fp32 products):
# a sanity check of the timed run, independent of the library's kernels. The
# parity proper is the test suite's comparison with the oracle.
def unpack_dequant(codes, scales, biases, gs, bits):
    """w = scale * code + bias in fp32, [..., rows, cols], with torch ops."""
    per = 32 // bits
    c = codes.to(torch.int64) & 0xFFFFFFFF
    sh = torch.arange(per, device=codes.device, dtype=torch.int64) * bits
    v = ((c.unsqueeze(-1) >> sh) & ((1 << bits) - 1)).flatten(-2).to(torch.float32)
    return v * scales.float().repeat_interleave(gs, -1) + biases.float().repeat_interleave(gs, -1)


def worst_ratio(y, x, w):
    """max |y - x.w^T| / (4e-3 * sum|x||w| + 1e-5); <= 1 passes (bf16 tolerance)."""
    ref = x.float() @ w.T
    tol = 4e-3 * (x.float().abs() @ w.abs().T) + 1e-5
    return float(((y.float() - ref).abs() / tol).max())


def _fp_tables(dev):
    """Values of every E2M1 code (16) and E4M3 code (256), from the bit fields."""
    e2 = []
    for c in range(16):
        e, m = (c >> 1) & 3, c & 1
        v = 0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
        e2.append(-v if c & 8 else v)
    e4 = []
    for c in range(256):
        e, m = (c >> 3) & 15, c & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        if e == 15 and m == 7:
            v = float("nan")
        e4.append(-v if c & 128 else v)
    return torch.tensor(e2, device=dev), torch.tensor(e4, device=dev)


def unpack_fp(codes, scales, mode):
    """Dequantized floating-point-mode weights in fp32 with torch ops (codes by
    shifts and masks, values by table lookup, times the scale)."""
    e2, e4 = _fp_tables(codes.device)
    bits = 8 if mode == "mxfp8" else 4
    gs = 16 if mode == "nvfp4" else 32
    per = 32 // bits
    c = codes.to(torch.int64) & 0xFFFFFFFF
    sh = torch.arange(per, device=codes.device, dtype=torch.int64) * bits
    q = ((c.unsqueeze(-1) >> sh) & ((1 << bits) - 1)).flatten(-2)
    v = (e4 if bits == 8 else e2)[q]
    sc = scales.to(torch.int64)
    sv = e4[sc] if mode == "nvfp4" else torch.exp2(sc.to(torch.float32) - 127)
    return v * sv.repeat_interleave(gs, -1)


def check_decode(wl, rows=None):
    c, s, b = wl.ws[0]
    w = unpack_dequant(c, s, b, wl.gs, wl.bits)
    if not wl.t:  # stored [K, N]: the product is x . w
        w = w.T
    x, y = wl.x, wl.y
    if rows is not None:
        x, y = x[rows], y[rows]
    return worst_ratio(y, x, w)


def check_gather(wl, samples=64):
    c, s, b = wl.ws[0]
    g = torch.Generator(device="cpu").manual_seed(5)
    pick = torch.randperm(wl.R, generator=g)[:samples].tolist()
    worst = 0.0
    for r in pick:
        e, t = int(wl.rhs[r]), int(wl.lhs[r])
        w = unpack_dequant(c[e], s[e], b[e], 64, 4)
        if not getattr(wl, "transpose", True):
            w = w.t()
        worst = max(worst, worst_ratio(wl.y[r:r + 1], wl.x[t:t + 1], w))
    return worst


def check_dequant(wl):
    c, s, b = wl.ws[0]
    ref = unpack_dequant(c, s, b, wl.gs, wl.bits).to(wl.out.dtype)
    return 0.0 if torch.equal(ref, wl.out) else float("inf")


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 6:
                    try:
                        rows.append((float(parts[0]), float(parts[1]), parts[2:]))
                    except ValueError:
                        pass
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, _, r in rows for n, v in zip(names, r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def timed_graph(fn_step, steps: int, warmup: int, stream, chunk: int = 512):
    """Warm up, capture the steps in CUDA graphs, time K steps with CUDA events
    on `stream`. fn_step(i) enqueues step i on the current stream. Returns ms."""
    with torch.cuda.stream(stream):
        for i in range(warmup):
            fn_step(i)
    stream.synchronize()
    graphs = []
    done = 0
    while done < steps:
        n = min(chunk, steps - done)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(done, done + n):
                fn_step(i)
        graphs.append(g)
        done += n
    for g in graphs:  # one untimed replay: graph upload
        g.replay()
    stream.synchronize()
    return graphs


def stream_timed(fn_step, steps: int, warmup: int, stream, barrier):
    """Warm up, then time K steps launched straight onto `stream` (no graph)
    with CUDA events on it. Returns ms."""
    for i in range(warmup):
        fn_step(i)
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        fn_step(i)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    return start.elapsed_time(end)


def replay_timed(graphs, stream, barrier):
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for g in graphs:
            g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    barrier()
    return start.elapsed_time(end)


# Sources of each profiled kernel (its .cu file and the headers it includes).
KERNEL_SOURCES = {
    "qmv_decode_b4_g64": ["csrc/qmv.cu", "csrc/common.cuh", "csrc/kernels.cuh", "csrc/tma.cuh",
                          "../include/nvq.h"],
}


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed: a comment
    edit does not change the kernel the counters were taken on."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_hash(kernel_key: str = "qmv_decode_b4_g64"):
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "group_wise_affine_dequant_b200")
    for f in KERNEL_SOURCES[kernel_key]:
        with open(os.path.normpath(os.path.join(pkg, f)), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current sources of that kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("src_hash") != kernel_hash(kernel_key):
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- workloads
class Decode:
    """x [M, K] . W[N, K]^T (transpose) or x . W[K, N], quantized (bits, gs)."""

    def __init__(self, dev, N=14336, K=4096, M=1, bits=4, gs=64, transpose=True, l2_bytes=None):
        import group_wise_affine_dequant_b200 as nvq
        self.nvq = nvq
        self.N, self.K, self.M, self.bits, self.gs, self.t = N, K, M, bits, gs, transpose
        shape = (N, K) if transpose else (K, N)
        w = W.normal(shape, 0.02, 0, "bf16").to(dev)
        c, s, b = nvq.nv_quantize_affine(w, gs, bits)
        del w
        wbytes = qbytes(N, K, bits, gs)
        l2 = l2_bytes or torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))  # 3x L2 between reuses of a copy
        self.ws = [(c.clone(), s.clone(), b.clone()) for _ in range(self.copies)]
        self.x = W.activations(M, K).to(dev)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.bytes = wbytes + 2 * M * (K + N)
        self.flops = 2 * M * N * K

    def call(self, j):
        c, s, b = self.ws[j]
        self.nvq.nv_qmm(self.x, c, s, b, self.gs, self.bits, self.t, out=self.y)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)

    def bind(self, stream, outs=None):
        """Arguments of nv_qmm for each weight copy, bound once for launches on
        `stream` straight through the C ABI (c_step)."""
        from group_wise_affine_dequant_b200 import binding
        self.fn = binding.lib().nv_qmm
        h = ctypes.c_void_p(stream.cuda_stream)
        outs = outs or [self.y] * self.copies
        self.cargs = [(self.x.data_ptr(), 1, self.M, self.K, self.N, c.data_ptr(), s.data_ptr(),
                       b.data_ptr(), self.gs, self.bits, int(self.t), 0, outs[j].data_ptr(), h)
                      for j, (c, s, b) in enumerate(self.ws)]
        self.status = 0
        return self

    def c_step(self, i):
        fn = self.fn
        for a in self.cargs:
            self.status |= fn(*a)


class DecodeE2E(Decode):
    """The same step from host buffers: each step copies its input x from pinned
    host memory, runs the product with every weight copy (one output row block
    per copy) and reads all the step's outputs back into pinned host memory."""

    def __init__(self, dev, **kw):
        super().__init__(dev, **kw)
        self.xh = self.x.cpu().pin_memory()
        self.yall = torch.empty(self.copies, self.M, self.N, dtype=torch.bfloat16, device=dev)
        self.yh = torch.empty(self.copies, self.M, self.N, dtype=torch.bfloat16).pin_memory()
        self.h2d = self.xh.numel() * 2
        self.d2h = self.yh.numel() * 2

    def step(self, i):
        self.x.copy_(self.xh, non_blocking=True)
        for j in range(self.copies):
            c, s, b = self.ws[j]
            self.nvq.nv_qmm(self.x, c, s, b, self.gs, self.bits, self.t, out=self.yall[j])
        self.yh.copy_(self.yall, non_blocking=True)

    def bind_e2e(self, stream):
        self.stream = stream
        return self.bind(stream, outs=list(self.yall))

    def c_step(self, i):
        """The step through the C ABI on the bound stream: x in, every copy, y out."""
        with torch.cuda.stream(self.stream):
            self.x.copy_(self.xh, non_blocking=True)
            fn = self.fn
            for a in self.cargs:
                self.status |= fn(*a)
            self.yh.copy_(self.yall, non_blocking=True)


class DecodeFp:
    """x [M, K] . W[N, K]^T with W in a floating-point mode (MXFP4, MXFP8, NVFP4)."""

    def __init__(self, dev, N=14336, K=4096, M=1, mode="mxfp4"):
        import group_wise_affine_dequant_b200 as nvq
        self.nvq = nvq
        self.N, self.K, self.M, self.mode = N, K, M, mode
        w = W.normal((N, K), 0.02, 0, "bf16").to(dev)
        c, s = nvq.nv_quantize_fp(w, mode)
        del w
        bits, gs = (8, 32) if mode == "mxfp8" else (4, 16 if mode == "nvfp4" else 32)
        wbytes = N * K * bits // 8 + N * (K // gs)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))
        self.ws = [(c.clone(), s.clone()) for _ in range(self.copies)]
        self.x = W.activations(M, K).to(dev)
        self.y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        self.bytes = wbytes + 2 * M * (K + N)
        self.flops = 2 * M * N * K

    def call(self, j):
        c, s = self.ws[j]
        self.nvq.nv_qmm_fp(self.x, c, s, self.mode, out=self.y)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)


def check_decode_fp(wl, rows=None):
    c, s = wl.ws[0]
    w = unpack_fp(c, s, wl.mode)
    x, y = wl.x, wl.y
    if rows is not None:
        x, y = x[rows], y[rows]
    return worst_ratio(y, x, w)


class Dequant:
    """w = scale * code + bias for W [N, K] (4-bit g64 codes) into bf16."""

    def __init__(self, dev, N=14336, K=4096, bits=4, gs=64):
        import group_wise_affine_dequant_b200 as nvq
        self.nvq = nvq
        self.bits, self.gs = bits, gs
        w = W.normal((N, K), 0.02, 0, "bf16").to(dev)
        c, s, b = nvq.nv_quantize_affine(w, gs, bits)
        del w
        wbytes = qbytes(N, K, bits, gs)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))
        self.ws = [(c.clone(), s.clone(), b.clone()) for _ in range(self.copies)]
        self.out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        self.bytes = wbytes + N * K * 2

    def call(self, j):
        c, s, b = self.ws[j]
        self.nvq.nv_dequantize_affine(c, s, b, self.gs, self.bits, out=self.out)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)


class GatherMM:
    """Mixture of experts with full-precision bf16 experts [64, 1536, 2048]."""

    def __init__(self, dev):
        import group_wise_affine_dequant_b200 as nvq
        self.nvq = nvq
        m = W.MOE
        self.E, self.N, self.K, self.T = m["E"], m["N"], m["K"], m["tokens"]
        w = W.normal((self.E, self.N, self.K), 0.02, 0, "bf16").to(dev)
        wbytes = w.numel() * 2
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))
        self.ws = [w] + [w.clone() for _ in range(self.copies - 1)]
        ids = W.expert_ids(self.T, self.E, m["top_k"], 2)
        lhs, rhs = W.flatten_pairs(ids)
        self.lhs = lhs.to(torch.int32).to(dev)
        self.rhs = rhs.to(torch.int32).to(dev)
        self.R = rhs.numel()
        self.x = W.normal((self.T, self.K), 1.0, 1, "bf16").to(dev)
        self.y = torch.empty(self.R, self.N, dtype=torch.bfloat16, device=dev)
        self.wsp = torch.empty(nvq.nv_gather_qmm_workspace_size(self.R, self.E), dtype=torch.uint8,
                               device=dev)
        self.bytes = wbytes + self.T * self.K * 2 + self.R * self.N * 2 + self.R * 8

    def call(self, j):
        self.nvq.nv_gather_mm(self.x, self.ws[j], self.rhs, self.lhs,
                              workspace=self.wsp, out=self.y)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)


def check_gather_mm(wl, samples=64):
    g = torch.Generator(device="cpu").manual_seed(5)
    pick = torch.randperm(wl.R, generator=g)[:samples].tolist()
    worst = 0.0
    for r in pick:
        e, t = int(wl.rhs[r]), int(wl.lhs[r])
        worst = max(worst, worst_ratio(wl.y[r:r + 1], wl.x[t:t + 1], wl.ws[0][e].float()))
    return worst


class Gather:
    """Mixture of experts: 64 experts [1536, 2048] 4-bit g64, 512 tokens x top-4
    (transpose False: the experts stored [2048, 1536], grouped along N)."""

    def __init__(self, dev, sorted_pairs: bool, row_exact: bool = False, transpose: bool = True):
        import group_wise_affine_dequant_b200 as nvq
        self.row_exact = row_exact
        self.transpose = transpose
        self.nvq = nvq
        m = W.MOE
        self.E, self.N, self.K, self.T = m["E"], m["N"], m["K"], m["tokens"]
        shape = (self.E, self.N, self.K) if transpose else (self.E, self.K, self.N)
        w = W.normal(shape, 0.02, 0, "bf16").to(dev)
        c, s, b = nvq.nv_quantize_affine(w, 64, 4)
        del w
        wbytes = qbytes(self.E * self.N, self.K, 4, 64)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))
        self.ws = [(c.clone(), s.clone(), b.clone()) for _ in range(self.copies)]
        ids = W.expert_ids(self.T, self.E, m["top_k"], 2)
        lhs, rhs = W.flatten_pairs(ids)
        if sorted_pairs:
            lhs, rhs, _ = W.stable_sort_pairs(lhs, rhs)
        self.sorted = sorted_pairs
        self.lhs = lhs.to(torch.int32).to(dev)
        self.rhs = rhs.to(torch.int32).to(dev)
        self.R = rhs.numel()
        self.x = W.normal((self.T, self.K), 1.0, 1, "bf16").to(dev)
        self.y = torch.empty(self.R, self.N, dtype=torch.bfloat16, device=dev)
        self.wsp = torch.empty(nvq.nv_gather_qmm_workspace_size(self.R, self.E), dtype=torch.uint8,
                               device=dev)
        self.bytes = wbytes + self.T * self.K * 2 + self.R * self.N * 2 + self.R * 8

    def call(self, j):
        c, s, b = self.ws[j]
        self.nvq.nv_gather_qmm(self.x, c, s, b, self.rhs, self.lhs, 64, 4, self.transpose, self.sorted,
                               self.row_exact, workspace=self.wsp, out=self.y)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)


class MoeBlock:
    """The routed SwiGLU block: 64 experts, gate/up [1536, 2048] and down
    [2048, 1536] 4-bit g64, 512 tokens x top-4 (uniform without replacement),
    normalized uniform routing weights."""

    def __init__(self, dev):
        import group_wise_affine_dequant_b200 as nvq
        self.nvq = nvq
        m = W.MOE
        self.E, self.I, self.K, self.T, self.top = m["E"], m["N"], m["K"], m["tokens"], m["top_k"]
        qs = []
        for seed, shape in ((0, (self.E, self.I, self.K)), (3, (self.E, self.I, self.K)),
                            (4, (self.E, self.K, self.I))):
            w = W.normal(shape, 0.02, seed, "bf16").to(dev)
            qs.append(nvq.nv_quantize_affine(w, 64, 4))
            del w
        wbytes = 3 * qbytes(self.E * self.I, self.K, 4, 64)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.copies = max(2, -(-3 * l2 // wbytes))
        self.ws = [tuple(tuple(t.clone() for t in q) for q in qs) for _ in range(self.copies)]
        self.ids = W.expert_ids(self.T, self.E, self.top, 2).to(torch.int32).to(dev)
        g = torch.Generator().manual_seed(6)
        rw = torch.rand(self.T, self.top, generator=g)
        self.rw = (rw / rw.sum(1, keepdim=True)).to(torch.float32).to(dev)
        self.x = W.normal((self.T, self.K), 1.0, 1, "bf16").to(dev)
        self.y = torch.empty(self.T, self.K, dtype=torch.bfloat16, device=dev)
        self.wsp = torch.empty(nvq.nv_moe_swiglu_workspace_size(self.T, self.top, self.E, self.I,
                                                                self.K),
                               dtype=torch.uint8, device=dev)
        self.bytes = wbytes + 2 * self.T * self.K * 2 + self.T * self.top * 8

    def call(self, j):
        gate, up, down = self.ws[j]
        self.nvq.nv_moe_swiglu(self.x, gate, up, down, self.ids, self.rw, 64, 4,
                               workspace=self.wsp, out=self.y)

    def step(self, i):
        for j in range(self.copies):
            self.call(j)


def check_moe(wl, tokens=8):
    """A few tokens' outputs against the block in plain torch arithmetic (fp32,
    codes unpacked by shifts and masks)."""
    gate, up, down = wl.ws[0]
    worst = 0.0
    for t in range(tokens):
        x = wl.x[t:t + 1].float()
        acc = torch.zeros(1, wl.K, device=x.device)
        mag = torch.zeros(1, wl.K, device=x.device)
        for j in range(wl.top):
            e = int(wl.ids[t, j])
            wg = unpack_dequant(gate[0][e], gate[1][e], gate[2][e], 64, 4)
            wu = unpack_dequant(up[0][e], up[1][e], up[2][e], 64, 4)
            wd = unpack_dequant(down[0][e], down[1][e], down[2][e], 64, 4)
            g, u = x @ wg.T, x @ wu.T
            ag, au = x.abs() @ wg.abs().T, x.abs() @ wu.abs().T
            sg = torch.sigmoid(g)
            h = g * sg * u
            # the product tolerance carried through silu(g) * u (as the oracle's)
            eh = 2 * (h.abs() + (sg * (1 + g * (1 - sg)) * u).abs() * ag + (g * sg).abs() * au)
            acc += float(wl.rw[t, j]) * (h @ wd.T)
            mag += abs(float(wl.rw[t, j])) * (eh @ wd.abs().T)
        tol = 4e-3 * mag + 1e-5
        worst = max(worst, float(((wl.y[t:t + 1].float() - acc).abs() / tol).max()))
    return worst


# --------------------------------------------------------------------------- arms
def run_nvq(args):
    import torch.distributed as dist
    ws, rank, local = dist_env()
    if ws > 1:
        dist.init_process_group("nccl", device_id=torch.device(f"cuda:{local}"),
                                timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device(f"cuda:{local}")
    stream = torch.cuda.Stream(dev)

    def barrier():
        if ws > 1:
            dist.barrier(device_ids=[local])

    def max_ms(v: float) -> float:
        return max_over_ranks(v, ws, dev)

    pk, pk_kind = peaks()
    K, Wm = args.steps, args.warmup

    # ---- headline: 4-bit g64 decode, launched straight onto the stream through
    # the C ABI (graph replay keeps the programmatic launch edges but measured
    # ~13% slower; it is reported beside, as decode_graph_replay_gbs)
    dec = Decode(dev).bind(stream)
    with ClockSampler(local) as clk:
        ms = stream_timed(dec.c_step, K, Wm, stream, barrier)
        # keep the clock sampler fed for at least ~0.5 s of load
        t_end = time.time() + max(0.0, 0.6 - ms / 1e3)
        while time.time() < t_end:
            stream_timed(dec.c_step, K, 0, stream, lambda: None)
    if dec.status != 0:
        raise SystemExit(f"nv_qmm returned status {dec.status}")
    graphs = timed_graph(dec.step, K, Wm, stream)
    ms_graph = max_ms(replay_timed(graphs, stream, barrier))
    del graphs
    chk = (lambda f, *a, **k: 0.0) if args.no_output_check else (lambda f, *a, **k: f(*a, **k))
    checks = {"decode": round(chk(check_decode, dec), 4)}
    ms = max_ms(ms)
    # the timed region holds K * copies launches of the decode kernel, nothing else
    per_launch_s = ms / 1e3 / (K * dec.copies)
    value = replica_rate(ws, dec.bytes * dec.copies, K, ms) / 1e9
    achieved = dec.bytes / per_launch_s / 1e9
    clocks = clk.summary()

    # ---- end to end through host buffers, the same launches
    e2e = DecodeE2E(dev).bind_e2e(stream)
    ms_e2e = max_ms(stream_timed(e2e.c_step, K, Wm, stream, barrier))
    if e2e.status != 0:
        raise SystemExit(f"nv_qmm returned status {e2e.status}")
    e2e_value = replica_rate(ws, e2e.bytes * e2e.copies, K, ms_e2e) / 1e9

    # ---- the other workloads, same rules (fewer steps)
    also = {}
    also["decode_graph_replay_gbs"] = round(replica_rate(ws, dec.bytes * dec.copies, K, ms_graph) / 1e9, 1)
    ks = max(3, min(K, 40))
    for name, mk in (("decode_8bit_gbs", lambda: Decode(dev, bits=8)),
                     ("decode_transposed_gbs", lambda: Decode(dev, N=14336, K=4096, transpose=False)),
                     ("decode_transposed_8bit_gbs", lambda: Decode(dev, transpose=False, bits=8)),
                     ("fewrow_m8_14336x4096_gbs", lambda: Decode(dev, M=8)),
                     ("fewrow_m8_4096x4096_gbs", lambda: Decode(dev, N=4096, M=8))):
        wl = mk()
        g = timed_graph(wl.step, ks, Wm, stream)
        t = max_ms(replay_timed(g, stream, barrier))
        also[name] = round(replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9, 1)
        checks[name.replace("_gbs", "")] = round(chk(check_decode, wl), 4)
        del g, wl
    # split-K: a small output with a long inner dimension (HBM-bound: 10.2 MB
    # moved against 1.9 GFLOP)
    wl = Decode(dev, N=1024, K=14336, M=64)
    g = timed_graph(wl.step, ks, Wm, stream)
    t = max_ms(replay_timed(g, stream, barrier))
    sk = replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9
    also["splitk_64x1024x14336_b4g64_gbs"] = round(sk, 1)
    also["splitk_64x1024x14336_b4g64_tflops"] = round(
        replica_rate(ws, wl.flops * wl.copies, ks, t) / 1e12, 1)
    also["splitk_frac_of_hbm"] = round(sk / ws / pk["hbm_gbs"], 4)
    also["splitk_partitions"] = wl.nvq.nv_qmm_splits(64, 14336, 1024, 4, 64)
    checks["splitk_64x1024x14336"] = round(chk(check_decode, wl), 4)
    del g, wl
    wl = Dequant(dev)
    g = timed_graph(wl.step, ks, Wm, stream)
    t = max_ms(replay_timed(g, stream, barrier))
    dq = replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9
    also["dequantize_14336x4096_b4g64_bf16_gbs"] = round(dq, 1)
    also["dequantize_frac_of_hbm"] = round(dq / ws / pk["hbm_gbs"], 4)
    checks["dequantize"] = chk(check_dequant, wl)
    del g, wl
    for name, srt, rx, tr in (("gather_sorted", True, False, True), ("gather_unsorted", False, False, True),
                              ("gather_row_exact", False, True, True),
                              ("gather_kn_sorted", True, False, False)):
        wl = Gather(dev, srt, rx, tr)
        g = timed_graph(wl.step, ks, Wm, stream)
        t = max_ms(replay_timed(g, stream, barrier))
        also[name + "_tok_s"] = round(replica_rate(ws, wl.T * wl.copies, ks, t), 1)
        also[name + "_gbs"] = round(replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9, 1)
        checks[name] = round(chk(check_gather, wl), 4)
        del g, wl
    wl = MoeBlock(dev)
    g = timed_graph(wl.step, ks, Wm, stream)
    t = max_ms(replay_timed(g, stream, barrier))
    also["moe_swiglu_tok_s"] = round(replica_rate(ws, wl.T * wl.copies, ks, t), 1)
    mb = replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9
    also["moe_swiglu_gbs"] = round(mb, 1)
    also["moe_swiglu_frac_of_hbm"] = round(mb / ws / pk["hbm_gbs"], 4)
    checks["moe_swiglu"] = round(chk(check_moe, wl), 4)
    del g, wl
    wl = GatherMM(dev)
    g = timed_graph(wl.step, ks, Wm, stream)
    t = max_ms(replay_timed(g, stream, barrier))
    also["gather_mm_bf16_tok_s"] = round(replica_rate(ws, wl.T * wl.copies, ks, t), 1)
    gm = replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9
    also["gather_mm_bf16_gbs"] = round(gm, 1)
    also["gather_mm_frac_of_hbm"] = round(gm / ws / pk["hbm_gbs"], 4)
    checks["gather_mm_bf16"] = round(chk(check_gather_mm, wl), 4)
    del g, wl
    for bits, gs in W.PREFILL_VARIANTS:
        wl = Decode(dev, N=14336, K=4096, M=2048, bits=bits, gs=gs)
        kp = max(3, min(K, 10))
        g = timed_graph(wl.step, kp, Wm, stream)
        t = max_ms(replay_timed(g, stream, barrier))
        tf = replica_rate(ws, wl.flops * wl.copies, kp, t) / 1e12
        key = "prefill_tflops" if (bits, gs) == (4, 64) else f"prefill_b{bits}_g{gs}_tflops"
        also[key] = round(tf, 1)
        if (bits, gs) == (4, 64):
            also["prefill_frac_of_bf16_peak"] = round(tf / pk["bf16_tflops"], 4)
        checks[key.replace("_tflops", "")] = round(chk(check_decode, wl, rows=torch.arange(0, 2048, 128)), 4)
        del g, wl
    # floating-point modes: decode (GB/s) at 14336 x 4096, and MXFP4 prefill (TFLOP/s)
    for mode in ("mxfp4", "nvfp4", "mxfp8"):
        wl = DecodeFp(dev, mode=mode)
        g = timed_graph(wl.step, ks, Wm, stream)
        t = max_ms(replay_timed(g, stream, barrier))
        gb = replica_rate(ws, wl.bytes * wl.copies, ks, t) / 1e9
        also[f"decode_{mode}_gbs"] = round(gb, 1)
        also[f"decode_{mode}_frac_of_hbm"] = round(gb / ws / pk["hbm_gbs"], 4)
        checks[f"decode_{mode}"] = round(chk(check_decode_fp, wl), 4)
        del g, wl
    wl = DecodeFp(dev, M=2048, mode="mxfp4")
    kp = max(3, min(K, 10))
    g = timed_graph(wl.step, kp, Wm, stream)
    t = max_ms(replay_timed(g, stream, barrier))
    also["prefill_mxfp4_tflops"] = round(replica_rate(ws, wl.flops * wl.copies, kp, t) / 1e12, 1)
    checks["prefill_mxfp4"] = round(chk(check_decode_fp, wl, rows=torch.arange(0, 2048, 128)), 4)
    del g, wl

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(ms / K, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
        "pct_of_8tbs": round(100 * achieved / HBM_NOMINAL_GBS, 2),
        "config": {"workload": "decode x[1,4096] . W[14336,4096]^T, affine 4-bit g64, bf16",
                   "M": 1, "N": 14336, "K": 4096, "bits": 4, "group_size": 64,
                   "products_per_step": dec.copies, "bytes_per_product": dec.bytes,
                   "bytes_per_step": dec.bytes * dec.copies, "parallelism": f"replicas x{ws}",
                   "l2": f"a step multiplies by each of {dec.copies} weight copies in turn "
                         f"(> 3x L2 between reuses of a copy)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "peak_kind": pk_kind, "unit": "GB/s",
                     "frac": round(achieved / pk["hbm_gbs"], 4),
                     "traffic": traffic_for("qmv_decode_b4_g64")},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": e2e.h2d,
                "d2h_bytes_per_step": e2e.d2h},
        "gpu_launches": K * dec.copies,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"]},
        "also": also,
        "output_check": {"rule": "worst |y - torch fp32 reference| / (4e-3 sum|x w| + 1e-5) per timed "
                                 "workload (prefill: 16 rows; gather: 64 pairs; dequantize: 0 = bitwise "
                                 "equal); <= 1 passes",
                         "worst": checks, "pass": all(v <= 1.0 for v in checks.values()),
                         "skipped": bool(args.no_output_check)},
        "cpu_baseline": None,
    }
    if ws == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def cpu_baseline(budget_s: float = 10.0, steps: int | None = None):
    """The oracle on the host's cores, on the decode workload: whole products
    (all 14336 outputs) repeated for about budget_s seconds."""
    import oracle as O
    w = W.decode_weight()
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.activations(1, 4096)
    bytes_ = qbytes(14336, 4096, 4, 64) + 2 * (4096 + 14336)
    t0 = time.perf_counter()
    O.qmm(x, c, s, b, 64, 4, True)
    one = time.perf_counter() - t0
    reps = steps or max(1, int(budget_s / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        O.qmm(x, c, s, b, 64, 4, True)
    dt = time.perf_counter() - t0
    return {"value": round(reps * bytes_ / dt / 1e9, 4), "unit": "GB/s", "cores": O.threads(),
            "kind": "oracle",
            "sample": f"{reps} whole decode products x[1,4096] . W[14336,4096]^T (4-bit g64), "
                      f"fp64 dequantize-then-dot, {dt:.1f} s"}


def run_reference(args):
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import oracle as O
    w = W.decode_weight()
    c, s, b = O.quantize_affine(w, 64, 4)
    x = W.activations(1, 4096)
    N, K = 14336, 4096
    # each step: a bounded, fixed sample of output rows, so K steps end in minutes
    t0 = time.perf_counter()
    O.qmm_sampled(x, c, s, b, 64, 4, True, torch.zeros(1024, dtype=torch.int64),
                  torch.arange(1024))
    per_row = (time.perf_counter() - t0) / 1024
    total_budget = 60.0
    rows = int(max(64, min(N, total_budget / max(1, args.steps + args.warmup) / max(per_row, 1e-9))))
    n_idx = torch.arange(rows, dtype=torch.int64)
    m_idx = torch.zeros(rows, dtype=torch.int64)
    for _ in range(args.warmup):
        O.qmm_sampled(x, c, s, b, 64, 4, True, m_idx, n_idx)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.qmm_sampled(x, c, s, b, 64, 4, True, m_idx, n_idx)
    dt = time.perf_counter() - t0
    bytes_per_step = rows * (K * 4 // 8 + 2 * 2 * K // 64) + 2 * K + 2 * rows
    value = args.steps * bytes_per_step / dt / 1e9
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
        "config": {"workload": "decode x[1,4096] . W[14336,4096]^T, affine 4-bit g64, bf16",
                   "M": 1, "N": N, "K": K, "bits": 4, "group_size": 64,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": O.threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {N} output rows per step (fp64 oracle)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PROFILE_WORKLOADS = {
    "decode": lambda dev: Decode(dev),
    "decode8": lambda dev: Decode(dev, bits=8),
    "decode_t0": lambda dev: Decode(dev, transpose=False),
    "fewrow8": lambda dev: Decode(dev, M=8),
    "gather": lambda dev: Gather(dev, sorted_pairs=False),
    "gather_kn": lambda dev: Gather(dev, sorted_pairs=True, transpose=False),
    "prefill": lambda dev: Decode(dev, N=14336, K=4096, M=2048, bits=4, gs=64),
    "splitk": lambda dev: Decode(dev, N=1024, K=14336, M=64),
    "prefill8": lambda dev: Decode(dev, N=14336, K=4096, M=2048, bits=8, gs=64),
    "dequant": lambda dev: Dequant(dev),
    "gather_mm": lambda dev: GatherMM(dev),
    "moe": lambda dev: MoeBlock(dev),
    "decode_mxfp4": lambda dev: DecodeFp(dev, mode="mxfp4"),
    "prefill_mxfp4": lambda dev: DecodeFp(dev, M=2048, mode="mxfp4"),
}


def run_profile(name: str, launches: int):
    """Plain stream launches of one workload's product (no graphs), so that a
    profiler sees one kernel per product (the router and the grouped kernel for
    a gather). Prints the mean time per product from CUDA events: not a bench
    value when the process runs under a profiler."""
    if name not in PROFILE_WORKLOADS:
        raise SystemExit(f"unknown workload {name!r}; one of {sorted(PROFILE_WORKLOADS)}")
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    wl = PROFILE_WORKLOADS[name](dev)
    for j in range(3):
        wl.call(j % wl.copies)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for j in range(launches):
        wl.call(j % wl.copies)
    e1.record()
    torch.cuda.synchronize()
    print(f"{name}: {launches} products, {e0.elapsed_time(e1) / launches * 1e3:.1f} us per product")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="nvq", choices=["nvq", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-output-check", action="store_true",
                    help="skip the torch checks of the timed outputs (for profiler launch lists)")
    ap.add_argument("--profile", metavar="WORKLOAD", default=None,
                    help="launch one workload's product --launches times for a profiler "
                         f"(one of {', '.join(PROFILE_WORKLOADS)}) instead of benchmarking")
    ap.add_argument("--launches", type=int, default=10)
    args = ap.parse_args()
    if args.profile:
        run_profile(args.profile, args.launches)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_nvq(args)


if __name__ == "__main__":
    main()
