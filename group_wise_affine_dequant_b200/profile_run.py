"""Launch one of the benchmark workloads a fixed number of times, for profilers.

    python -m group_wise_affine_dequant_b200.profile_run WORKLOAD [LAUNCHES]

WORKLOAD is one of decode (x[1,4096] . W[14336,4096]^T, 4-bit g64), decode8
(the same at 8 bits), gather (64 experts [1536,2048] 4-bit g64, 512 tokens x
top-4, unsorted), prefill (x[2048,4096] . W[14336,4096]^T, 4-bit g64),
dequant (W[14336,4096] 4-bit g64 codes to bf16), gather_mm (the mixture of
experts with bf16 experts). The
workloads are bench.py's (same shapes, seeds and weight-copy rotation); the
launches are plain stream launches (no graphs), so that a profiler sees one
kernel per product (two plus the router for a gather). Prints the mean time per
launch from CUDA events; that number is not a benchmark result when the process
runs under a profiler.
"""
from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def make(name: str, dev):
    if name == "decode":
        return bench.Decode(dev)
    if name == "decode8":
        return bench.Decode(dev, bits=8)
    if name == "gather":
        return bench.Gather(dev, sorted_pairs=False)
    if name == "prefill":
        return bench.Decode(dev, N=14336, K=4096, M=2048, bits=4, gs=64)
    if name == "dequant":
        return bench.Dequant(dev)
    if name == "gather_mm":
        return bench.GatherMM(dev)
    raise SystemExit(f"unknown workload {name!r}")


def main(argv):
    if len(argv) < 2:
        raise SystemExit(__doc__)
    name = argv[1]
    launches = int(argv[2]) if len(argv) > 2 else 20
    dev = torch.device("cuda:0")
    wl = make(name, dev)
    for i in range(3):
        wl.step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(launches):
        wl.step(i)
    e1.record()
    torch.cuda.synchronize()
    print(f"{name}: {launches} launches, {e0.elapsed_time(e1) / launches * 1e3:.1f} us per product")


if __name__ == "__main__":
    main(sys.argv)
