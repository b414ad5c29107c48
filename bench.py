"""Benchmark of the W4A16 linear layer on B200.

One step = one pass over the Llama-7B-shaped decode GEMVs: the four layer
shapes (K, N) in {(4096,12288), (4096,4096), (4096,22016), (11008,4096)} at
M in {1, 4, 16} (12 calls of w4a16_gemm), INT4 asymmetric RTN, group 128,
weights ~N(0, 0.02^2), bf16 activations ~N(0,1) with 0.1% outlier channels
x50.  Weights are quantized and prepacked on the GPU first; every call of a
step reads a different replica of its layer's packed weights, and the
replicas total more than 4x the L2 size, so no call finds its weights in L2.

metric: achieved HBM TB/s = algorithmic bytes / time, with algorithmic bytes
per call = N*K/2 (codes) + N*(K/G)*2.5 (fp16 scale + 4-bit zero) + 2*M*K (X)
+ 2*M*N (Y).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
       [--no-rows]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_bit_gemm_b200 import synthetic as S  # noqa: E402

METRIC = "W4A16 linear: achieved HBM TB/s (decode M<=16) and TFLOP/s (prefill) vs roofline"
WL = S.LLAMA7B_DECODE
WORKLOAD = ("Llama-7B-shaped decode GEMVs (K,N) in {(4096,12288),(4096,4096),(4096,22016),"
            "(11008,4096)} x M in {1,4,16}; INT4 asym RTN g128; W~N(0,0.02^2); X bf16 N(0,1) "
            "with 0.1% K-channels x50")


def int4_bytes(M, N, K, G):
    return N * K / 2 + N * (K // G) * 2.5 + 2 * M * K + 2 * M * N


def nf4_bytes(M, N, K):
    nb = N * K // 64
    return N * K / 2 + nb + 4 * -(-nb // 256) + 2 * M * K + 2 * M * N


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "samples": len(rows),
                "reasons": reasons}


# --------------------------------------------------------------------- setup

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, v: float) -> float:
    if pg is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(pg, v: float) -> float:
    if pg is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device="cuda")
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return float(t.item())


def bf16_dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


class DecodeStep:
    """The 12 decode calls of one step, with rotating weight replicas."""

    def __init__(self, w4, seed=0):
        self.w4 = w4
        G = WL["G"]
        self.G = G
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
        packed = {}
        for (K, N) in WL["shapes"]:
            W = torch.from_numpy(S.layer_w(WL, K, N, seed)).cuda()
            Wq, sc, zr = w4.quantize_rtn(W, G)
            packed[(K, N)] = w4.prepack(Wq, sc, zr, G)
            del W, Wq, sc, zr
        set_bytes = sum(p.numel() for p in packed.values())
        # call i of a step reads replica i % R of its layer: a layer's three
        # calls (M = 1, 4, 16 are 4 calls apart) read three different
        # replicas, and R >= 4 x L2 / set size
        R = max(3, -(-4 * l2 // set_bytes))
        if R in (4, 8):
            R += 1
        self.replicas = R
        self.wp = {s_: [p] + [p.clone() for _ in range(R - 1)] for s_, p in packed.items()}
        self.replica_bytes = set_bytes * R
        self.calls = []
        c = 0
        for M in WL["Ms"]:
            for (K, N) in WL["shapes"]:
                xb = S.layer_x(WL, M, K, N, seed)
                X = bf16_dev(xb)
                Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
                self.calls.append(dict(M=M, K=K, N=N, X=X, Y=Y, xbits=xb,
                                       bytes=int4_bytes(M, N, K, G)))
                c += 1
        self.ws_bytes = max(w4.workspace_bytes(c_["M"], c_["N"], c_["K"], G)
                            for c_ in self.calls)
        self.ws = torch.zeros(self.ws_bytes + 256, dtype=torch.uint8, device="cuda")
        self.step_bytes = sum(c_["bytes"] for c_ in self.calls)

    def run_one(self, i, X=None, Y=None):
        c = self.calls[i]
        wp = self.wp[(c["K"], c["N"])][i % self.replicas]
        self.w4.w4a16_gemm(c["X"] if X is None else X, wp, c["N"], c["K"], self.G,
                           out=c["Y"] if Y is None else Y, workspace=self.ws)

    def run(self, events=None, X_override=None, Y_override=None):
        for i, c in enumerate(self.calls):
            wp = self.wp[(c["K"], c["N"])][i % self.replicas]
            X = c["X"] if X_override is None else X_override[i]
            Y = c["Y"] if Y_override is None else Y_override[i]
            if events is not None:
                events[i][0].record()
            self.w4.w4a16_gemm(X, wp, c["N"], c["K"], self.G, out=Y, workspace=self.ws)
            if events is not None:
                events[i][1].record()


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g
def sleep_gpu(ms: float):
    """Keep the stream busy while the host queues the next launches, so that
    per-call events measure kernel time, not host launch latency."""
    torch.cuda._sleep(int(ms * 2.0e6))


def time_calls(calls, reps: int, warm: int = 2):
    """Per-call device time (ms, averaged over `reps`) of closures run in order
    on the current stream, each bracketed by CUDA events."""
    for _ in range(warm):
        for f in calls:
            f()
    torch.cuda.synchronize()
    tot = [0.0] * len(calls)
    for _ in range(reps):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in calls]
        sleep_gpu(1.0 + 0.05 * len(calls))
        for (a, b), f in zip(ev, calls):
            a.record()
            f()
            b.record()
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(ev):
            tot[i] += a.elapsed_time(b)
    return [t / reps for t in tot]


def measure_decode(step, args, pg, local):
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(3):
            step.run()
    stream.synchronize()
    # per-call kernel durations (one kernel per call)
    with torch.cuda.stream(stream):
        per_call = time_calls([(lambda i=i: step.run_one(i)) for i in range(len(step.calls))],
                              reps=20)
    g = capture(step.run, stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    stream.synchronize()
    barrier(pg)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier(pg)
        with torch.cuda.stream(stream):
            start.record()
            for _ in range(args.steps):
                g.replay()
            end.record()
        end.synchronize()
        torch.cuda.synchronize()
        barrier(pg)
    ms = start.elapsed_time(end)
    del g
    return ms, per_call, clk.summary()


def measure_e2e(step, args, pg):
    """Same step through the public API with host buffers: pinned-host X ->
    device, the 12 calls, device Y -> pinned host, all inside the timed region."""
    hx = [c["X"].cpu().pin_memory() for c in step.calls]
    hy = [torch.empty(c["Y"].shape, dtype=torch.bfloat16).pin_memory() for c in step.calls]
    dx = [torch.empty_like(c["X"]) for c in step.calls]
    dy = [torch.empty_like(c["Y"]) for c in step.calls]
    stream = torch.cuda.Stream()

    def e2e_step():
        for d, h in zip(dx, hx):
            d.copy_(h, non_blocking=True)
        step.run(X_override=dx, Y_override=dy)
        for h, d in zip(hy, dy):
            h.copy_(d, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
    stream.synchronize()
    g = capture(e2e_step, stream)
    n = max(1, min(args.steps, 2000))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    stream.synchronize()
    barrier(pg)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record()
        for _ in range(n):
            g.replay()
        end.record()
    end.synchronize()
    ms = max_over_ranks(pg, start.elapsed_time(end))
    # results really arrived on the host
    assert torch.equal(hy[0], dy[0].cpu())
    h2d = sum(t.numel() * 2 for t in hx)
    d2h = sum(t.numel() * 2 for t in hy)
    del g
    return ms, n, h2d, d2h
