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


# DRAM bytes of one decode-kernel launch from an ncu capture, valid only for
# the kernel source it was taken on (sha256 of w4_gemv_kernel.cuh).
TRAFFIC_CAPTURE = {
    "kernel_sha256": "3350610e925e15b1f6723d157b6f41ca8c1120b404bc54b17516d4155ee8b0f5",
    "shape": {"M": 1, "N": 12288, "K": 4096, "G": 128},
    "dram_bytes": 26182656,
}


def gemv_kernel_sha256():
    import hashlib
    path = os.path.join(ROOT, "weight_only_bit_gemm_b200", "csrc", "w4_gemv_kernel.cuh")
    return hashlib.sha256(open(path, "rb").read()).hexdigest()


def traffic_per_launch(step):
    """Measured DRAM bytes scaled to the step's mean launch (traffic tracks the
    algorithmic bytes, so scale by their ratio); None if the kernel changed."""
    cap = TRAFFIC_CAPTURE
    if cap["dram_bytes"] is None or cap["kernel_sha256"] != gemv_kernel_sha256():
        return None
    sh = cap["shape"]
    ratio = cap["dram_bytes"] / int4_bytes(sh["M"], sh["N"], sh["K"], sh["G"])
    return ratio * step.step_bytes / len(step.calls)


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


def _reduce(pg, v: float, op) -> float:
    # NCCL reduces device tensors; gloo (the CPU tests of this logic) host ones
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(pg, v: float) -> float:
    """The slowest rank's time: the job is done when the last rank is."""
    return v if pg is None else _reduce(pg, v, pg.ReduceOp.MAX)


def sum_over_ranks(pg, v: float) -> float:
    """Whole-job totals (bytes processed by all ranks)."""
    return v if pg is None else _reduce(pg, v, pg.ReduceOp.SUM)


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


def time_graph(calls, reps: int = 5, warm: int = 2):
    """Device time (ms) of one pass over `calls` (closures, run in order on the
    current stream) captured as one CUDA graph, averaged over `reps` replays;
    the calls are run once eagerly first so that nothing allocates during the
    capture.  Comparable with the graph-timed decode step: launch latency is
    hidden and consecutive kernels overlap through programmatic dependent
    launch."""
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for f in calls:
            f()
    stream.synchronize()

    def run_all():
        for f in calls:
            f()
    g = capture(run_all, stream)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
    b.synchronize()
    del g
    return a.elapsed_time(b) / reps


def time_per_call(f, n: int = 5):
    """Device time (ms) of one call of f, from a CUDA graph of n back-to-back
    calls (launch latency hidden, as in the decode step's timing)."""
    return time_graph([f] * n) / n


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
    """Same step through the public API with host buffers: every step copies
    its 12 activation inputs from pinned host memory to the device, runs the
    12 calls, and reads the 12 outputs back into pinned host memory, all
    inside the timed region.  Copies run on their own streams and are double
    buffered, so that step k's outputs travel back and step k+1's inputs
    travel in while the calls of another step run."""
    n_calls = len(step.calls)
    x_sizes = [c["X"].numel() for c in step.calls]
    y_sizes = [c["Y"].numel() for c in step.calls]
    hx = torch.cat([c["X"].reshape(-1).cpu() for c in step.calls]).pin_memory()
    hy = torch.empty(sum(y_sizes), dtype=torch.bfloat16).pin_memory()

    def views(buf, sizes, shapes):
        out, o = [], 0
        for n, sh in zip(sizes, shapes):
            out.append(buf[o:o + n].view(sh))
            o += n
        return out

    dx = [torch.empty_like(hx, device="cuda") for _ in range(2)]
    dy = [torch.empty(hy.shape, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    xv = [views(dx[b], x_sizes, [c["X"].shape for c in step.calls]) for b in range(2)]
    yv = [views(dy[b], y_sizes, [c["Y"].shape for c in step.calls]) for b in range(2)]
    cs, xs, ys = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    graphs = []
    for b in range(2):
        with torch.cuda.stream(cs):
            step.run(X_override=xv[b], Y_override=yv[b])
        cs.synchronize()
        graphs.append(capture(lambda b=b: step.run(X_override=xv[b], Y_override=yv[b]), cs))
    x_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    y_free = [torch.cuda.Event() for _ in range(2)]

    def one_step(k):
        b = k % 2
        if k >= 2:
            xs.wait_event(done[b])        # the calls of step k-2 have read dx[b]
        with torch.cuda.stream(xs):
            dx[b].copy_(hx, non_blocking=True)
        x_ready[b].record(xs)
        cs.wait_event(x_ready[b])
        if k >= 2:
            cs.wait_event(y_free[b])      # step k-2's outputs have left dy[b]
        with torch.cuda.stream(cs):
            graphs[b].replay()
        done[b].record(cs)
        ys.wait_event(done[b])
        with torch.cuda.stream(ys):
            hy.copy_(dy[b], non_blocking=True)
        y_free[b].record(ys)

    n = max(2, min(args.steps, 2000))
    for k in range(args.warmup):
        one_step(k)
    torch.cuda.synchronize()
    barrier(pg)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(xs)
    cs.wait_event(start)
    ys.wait_event(start)
    for k in range(n):
        one_step(k)
    cs.wait_event(y_free[(n - 1) % 2])
    end.record(cs)
    end.synchronize()
    ms = max_over_ranks(pg, start.elapsed_time(end))
    # the outputs really arrived on the host: the last step's buffer
    assert torch.equal(hy, dy[(n - 1) % 2].cpu())
    for g in graphs:
        del g
    h2d = hx.numel() * 2
    d2h = hy.numel() * 2
    return ms, n, h2d, d2h


# --------------------------------------------------------------------- other rows

def _replicas_for(nbytes_each: int, l2: int) -> int:
    return max(2, -(-4 * l2 // max(1, nbytes_each)))


def measure_rows(w4, peaks):
    """The other steps of the path, each timed alone (device time, CUDA events;
    the standalone kernels as CUDA graphs of 5 back-to-back calls)."""
    rows = {}
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    hbm = peaks["hbm_gbs"]

    # a1+a2: INT4 RTN quantize + pack, and a6: standalone dequant, a4: prepack
    K, N, G = 4096, 22016, 128
    W = torch.from_numpy(S.layer_w(WL, K, N)).cuda()
    Wq, sc, zr = w4.quantize_rtn(W, G)
    t = time_per_call(lambda: w4.quantize_rtn(W, G))
    qb = N * K * 4 + N * K / 2 + N * (K // G) * 3
    rows["quantize_rtn"] = {"shape": [N, K], "G": G, "ms": t, "GB/s": qb / t / 1e6,
                            "frac_of_hbm": qb / t / 1e6 / hbm}
    t = time_per_call(lambda: w4.dequant(Wq, sc, zr, G))
    db = N * K / 2 + N * (K // G) * 3 + N * K * 2
    rows["dequant"] = {"shape": [N, K], "G": G, "ms": t, "GB/s": db / t / 1e6,
                       "frac_of_hbm": db / t / 1e6 / hbm}
    t = time_per_call(lambda: w4.prepack(Wq, sc, zr, G))
    pb = 2 * (N * K / 2 + N * (K // G) * 2.5)
    rows["prepack"] = {"shape": [N, K], "G": G, "ms": t, "GB/s": pb / t / 1e6}
    del W, Wq, sc, zr

    # a5: NF4 quantize; a7: NF4 decode / small batch
    nf = S.NF4_DECODE
    calls, nbytes = [], []
    for (K, N) in nf["shapes"]:
        W = torch.from_numpy(S.layer_w(nf, K, N)).cuda()
        q4, c4, s24 = w4.nf4_quantize(W)
        if (K, N) == nf["shapes"][0]:
            t = time_per_call(lambda: w4.nf4_quantize(W))
            b = N * K * 4 + N * K / 2 + N * K / 64
            rows["nf4_quantize"] = {"shape": [N, K], "ms": t, "GB/s": b / t / 1e6}
        wp = w4.nf4_prepack(q4, c4)
        reps = [wp] + [wp.clone() for _ in range(_replicas_for(wp.numel(), l2) - 1)]
        for M in nf["Ms"]:
            X = bf16_dev(S.layer_x(nf, M, K, N))
            for r in reps:
                calls.append(lambda X=X, r=r, s=s24, N=N, K=K: w4.nf4_gemm(X, r, s, N, K))
                nbytes.append(nf4_bytes(M, N, K))
        del W
    tg = time_graph(calls)
    ts = time_calls(calls, reps=5)
    rows["nf4_gemm_decode"] = {"configs": "(K,N) in {(4096,14336),(14336,4096)} x M in {1,8,32}",
                               "timing": "CUDA graph of all calls",
                               "TB/s": sum(nbytes) / tg / 1e9,
                               "frac_of_hbm": sum(nbytes) / tg / 1e6 / hbm,
                               "eager_TB/s": sum(nbytes) / sum(ts) / 1e9}

    # NEXT row: NF4 with mean-offset double quantization of the constants,
    # same shapes (8 bytes of constants per run instead of 4)
    calls, nbytes = [], []
    for (K, N) in nf["shapes"]:
        W = torch.from_numpy(S.layer_w(nf, K, N)).cuda()
        q4, c4, m4, s24 = w4.nf4_quantize_meandq(W)
        if (K, N) == nf["shapes"][0]:
            t = time_per_call(lambda: w4.nf4_quantize_meandq(W))
            b = N * K * 4 + N * K / 2 + N * K / 64
            rows["nf4_meandq_quantize"] = {"shape": [N, K], "ms": t, "GB/s": b / t / 1e6}
        wp = w4.nf4_prepack(q4, c4.view(torch.uint8))
        reps = [wp] + [wp.clone() for _ in range(_replicas_for(wp.numel(), l2) - 1)]
        for M in nf["Ms"]:
            X = bf16_dev(S.layer_x(nf, M, K, N))
            for r in reps:
                calls.append(lambda X=X, r=r, m=m4, s=s24, N=N, K=K:
                             w4.nf4_gemm_meandq(X, r, m, s, N, K))
                nbytes.append(nf4_bytes(M, N, K) + 4 * -(-(N * K // 64) // 256))
        del W
    tg = time_graph(calls)
    rows["nf4_meandq_gemm_decode"] = {
        "configs": "(K,N) in {(4096,14336),(14336,4096)} x M in {1,8,32}, mean-offset constants",
        "timing": "CUDA graph of all calls",
        "TB/s": sum(nbytes) / tg / 1e9, "frac_of_hbm": sum(nbytes) / tg / 1e6 / hbm}

    # NEXT row: FP4 (E2M1) table in the NF4 kernels, same shapes
    f4 = S.FP4_DECODE
    calls, nbytes = [], []
    for (K, N) in f4["shapes"]:
        W = torch.from_numpy(S.layer_w(f4, K, N)).cuda()
        q4, c4, s24 = w4.fp4_quantize(W)
        if (K, N) == f4["shapes"][0]:
            t = time_per_call(lambda: w4.fp4_quantize(W))
            b = N * K * 4 + N * K / 2 + N * K / 64
            rows["fp4_quantize"] = {"shape": [N, K], "ms": t, "GB/s": b / t / 1e6}
        wp = w4.nf4_prepack(q4, c4)
        reps = [wp] + [wp.clone() for _ in range(_replicas_for(wp.numel(), l2) - 1)]
        for M in f4["Ms"]:
            X = bf16_dev(S.layer_x(f4, M, K, N))
            for r in reps:
                calls.append(lambda X=X, r=r, s=s24, N=N, K=K: w4.fp4_gemm(X, r, s, N, K))
                nbytes.append(nf4_bytes(M, N, K))
        del W
    tg = time_graph(calls)
    ts = time_calls(calls, reps=5)
    rows["fp4_gemm_decode"] = {"configs": "(K,N) in {(4096,14336),(14336,4096)} x M in {1,8,32}",
                               "timing": "CUDA graph of all calls",
                               "TB/s": sum(nbytes) / tg / 1e9,
                               "frac_of_hbm": sum(nbytes) / tg / 1e6 / hbm,
                               "eager_TB/s": sum(nbytes) / sum(ts) / 1e9}

    # a3: act-order (g_idx) decode and M=256, group 32 and the 64 / 128 sweep
    ao = S.ACT_ORDER_13B
    sweep = {}
    for G in [ao["G"], *ao["G_sweep"]]:
        dec_calls, dec_bytes, big_calls, big_flops = [], [], [], []
        for (K, N) in ao["shapes"]:
            W = torch.from_numpy(S.layer_w(ao, K, N)).cuda()
            g_idx = torch.from_numpy(
                S.act_order_g_idx(S.draw_perm(K, tag=ao["tag"], N=N), G)).cuda()
            Wq, sc, zr = w4.quantize_rtn(W, G, g_idx)
            wp = w4.prepack(Wq, sc, zr, G, g_idx)
            reps = [wp] + [wp.clone() for _ in range(_replicas_for(wp.numel(), l2) - 1)]
            for M in ao["Ms"]:
                X = bf16_dev(S.layer_x(ao, M, K, N))
                for r in reps:
                    f = (lambda X=X, r=r, N=N, K=K, G=G: w4.w4a16_gemm(X, r, N, K, G, True))
                    if M <= 16:
                        dec_calls.append(f)
                        dec_bytes.append(int4_bytes(M, N, K, G) + 4 * K)
                    else:
                        big_calls.append(f)
                        big_flops.append(2.0 * M * N * K)
            del W, Wq, sc, zr
        tg = time_graph(dec_calls)
        te = sum(time_calls(dec_calls, reps=5))
        tb = time_graph(big_calls)
        sweep[f"G{G}"] = {"decode_TB/s": sum(dec_bytes) / tg / 1e9,
                          "decode_frac_of_hbm": sum(dec_bytes) / tg / 1e6 / hbm,
                          "decode_eager_TB/s": sum(dec_bytes) / te / 1e9,
                          "m256_TFLOP/s": sum(big_flops) / tb / 1e9,
                          "m256_frac_of_bf16_peak": sum(big_flops) / tb / 1e9 / peaks["bf16_tflops"]}
        del dec_calls, big_calls, reps, wp
        torch.cuda.empty_cache()
    rows["act_order"] = {"configs": "(K,N) in {(5120,13824),(13824,5120)}; decode M in {1,16}, "
                                    "prefill M=256; g_idx from a seeded permutation",
                         "timing": "CUDA graph of all calls of a group size",
                         "per_G": sweep}

    # NEXT row: symmetric INT4 after the AWQ factor (decode shapes of Llama-7B)
    aw = S.AWQ_SYM_DECODE
    awq_calls, plain_calls, awq_bytes = [], [], []
    for (K, N) in aw["shapes"]:
        G = aw["G"]
        W = torch.from_numpy(S.layer_w(aw, K, N)).cuda()
        sd = torch.from_numpy(S.layer_awq_s(aw, K, N)).cuda()
        Ws = w4.awq_scale_weights(W, sd)
        Wq, sc, zr = w4.quantize_sym(Ws, G)
        if (K, N) == (4096, 22016):
            t = time_per_call(lambda: w4.awq_scale_weights(W, sd, out=Ws))
            b = 2 * N * K * 4 + K * 4
            rows["awq_scale_weights"] = {"shape": [N, K], "ms": t, "GB/s": b / t / 1e6,
                                         "frac_of_hbm": b / t / 1e6 / hbm}
            t = time_per_call(lambda: w4.quantize_sym(Ws, G))
            qb = N * K * 4 + N * K / 2 + N * (K // G) * 3
            rows["quantize_sym"] = {"shape": [N, K], "G": G, "ms": t, "GB/s": qb / t / 1e6,
                                    "frac_of_hbm": qb / t / 1e6 / hbm}
        wp = w4.prepack(Wq, sc, zr, G)
        reps = [wp] + [wp.clone() for _ in range(_replicas_for(wp.numel(), l2) - 1)]
        for M in aw["Ms"]:
            X = bf16_dev(S.layer_x(aw, M, K, N))
            for r in reps:
                awq_calls.append(lambda X=X, r=r, N=N, K=K, G=G, sd=sd:
                                 w4.w4a16_awq_gemm(X, sd, r, N, K, G))
                plain_calls.append(lambda X=X, r=r, N=N, K=K, G=G: w4.w4a16_gemm(X, r, N, K, G))
                awq_bytes.append(int4_bytes(M, N, K, G) + 4 * K)
        del W, Ws, Wq, sc, zr
    tg = time_graph(awq_calls)
    tpg = time_graph(plain_calls)
    ts = time_calls(awq_calls, reps=5)
    rows["awq_sym_decode"] = {
        "configs": "(K,N) in {(4096,12288),(4096,4096),(4096,22016),(11008,4096)} x M in {1,4,16}, "
                   "G=128, symmetric codes, AWQ factor on X",
        "timing": "CUDA graph of all calls",
        "TB/s": sum(awq_bytes) / tg / 1e9,
        "frac_of_hbm": sum(awq_bytes) / tg / 1e6 / hbm,
        "same_weights_without_factor_TB/s": sum(awq_bytes) / tpg / 1e9,
        "eager_TB/s": sum(awq_bytes) / sum(ts) / 1e9}

    # NEXT row: LLM.int8 mixed decomposition on the Llama-7B decode inputs
    # (0.1% of channels x50, i.e. outliers above the 6.0 threshold)
    i8_calls, i8_bytes = [], []
    for (K, N) in WL["shapes"]:
        W = torch.from_numpy(S.layer_w(WL, K, N)).cuda()
        qw, sw = w4.llm_int8_quantize_weights(W)
        if (K, N) == (4096, 22016):
            t = time_per_call(lambda: w4.llm_int8_quantize_weights(W))
            b = N * K * 4 + N * K + 4 * N
            rows["llm_int8_quantize"] = {"shape": [N, K], "ms": t, "GB/s": b / t / 1e6}
        reps = [qw] + [qw.clone() for _ in range(_replicas_for(qw.numel(), l2) - 1)]
        for M in WL["Ms"]:
            X = bf16_dev(S.layer_x(WL, M, K, N))
            for r in reps:
                i8_calls.append(lambda X=X, r=r, sw=sw: w4.llm_int8_gemm(X, r, sw))
                i8_bytes.append(N * K + 4 * N + 2 * M * K + 2 * M * N)
        del W
    tg = time_graph(i8_calls)
    ts = time_calls(i8_calls, reps=5)
    rows["llm_int8_decode"] = {
        "configs": "(K,N) in {(4096,12288),(4096,4096),(4096,22016),(11008,4096)} x M in {1,4,16}, "
                   "threshold 6.0",
        "timing": "CUDA graph of all calls",
        "TB/s": sum(i8_bytes) / tg / 1e9,
        "frac_of_hbm": sum(i8_bytes) / tg / 1e6 / hbm,
        "eager_TB/s": sum(i8_bytes) / sum(ts) / 1e9}

    # NEXT row: LLM.int8 at prefill sizes (the tensor-core kind::i8 product)
    pre = {}
    for (K, N) in [(4096, 12288), (11008, 4096)]:
        W = torch.from_numpy(S.layer_w(WL, K, N)).cuda()
        qw, sw = w4.llm_int8_quantize_weights(W)
        del W
        for M in (256, 2048):
            X = bf16_dev(S.layer_x(WL, M, K, N))
            t = time_graph([lambda X=X, qw=qw, sw=sw: w4.llm_int8_gemm(X, qw, sw)])
            pre[f"K{K}_N{N}_M{M}"] = {"us": t * 1e3, "TOPS": 2.0 * M * N * K / t / 1e9}
            del X
        del qw, sw
    rows["llm_int8_prefill"] = {"timing": "CUDA graph of one call (3 launches)", "per_shape": pre}

    # NEXT row: GPTQ at quantization time (13B MLP up-projection, act-order, G = 32,
    # 512 calibration tokens): Hessian, then the compensated quantization
    K, N, G, ncal = 5120, 13824, ao["G"], 512
    W = torch.from_numpy(S.layer_w(ao, K, N)).cuda()
    xc = bf16_dev(S.draw_calib_x(ncal, K, tag=ao["tag"]))
    t_h = time_calls([lambda: w4.gptq_hessian(xc)], reps=3)[0]
    H = w4.gptq_hessian(xc)
    t_q = time_calls([lambda: w4.gptq_quantize(W, H, G, True)], reps=2, warm=1)[0]
    fl_h = 2.0 * ncal * K * K
    fl_q = 2.0 * K ** 3 / 3 + 1.0 * N * K * K   # factor + inverse, column updates
    rows["gptq"] = {"shape": [N, K], "G": G, "act_order": True, "calib_tokens": ncal,
                    "hessian_ms": t_h, "hessian_TFLOP/s": fl_h / t_h / 1e9,
                    "quantize_ms": t_q, "quantize_TFLOP/s": fl_q / t_q / 1e9}
    del W, xc, H
    torch.cuda.empty_cache()

    # a8: prefill tensor-core GEMM (70B MLP shapes)
    pf = S.PREFILL_70B
    out = {}
    for (K, N) in pf["shapes"]:
        G = pf["G"]
        W = torch.from_numpy(S.layer_w(pf, K, N)).cuda()
        Wq, sc, zr = w4.quantize_rtn(W, G)
        wp = w4.prepack(Wq, sc, zr, G)
        Wd = w4.dequant(Wq, sc, zr, G)
        del W, Wq, sc, zr
        for M in pf["Ms"]:
            X = bf16_dev(S.layer_x(pf, M, K, N))
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            t = time_calls([lambda: w4.w4a16_gemm(X, wp, N, K, G, out=Y)], reps=3)[0]
            tc = time_calls([lambda: torch.matmul(X, Wd.t())], reps=3)[0]
            fl = 2.0 * M * N * K
            out[f"K{K}_N{N}_M{M}"] = {"ms": t, "flops": fl, "TFLOP/s": fl / t / 1e9,
                                      "frac_of_bf16_peak": fl / t / 1e9 / peaks["bf16_tflops"],
                                      "cublas_bf16_dense_TFLOP/s": fl / tc / 1e9}
            del X, Y
        del Wd, wp
        torch.cuda.empty_cache()
    tot_fl = sum(v["flops"] for v in out.values())
    tot_ms = sum(v["ms"] for v in out.values())
    rows["prefill_gemm"] = {"per_shape": out, "TFLOP/s": tot_fl / tot_ms / 1e9,
                            "frac_of_bf16_peak": tot_fl / tot_ms / 1e9 / peaks["bf16_tflops"]}
    return rows


# --------------------------------------------------------------------- CPU oracle

def _oracle_layer(K, N, rows):
    """Oracle-side data for the first `rows` output rows of a decode layer
    (rows are independent, so a row subset is a faithful sample)."""
    import oracle as O
    W = S.layer_w(WL, K, N)[:rows]
    q, s, z = O.quantize_rtn(W, WL["G"])             # offline step, not timed
    return O.pack_nibbles(q), s, z, S.layer_x(WL, 1, K, N)


def _oracle_call(Wq, s, z, xb):
    import oracle as O
    O.matmul_ref(xb, O.dequant_rtn(Wq, s, z, WL["G"]))


def blas_threads() -> int:
    """Threads NumPy's BLAS runs the oracle's fp64 product on (its default:
    every core this process may use)."""
    from threadpoolctl import threadpool_info
    n = [int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas"]
    return max(n) if n else 1


def oracle_sample(rows=4096):
    """Time the CPU oracle (dequant + fp64 matmul) on the decode workload: the
    first `rows` output rows of each of the 4 layer shapes at M = 1, on the
    host's cores (BLAS default threads).  Returns (bytes, seconds, description)."""
    tot_b, tot_s = 0.0, 0.0
    for (K, N) in WL["shapes"]:
        r = min(rows, N)
        Wq, s, z, xb = _oracle_layer(K, N, r)
        t0 = time.perf_counter()
        _oracle_call(Wq, s, z, xb)
        tot_s += time.perf_counter() - t0
        tot_b += int4_bytes(1, r, K, WL["G"])
    return tot_b, tot_s, (f"first {rows} output rows of each of the 4 layer shapes at M=1: "
                          f"numpy dequant + fp64 matmul, BLAS on {blas_threads()} threads")


def oracle_prefill_sample(tokens=256, rows=4096):
    """The oracle on a bounded prefill sample: tokens 0..tokens-1 of the 70B
    M = 512 activations against the first `rows` output rows of the
    K = 8192, N = 28672 layer.  Returns (flops, seconds, description)."""
    import oracle as O
    pf = S.PREFILL_70B
    K, N = pf["shapes"][0]
    W = S.layer_w(pf, K, N)[:rows]
    q, s, z = O.quantize_rtn(W, pf["G"])                # offline step, not timed
    Wq = O.pack_nibbles(q)
    xb = S.layer_x(pf, pf["Ms"][0], K, N)[:tokens]
    t0 = time.perf_counter()
    O.matmul_ref(xb, O.dequant_rtn(Wq, s, z, pf["G"]))
    sec = time.perf_counter() - t0
    return (2.0 * tokens * rows * K, sec,
            f"tokens 0..{tokens - 1} of the M={pf['Ms'][0]} input x first {rows} output rows of "
            f"K={K}, N={N}: numpy dequant + fp64 matmul, BLAS on {blas_threads()} threads")


def run_reference(args, world, rank):
    """`--impl reference`: the CPU oracle as the reference arm, same metric and
    config.  Each step is one oracle decode call at M = 1 on a row subset of a
    layer (rotating over the 4 shapes), the subset sized so that the whole run
    takes about two minutes."""
    if rank != 0:
        return
    n_total = args.warmup + args.steps
    budget = max(0.002, 90.0 / n_total)             # seconds per step
    # calibrate seconds per row on a 1024-row slice of the deepest layer
    Wq, s, z, xb = _oracle_layer(11008, 4096, 1024)
    _oracle_call(Wq, s, z, xb)
    t0 = time.perf_counter()
    _oracle_call(Wq, s, z, xb)
    per_row = 1.5 * (time.perf_counter() - t0) / 1024
    rows = int(max(8, min(4096, budget / max(per_row, 1e-9))))
    prepared = [(K, N, *_oracle_layer(K, N, min(rows, N))) for (K, N) in WL["shapes"]]
    tot_b, tot_s = 0.0, 0.0
    for i in range(n_total):
        K, N, Wq, s, z, xb = prepared[i % len(prepared)]
        t0 = time.perf_counter()
        _oracle_call(Wq, s, z, xb)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            tot_s += dt
            tot_b += int4_bytes(1, Wq.shape[0], K, WL["G"])
    v = tot_b / tot_s / 1e12
    cores = blas_threads()
    sample = (f"one M=1 decode call per step on the first {rows} output rows of a layer, "
              f"4 layer shapes rotating; numpy dequant + fp64 matmul, BLAS on {cores} threads")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_s * 1e3 / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": v, "unit": "TB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_single(w4, args):
    fmt, K, N, M = args.single[0], *map(int, args.single[1:])
    if fmt in ("nf4", "fp4"):
        wl = S.NF4_DECODE if fmt == "nf4" else S.FP4_DECODE
        W = torch.from_numpy(S.layer_w(wl, K, N)).cuda()
        q, c, s2 = (w4.nf4_quantize if fmt == "nf4" else w4.fp4_quantize)(W)
        wp = w4.nf4_prepack(q, c)
        X = bf16_dev(S.layer_x(wl, M, K, N))
        gemm = w4.nf4_gemm if fmt == "nf4" else w4.fp4_gemm
        f = (lambda: gemm(X, wp, s2, N, K))
        nbytes, flops = nf4_bytes(M, N, K), 2.0 * M * N * K
    elif fmt in ("quant", "nf4q"):
        # the quantize kernels alone (M unused): INT4 RTN g128, or NF4 with
        # double-quantized constants
        wl = WL if fmt == "quant" else S.NF4_DECODE
        W = torch.from_numpy(S.layer_w(wl, K, N)).cuda()
        f = ((lambda W=W: w4.quantize_rtn(W, WL["G"])) if fmt == "quant"
             else (lambda W=W: w4.nf4_quantize(W)))
        nbytes = N * K * 4 + N * K / 2 + (N * (K // WL["G"]) * 3 if fmt == "quant" else N * K // 64)
        flops = 0.0
    elif fmt == "gptq":
        # M = calibration tokens; act-order, G = 32 (the 13B act-order family)
        G = S.ACT_ORDER_13B["G"]
        W = torch.from_numpy(S.layer_w(S.ACT_ORDER_13B, K, N)).cuda()
        xc = bf16_dev(S.draw_calib_x(M, K, tag=S.ACT_ORDER_13B["tag"]))
        H = w4.gptq_hessian(xc)
        f = (lambda W=W, H=H: w4.gptq_quantize(W, H, G, True))
        nbytes, flops = N * K * 4, 2.0 * K ** 3 / 3 + 1.0 * N * K * K
    elif fmt == "int8":
        W = torch.from_numpy(S.layer_w(WL, K, N)).cuda()
        qw, sw = w4.llm_int8_quantize_weights(W)
        X = bf16_dev(S.layer_x(WL, M, K, N))
        f = (lambda: w4.llm_int8_gemm(X, qw, sw))
        nbytes, flops = N * K + 4 * N + 2 * M * K + 2 * M * N, 2.0 * M * N * K
    elif fmt == "awq":
        aw = S.AWQ_SYM_DECODE
        G = aw["G"]
        W = torch.from_numpy(S.layer_w(aw, K, N)).cuda()
        sd = torch.from_numpy(S.layer_awq_s(aw, K, N)).cuda()
        Wq, sc, zr = w4.quantize_sym(w4.awq_scale_weights(W, sd), G)
        wp = w4.prepack(Wq, sc, zr, G)
        X = bf16_dev(S.layer_x(aw, M, K, N))
        f = (lambda: w4.w4a16_awq_gemm(X, sd, wp, N, K, G))
        nbytes, flops = int4_bytes(M, N, K, G) + 4 * K, 2.0 * M * N * K
    else:
        G = WL["G"]
        W = torch.from_numpy(S.layer_w(WL, K, N)).cuda()
        Wq, sc, zr = w4.quantize_rtn(W, G)
        wp = w4.prepack(Wq, sc, zr, G)
        X = bf16_dev(S.layer_x(WL, M, K, N))
        f = (lambda: w4.w4a16_gemm(X, wp, N, K, G))
        nbytes, flops = int4_bytes(M, N, K, G), 2.0 * M * N * K
    del W
    t = time_calls([f], reps=max(1, args.steps), warm=args.warmup)[0]
    print(json.dumps({"single": [fmt, K, N, M], "us": t * 1e3, "TB/s": nbytes / t / 1e9,
                      "TFLOP/s": flops / t / 1e9}), flush=True)


def run_probe(name):
    """Compile a microbenchmark for sm_100a into a temporary directory and run it."""
    import subprocess
    import tempfile
    src = os.path.join(ROOT, "weight_only_bit_gemm_b200", "probes", name + ".cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, name)
        subprocess.run([os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O3", "-std=c++17", "-o", exe, src], check=True)
        subprocess.run([exe], check=True)


# --------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-rows", action="store_true", help="skip the other-row measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--probe", choices=["pipes", "tcgen05_mma"],
                    help="build and run one microbenchmark of weight_only_bit_gemm_b200/probes "
                         "(the measurements the kernels' design rests on) and print its table")
    ap.add_argument("--single", nargs=4, metavar=("FMT", "K", "N", "M"),
                    help="profiling aid: run one layer call (FMT int4|nf4|fp4|awq|gptq|int8, or the "
                         "quantize kernels quant|nf4q) warmup+steps times "
                         "eagerly and print its mean device time")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.probe:
        run_probe(args.probe)
        return

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return

    world, rank, local, pg = dist_setup()
    from weight_only_bit_gemm_b200 import build
    build.build()
    from weight_only_bit_gemm_b200 import w4

    if args.single:
        run_single(w4, args)
        return

    peaks = load_peaks()
    step = DecodeStep(w4)
    ms, per_call, clocks = measure_decode(step, args, pg, local)
    ms = max_over_ranks(pg, ms)
    total_bytes = sum_over_ranks(pg, step.step_bytes * args.steps)
    value = total_bytes / (ms * 1e-3) / 1e12
    e2e_ms, e2e_n, h2d, d2h = measure_e2e(step, args, pg)
    e2e_value = sum_over_ranks(pg, step.step_bytes * e2e_n) / (e2e_ms * 1e-3) / 1e12
    if w4.device_status() != w4.W4_OK:
        raise RuntimeError("device error during the benchmark")

    # every launch in the timed step is the decode kernel: its mean duration is
    # the step time over the launches in it
    launch_ms = (ms / args.steps) / len(step.calls)
    achieved = (step.step_bytes / len(step.calls)) / (launch_ms * 1e-3) / 1e9
    per_shape = {}
    for c, t in zip(step.calls, per_call):
        per_shape[f"K{c['K']}_N{c['N']}_M{c['M']}"] = {
            "us": round(t * 1e3, 3), "TB/s": round(c["bytes"] / (t * 1e-3) / 1e12, 3)}

    rows = None
    cpu = None
    if rank == 0 and world == 1:
        if not args.no_rows:
            rows = measure_rows(w4, peaks)
        if not args.no_cpu:
            b, sec, desc = oracle_sample()
            fl, psec, pdesc = oracle_prefill_sample()
            cpu = {"value": b / sec / 1e12, "unit": "TB/s", "cores": blas_threads(),
                   "kind": "oracle", "sample": desc, "seconds": sec,
                   "prefill": {"value": fl / psec / 1e12, "unit": "TFLOP/s", "sample": pdesc,
                               "seconds": psec}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "calls_per_step": len(step.calls),
                       "bytes_per_step": step.step_bytes,
                       "l2": f"inputs larger than L2: {step.replicas} weight replicas per layer, "
                             f"{step.replica_bytes / 1e6:.0f} MB total, each call reads its own",
                       "parallelism": f"replicas x{world} (independent problems per GPU)",
                       "timing": "CUDA graph of one step, CUDA events on the launching stream"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": traffic_per_launch(step), "peak_source": peaks["source"],
                         "kernel": "w4_gemv_kernel",
                         "launch_us": launch_ms * 1e3,
                         "algorithmic_bytes_per_launch": step.step_bytes / len(step.calls),
                         "per_call_isolated": per_shape},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * len(step.calls),
            "clocks": clocks,
        }
        if rows is not None:
            line["rows"] = rows
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
