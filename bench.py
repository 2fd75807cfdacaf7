"""Benchmark of the NVFP4 W4A4 linear-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill]

Prints ONE JSON line (rank 0).  Default workload ("decode"): the decode GEMV
configuration -- M in {1,2,4,8,16}, (N,K) in {(4096,4096), (14336,4096),
(4096,14336)}, bf16 activations N(0,1) with 1% of channels x50 quantized online
(per-tensor amax, block scales, codes) and multiplied by pre-quantized NVFP4
weights N(0,0.02).  One step = all 15 (M, shape) linear calls, each
nvfp4_quantize + nvfp4_gemm.  Weights rotate through 4 copies per shape
(302 MB) so each call streams its weights from HBM, not L2.

value = aggregate algorithmic GB/s of a step (per call N*K*9/16 + M*K*(2+9/16)
+ 4*M*N bytes), device-timed with CUDA events around K graph-replayed steps.
Multi-GPU: replicas only (the decode path has no data-path exchange); value is
the bytes all ranks processed over the slowest rank's time.
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

METRIC = "NVFP4 linear µs/call & GB/s at M=1–16, TFLOP/s at M=8192; % of roofline"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "100", *sel], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.15)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts + frac, float(parts[2]), float(parts[3]), parts[6:10]))
            except Exception:
                continue
        os.unlink(self.f.name)
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.05 <= r[0] <= (self.t1 or 1e18) + 0.05]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(inside), "samples_total": len(rows)}


# ------------------------------------------------------------ distributed

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------ decode workload

def decode_bytes(M, N, K):
    """Algorithmic bytes of one online-quantized linear call: W codes+scales, X bf16
    read, X NVFP4 written/read once, Y fp32 written."""
    return N * K * 9 // 16 + M * K * 2 + M * K * 9 // 16 + 4 * M * N


def gemv_bytes(M, N, K):
    return N * K * 9 // 16 + M * K * 9 // 16 + 4 * M * N


class DecodeWorkload:
    """Decode step: 15 (M, shape) online-quantized linear calls.  Operands use
    TILED block scales, so nvfp4_gemm runs the tensor-core few-row path; a
    ROWMAJOR twin of every operand (same codes) serves to time the CUDA-core
    GEMV on the same data."""
    COPIES = 4

    def __init__(self, dev):
        import nvfp4_block_scaled_18_b200 as nv
        from nvfp4_block_scaled_18_b200 import workloads as wl
        self.nv, self.wl, self.dev = nv, wl, dev
        self.shapes = list(wl.DECODE_SHAPES)
        self.Ms = list(wl.DECODE_M)
        self.calls = [(M, N, K) for M in self.Ms for (N, K) in self.shapes]
        self.W, self.Wrm = {}, {}
        for (N, K) in self.shapes:
            w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
            q0 = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q0, workspace=nv.Workspace(N, K, dev))
            r0 = nv.NVFP4Tensor.empty(N, K, nv.SF_ROWMAJOR, device=dev)
            nv.nvfp4_quantize(w, r0, workspace=nv.Workspace(N, K, dev))
            del w
            tiled, rowm = [q0], [r0]
            for _ in range(self.COPIES - 1):
                c = q0.codes.clone()
                tiled.append(nv.NVFP4Tensor(c, q0.scales.clone(), q0.tensor_scale.clone(), N, K, nv.SF_TILED))
                rowm.append(nv.NVFP4Tensor(c, r0.scales.clone(), r0.tensor_scale.clone(), N, K, nv.SF_ROWMAJOR))
            self.W[(N, K)], self.Wrm[(N, K)] = tiled, rowm
        self.X, self.Xhost, self.QX, self.QXrm, self.WS, self.Y, self.Yhost = {}, {}, {}, {}, {}, {}, {}
        for M in self.Ms:
            for K in sorted({k for _, k in self.shapes}):
                x = wl.to_bf16(wl.decode_x(M, K))
                self.Xhost[(M, K)] = x.pin_memory()
                self.X[(M, K)] = x.to(dev)
                self.QX[(M, K)] = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
                self.QXrm[(M, K)] = nv.NVFP4Tensor.empty(M, K, nv.SF_ROWMAJOR, device=dev)
                self.WS[(M, K)] = nv.Workspace(M, K, dev)
            for (N, K) in self.shapes:
                self.Y[(M, N, K)] = torch.empty((M, N), dtype=torch.float32, device=dev)
                self.Yhost[(M, N, K)] = torch.empty((M, N), dtype=torch.float32).pin_memory()
        self.step_bytes = sum(decode_bytes(*c) for c in self.calls)
        self.launches_per_step = 3 * len(self.calls)  # amax + quantize + GEMV per call
        torch.cuda.synchronize()

    def copy_index(self, step, i):
        return ((step * len(self.calls) + i) // len(self.shapes)) % self.COPIES

    def run_step(self, step, e2e=False):
        nv = self.nv
        for i, (M, N, K) in enumerate(self.calls):
            if e2e:
                self.X[(M, K)].copy_(self.Xhost[(M, K)], non_blocking=True)
            nv.nvfp4_quantize(self.X[(M, K)], self.QX[(M, K)], workspace=self.WS[(M, K)])
            nv.nvfp4_gemm(self.QX[(M, K)], self.W[(N, K)][self.copy_index(step, i)], self.Y[(M, N, K)])
            if e2e:
                self.Yhost[(M, N, K)].copy_(self.Y[(M, N, K)], non_blocking=True)

    def h2d_bytes(self):
        return sum(M * K * 2 for (M, N, K) in self.calls)

    def d2h_bytes(self):
        return sum(M * N * 4 for (M, N, K) in self.calls)


def capture_graphs(wk, phases, e2e=False):
    graphs = []
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for p in range(phases):      # eager warm-up of every phase (sets kernel attributes)
            wk.run_step(p, e2e)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for p in range(phases):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            wk.run_step(p, e2e)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def time_graphs(graphs, steps, warmup, world, sampler=None):
    n = len(graphs)
    for i in range(warmup):
        graphs[i % n].replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark_start()
    start.record()
    for i in range(steps):
        graphs[i % n].replay()
    end.record()
    end.synchronize()
    if sampler:
        sampler.mark_end()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)


def time_gemv_launches(wk, rowmajor=False, reps=24):
    """Per-launch device time (ms) of the decode GEMM for every (M, shape):
    the tensor-core few-row kernel (TILED operands) or, with rowmajor=True, the
    CUDA-core GEMV on the same codes.  Weights rotate through the copies."""
    nv = wk.nv
    out = {}
    for (M, N, K) in wk.calls:
        qx = (wk.QXrm if rowmajor else wk.QX)[(M, K)]
        ws = (wk.Wrm if rowmajor else wk.W)[(N, K)]
        y = wk.Y[(M, N, K)]
        nv.nvfp4_quantize(wk.X[(M, K)], qx, workspace=wk.WS[(M, K)])
        i = [0]

        def call():
            nv.nvfp4_gemm(qx, ws[i[0] % wk.COPIES], y)
            i[0] += 1
        out[(M, N, K)] = time_launches(call, reps=reps)
    return out


# ------------------------------------------------------------ prefill workload

def fp4_peak_tflops(peaks, sustained=False):
    """Dense FP4 peak: the measured bf16 GEMM peak x 4 (nominal 9 / 2.25 PFLOP/s)."""
    return 4.0 * (peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"])


class PrefillWorkload:
    """Large prefill W4A4: M = 8192, (N,K) in {(14336,4096), (4096,14336), (28672,8192)},
    bf16 N(0,1) activations with 1% channels x50 quantized online (TILED scales),
    each shape with and without the S = 256 outlier-residue K extension
    (reorder + residue quantizer with no normalisation, W_aug of K+S columns)."""

    S = 256

    def __init__(self, dev):
        import nvfp4_block_scaled_18_b200 as nv
        from nvfp4_block_scaled_18_b200 import workloads as wl
        self.nv, self.dev = nv, dev
        self.M = wl.PREFILL_M
        self.shapes = list(wl.PREFILL_SHAPES)
        self.calls = []   # (name, M, N, Keff, S)
        self.buf = {}
        g = torch.Generator(device="cpu").manual_seed(0)
        for (N, K) in self.shapes:
            x = wl.to_bf16(wl.prefill_x(self.M, K)).to(dev)
            perm = torch.from_numpy(wl.calibrated_perm(wl.prefill_x(64, K))).to(dev)
            w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
            qw = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, qw, workspace=nv.Workspace(N, K, dev))
            w_aug = torch.cat([w[:, perm.long()], w[:, perm[: self.S].long()]], dim=1).contiguous()
            del w
            qwa = nv.NVFP4Tensor.empty(N, K + self.S, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w_aug, qwa, workspace=nv.Workspace(N, K + self.S, dev))
            del w_aug
            self.buf[(N, K)] = dict(
                x=x, perm=perm, qw=qw, qwa=qwa,
                qx=nv.NVFP4Tensor.empty(self.M, K, nv.SF_TILED, device=dev),
                qxa=nv.NVFP4Tensor.empty(self.M, K + self.S, nv.SF_TILED, device=dev),
                ws=nv.Workspace(self.M, K, dev),
                y=torch.empty((self.M, N), dtype=torch.float32, device=dev))
            self.calls.append(("plain", self.M, N, K, 0))
            self.calls.append(("k+s", self.M, N, K + self.S, self.S))
        torch.cuda.synchronize()

    def quantize(self, N, K, S):
        b = self.buf[(N, K)]
        if S == 0:
            self.nv.nvfp4_quantize(b["x"], b["qx"], workspace=b["ws"])
        else:
            self.nv.nvfp4_rmsnorm_reorder_quantize(b["x"], b["qxa"], perm=b["perm"], S=S, workspace=b["ws"])

    def gemm(self, N, K, S):
        b = self.buf[(N, K)]
        self.nv.nvfp4_gemm(b["qxa"] if S else b["qx"], b["qwa"] if S else b["qw"], b["y"])

    def run_step(self, step=0, e2e=False):
        for (_, M, N, Keff, S) in self.calls:
            K = Keff - S
            self.quantize(N, K, S)
            self.gemm(N, K, S)

    def h2d_bytes(self):
        return sum(M * (Keff - S) * 2 for (_, M, N, Keff, S) in self.calls)

    def d2h_bytes(self):
        return sum(M * N * 4 for (_, M, N, Keff, S) in self.calls)


def prefill_e2e(wk, steps):
    """End-to-end prefill step time (ms): each call's X copied from pinned host
    memory, quantized, multiplied, and Y copied back to pinned host memory."""
    host_x = {k: b["x"].cpu().pin_memory() for k, b in wk.buf.items()}
    host_y = {k: torch.empty(b["y"].shape, dtype=torch.float32).pin_memory() for k, b in wk.buf.items()}

    def step():
        for (_, M, N, Keff, S) in wk.calls:
            K = Keff - S
            b = wk.buf[(N, K)]
            b["x"].copy_(host_x[(N, K)], non_blocking=True)
            wk.quantize(N, K, S)
            wk.gemm(N, K, S)
            host_y[(N, K)].copy_(b["y"], non_blocking=True)

    step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step()
    end.record()
    end.synchronize()
    return start.elapsed_time(end)


def time_launches(fn, reps=8, rounds=3):
    """Median device time (ms) of fn() launches: CUDA events around each launch,
    all queued behind a sleep kernel so host gaps never enter the intervals."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    fn()
    times = []
    for _ in range(rounds):
        torch.cuda.synchronize()
        torch.cuda._sleep(20_000_000)
        for r in range(reps):
            ev[r][0].record()
            fn()
            ev[r][1].record()
        torch.cuda.synchronize()
        times += [a.elapsed_time(b) for a, b in ev]
    return statistics.median(times)


def measure_prefill_from(wk, peaks):
    """Per-launch GEMM and quantizer times on the prefill workload."""
    out, flops_total, gemm_ms_total = {}, 0.0, 0.0
    for (name, M, N, Keff, S) in wk.calls:
        K = Keff - S
        wk.quantize(N, K, S)
        g_ms = time_launches(lambda: wk.gemm(N, K, S))
        q_ms = time_launches(lambda: wk.quantize(N, K, S))
        flops = 2.0 * M * N * Keff
        q_bytes = 2 * M * K + M * Keff * 9 // 16
        flops_total += flops
        gemm_ms_total += g_ms
        out[f"M{M}_N{N}_K{K}" + (f"+S{S}" if S else "")] = {
            "gemm_us": round(g_ms * 1e3, 2), "gemm_TFLOPs": round(flops / (g_ms * 1e-3) / 1e12, 1),
            "gemm_frac_fp4_peak": round(flops / (g_ms * 1e-3) / 1e12 / fp4_peak_tflops(peaks), 4),
            "quant_us": round(q_ms * 1e3, 2), "quant_GBps": round(q_bytes / (q_ms * 1e-3) / 1e9, 1)}
    achieved = flops_total / (gemm_ms_total * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp4_peak_tflops(peaks), 1),
            "unit": "TFLOP/s", "frac": round(achieved / fp4_peak_tflops(peaks), 4), "traffic": None,
            "kernel": "k_gemm_nvf4 (6 prefill launches)",
            "peak_source": peaks["source"] + " bf16 x4 (dense FP4 / bf16 nominal ratio)"}
    return out, roof


# ------------------------------------------------------------ CPU baseline

def cpu_oracle_sample(workload: str = "decode", budget_s: float = 12.0):
    """Time the CPU oracle (as it stands) on the decode workload: (N,K)=(4096,4096),
    M in {1,16}; quantize X online, fp64 GEMM on the dequantized operands."""
    import oracle
    from nvfp4_block_scaled_18_b200 import workloads as wl
    oracle.build()
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    if workload == "prefill":
        # a 128-row slice of the M = 8192 activations against the full (14336, 4096) weight
        N, K, rows = 14336, 4096, 128
        qw = oracle.quantize(wl.weights_normal(N, K))
        x = wl.prefill_x(rows, K)
        flops, t_total, calls = 0.0, 0.0, 0
        t_start = time.perf_counter()
        while time.perf_counter() - t_start < budget_s or calls < 1:
            t0 = time.perf_counter()
            oracle.gemm(oracle.quantize(x), qw)
            t_total += time.perf_counter() - t0
            flops += 2.0 * rows * N * K
            calls += 1
        return {"value": round(flops / t_total / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                "sample": f"{calls} x (128 rows of X, M=8192 workload) against W (14336,4096): oracle quantize "
                          f"+ fp64 dequantized GEMM, {t_total:.1f} s"}
    N, K = 4096, 4096
    w = wl.weights_normal(N, K)
    qw = oracle.quantize(w)
    done_bytes, t_total, calls = 0, 0.0, 0
    Ms = [1, 16]
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s or calls < 2:
        M = Ms[calls % 2]
        x = wl.decode_x(M, K)
        t0 = time.perf_counter()
        qx = oracle.quantize(x)
        oracle.gemm(qx, qw)
        t_total += time.perf_counter() - t0
        done_bytes += decode_bytes(M, N, K)
        calls += 1
    return {"value": round(done_bytes / t_total / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{calls} linear calls on (N,K)=(4096,4096), M alternating 1/16: oracle quantize "
                      f"+ fp64 dequantized GEMM, {t_total:.1f} s"}


def reference_arm(args):
    """--impl reference: the CPU oracle timed as the comparison arm (rank 0 only)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    from nvfp4_block_scaled_18_b200 import workloads as wl
    oracle.build()
    budget = 150.0
    per_step = max(0.02, min(1.0, budget / max(1, args.steps + args.warmup)))
    shapes = list(wl.DECODE_SHAPES)
    Ms = list(wl.DECODE_M)
    cache = {}

    def sample(i):
        M, (N, K) = Ms[i % len(Ms)], shapes[(i // len(Ms)) % len(shapes)]
        if (N, K) not in cache:
            w = wl.weights_normal(N, K)
            cache[(N, K)] = (oracle.quantize(w), w.shape[0])
        qw, _ = cache[(N, K)]
        # bound the work of a step: a row subset of W sized to the per-step budget
        rows = max(8, min(N, int(per_step * 4e5 / max(1, K / 4096))))
        sub = oracle.QTensor(qw.codes[:rows], qw.scales[:rows], qw.s)
        x = wl.decode_x(M, K)
        t0 = time.perf_counter()
        oracle.gemm(oracle.quantize(x), sub)
        return time.perf_counter() - t0, decode_bytes(M, rows, K)

    for i in range(args.warmup):
        sample(i)
    t, b = 0.0, 0
    for i in range(args.steps):
        dt, db = sample(i)
        t += dt
        b += db
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    value = b / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode GEMV, M=1..16, (N,K)=(4096,4096),(14336,4096),(4096,14336); "
                                   "CPU oracle on a bounded row sample of W per step"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps, each one linear call on a W row subset"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="decode line without the prefill sub-measurement")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return reference_arm(args)

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    import nvfp4_block_scaled_18_b200 as nv
    nv.load_library()
    peaks = load_peaks()

    if args.workload == "decode":
        wk = DecodeWorkload(dev)
        phases = DecodeWorkload.COPIES
        unit, work_per_step = "GB/s", float(wk.step_bytes)
        scale = 1e9
        steps = args.steps
    else:
        wk = PrefillWorkload(dev)
        phases = 1
        unit, work_per_step = "TFLOP/s", float(sum(2.0 * M * N * Keff for (_, M, N, Keff, _) in wk.calls))
        scale = 1e12
        steps = max(1, min(args.steps, 40))
    graphs = capture_graphs(wk, phases)
    sampler = ClockSampler(torch.cuda.current_device())
    ms = time_graphs(graphs, steps, args.warmup, world, sampler)
    clocks = sampler.stop()
    ms_max = max_over_ranks(ms, world)
    value = sum_over_ranks(work_per_step * steps, world) / (ms_max * 1e-3) / scale
    ms_per_step = ms_max / steps

    # end to end: pinned host X -> device, quantize + GEMM, Y -> pinned host, every step
    e2e_steps = max(4 * phases, min(steps, 400)) if args.workload == "decode" else max(2, min(steps, 5))
    if args.workload == "decode":
        e2e_graphs = capture_graphs(wk, phases, e2e=True)
        ms_e2e = max_over_ranks(time_graphs(e2e_graphs, e2e_steps, args.warmup, world), world)
        h2d, d2h = wk.h2d_bytes(), wk.d2h_bytes()
    else:
        ms_e2e, h2d, d2h = prefill_e2e(wk, e2e_steps), wk.h2d_bytes(), wk.d2h_bytes()
        ms_e2e = max_over_ranks(ms_e2e, world)
        e2e_graphs = []
    e2e_value = sum_over_ranks(work_per_step * e2e_steps, world) / (ms_e2e * 1e-3) / scale

    line = {"metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5)}
    if args.workload == "decode":
        per = time_gemv_launches(wk)
        per_cc = time_gemv_launches(wk, rowmajor=True)
        g_bytes = sum(gemv_bytes(*c) for c in wk.calls)
        achieved = g_bytes / (sum(per.values()) * 1e-3) / 1e9
        achieved_cc = g_bytes / (sum(per_cc.values()) * 1e-3) / 1e9
        line["us_per_call"] = round(ms_per_step * 1e3 / len(wk.calls), 3)
        detail = {f"M{M}_N{N}_K{K}": {
            "tc_us": round(per[(M, N, K)] * 1e3, 3),
            "tc_GBps": round(gemv_bytes(M, N, K) / (per[(M, N, K)] * 1e-3) / 1e9, 1),
            "cuda_core_us": round(per_cc[(M, N, K)] * 1e3, 3),
            "cuda_core_GBps": round(gemv_bytes(M, N, K) / (per_cc[(M, N, K)] * 1e-3) / 1e9, 1)}
            for (M, N, K) in wk.calls}
        detail["cuda_core_gemv_aggregate"] = {"achieved_GBps": round(achieved_cc, 1),
                                              "frac": round(achieved_cc / peaks["hbm_gbs"], 4)}
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                    "kernel": "k_gemv_tc (tensor-core few-row GEMM, all 15 decode launches)",
                    "peak_source": peaks["source"]}
        config = {"workload": "decode GEMV (M in 1,2,4,8,16; (N,K) in (4096,4096),(14336,4096),(4096,14336)); "
                              "online bf16->NVFP4 activation quantization + NVFP4 GEMM, fp32 out",
                  "calls_per_step": len(wk.calls), "l2": "weights rotate through 4 copies per shape (302 MB > L2)",
                  "parallelism": f"replicas x{world}"}
        launches = wk.launches_per_step * steps
    else:
        detail, roofline = measure_prefill_from(wk, peaks)
        config = {"workload": "large prefill W4A4 GEMM, M=8192, (N,K) in (14336,4096),(4096,14336),(28672,8192), "
                              "each without and with the S=256 outlier-residue K extension; online quantization",
                  "calls_per_step": len(wk.calls), "l2": "inputs > L2 (X 67-235 MB, Y 134-940 MB per call)",
                  "parallelism": f"replicas x{world}"}
        launches = 3 * len(wk.calls) * steps
    line.update({"higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1",
                 "data": "synthetic", "config": config, "roofline": roofline,
                 "e2e": {"value": round(e2e_value, 2), "unit": unit, "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h},
                 "gpu_launches": launches, "clocks": clocks, "detail": detail})
    if args.workload == "decode" and not args.no_prefill:
        del graphs, e2e_graphs
        pw = PrefillWorkload(dev)
        pdetail, proof = measure_prefill_from(pw, peaks)
        line["prefill"] = {"roofline": proof, "detail": pdetail}
        del pw
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
