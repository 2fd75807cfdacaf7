"""Benchmark of the NVFP4 W4A4 linear-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill]

Prints ONE JSON line (rank 0).  Default workload ("decode"): the decode GEMV
configuration -- M in {1,2,4,8,16}, (N,K) in {(4096,4096), (14336,4096),
(4096,14336)}, bf16 activations N(0,1) with 1% of channels x50 quantized online
(per-tensor amax, block scales, codes) and multiplied by pre-quantized NVFP4
weights N(0,0.02).  One step = all 15 (M, shape) linear calls, each one
nvfp4_quantize_gemm (activation quantization and GEMM in one launch; Q(X) is
written as well).  Every shape has enough weight copies (>= 260 MB) that each
call streams its weights from HBM, not L2.

value = aggregate algorithmic GB/s of a step (per call N*K*9/16 + M*K*(2+9/16)
+ 4*M*N bytes), device-timed with CUDA events around K graph-replayed steps.
Per-call times in "detail" come from graphs of back-to-back calls of one shape
(the steady state of a chain of layers).  Multi-GPU: replicas only (the decode
path has no data-path exchange); value is the bytes all ranks processed over
the slowest rank's time.
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

def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU (torchrun env).  NCCL where CUDA is present, gloo
    otherwise (host-only runs and tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    use_cuda = torch.cuda.is_available()
    if backend is None:
        backend = "nccl" if use_cuda else "gloo"
    if use_cuda:
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _all_reduce_scalar(x: float, world: int, op) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    import torch.distributed as dist
    return _all_reduce_scalar(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x: float, world: int) -> float:
    import torch.distributed as dist
    return _all_reduce_scalar(x, world, dist.ReduceOp.SUM if world > 1 else None)


def replica_throughput(work: float, ms: float, world: int, scale: float):
    """Whole-job throughput of independent replicas: the work all ranks did over
    the slowest rank's time.  Returns (value in units/s / scale, max ms)."""
    ms_max = max_over_ranks(ms, world)
    total = sum_over_ranks(work, world)
    return total / (ms_max * 1e-3) / scale, ms_max


# ------------------------------------------------------------ decode workload

# DRAM traffic / algorithmic bytes of k_decode_tc from its ncu capture (None once the kernel
# changes after the capture)
DECODE_TRAFFIC_RATIO = 33.103104e6 / (4096 * 14336 * 9 / 16 + 1 * 14336 * (2 + 9 / 16) + 4 * 1 * 4096)


def decode_bytes(M, N, K):
    """Algorithmic bytes of one online-quantized linear call: W codes+scales, X bf16
    read, X NVFP4 written/read once, Y fp32 written."""
    return N * K * 9 // 16 + M * K * 2 + M * K * 9 // 16 + 4 * M * N


def gemv_bytes(M, N, K):
    return N * K * 9 // 16 + M * K * 9 // 16 + 4 * M * N


class DecodeWorkload:
    """Decode step: 15 (M, shape) linear calls, each nvfp4_quantize_gemm on TILED
    weights (tensor-core decode kernel, activation quantization fused).  Every
    shape keeps enough weight copies to exceed L2.  A ROWMAJOR twin of every
    weight (same codes) serves to time the CUDA-core GEMV on the same data."""
    L2_SPAN = 260e6

    def __init__(self, dev):
        import nvfp4_block_scaled_18_b200 as nv
        from nvfp4_block_scaled_18_b200 import workloads as wl
        self.nv, self.wl, self.dev = nv, wl, dev
        self.shapes = list(wl.DECODE_SHAPES)
        self.Ms = list(wl.DECODE_M)
        self.calls = [(M, N, K) for M in self.Ms for (N, K) in self.shapes]
        self.W, self.Wrm, self.copies = {}, {}, {}
        for (N, K) in self.shapes:
            w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
            q0 = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q0, workspace=nv.Workspace(N, K, dev))
            r0 = nv.NVFP4Tensor.empty(N, K, nv.SF_ROWMAJOR, device=dev)
            nv.nvfp4_quantize(w, r0, workspace=nv.Workspace(N, K, dev))
            del w
            n = max(4, int(np.ceil(self.L2_SPAN / (N * K * 9 / 16))))
            tiled, rowm = [q0], [r0]
            for _ in range(n - 1):
                c = q0.codes.clone()
                tiled.append(nv.NVFP4Tensor(c, q0.scales.clone(), q0.tensor_scale.clone(), N, K, nv.SF_TILED))
                rowm.append(nv.NVFP4Tensor(c, r0.scales.clone(), r0.tensor_scale.clone(), N, K, nv.SF_ROWMAJOR))
            self.W[(N, K)], self.Wrm[(N, K)], self.copies[(N, K)] = tiled, rowm, n
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
        # 1 launch per call when quantization is fused, 2 where quantize-then-GEMM is chosen
        self.plan = {c: nv.nvfp4_quantize_gemm_plan(*c) for c in self.calls}
        assert all(v in (1, 2) for v in self.plan.values()), self.plan
        self.launches_per_step = sum(self.plan.values())
        self.phases = max(self.copies.values())
        torch.cuda.synchronize()

    def weight(self, N, K, i, rowmajor=False):
        ws = (self.Wrm if rowmajor else self.W)[(N, K)]
        return ws[i % len(ws)]

    def call(self, M, N, K, i, mode="fused"):
        """One linear call with weight copy i: 'fused' (one launch), 'separate'
        (nvfp4_quantize + nvfp4_gemm) or 'cuda_core' (ROWMAJOR operands)."""
        nv = self.nv
        x, y = self.X[(M, K)], self.Y[(M, N, K)]
        if mode == "fused":
            nv.nvfp4_quantize_gemm(x, self.QX[(M, K)], self.weight(N, K, i), y)
        elif mode == "separate":
            nv.nvfp4_quantize(x, self.QX[(M, K)], workspace=self.WS[(M, K)])
            nv.nvfp4_gemm(self.QX[(M, K)], self.weight(N, K, i), y)
        else:
            nv.nvfp4_quantize(x, self.QXrm[(M, K)], workspace=self.WS[(M, K)])
            nv.nvfp4_gemm(self.QXrm[(M, K)], self.weight(N, K, i, rowmajor=True), y)

    def run_step(self, step, e2e=False):
        for (M, N, K) in self.calls:
            i = step * len(self.Ms) + self.Ms.index(M)   # every call of a step streams its own weight copy
            if e2e:   # pinned host X -> device, quantize + GEMM, Y -> pinned host: one C-ABI call
                self.nv.nvfp4_quantize_gemm_host(self.Xhost[(M, K)], self.X[(M, K)], self.QX[(M, K)],
                                                 self.weight(N, K, i), self.Y[(M, N, K)], self.Yhost[(M, N, K)])
            else:
                self.call(M, N, K, i)

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


class EagerStep:
    """Stands in for a captured step graph: replay() launches the step directly."""

    def __init__(self, wk, phase, e2e=False):
        self.wk, self.phase, self.e2e = wk, phase, e2e

    def replay(self):
        self.wk.run_step(self.phase, self.e2e)


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


def time_back_to_back(fn, n, reps=5):
    """Per-call device time (ms) of fn(0..n-1) captured back to back in one graph:
    median over reps replays of (replay time / n)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(n):
            fn(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b) / n)
    del g
    return statistics.median(times)


def time_decode_calls(wk, mode):
    """Per-call time (ms) of every decode (M, shape) in one mode, back to back
    over all weight copies of the shape (never L2-resident)."""
    out = {}
    for (M, N, K) in wk.calls:
        n = wk.copies[(N, K)]
        out[(M, N, K)] = time_back_to_back(lambda i: wk.call(M, N, K, i, mode), n)
    return out


class ResServeDecode:
    """ResServe decode (M in 1,4,16; (N,K) in (5120,5120),(27648,5120),(5120,27648);
    Student-t(3) x 0.5 activations): fused plain vs fused residue-compensated
    linear, to report the latency overhead of the residue at M <= 16.  M=64
    (quantize, then the tcgen05 GEMV) is reported beside it."""
    L2_SPAN = 260e6

    def __init__(self, dev):
        import nvfp4_block_scaled_18_b200 as nv
        from nvfp4_block_scaled_18_b200 import workloads as wl
        self.nv = nv
        self.Ms = [m for m in wl.RESSERVE_M if m <= 16]
        self.big_Ms = [m for m in wl.RESSERVE_M if m > 16]
        self.shapes = list(wl.RESSERVE_SHAPES)
        self.W, self.buf = {}, {}
        for (N, K) in self.shapes:
            w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
            q0 = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q0, workspace=nv.Workspace(N, K, dev))
            del w
            n = max(2, int(np.ceil(self.L2_SPAN / (N * K * 9 / 16))))
            self.W[(N, K)] = [q0] + [nv.NVFP4Tensor(q0.codes.clone(), q0.scales.clone(), q0.tensor_scale.clone(),
                                                    N, K, nv.SF_TILED) for _ in range(n - 1)]
            for M in self.Ms + self.big_Ms:
                self.buf[(M, N, K)] = dict(
                    x=wl.to_bf16(wl.resserve_x(M, K)).to(dev),
                    q=nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev),
                    r=nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev),
                    y=torch.empty((M, N), dtype=torch.float32, device=dev),
                    ws=nv.Workspace(M, K, dev))
        torch.cuda.synchronize()

    def measure(self):
        out = {}
        for (N, K) in self.shapes:
            ws = self.W[(N, K)]
            for M in self.Ms:
                b = self.buf[(M, N, K)]
                t0 = time_back_to_back(lambda i: self.nv.nvfp4_quantize_gemm(b["x"], b["q"], ws[i % len(ws)], b["y"]),
                                       len(ws))
                t1 = time_back_to_back(lambda i: self.nv.nvfp4_quantize_residue_gemm(b["x"], b["q"], b["r"],
                                                                                     ws[i % len(ws)], b["y"]),
                                       len(ws))
                # the residue's tensor scale given (e.g. calibrated offline): no second maximum
                t2 = time_back_to_back(lambda i: self.nv.nvfp4_quantize_residue_gemm(
                    b["x"], b["q"], b["r"], ws[i % len(ws)], b["y"], rscale_in=b["r"].tensor_scale), len(ws))
                out[f"M{M}_N{N}_K{K}"] = {"plain_us": round(t0 * 1e3, 3), "residue_us": round(t1 * 1e3, 3),
                                          "overhead_pct": round((t1 - t0) / t0 * 100.0, 1),
                                          "residue_given_scale_us": round(t2 * 1e3, 3),
                                          "overhead_given_scale_pct": round((t2 - t0) / t0 * 100.0, 1)}
        worst = max(v["overhead_pct"] for v in out.values())
        mean = float(np.mean([v["overhead_pct"] for v in out.values()]))
        worst_g = max(v["overhead_given_scale_pct"] for v in out.values())
        mean_g = float(np.mean([v["overhead_given_scale_pct"] for v in out.values()]))
        big = {}
        for (N, K) in self.shapes:
            ws = self.W[(N, K)]
            for M in self.big_Ms:
                b = self.buf[(M, N, K)]

                def plain(i):
                    self.nv.nvfp4_quantize(b["x"], b["q"], workspace=b["ws"])
                    self.nv.nvfp4_gemm(b["q"], ws[i % len(ws)], b["y"])

                def residue(i):
                    self.nv.nvfp4_quantize_residue(b["x"], b["q"], b["r"], workspace=b["ws"])
                    self.nv.nvfp4_gemm_residue(b["q"], b["r"], ws[i % len(ws)], b["y"])
                t0 = time_back_to_back(plain, len(ws))
                t1 = time_back_to_back(residue, len(ws))
                big[f"M{M}_N{N}_K{K}"] = {"plain_us": round(t0 * 1e3, 3), "residue_us": round(t1 * 1e3, 3),
                                          "overhead_pct": round((t1 - t0) / t0 * 100.0, 1)}
        return {"per_call": out, "overhead_pct_max": worst, "overhead_pct_mean": round(mean, 1),
                "given_scale": {"overhead_pct_max": worst_g, "overhead_pct_mean": round(mean_g, 1),
                                "note": "residue tensor scale passed in (rscale_in): a separate line, "
                                        "the computed-scale numbers above stand"},
                "target": "<= 10% extra latency at M <= 16",
                "m64_quantize_then_gemm": big}


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
            perm = torch.from_numpy(wl.prefill_perm(K)).to(dev)
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


def measure_arcquant(nv, dev, peaks):
    """ARCQuant prefill: X 2048 x 4096 bf16 (2% channels x30), gamma, a perm from
    512 calibration rows, W 11008 x 4096. For S in {0, 128, 256, 512}: the fused
    RMSNorm + reorder + K->K+S quantizer, rotating over 16 activation copies
    (268 MB, > 2x L2), and the augmented GEMM Y = s_aug s_w [QX|QR][QW|QW_o]^T
    (tensor-bound; one operand copy)."""
    from nvfp4_block_scaled_18_b200 import workloads as wl
    M, K, N = wl.ARC_M, wl.ARC_K, wl.ARC_N
    x, gamma, perm = wl.arc_inputs()
    ncopy = 16
    xs = [wl.to_bf16(x).to(dev) for _ in range(ncopy)]
    g = wl.to_bf16(gamma).to(dev)
    p = torch.from_numpy(np.ascontiguousarray(perm, dtype=np.int32)).to(dev)
    w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
    y = torch.empty((M, N), dtype=torch.float32, device=dev)
    ws = nv.Workspace(M, K, dev)
    out = {"shape": f"M{M}_N{N}_K{K}"}
    for S in (0, 128, 256, 512):
        qs = [nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED, device=dev) for _ in range(ncopy)]
        w_aug = torch.cat([w[:, p.long()], w[:, p[:S].long()]], dim=1).contiguous()
        qw = nv.NVFP4Tensor.empty(N, K + S, nv.SF_TILED, device=dev)
        nv.nvfp4_quantize(w_aug, qw, workspace=nv.Workspace(N, K + S, dev))
        del w_aug
        t_q = time_back_to_back(lambda i: nv.nvfp4_rmsnorm_reorder_quantize(
            xs[i], qs[i], gamma=g, eps=1e-5, perm=p, S=S, workspace=ws), ncopy)
        t_g = time_back_to_back(lambda i: nv.nvfp4_gemm(qs[i % ncopy], qw, y), 4)
        q_bytes = 2 * M * K + M * (K + S) * 9 // 16 + 6 * K
        flops = 2.0 * M * N * (K + S)
        out[f"S{S}"] = {"quant_us": round(t_q * 1e3, 2), "quant_GBps": round(q_bytes / (t_q * 1e-3) / 1e9, 1),
                        "quant_frac_hbm": round(q_bytes / (t_q * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                        "gemm_us": round(t_g * 1e3, 2), "gemm_TFLOPs": round(flops / (t_g * 1e-3) / 1e12, 1),
                        "gemm_frac_fp4_peak": round(flops / (t_g * 1e-3) / 1e12 / fp4_peak_tflops(peaks), 4)}
        del qs, qw
    base = out["S0"]["quant_us"] + out["S0"]["gemm_us"]
    for S in (128, 256, 512):
        o = out[f"S{S}"]
        o["overhead_pct_vs_S0"] = round(100.0 * ((o["quant_us"] + o["gemm_us"]) / base - 1.0), 1)
    return out


def measure_prefill_from(wk, peaks):
    """Per-launch GEMM and quantizer times on the prefill workload."""
    out, flops_total, gemm_ms_total = {}, 0.0, 0.0
    for (name, M, N, Keff, S) in wk.calls:
        K = Keff - S
        wk.quantize(N, K, S)
        g_ms = time_back_to_back(lambda i: wk.gemm(N, K, S), 4)
        q_ms = time_back_to_back(lambda i: wk.quantize(N, K, S), 4)
        flops = 2.0 * M * N * Keff
        q_bytes = 2 * M * K + M * Keff * 9 // 16
        flops_total += flops
        gemm_ms_total += g_ms
        out[f"M{M}_N{N}_K{K}" + (f"+S{S}" if S else "")] = {
            "gemm_us": round(g_ms * 1e3, 2), "gemm_TFLOPs": round(flops / (g_ms * 1e-3) / 1e12, 1),
            "gemm_frac_fp4_peak": round(flops / (g_ms * 1e-3) / 1e12 / fp4_peak_tflops(peaks), 4),
            "quant_us": round(q_ms * 1e3, 2), "quant_GBps": round(q_bytes / (q_ms * 1e-3) / 1e9, 1)}
    # MXFP4 quantizer (a NEXT row: 32-element blocks, E8M0 scales, one pass) on the
    # first shape's activations, plain and with the residue
    (_, M, N, Keff, S) = wk.calls[0]
    x = wk.buf[(N, Keff - S)]["x"]
    K = Keff - S
    mc = torch.empty(M * K // 2, dtype=torch.uint8, device=x.device)
    ms = torch.empty(M * K // 32, dtype=torch.uint8, device=x.device)
    rc, rs = torch.empty_like(mc), torch.empty_like(ms)
    mx_bytes = M * K * (2 + 0.5 + 1 / 32)
    t_mx = time_back_to_back(lambda i: wk.nv.nvfp4_mx_quantize(x, mc, ms), 4)
    t_mxr = time_back_to_back(lambda i: wk.nv.nvfp4_mx_quantize(x, mc, ms, rc, rs), 4)
    out["mxfp4_quantize"] = {"shape": f"{M}x{K} bf16", "us": round(t_mx * 1e3, 2),
                             "GBps": round(mx_bytes / (t_mx * 1e-3) / 1e9, 1),
                             "residue_us": round(t_mxr * 1e3, 2),
                             "residue_GBps": round((mx_bytes + M * K * (0.5 + 1 / 32)) / (t_mxr * 1e-3) / 1e9, 1)}
    nv = wk.nv
    # ResServe residue on the large-M GEMM (two accumulation passes per tile) on the same shape
    q_r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=x.device)
    r_r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=x.device)
    nv.nvfp4_quantize_residue(x, q_r, r_r, workspace=wk.buf[(N, K)]["ws"])
    qw_r, y_r = wk.buf[(N, K)]["qw"], wk.buf[(N, K)]["y"]
    t_p = time_back_to_back(lambda i: nv.nvfp4_gemm(q_r, qw_r, y_r), 4)
    t_r = time_back_to_back(lambda i: nv.nvfp4_gemm_residue(q_r, r_r, qw_r, y_r), 4)
    out["resserve_gemm"] = {"shape": f"M{M}_N{N}_K{K}", "plain_us": round(t_p * 1e3, 2),
                            "residue_us": round(t_r * 1e3, 2),
                            "overhead_pct": round(100.0 * (t_r / t_p - 1.0), 1),
                            "residue_TFLOPs": round(4.0 * M * N * K / (t_r * 1e-3) / 1e12, 1)}
    del q_r, r_r
    # MXFP4 GEMM (kind::mxf4, one E8M0 scale per 32 elements) on the same shape:
    # both operands quantized on the device with TILED scales
    from nvfp4_block_scaled_18_b200 import workloads as wl
    w = torch.from_numpy(wl.weights_normal(N, K)).to(x.device)
    wc = torch.empty((N, K // 2), dtype=torch.uint8, device=x.device)
    wsc = torch.empty(nv.mx_scales_bytes(N, K, nv.SF_TILED), dtype=torch.uint8, device=x.device)
    nv.nvfp4_mx_quantize(w, wc.view(-1), wsc, sf_layout=nv.SF_TILED)
    del w
    xsc = torch.empty(nv.mx_scales_bytes(M, K, nv.SF_TILED), dtype=torch.uint8, device=x.device)
    nv.nvfp4_mx_quantize(x, mc, xsc, sf_layout=nv.SF_TILED)
    y = wk.buf[(N, K)]["y"]
    t_mg = time_back_to_back(lambda i: nv.nvfp4_mx_gemm(mc.view(M, -1), xsc, wc, wsc, y), 4)
    out["mxfp4_gemm"] = {"shape": f"M{M}_N{N}_K{K}", "us": round(t_mg * 1e3, 2),
                         "TFLOPs": round(2.0 * M * N * K / (t_mg * 1e-3) / 1e12, 1),
                         "frac_fp4_peak": round(2.0 * M * N * K / (t_mg * 1e-3) / 1e12 / fp4_peak_tflops(peaks), 4)}
    # the compensated MXFP4 linear: X with its residue, the residue's K-tiles in the same accumulation
    rsc = torch.empty_like(xsc)
    nv.nvfp4_mx_quantize(x, mc, xsc, rc, rsc, sf_layout=nv.SF_TILED)
    t_mgr = time_back_to_back(lambda i: nv.nvfp4_mx_gemm_residue(mc.view(M, -1), xsc, rc.view(M, -1), rsc, wc, wsc,
                                                                 y), 4)
    out["mxfp4_gemm"].update({"residue_us": round(t_mgr * 1e3, 2),
                              "residue_overhead_pct": round(100.0 * (t_mgr / t_mg - 1.0), 1)})
    del wc, wsc, xsc, rsc
    try:
        out["arcquant_prefill"] = measure_arcquant(nv, x.device, peaks)
    except Exception as e:   # a detail leg: record the failure, keep the line
        out["arcquant_prefill"] = {"error": f"{type(e).__name__}: {e}"}
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


def arm_config(workload: str, world: int, calls_per_step: int) -> dict:
    """The `config` of a bench line; both arms report the same one."""
    if workload == "decode":
        return {"workload": "decode GEMV (M in 1,2,4,8,16; (N,K) in (4096,4096),(14336,4096),(4096,14336)); "
                            "online bf16->NVFP4 activation quantization + NVFP4 GEMM in one launch, fp32 out",
                "calls_per_step": calls_per_step,
                "l2": "every call streams its own weight copy; >= 260 MB of copies per shape (> L2)",
                "parallelism": f"replicas x{world}"}
    return {"workload": "large prefill W4A4 GEMM, M=8192, (N,K) in (14336,4096),(4096,14336),(28672,8192), "
                        "each without and with the S=256 outlier-residue K extension; online quantization",
            "calls_per_step": calls_per_step, "l2": "inputs > L2 (X 67-235 MB, Y 134-940 MB per call)",
            "parallelism": f"replicas x{world}"}


def reference_arm(args):
    """--impl reference: the CPU oracle, as it stands, timed as the comparison arm
    on the same workload, metric and unit (rank 0 only). Each step is one call of
    the workload on a bounded sample: a row subset of W (decode), or a row subset
    of X and of W (prefill), sized so that the whole run stays within minutes."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    from nvfp4_block_scaled_18_b200 import workloads as wl
    oracle.build()
    budget = 120.0        # seconds of timed oracle work over warm-up and timed steps
    per_step = max(0.02, min(1.0, budget / max(1, args.steps + args.warmup)))
    cache = {}
    # the W row subset of a step is sized by the oracle's cost per W element
    # (dequantization to fp64 dominates): about 10 ns (decode), 20 ns (32 rows of X)
    if args.workload == "decode":
        shapes, Ms = list(wl.DECODE_SHAPES), list(wl.DECODE_M)
        calls_per_step, unit, scale = len(shapes) * len(Ms), "GB/s", 1e9

        def sample(i):
            M, (N, K) = Ms[i % len(Ms)], shapes[(i // len(Ms)) % len(shapes)]
            rows = max(8, min(N, int(per_step / (1e-8 * K))))
            if (N, K) not in cache:      # the first rows of the workload's W
                cache[(N, K)] = oracle.quantize(wl.weights_normal(rows, K))
            sub = cache[(N, K)]
            x = wl.decode_x(M, K)
            t0 = time.perf_counter()
            oracle.gemm(oracle.quantize(x), sub)
            return time.perf_counter() - t0, decode_bytes(M, rows, K)
        what = "one linear call per step (M 1..16 cycling over the shapes) on a W row subset"
    else:
        calls = [(N, K, S) for (N, K) in wl.PREFILL_SHAPES for S in (0, 256)]
        calls_per_step, unit, scale = len(calls), "TFLOP/s", 1e12
        x_rows = 32

        def sample(i):
            N, K, S = calls[i % len(calls)]
            w_rows = max(16, min(N, int(per_step / (2e-8 * (K + S)))))
            if (N, K, S) not in cache:   # the first rows of the workload's W
                w = wl.weights_normal(w_rows, K)
                if S:
                    perm = wl.calibrated_perm(wl.prefill_x(64, K))
                    cache[(N, K, S)] = (oracle.quantize(oracle.augment_weight(w, perm, S)), perm)
                else:
                    cache[(N, K, S)] = (oracle.quantize(w), None)
            qw, perm = cache[(N, K, S)]
            x = wl.prefill_x(x_rows, K)
            t0 = time.perf_counter()
            qx = oracle.rmsnorm_reorder_quantize(x, None, 1e-5, perm, S) if S else oracle.quantize(x)
            oracle.gemm(qx, qw)
            return time.perf_counter() - t0, 2.0 * x_rows * qw.codes.shape[0] * (K + S)
        what = (f"one of the 6 prefill calls per step: {x_rows} rows of X (quantized, reordered for K+S) "
                "against a W row subset")

    for i in range(args.warmup):
        sample(i)
    t, work = 0.0, 0.0
    for i in range(args.steps):
        dt, dw = sample(i)
        t += dt
        work += dw
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    value = work / t / scale
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(args.workload, world, calls_per_step),
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps, {what}; oracle quantize + fp64 dequantized GEMM"},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ profiling cases

def profile_case(case: str) -> int:
    """A handful of launches of one kernel, inputs just above L2, for ncu:
    decode   -- nvfp4_quantize_gemm, M=1, (N,K)=(4096,14336), 5 weight copies (147 MB)
    decode_res -- nvfp4_quantize_residue_gemm (computed residue scale), M=4, (N,K)=(5120,5120)
                (ResServe decode), Student-t activations, 12 weight copies (177 MB)
    prefill  -- nvfp4_gemm, M=8192, (N,K)=(14336,4096) (A 19 MB, W 33 MB, Y 470 MB)
    quantize -- nvfp4_quantize of the 8192x4096 bf16 prefill activations (67 MB)
    reorder  -- nvfp4_rmsnorm_reorder_quantize of the same activations, S=256
    mxgemm   -- nvfp4_mx_gemm, M=8192, (N,K)=(14336,4096), MXFP4 operands with TILED scales
    arcquant -- nvfp4_rmsnorm_reorder_quantize on the ARCQuant prefill activations
                (2048x4096 bf16, gamma, calibrated perm, S=256)
    gemv     -- nvfp4_gemm on ROWMAJOR operands (CUDA-core GEMV), M=1, (N,K)=(4096,14336),
                5 weight copies (165 MB)
    gemv_tc  -- nvfp4_gemm_residue, M=64, (N,K)=(5120,27648) (ResServe decode), TILED
                operands, 3 weight copies (239 MB)
    mxquant  -- nvfp4_mx_quantize of the 8192x4096 bf16 prefill activations (67 MB), TILED."""
    import nvfp4_block_scaled_18_b200 as nv
    from nvfp4_block_scaled_18_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    nv.load_library()
    if case == "decode":
        M, N, K = 1, 4096, 14336
        w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
        ws = []
        for _ in range(5):
            q = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q, workspace=nv.Workspace(N, K, dev))
            ws.append(q)
        x = wl.to_bf16(wl.decode_x(M, K)).to(dev)
        qx = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        y = torch.empty((M, N), device=dev)
        for i in range(10):
            nv.nvfp4_quantize_gemm(x, qx, ws[i % 5], y)
    elif case == "decode_res":
        M, N, K = 4, 5120, 5120
        w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
        ws = []
        for _ in range(12):
            q = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q, workspace=nv.Workspace(N, K, dev))
            ws.append(q)
        x = wl.to_bf16(wl.resserve_x(M, K)).to(dev)
        qx = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        rx = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        y = torch.empty((M, N), device=dev)
        for i in range(12):
            nv.nvfp4_quantize_residue_gemm(x, qx, rx, ws[i], y)
    elif case == "prefill":
        M, N, K = 8192, 14336, 4096
        qa = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        qw = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
        nv.nvfp4_quantize(wl.to_bf16(wl.prefill_x(M, K)).to(dev), qa, workspace=nv.Workspace(M, K, dev))
        nv.nvfp4_quantize(torch.from_numpy(wl.weights_normal(N, K)).to(dev), qw, workspace=nv.Workspace(N, K, dev))
        y = torch.empty((M, N), device=dev)
        for _ in range(3):
            nv.nvfp4_gemm(qa, qw, y)
    elif case == "mxgemm":
        M, N, K = 8192, 14336, 4096
        ops = []
        for v in (wl.to_bf16(wl.prefill_x(M, K)).to(dev), torch.from_numpy(wl.weights_normal(N, K)).to(dev)):
            rows = v.shape[0]
            c = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev)
            sc = torch.empty(nv.mx_scales_bytes(rows, K, nv.SF_TILED), dtype=torch.uint8, device=dev)
            nv.nvfp4_mx_quantize(v, c.view(-1), sc, sf_layout=nv.SF_TILED)
            ops.append((c, sc))
            del v
        y = torch.empty((M, N), device=dev)
        for _ in range(3):
            nv.nvfp4_mx_gemm(ops[0][0], ops[0][1], ops[1][0], ops[1][1], y)
    elif case == "arcquant":
        x, gamma, perm = wl.arc_inputs()
        M, K, S = wl.ARC_M, wl.ARC_K, 256
        xs = [wl.to_bf16(x).to(dev) for _ in range(8)]   # 134 MB of activation copies (> L2)
        g = wl.to_bf16(gamma).to(dev)
        p = torch.from_numpy(np.ascontiguousarray(perm, dtype=np.int32)).to(dev)
        q = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED, device=dev)
        ws = nv.Workspace(M, K, dev)
        for i in range(3):
            nv.nvfp4_rmsnorm_reorder_quantize(xs[i], q, gamma=g, eps=1e-5, perm=p, S=S, workspace=ws)
    elif case == "gemv":
        M, N, K = 1, 4096, 14336
        w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
        ws = []
        for _ in range(5):
            q = nv.NVFP4Tensor.empty(N, K, nv.SF_ROWMAJOR, device=dev)
            nv.nvfp4_quantize(w, q, workspace=nv.Workspace(N, K, dev))
            ws.append(q)
        qx = nv.NVFP4Tensor.empty(M, K, nv.SF_ROWMAJOR, device=dev)
        nv.nvfp4_quantize(wl.to_bf16(wl.decode_x(M, K)).to(dev), qx, workspace=nv.Workspace(M, K, dev))
        y = torch.empty((M, N), device=dev)
        for i in range(10):
            nv.nvfp4_gemm(qx, ws[i % 5], y)
    elif case == "gemv_tc":
        M, N, K = 64, 5120, 27648
        w = torch.from_numpy(wl.weights_normal(N, K)).to(dev)
        ws = []
        for _ in range(3):
            q = nv.NVFP4Tensor.empty(N, K, nv.SF_TILED, device=dev)
            nv.nvfp4_quantize(w, q, workspace=nv.Workspace(N, K, dev))
            ws.append(q)
        q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        r = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        nv.nvfp4_quantize_residue(wl.to_bf16(wl.resserve_x(M, K)).to(dev), q, r, workspace=nv.Workspace(M, K, dev))
        y = torch.empty((M, N), device=dev)
        for i in range(6):
            nv.nvfp4_gemm_residue(q, r, ws[i % 3], y)
    elif case == "mxquant":
        M, K = 8192, 4096
        x = wl.to_bf16(wl.prefill_x(M, K)).to(dev)
        c = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty(nv.mx_scales_bytes(M, K, nv.SF_TILED), dtype=torch.uint8, device=dev)
        for _ in range(3):
            nv.nvfp4_mx_quantize(x, c.view(-1), sc, sf_layout=nv.SF_TILED)
    elif case == "reorder":
        M, K, S = 8192, 4096, 256
        x = wl.to_bf16(wl.prefill_x(M, K)).to(dev)
        perm = torch.from_numpy(wl.prefill_perm(K)).to(dev)
        q = nv.NVFP4Tensor.empty(M, K + S, nv.SF_TILED, device=dev)
        ws = nv.Workspace(M, K, dev)
        for _ in range(3):
            nv.nvfp4_rmsnorm_reorder_quantize(x, q, perm=perm, S=S, workspace=ws)
    else:
        M, K = 8192, 4096
        x = wl.to_bf16(wl.prefill_x(M, K)).to(dev)
        q = nv.NVFP4Tensor.empty(M, K, nv.SF_TILED, device=dev)
        ws = nv.Workspace(M, K, dev)
        for _ in range(3):
            nv.nvfp4_quantize(x, q, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "ok": True}), flush=True)
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
    ap.add_argument("--eager", action="store_true",
                    help="decode: launch every step directly on the stream (no CUDA graphs) and skip the "
                         "per-call detail; for profilers that cannot follow graph replays")
    ap.add_argument("--profile-case", choices=["decode", "decode_res", "prefill", "quantize", "reorder", "mxgemm", "arcquant",
                                               "gemv", "gemv_tc", "mxquant"],
                    help="run a few launches of one kernel on a small case (for ncu captures) and exit")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile_case:
        return profile_case(args.profile_case)

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    import nvfp4_block_scaled_18_b200 as nv
    nv.load_library()
    peaks = load_peaks()

    if args.workload == "decode":
        wk = DecodeWorkload(dev)
        phases = wk.phases
        unit, work_per_step = "GB/s", float(wk.step_bytes)
        scale = 1e9
        steps = args.steps
    else:
        wk = PrefillWorkload(dev)
        phases = 1
        unit, work_per_step = "TFLOP/s", float(sum(2.0 * M * N * Keff for (_, M, N, Keff, _) in wk.calls))
        scale = 1e12
        steps = max(1, min(args.steps, 40))
    eager = args.eager and args.workload == "decode"
    graphs = [EagerStep(wk, p) for p in range(phases)] if eager else capture_graphs(wk, phases)
    sampler = ClockSampler(torch.cuda.current_device())
    ms = time_graphs(graphs, steps, args.warmup, world, sampler)
    clocks = sampler.stop()
    value, ms_max = replica_throughput(work_per_step * steps, ms, world, scale)
    ms_per_step = ms_max / steps

    # end to end: pinned host X -> device, quantize + GEMM, Y -> pinned host, every step
    e2e_steps = max(4 * phases, min(steps, 400)) if args.workload == "decode" else max(2, min(steps, 5))
    if args.workload == "decode":
        e2e_graphs = [EagerStep(wk, p, True) for p in range(phases)] if eager else capture_graphs(wk, phases, e2e=True)
        ms_e2e = time_graphs(e2e_graphs, e2e_steps, args.warmup, world)
        h2d, d2h = wk.h2d_bytes(), wk.d2h_bytes()
    else:
        ms_e2e, h2d, d2h = prefill_e2e(wk, e2e_steps), wk.h2d_bytes(), wk.d2h_bytes()
        e2e_graphs = []
    e2e_value, _ = replica_throughput(work_per_step * e2e_steps, ms_e2e, world, scale)

    line = {"metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5)}
    if eager:
        detail = {"mode": "eager launches, no per-call detail"}
        roofline = {"bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": None,
                    "traffic": None, "kernel": "k_decode_tc", "peak_source": peaks["source"]}
        config = {"workload": "decode GEMV (eager launches)", "calls_per_step": len(wk.calls),
                  "parallelism": f"replicas x{world}"}
        launches = wk.launches_per_step * steps
    elif args.workload == "decode":
        per = time_decode_calls(wk, "fused")
        per_sep = time_decode_calls(wk, "separate")
        per_cc = time_decode_calls(wk, "cuda_core")
        tot = lambda d: sum(d.values())
        achieved = wk.step_bytes / (tot(per) * 1e-3) / 1e9
        line["us_per_call"] = round(ms_per_step * 1e3 / len(wk.calls), 3)
        gbps = lambda c, t: round(decode_bytes(*c) / (t * 1e-3) / 1e9, 1)
        detail = {f"M{M}_N{N}_K{K}": {
            "fused_us": round(per[(M, N, K)] * 1e3, 3), "fused_GBps": gbps((M, N, K), per[(M, N, K)]),
            "separate_us": round(per_sep[(M, N, K)] * 1e3, 3),
            "cuda_core_us": round(per_cc[(M, N, K)] * 1e3, 3), "cuda_core_GBps": gbps((M, N, K), per_cc[(M, N, K)])}
            for (M, N, K) in wk.calls}
        for name, d in (("fused", per), ("separate", per_sep), ("cuda_core", per_cc)):
            a = wk.step_bytes / (tot(d) * 1e-3) / 1e9
            detail[f"{name}_aggregate"] = {"us_per_call": round(tot(d) * 1e3 / len(wk.calls), 3),
                                           "GBps": round(a, 1), "frac_hbm": round(a / peaks["hbm_gbs"], 4)}
        detail["per_call_timing"] = "graphs of back-to-back calls of one shape over all its weight copies"
        del graphs
        rs = ResServeDecode(dev)
        detail["resserve_residue_overhead"] = rs.measure()
        del rs
        # DRAM bytes per launch from the ncu capture of k_decode_tc (M=1, (4096,14336)):
        # 33.094 MB measured against 33.083 MB algorithmic; scaled to the average call of a step
        traffic = wk.step_bytes / len(wk.calls) * DECODE_TRAFFIC_RATIO if DECODE_TRAFFIC_RATIO else None
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": None if traffic is None else round(traffic),
                    "traffic_basis": "bytes per average call of a step: algorithmic x (measured/algorithmic) "
                                     "of the profiled launch (profiles/k_decode_tc_m1_4096x14336.md)",
                    "kernel": "k_decode_tc (fused quantize + GEMM; plain GEMM after the quantizer on the calls "
                              "where that is estimated faster), all 15 decode calls back to back",
                    "launches_per_step": wk.launches_per_step,
                    "peak_source": peaks["source"]}
        config = arm_config("decode", world, len(wk.calls))
        launches = wk.launches_per_step * steps
    else:
        detail, roofline = measure_prefill_from(wk, peaks)
        config = arm_config("prefill", world, len(wk.calls))
        launches = 3 * len(wk.calls) * steps
    line.update({"higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1",
                 "data": "synthetic", "config": config, "roofline": roofline,
                 "e2e": {"value": round(e2e_value, 2), "unit": unit, "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h,
                         "call": ("nvfp4_quantize_gemm_host (C ABI, pinned host buffers)"
                                  if args.workload == "decode" else "torch host copies around the C-ABI calls")},
                 "gpu_launches": launches, "clocks": clocks, "detail": detail})
    if args.workload == "decode" and not args.no_prefill and not eager:
        del e2e_graphs
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
