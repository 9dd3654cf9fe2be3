#!/usr/bin/env python
"""Benchmark of the int8 quantized linears on B200.

Headline workload: the W8A16 decode sweep -- bf16 activations (M in {1, 4, 16}) times int8
per-channel weights of shapes (K, N) in {(960, 2560), (2048, 8192), (4096, 11008),
(4096, 32000)}, bf16 output.  One step runs every (shape, M) case once, as one CUDA graph
of 12 GEMV launches; the metric is algorithmic bytes moved (int8 weights + fp32 scales +
bf16 activations + bf16 outputs) per second.  Two copies of every weight rotate between
steps (390 MB, over 3x the 126 MB L2), and within a step cases run M-major, so a weight
is never re-read from L2.

Extra sub-benchmarks (same JSON line, key "paths"): the sweep with a bias, the NVFP4
weight-only twin on the sweep's shapes, W8A8 static int8 linear (K = 960) and prefill
(M = 4096, also with a bias), 8da4w, the quantizers (both weight grids), a Llama-shaped
stack and the offline GPTQ path (calibration Hessian + GPTQ of one 11008 x 4096 layer).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched under torch.distributed.run) every rank runs an independent replica
(the path has no exchange step); time is the max over ranks and the value counts all ranks.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import q8_workloads as wl  # noqa: E402

METRIC = "W8A16 decode GB/s (% of HBM peak); W8A8/8da4w prefill TOPS (% int8 peak)"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-paths", action="store_true", help="skip the sub-benchmarks")
    p.add_argument("--eager", action="store_true",
                   help="launch the timed steps one by one instead of replaying CUDA graphs "
                        "(for profilers that cannot replay graph-captured launches)")
    p.add_argument("--profile", choices=["w8a16", "w8a8", "q4", "w4a16", "quant"], default=None,
                   help="run only one kernel case --reps times (for ncu captures), then exit")
    p.add_argument("--pM", type=int, default=16)
    p.add_argument("--pN", type=int, default=32000)
    p.add_argument("--pK", type=int, default=4096)
    p.add_argument("--pG", type=int, default=32, help="8da4w group size (--profile q4)")
    p.add_argument("--reps", type=int, default=3)
    p.add_argument("--ptwo", type=int, default=1, help="W8A8 two-pass (1) or one pass (0)")
    return p.parse_args()


# ----------------------------------------------------------------------------- distributed


class Dist:
    """One process per GPU (replicas: the path has no exchange step).  The process group
    only carries the barriers around the timed region and the max-over-ranks time; it is
    NCCL on GPUs and gloo on the host (the multi-rank tests run it on CPU)."""

    def __init__(self, gpus: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.dev = torch.device("cuda", self.local) if backend == "nccl" else torch.device("cpu")
        if self.world > 1:
            import torch.distributed as dist

            if backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                        device_id=self.dev)
            else:
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
            self.pg = dist
        elif backend == "nccl":
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def job_throughput(world: int, steps: int, units_per_step: float, max_ms: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return world * steps * units_per_step / (max_ms * 1e-3)


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampled every 20 ms on this rank's GPU while the timed region runs."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="q8clk_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = list(csv.reader(io.StringIO(open(self.path).read())))
        os.unlink(self.path)
        return rows

    @staticmethod
    def summarize(rows, t0: float, t1: float) -> dict:
        def ts(r):
            try:
                return datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                return None

        good = [r for r in rows if len(r) >= 10]
        inside = [r for r in good if ts(r) is not None and t0 <= ts(r) <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside, window = good, "warm-up + timed region (timed region shorter than 3 samples)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in inside]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            for name, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(inside[0][3]),
                "reasons": sorted(reasons), "samples": len(inside), "window": window,
                "power_w_max": max(float(r[4]) for r in inside)}


def sweep_traffic():
    """Per-launch DRAM traffic of the headline kernel from the committed ncu capture
    (profiles/w8a16_sweep_traffic.txt), or None if the kernel source changed since."""
    import hashlib

    prof = os.path.join(ROOT, "profiles", "w8a16_sweep_traffic.txt")
    src = os.path.join(ROOT, "int8_quantized_linear_q8_b200", "csrc", "k_gemv_tma.cu")
    if not (os.path.exists(prof) and os.path.exists(src)):
        return None
    kv = dict(line.strip().split("=", 1) for line in open(prof)
              if "=" in line and not line.startswith("#"))
    cur = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if kv.get("kernel_source_sha256_16") != cur:
        return None
    return int(kv["traffic_bytes_per_launch_avg"])


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- workloads


def w8a16_bytes(M, N, K):
    return N * K + 4 * N + 2 * M * K + 2 * M * N


class W8A16Sweep:
    """Device-resident W8A16 decode sweep: 2 rotating copies of every weight."""

    COPIES = 2

    def __init__(self, dev):
        import int8_quantized_linear_q8_b200 as q8

        self.q8 = q8
        g = torch.Generator(device=dev)
        self.shapes = []
        for i, sh in enumerate(wl.W8A16_SWEEP_SHAPES):
            g.manual_seed(wl.W8A16_SWEEP_SEED_W * 1000 + i)
            W = torch.randn(sh.N, sh.K, generator=g, device=dev) * 0.02
            q, s, _ = q8.q8_quantize_weight(W, want_wsum=False)
            del W
            copies = [q] + [q.clone() for _ in range(self.COPIES - 1)]
            self.shapes.append((sh, copies, s))
        self.xs, self.ys = {}, {}
        for M in wl.W8A16_SWEEP_M:
            for i, (sh, _, _) in enumerate(self.shapes):
                g.manual_seed(wl.W8A16_SWEEP_SEED_X * 1000 + 10 * i + M)
                self.xs[(i, M)] = torch.randn(M, sh.K, generator=g, device=dev).to(torch.bfloat16)
                self.ys[(i, M)] = torch.empty(M, sh.N, dtype=torch.bfloat16, device=dev)
        self.cases = [(i, M) for M in wl.W8A16_SWEEP_M for i in range(len(self.shapes))]
        self.step_bytes = sum(w8a16_bytes(M, self.shapes[i][0].N, self.shapes[i][0].K)
                              for i, M in self.cases)
        self.weight_bytes = sum(sh.N * sh.K * self.COPIES for sh, _, _ in self.shapes)
        torch.cuda.synchronize()

    def launch(self, i, M, copy):
        sh, copies, s = self.shapes[i]
        self.q8.q8_linear_w8a16(self.xs[(i, M)], copies[copy], s, y=self.ys[(i, M)])

    def step(self, copy):
        for i, M in self.cases:
            self.launch(i, M, copy)

    def graphs(self):
        """One CUDA graph per weight copy, each one full step."""
        out = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for c in range(self.COPIES):
                self.step(c)   # warm the launch path outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for c in range(self.COPIES):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                self.step(c)
            out.append(gr)
        torch.cuda.synchronize()
        return out


class _EagerStep:
    """Stands in for a captured step graph: replay() launches the step's kernels directly."""

    def __init__(self, sweep, copy):
        self.sweep, self.copy = sweep, copy

    def replay(self):
        self.sweep.step(self.copy)


def time_graphs(graphs, steps: int, warmup: int, dist: Dist):
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(st)
    for i in range(steps):
        graphs[i % len(graphs)].replay()
    e1.record(st)
    torch.cuda.synchronize()
    t1 = time.time()
    dist.barrier()
    ms = e0.elapsed_time(e1)
    return dist.max(ms), t0, t1


def per_case_times(sweep: W8A16Sweep, reps: int = 20, launch=None):
    """Average device time of each case's kernel, alone, from a graph of `reps` launches
    alternating weight copies (events on the launching stream).  `launch(i, M, copy)`
    defaults to the sweep's own q8_linear_w8a16 launch."""
    launch = launch or sweep.launch
    out = []
    for i, M in sweep.cases:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            launch(i, M, 0)
        torch.cuda.current_stream().wait_stream(s)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for r in range(reps):
                launch(i, M, r % sweep.COPIES)
        gr.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(2):
            gr.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (2 * reps)
        sh = sweep.shapes[i][0]
        b = w8a16_bytes(M, sh.N, sh.K)
        out.append({"K": sh.K, "N": sh.N, "M": M, "us": round(us, 3),
                    "GBps": round(b / us / 1e3, 1)})
        del gr
    return out


def e2e_w8a16(sweep: W8A16Sweep, steps: int, warmup: int, dist: Dist):
    """Same metric through the public API with host buffers: every step copies all the
    cases' activations host->device (one pinned buffer), runs the 12 calls on views of it,
    and reads all the outputs back device->host (one pinned buffer).  The two copies run on
    their own streams with double-buffered device and host buffers, so a step's output read
    and the next step's input copy overlap the kernels, as in a serving loop; the timed
    region ends when the last step's outputs are in host memory."""
    q8 = sweep.q8
    dev = next(iter(sweep.xs.values())).device
    keys = list(sweep.cases)
    nx = [sweep.xs[k].numel() for k in keys]
    ny = [sweep.ys[k].numel() for k in keys]
    hx0 = torch.cat([sweep.xs[k].reshape(-1).cpu() for k in keys])
    hx = [hx0.clone().pin_memory() for _ in range(2)]
    hy = [torch.empty(sum(ny), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    dxa = [torch.empty(sum(nx), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dya = [torch.empty(sum(ny), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dx, dy = [{}, {}], [{}, {}]
    for b in range(2):
        ox = oy = 0
        for k, a, c in zip(keys, nx, ny):
            dx[b][k] = dxa[b][ox:ox + a].view(sweep.xs[k].shape)
            dy[b][k] = dya[b][oy:oy + c].view(sweep.ys[k].shape)
            ox, oy = ox + a, oy + c
    h2d = hx[0].numel() * hx[0].element_size()
    d2h = hy[0].numel() * hy[0].element_size()
    comp = torch.cuda.current_stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, used, ran, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for b in range(2):                  # every event recorded once before its first wait
        for e in (used[b], out_done[b]):
            e.record(comp)

    def step(c, b):
        cin.wait_event(used[b])         # the kernels that read dxa[b] two steps ago are done
        with torch.cuda.stream(cin):
            dxa[b].copy_(hx[b], non_blocking=True)
        in_done[b].record(cin)
        comp.wait_event(in_done[b])
        comp.wait_event(out_done[b])    # dya[b]'s previous contents have been read back
        for i, M in keys:
            sh, copies, s = sweep.shapes[i]
            q8.q8_linear_w8a16(dx[b][(i, M)], copies[c], s, y=dy[b][(i, M)])
        used[b].record(comp)
        cout.wait_event(used[b])
        with torch.cuda.stream(cout):
            hy[b].copy_(dya[b], non_blocking=True)
        out_done[b].record(cout)

    for i in range(warmup):
        step(i % sweep.COPIES, i % 2)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    cin.wait_event(e0)
    for i in range(steps):
        step(i % sweep.COPIES, i % 2)
    comp.wait_event(out_done[(steps - 1) % 2])
    e1.record(comp)
    torch.cuda.synchronize()
    ms = dist.max(e0.elapsed_time(e1))
    value = dist.world * steps * sweep.step_bytes / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / steps, 4),
            "copies": "one pinned H2D and one D2H per step, on copy streams overlapping the "
                      "kernels (double-buffered)"}


def cpu_baseline_w8a16(sweep: W8A16Sweep, budget_s: float = 12.0):
    """The oracle, as it stands, on the host cores: the M = 1 case of each sweep shape
    (full weights), repeated until about `budget_s` seconds have passed."""
    import oracle

    hq = [(sh, copies[0].cpu().numpy(), s.cpu().numpy()) for sh, copies, s in sweep.shapes]
    hx = {i: sweep.xs[(i, 1)].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
          for i in range(len(hq))}
    done_bytes, t0, reps = 0, time.perf_counter(), 0
    while True:
        for i, (sh, q, s) in enumerate(hq):
            oracle.linear_w8a16(hx[i], q, s)
            done_bytes += w8a16_bytes(1, sh.N, sh.K)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": round(done_bytes / el / 1e9, 3), "unit": UNIT,
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"M=1 case of each of the 4 sweep shapes (full weights), {reps} passes, "
                      f"{el:.1f} s"}


# ----------------------------------------------------------------------------- sub-benchmarks


def bench_w8a8_paths(dev, reps=30):
    """W8A8 static (K = 960, N in {960, 2560}, M in {1, 256, 2048}; one and two passes):
    achieved int8 TOPS (2 M N K per pass) and GB/s (fp32 x in, fp32 y out, int8 W)."""
    import int8_quantized_linear_q8_b200 as q8

    out = []
    K = wl.W8A8_K
    x_all, calib = wl.w8a8_inputs(max(wl.W8A8_M), K=K)
    mm = torch.empty(2, device=dev)
    q8.q8_observe_minmax(calib.to(dev), mm, reset=True)
    first = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
    second = (float(np.float32(first[0]) / np.float32(255.0)), 0)
    for N in wl.W8A8_N:
        W = wl.weight(N, K, seed=wl.W8A8_SEED_W).to(dev)
        q, s, ws = q8.q8_quantize_weight(W)
        for M in wl.W8A8_M:
            x = x_all[:M].contiguous().to(dev)
            y = torch.empty(M, N, device=dev)
            for two in (False, True):
                sec = second if two else None
                wsb = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, M, N, K, int(two))
                work = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
                fn = lambda: q8.q8_linear_w8a8(x, first, q, ws, s, second=sec, y=y, workspace=work)
                us = _graph_time(fn, reps)
                ops = 2.0 * M * N * K * (2 if two else 1)
                byts = 4 * M * K + N * K + 8 * N + 4 * M * N
                out.append({"K": K, "N": N, "M": M, "two_pass": two, "us": round(us, 2),
                            "TOPS": round(ops / us / 1e6, 2), "GBps": round(byts / us / 1e3, 1)})
    return out


def int8_peak_tops(peaks) -> float:
    """Dense int8 tensor peak: the measured bf16 peak times NVIDIA's nominal int8:bf16
    dense ratio (2:1, the fp8 = int8 rate)."""
    return 2.0 * peaks["bf16_tflops"]


def bench_w8a8_prefill(dev, peaks, reps=5):
    """W8A8 (static per-tensor activations) at M = 4096 on the Llama-shaped linears
    (tcgen05 int8 GEMM incl. its activation-code pre-kernel), one and two passes, and the
    4096 x 11008 case once more with a bias."""
    import int8_quantized_linear_q8_b200 as q8

    out = []
    M = wl.LLAMA_PREFILL_M
    g = torch.Generator(device=dev)
    for (K, N) in [(4096, 4096), (4096, 11008), (11008, 4096)]:
        g.manual_seed(31 * K + N)
        x = torch.randn(M, K, generator=g, device=dev)
        W = torch.randn(N, K, generator=g, device=dev) * 0.02
        q, s, ws = q8.q8_quantize_weight(W)
        del W
        mm = torch.empty(2, device=dev)
        q8.q8_observe_minmax(x, mm, reset=True)
        first = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
        second = (float(np.float32(first[0]) / np.float32(255.0)), 0)
        y = torch.empty(M, N, device=dev)
        for two in (False, True):
            sec = second if two else None
            nb = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, M, N, K, int(two))
            work = torch.empty(nb, dtype=torch.uint8, device=dev)
            fn = lambda: q8.q8_linear_w8a8(x, first, q, ws, s, second=sec, y=y, workspace=work)
            us = _graph_time(fn, reps)
            ops = 2.0 * M * N * K * (2 if two else 1)
            tops = ops / us / 1e6
            out.append({"M": M, "K": K, "N": N, "two_pass": two, "us": round(us, 1),
                        "TOPS": round(tops, 1),
                        "frac_int8_peak": round(tops / int8_peak_tops(peaks), 4)})
            if N == 11008:
                b = torch.randn(N, generator=g, device=dev)
                fn = lambda: q8.q8_linear_w8a8(x, first, q, ws, s, second=sec, y=y,
                                               workspace=work, bias=b)
                us = _graph_time(fn, reps)
                tops = ops / us / 1e6
                out.append({"M": M, "K": K, "N": N, "two_pass": two, "bias": True,
                            "us": round(us, 1), "TOPS": round(tops, 1),
                            "frac_int8_peak": round(tops / int8_peak_tops(peaks), 4)})
        del x, q, s, ws, y, work
    return out


def bias_case_times(sweep: W8A16Sweep):
    """The sweep's cases through q8_linear_w8a16 with an fp32 bias [N] (4 N more bytes),
    timed like the headline's per-case times."""
    q8 = sweep.q8
    g = torch.Generator(device=sweep.shapes[0][1][0].device)
    g.manual_seed(91)
    bias = [torch.randn(sh.N, generator=g, device=g.device) for sh, _, _ in sweep.shapes]

    def launch(i, M, copy):
        sh, copies, s = sweep.shapes[i]
        q8.q8_linear_w8a16(sweep.xs[(i, M)], copies[copy], s, y=sweep.ys[(i, M)], bias=bias[i])

    out = per_case_times(sweep, launch=launch)
    for c in out:
        c["GBps"] = round((w8a16_bytes(c["M"], c["N"], c["K"]) + 4 * c["N"]) / c["us"] / 1e3, 1)
    total_b = sum(w8a16_bytes(c["M"], c["N"], c["K"]) + 4 * c["N"] for c in out)
    total_us = sum(c["us"] for c in out)
    return {"cases": out, "GBps_sum_of_cases": round(total_b / total_us / 1e3, 1)}


def bench_q4(dev, peaks, reps=5):
    """8da4w: x bf16 [M, 4096] (M in 1, 64, 512, 4096), int4 weights [11008, 4096] with
    fp32 group scales (G in 32, 128; and G = 256 at M = 512, 4096, where the int8 GEMM runs
    at every M); incl. the per-row qparams pre-kernel."""
    import int8_quantized_linear_q8_b200 as q8

    out = []
    K, N = wl.Q4_K, wl.Q4_N
    g = torch.Generator(device=dev)
    g.manual_seed(wl.Q4_SEED_W)
    W = torch.randn(N, K, generator=g, device=dev) * 0.02
    cases = [(G, wl.Q4_M) for G in wl.Q4_G] + [(256, (512, 4096))]
    for G, Ms in cases:
        q4, gs = q8.q8_quantize_weight_q4gs(W, G)
        for M in Ms:
            g.manual_seed(wl.Q4_SEED_X + M)
            x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
            y = torch.empty(M, N, device=dev)
            nb = q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_DQ8CA_Q4GSW, M, N, K, G)
            work = torch.empty(nb, dtype=torch.uint8, device=dev)
            fn = lambda: q8.q8_linear_dq8ca_q4gsw(x, q4, gs, G, y=y, workspace=work)
            us = _graph_time(fn, reps if M >= 512 else 4 * reps)
            ops = 2.0 * M * N * K
            byts = N * K // 2 + 4 * N * (K // G) + 2 * M * K + 4 * M * N
            out.append({"M": M, "G": G, "us": round(us, 2), "TOPS": round(ops / us / 1e6, 2),
                        "GBps": round(byts / us / 1e3, 1),
                        "frac_int8_peak": round(ops / us / 1e6 / int8_peak_tops(peaks), 4),
                        "frac_hbm": round(byts / us / 1e3 / peaks["hbm_gbs"], 4)})
    return out


def bench_w4a16(dev, peaks, reps=20):
    """The NVFP4 weight-only twin on the W8A16 sweep's shapes and rows (same seeded weights,
    quantized to E2M1 codes with E4M3 block scales): per-case device time from a graph of
    `reps` launches alternating two weight copies; bytes = N*K/2 codes + N*K/16 scale bytes +
    2MK + 2MN."""
    import int8_quantized_linear_q8_b200 as q8

    out = []
    g = torch.Generator(device=dev)
    for i, sh in enumerate(wl.W8A16_SWEEP_SHAPES):
        g.manual_seed(wl.W8A16_SWEEP_SEED_W * 1000 + i)
        W = torch.randn(sh.N, sh.K, generator=g, device=dev) * 0.02
        copies = [q8.q8_quantize_weight_nvfp4(W), q8.q8_quantize_weight_nvfp4(W.clone())]
        del W
        for M in wl.W8A16_SWEEP_M:
            g.manual_seed(wl.W8A16_SWEEP_SEED_X * 1000 + 10 * i + M)
            x = torch.randn(M, sh.K, generator=g, device=dev).to(torch.bfloat16)
            y = torch.empty(M, sh.N, dtype=torch.bfloat16, device=dev)
            state = {"c": 0}

            def fn():
                q4, sf, gsc = copies[state["c"] % 2]
                state["c"] += 1
                q8.q8_linear_w4a16_nvfp4(x, q4, sf, gsc, y=y)

            us = _graph_time(fn, reps)
            b = sh.N * sh.K // 2 + sh.N * sh.K // 16 + 2 * M * sh.K + 2 * M * sh.N
            out.append({"K": sh.K, "N": sh.N, "M": M, "us": round(us, 3),
                        "GBps": round(b / us / 1e3, 1),
                        "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
        del copies
    return out


def bench_quantizers(dev, peaks, reps=5):
    """The quantizers as HBM streams: weight codes on both grids (fp32 32000x4096 in),
    per-row activation qparams + codes (bf16 4096x4096), static activation codes with the
    residual pass, and the residual calibration observer (fp32 4096x4096)."""
    import int8_quantized_linear_q8_b200 as q8

    g = torch.Generator(device=dev)
    g.manual_seed(77)
    out = []
    W = torch.randn(32000, 4096, generator=g, device=dev) * 0.02
    q = torch.empty(32000, 4096, dtype=torch.int8, device=dev)
    sw = torch.empty(32000, device=dev)
    ws = torch.empty(32000, dtype=torch.int32, device=dev)
    us = _graph_time(lambda: q8.q8_quantize_weight(W, q=q, s_w=sw, wsum=ws), reps)
    b = 32000 * 4096 * 5 + 32000 * 8
    out.append({"op": "quantize_weight", "shape": [32000, 4096], "us": round(us, 1),
                "GBps": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
    us = _graph_time(lambda: q8.q8_quantize_weight(W, q=q, s_w=sw, wsum=ws, grid="full128"),
                     reps)
    out.append({"op": "quantize_weight_full128", "shape": [32000, 4096], "us": round(us, 1),
                "GBps": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
    del W, q
    xb = torch.randn(4096, 4096, generator=g, device=dev).to(torch.bfloat16)
    s = torch.empty(4096, device=dev)
    z = torch.empty(4096, dtype=torch.int32, device=dev)
    xq = torch.empty(4096, 4096, dtype=torch.int8, device=dev)
    us = _graph_time(lambda: q8.q8_choose_qparams(xb, s=s, z=z, xq=xq), reps)
    b = 4096 * 4096 * 3 + 4096 * 8
    out.append({"op": "choose_qparams", "shape": [4096, 4096], "us": round(us, 1),
                "GBps": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
    xf = torch.randn(4096, 4096, generator=g, device=dev) * 4
    xq2 = torch.empty(4096, 4096, dtype=torch.int8, device=dev)
    us = _graph_time(lambda: q8.q8_quantize_static(xf, (0.05, 3), (0.05 / 255, 0), xq1=xq, xq2=xq2),
                     reps)
    b = 4096 * 4096 * 6
    out.append({"op": "quantize_static_two_pass", "shape": [4096, 4096], "us": round(us, 1),
                "GBps": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
    mm = torch.empty(2, device=dev)
    us = _graph_time(lambda: q8.q8_observe_residual_minmax(xf, (0.05, 3), mm, reset=True), reps)
    b = 4096 * 4096 * 4
    out.append({"op": "observe_residual_minmax", "shape": [4096, 4096], "us": round(us, 1),
                "GBps": round(b / us / 1e3, 1), "frac_hbm": round(b / us / 1e3 / peaks["hbm_gbs"], 4)})
    return out


def bench_gptq(dev):
    """The offline GPTQ path on one Llama MLP up-projection (N = 11008, K = 4096): the
    calibration Hessian of 4096 fp32 rows (float64 x^T x), then GPTQ on the int8 grid
    (float64 factorisations and updates).  Event-timed, one run each after a warm-up."""
    import int8_quantized_linear_q8_b200 as q8

    N, K, R = 11008, 4096, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(93)
    x = torch.randn(R, K, generator=g, device=dev)
    W = torch.randn(N, K, generator=g, device=dev) * 0.02
    H = torch.empty(K, K, dtype=torch.float64, device=dev)
    nb = q8.q8_workspace_bytes(q8.Q8_OP_GPTQ_INT8, 0, N, K, 128)
    work = torch.empty(nb, dtype=torch.uint8, device=dev)
    q = torch.empty(N, K, dtype=torch.int8, device=dev)
    s = torch.empty(N, device=dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    ms_h = timed(lambda: q8.q8_hessian_accumulate(x, H, reset=True))
    ms_g = timed(lambda: q8.q8_gptq_int8(W, H, q=q, s_w=s, want_wsum=False, workspace=work))
    out = {"hessian": {"R": R, "K": K, "ms": round(ms_h, 2),
                       "fp64_Gops": round(R * K * (K + 1) / 2 * 2 / ms_h / 1e6, 1)},
           "gptq": {"N": N, "K": K, "block": 128, "ms": round(ms_g, 1),
                    "fp64_Gops": round((K ** 3 + N * K * K) * 2 / ms_g / 1e6, 1)}}
    del x, W, H, work, q, s
    return out


def bench_llama_stack(dev, peaks, prefill=True):
    """Llama-shaped stack, 32 layers x (q, k, v, o 4096x4096; gate, up 4096->11008; down
    11008->4096): decode at M = 1 through the W8A16 GEMV (6.5 GB of int8 weights per pass,
    one CUDA graph of 224 launches) and prefill at M = 4096 through the W8A8 GEMM."""
    import int8_quantized_linear_q8_b200 as q8

    g = torch.Generator(device=dev)
    layers = []
    for li in range(wl.LLAMA_LAYERS):
        lin = []
        for j, (name, K, N) in enumerate(wl.LLAMA_LINEARS):
            g.manual_seed(8 + li * 16 + j)
            W = torch.randn(N, K, generator=g, device=dev) * 0.02
            q, s, ws = q8.q8_quantize_weight(W)
            del W
            lin.append((K, N, q, s, ws))
        layers.append(lin)
    wbytes = sum(K * N for lin in layers for (K, N, _, _, _) in lin)
    res = {"layers": wl.LLAMA_LAYERS, "weight_bytes": wbytes}
    # decode
    xs = {K: torch.randn(1, K, generator=g, device=dev).to(torch.bfloat16) for K in (4096, 11008)}
    ys = {N: torch.empty(1, N, dtype=torch.bfloat16, device=dev) for N in (4096, 11008)}

    def decode():
        for lin in layers:
            for (K, N, q, s, ws) in lin:
                q8.q8_linear_w8a16(xs[K], q, s, y=ys[N])

    us = _graph_time(decode, 1)
    byts = sum(K * N + 4 * N + 2 * K + 2 * N for lin in layers for (K, N, _, _, _) in lin)
    res["decode"] = {"M": 1, "us_per_pass": round(us, 1), "GBps": round(byts / us / 1e3, 1),
                     "frac_hbm": round(byts / us / 1e3 / peaks["hbm_gbs"], 4),
                     "launches": 7 * wl.LLAMA_LAYERS}
    if prefill:
        M = wl.LLAMA_PREFILL_M
        xf = {K: torch.randn(M, K, generator=g, device=dev) for K in (4096, 11008)}
        qp = {}
        mm = torch.empty(2, device=dev)
        for K, x in xf.items():
            q8.q8_observe_minmax(x, mm, reset=True)
            qp[K] = q8.q8_qparams_from_minmax(*mm.cpu().tolist())
        yf = {N: torch.empty(M, N, device=dev) for N in (4096, 11008)}
        work = torch.empty(q8.q8_workspace_bytes(q8.Q8_OP_LINEAR_W8A8, M, 4096, 11008, 0),
                           dtype=torch.uint8, device=dev)

        def pre():
            for lin in layers:
                for (K, N, q, s, ws) in lin:
                    q8.q8_linear_w8a8(xf[K], qp[K], q, ws, s, y=yf[N], workspace=work)

        us = _graph_time(pre, 1)
        ops = sum(2.0 * M * N * K for lin in layers for (K, N, _, _, _) in lin)
        res["prefill"] = {"M": M, "ms_per_pass": round(us / 1e3, 2),
                          "TOPS": round(ops / us / 1e6, 1),
                          "frac_int8_peak": round(ops / us / 1e6 / int8_peak_tops(peaks), 4),
                          "launches": 2 * 7 * wl.LLAMA_LAYERS}
        del xf, yf, work
    del layers
    torch.cuda.empty_cache()
    return res


def _graph_time(fn, reps):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for _ in range(reps):
            fn()
    gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        gr.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1000.0 / (3 * reps)


# ----------------------------------------------------------------------------- arms


def run_ours(args):
    dist = Dist(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    import int8_quantized_linear_q8_b200 as q8
    from int8_quantized_linear_q8_b200 import build as q8build

    if dist.rank == 0:
        q8build.build()
    dist.barrier()
    q8.lib()

    sweep = W8A16Sweep(dev)
    if args.eager:
        graphs = [_EagerStep(sweep, c) for c in range(sweep.COPIES)]
    else:
        graphs = sweep.graphs()
    clk = ClockSampler(dist.local)
    clk.start()
    ms, t0, t1 = time_graphs(graphs, args.steps, args.warmup, dist)
    rows = clk.stop()
    clocks = ClockSampler.summarize(rows, t0, t1) if isinstance(rows, list) else rows
    del graphs
    ms_per_step = ms / args.steps
    value = job_throughput(dist.world, args.steps, sweep.step_bytes, ms) / 1e9
    peaks = measured_peaks()
    per_rank_gbps = args.steps * sweep.step_bytes / (ms * 1e-3) / 1e9

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 activations; N(0,0.02^2) fp32 weights "
                "quantized per channel on the GPU)",
        "config": {"workload": SWEEP_WORKLOAD,
                   "step": "12 GEMV launches (every shape x M), " +
                           ("launched eagerly" if args.eager else "one CUDA graph"),
                   "bytes_per_step": sweep.step_bytes,
                   "l2": f"inputs larger than L2: {sweep.COPIES} rotating weight copies "
                         f"({sweep.weight_bytes / 1e6:.0f} MB) vs 126 MB L2; M-major order",
                   "parallelism": f"replicas x{dist.world}"},
        "roofline": {"bound": "hbm", "kernel": "k_w8a16_tma",
                     "achieved": round(per_rank_gbps, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(per_rank_gbps / peaks["hbm_gbs"], 4),
                     "peak_source": peaks["source"], "traffic": sweep_traffic(),
                     "bytes_per_launch_avg": sweep.step_bytes // len(sweep.cases),
                     "note": "achieved = algorithmic bytes of the 12 launches / event time of "
                             "the timed steps (the step is only these launches)"},
        "gpu_launches": args.steps * len(sweep.cases),
        "clocks": clocks,
    }
    if dist.rank == 0 and not args.eager:
        result["cases"] = per_case_times(sweep)
    result["e2e"] = e2e_w8a16(sweep, max(10, min(args.steps // 10, 200)), 3, dist)
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline_w8a16(sweep)
    if dist.rank == 0 and not args.no_paths:
        result["paths"] = {
            "w8a16_bias": bias_case_times(sweep),
            "w4a16_nvfp4": bench_w4a16(dev, peaks),
            "w8a8_static_k960": bench_w8a8_paths(dev),
            "w8a8_prefill_m4096": bench_w8a8_prefill(dev, peaks),
            "dq8ca_q4gsw": bench_q4(dev, peaks),
            "quantizers": bench_quantizers(dev, peaks),
            "llama_stack": bench_llama_stack(dev, peaks),
            "gptq_offline": bench_gptq(dev),
        }
    dist.barrier()
    if dist.rank == 0:
        print(json.dumps(result), flush=True)
    dist.close()


SWEEP_WORKLOAD = ("W8A16 decode sweep: bf16 x [M,K] (M in 1,4,16) times int8 W [N,K], (K,N) in "
                  "(960,2560),(2048,8192),(4096,11008),(4096,32000); bf16 out")


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores, on the same metric
    (W8A16 decode GB/s).  Each step is a bounded sample of the workload: the M = 1 case of
    each sweep shape restricted to its first 256 output channels."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle

    shapes = wl.W8A16_SWEEP_SHAPES
    data = []
    rows = 256
    for i, sh in enumerate(shapes):
        W = wl.weight(rows, sh.K, seed=wl.W8A16_SWEEP_SEED_W * 1000 + i)
        q, s, _ = oracle.quantize_weight(W.numpy())
        x = wl.bf16_bits(wl.normal_bf16((1, sh.K), 1.0, seed=wl.W8A16_SWEEP_SEED_X * 1000 + i))
        data.append((sh, q, s, x))
    step_bytes = sum(w8a16_bytes(1, rows, sh.K) for sh, _, _, _ in data)

    def step():
        for sh, q, s, x in data:
            oracle.linear_w8a16(x, q, s)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = args.steps * step_bytes / el / 1e9
    sample = "per step: M=1 case of each of the 4 sweep shapes, first 256 output channels"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": SWEEP_WORKLOAD, "sample": sample,
                                        "bytes_per_step": step_bytes,
                                        "parallelism": "replicas x1 (rank 0 only)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile(args):
    """One kernel case, launched --reps times on fresh data (ncu capture target)."""
    import int8_quantized_linear_q8_b200 as q8

    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    M, N, K = args.pM, args.pN, args.pK
    W = torch.randn(N, K, generator=g, device=dev) * 0.02
    q, s, ws = q8.q8_quantize_weight(W)
    del W
    if args.profile == "w8a16":
        x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for _ in range(args.reps):
            q8.q8_linear_w8a16(x, q, s, y=y)
    elif args.profile == "w8a8":
        x = torch.randn(M, K, generator=g, device=dev) * 4
        y = torch.empty(M, N, device=dev)
        sec = (0.05 / 255, 0) if args.ptwo else None
        for _ in range(args.reps):
            q8.q8_linear_w8a8(x, (0.05, 3), q, ws, s, second=sec, y=y)
    elif args.profile == "w4a16":
        W = torch.randn(N, K, generator=g, device=dev) * 0.02
        q4, sf, gsc = q8.q8_quantize_weight_nvfp4(W)
        del W
        x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for _ in range(args.reps):
            q8.q8_linear_w4a16_nvfp4(x, q4, sf, gsc, y=y)
    elif args.profile == "quant":
        # the quantizers on an fp32 [N, K] weight and fp32 / bf16 [M, K] activations
        W = torch.randn(N, K, generator=g, device=dev) * 0.02
        xf = torch.randn(M, K, generator=g, device=dev) * 4
        xb = xf.to(torch.bfloat16)
        for _ in range(args.reps):
            q8.q8_quantize_weight(W, q=q, s_w=s, wsum=ws)
            q8.q8_choose_qparams(xb)
            q8.q8_quantize_static(xf, (0.05, 3), second=(0.05 / 255, 0))
    else:
        W = torch.randn(N, K, generator=g, device=dev) * 0.02
        q4, gs = q8.q8_quantize_weight_q4gs(W, args.pG)
        del W
        x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, device=dev)
        for _ in range(args.reps):
            q8.q8_linear_dq8ca_q4gsw(x, q4, gs, args.pG, y=y)
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "M": M, "N": N, "K": K, "reps": args.reps}))


def main():
    args = parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
