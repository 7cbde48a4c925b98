#!/usr/bin/env python3
"""Benchmark of the quantized decode-step linear layer on B200.

Default workload: a synthetic Q4_0 dense decode layer stack shaped like a 4B model at M = 1:
36 layers of hidden 2560, each with the projections q/k/v (2560 -> 4096/1024/1024, packed and
launched as one fused 6144-row GEMV), o (4096 -> 2560), gate_up (2560 -> 2 x 9728, fused SiLU gate)
and down (9728 -> 2560).  One step = one decode token through all 36 layers: the 144 GEMVs run as
one persistent qlin_gemv_chain launch, captured in a CUDA graph and replayed.  Attention, norms,
embeddings and the LM head are not part of the path and are not run.

Metric: quantized GEMV weight-stream GB/s (algorithmic bytes: packed codes + scales + activations
+ outputs, each once) and the equivalent decode tokens/s; one JSON line on stdout (rank 0).  With
one GPU the line also carries a "configs" object: the other workloads (the Q8_0 GEMV, the NVFP4
27B-shaped MLP at M = 1 and 4, the Q4_0 8B-A1B-shaped MoE layer at M = 1 and 8, the NVFP4 prefill
chunk at M = 512 and 64 plus an M sweep), each with its value, roofline, clocks and CPU baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlin|reference] [--config NAME]

--impl reference times the fp64 CPU oracle (the test reference) on a bounded sample of the same
workload; the oracle is used nowhere else in this file except the cpu_baseline legs.
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
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "quantized GEMV weight-stream GB/s (% of B200 HBM peak); synthetic decode tok/s"
HIDDEN, LAYERS = 2560, 36
# (name, N, K, epilogue) per layer; q/k/v share their input and are packed as one 6144-row matrix
STACK = [("qkv", 4096 + 1024 + 1024, 2560, 0), ("o", 2560, 4096, 0),
         ("gate_up", 2 * 9728, 2560, 1), ("down", 2560, 9728, 0)]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def fp4_peaks():
    """FP4 dense tensor denominators (TFLOP/s): the measured cuBLAS bf16 burst x 4 (NVIDIA's nominal
    fp4/bf16 ratio) as the roofline peak, and the 9 PFLOP/s dense spec beside it."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
        return 4 * bf16, "measured bf16 burst (cuBLAS) x 4, the nominal fp4/bf16 ratio", 9000.0
    except Exception:
        return 4 * 1590.0, "fallback bf16 x 4", 9000.0


def bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16 burst (cuBLAS)"
    except Exception:
        return 1590.0, "fallback bf16"


def sources_sha(names):
    """Short hash of library sources, so a recorded ncu traffic figure is used only for the
    kernel it was captured from."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "gemm_dequant_gemv_q8_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(key):
    """dram read + write bytes per launch from profiles/traffic.json, or None when the capture is
    of other sources than the current ones (the figure is then stale)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(key)
        if not e or e.get("sources_sha") != sources_sha(e["sources"]):
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled every ~2 ms through NVML (read-only
    queries) while the timed region runs; nvidia-smi is the fallback when NVML is unavailable."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []
        self.stop = threading.Event()
        self.t = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.index]) if vis and vis.split(",")[0].isdigit() else self.index
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _poll_nvml(self, nv, h):
        bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                flags = ["Active" if r & b else "Not Active" for b in bits]
                self.lines.append(f"{self.index}, {sm}, {mx}, {pw}, {r:#x}, " + ", ".join(flags))
            except Exception:
                break
            time.sleep(0.001)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.t = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.t.start()
            t0 = time.perf_counter()
            while not self.lines and time.perf_counter() - t0 < 2.0:  # sampling is running
                time.sleep(0.001)
            self.lines.clear()  # keep only samples taken inside the timed region
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(1.0)  # nvidia-smi's first sample
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        elif self.t is not None:
            self.t.join(timeout=1.0)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [t.strip() for t in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workloads
class DenseStack:
    """The packed layer stack on one GPU, with its inputs and outputs resident in HBM.

    All per-layer activations live in one device buffer (xbuf) and all per-layer outputs that
    leave the step (qkv, o, down) in another (ybuf), so the end-to-end leg moves them with one
    host->device and one device->host copy per step."""

    MODES = ("chain", "layer_chain", "launches")

    DATAFLOWS = ("stated", "serial")

    def __init__(self, fmt, layers, M=1, device="cuda", mode="chain", dataflow="stated", share=None):
        """mode: "chain" = the whole step as qlin_gemv_chain launches of up to
        qlin_chain_max_ops() ops (one for 36 layers); "layer_chain" = one chain of four ops per
        layer; "launches" = one qlin_gemv per projection.
        dataflow: "stated" = every projection reads its own N(0,1) activations except down, which
        reads its layer's h; "serial" = every projection reads the previous one's output, as in a
        decode step (o reads the first 4096 of the 6144 qkv outputs, qkv of layer l+1 reads down
        of layer l), so each op waits for the one before it.
        share: another DenseStack whose packed weights and buffers this one reuses."""
        import gemm_dequant_gemv_q8_b200 as q
        assert mode in self.MODES and dataflow in self.DATAFLOWS
        self.q, self.fmt, self.M, self.layers, self.mode = q, fmt, M, layers, mode
        self.dataflow = dataflow
        self.packed, self.ws = [], []
        self.weight_bytes = 0
        xs = [(l, pi, K) for l in range(layers) for pi, (n_, N, K, e) in enumerate(STACK) if n_ != "down"]
        ys = [(l, pi, N) for l in range(layers) for pi, (n_, N, K, e) in enumerate(STACK) if n_ != "gate_up"]
        if share is not None:
            self.xbuf, self.ybuf, self.hbuf = share.xbuf, share.ybuf, share.hbuf
        else:
            self.xbuf = torch.empty(M, sum(k for _, _, k in xs), device=device)
            self.ybuf = torch.empty(M, sum(n for _, _, n in ys), device=device)
            self.hbuf = torch.empty(layers, M, STACK[2][1] // 2, device=device)
        self.x, self.y = {}, {}
        off = 0
        for l, pi, K in xs:
            self.x[(l, pi)] = self.xbuf[:, off:off + K]
            off += K
        off = 0
        for l, pi, N in ys:
            self.y[(l, pi)] = self.ybuf[:, off:off + N]
            off += N
        for l in range(layers):
            self.x[(l, 3)] = self.hbuf[l]
            self.y[(l, 2)] = self.hbuf[l]
            if share is not None:
                continue
            lp, lw = [], []
            for pi, (name, N, K, epi) in enumerate(STACK):
                g = synth.gen(synth.seed_for(2, l, pi), device=device)
                blocks, scales, gs = synth.weights(fmt, N, K, g, device=device)
                pf = q.QLIN_PACK_GATE_UP if epi else q.QLIN_PACK_DEFAULT
                lp.append(q.qlin_pack_weights(fmt, N, K, blocks, scales, gs, pf))
                del blocks, scales
                self.weight_bytes += q.qlin_packed_bytes(fmt, N, K, pf) - 256
                lw.append(q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, N, K), device))
                if name != "down":
                    self.x[(l, pi)].copy_(synth.activations(
                        M, K, synth.gen(synth.seed_for(2, l, 5 + pi), device=device), device=device))
            self.packed.append(lp)
            self.ws.append(lw)
        if share is not None:
            self.packed, self.ws, self.weight_bytes = share.packed, share.ws, share.weight_bytes
        torch.cuda.synchronize()
        # algorithmic bytes per step: weights once + every activation read + every output written
        act = 0
        for (name, N, K, epi) in STACK:
            act += 4 * M * K + 4 * M * (N // 2 if epi else N)
        self.act_bytes = act * layers
        self.step_bytes = self.weight_bytes + self.act_bytes
        deps = {}  # (l, pi) -> the projection whose output it reads
        for l in range(layers):
            deps[(l, 3)] = (l, 2)
            if dataflow == "serial":
                if l > 0:
                    self.x[(l, 0)] = self.y[(l - 1, 3)]
                    deps[(l, 0)] = (l - 1, 3)
                self.x[(l, 1)] = self.y[(l, 0)][:, :STACK[1][2]]
                self.x[(l, 2)] = self.y[(l, 1)]
                deps[(l, 1)], deps[(l, 2)] = (l, 0), (l, 1)
        self.chains = []  # (ops, workspace) per launch
        if mode != "launches":
            ops, index = [], {}
            for l in range(layers):
                for pi, (name, N, K, epi) in enumerate(STACK):
                    if pi == 0 and ops and (mode == "layer_chain" or
                                            len(ops) + len(STACK) > q.qlin_chain_max_ops()):
                        self.chains.append(ops)
                        ops, index = [], {}
                    wait = index.get(deps.get((l, pi)), -1)  # an op of an earlier launch is done
                    index[(l, pi)] = len(ops)
                    ops.append(q.gemv_op(self.packed[l][pi], N, K, self.x[(l, pi)], self.y[(l, pi)],
                                         q.QLIN_EPI_SILU_GATE if epi else q.QLIN_EPI_NONE, wait))
            self.chains.append(ops)
            self.chains = [(o, q.workspace(q.qlin_chain_workspace_bytes(fmt, M, o), device)) for o in self.chains]
            self.launches_per_step = len(self.chains)
        else:
            self.launches_per_step = len(STACK) * layers

    def step(self, pdl=True):
        q = self.q
        fl = q.QLIN_FLAG_PDL if pdl else 0
        if self.chains:
            for ops, ws in self.chains:
                q.qlin_gemv_chain(self.fmt, q.QLIN_F32, self.M, ops, flags=fl, ws=ws)
            return
        for l in range(self.layers):
            P, W = self.packed[l], self.ws[l]
            for pi, (name, N, K, epi) in enumerate(STACK):
                q.qlin_gemv(self.fmt, P[pi], N, K, self.x[(l, pi)], y=self.y[(l, pi)], ws=W[pi],
                            flags=fl | (q.QLIN_EPI_SILU_GATE if epi else 0))

    def capture(self, pdl=True, host_io=None):
        """CUDA graph of one step; with host_io=(pinned_x, pinned_y) the graph also copies the
        step's inputs in and its outputs out."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step(pdl)  # warm (attributes, module load)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if host_io:
                self.xbuf.copy_(host_io[0], non_blocking=True)
            self.step(pdl)
            if host_io:
                host_io[1].copy_(self.ybuf, non_blocking=True)
        torch.cuda.synchronize()
        return g


def max_over_ranks(v, world, device="cuda"):
    """The largest of every rank's value (every rank calls it, in the same order)."""
    t = torch.tensor([float(v)], device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(step_bytes, world, ms):
    """Whole-job throughput: every rank streams step_bytes per step, the job takes the slowest rank's
    time (replicas: the work per GPU is fixed as the GPU count grows)."""
    return world * step_bytes / (ms * 1e-3) / 1e9


def time_graph(graph, steps, warmup):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        graph.replay()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / steps


def time_chain_kernel(stack, reps=4):
    """Average duration of one chain launch: `reps` steps' chain launches (no PDL, so launches do
    not overlap) captured in one CUDA graph, timed with CUDA events on the stream that replays it.
    Returns (ms per launch, algorithmic bytes per launch)."""
    q = stack.q

    def run():
        for _ in range(reps):
            for ops, ws in stack.chains:
                q.qlin_gemv_chain(stack.fmt, q.QLIN_F32, stack.M, ops, ws=ws)

    ms = _time_graph_of(run, 3, 2) / (reps * len(stack.chains))
    return ms, stack.step_bytes / len(stack.chains)


def time_dominant_kernel(stack, reps=3):
    """Average duration of the gate_up + SiLU GEMV launch (the largest per-launch share): a graph of
    every layer's gate_up launch (1 GB of weights at 36 layers, so every launch streams from HBM),
    timed with CUDA events."""
    q = stack.q
    name, N, K, epi = STACK[2]

    def run():
        for l in range(stack.layers):
            q.qlin_gemv(stack.fmt, stack.packed[l][2], N, K, stack.x[(l, 2)], y=stack.y[(l, 2)],
                        ws=stack.ws[l][2], flags=q.QLIN_EPI_SILU_GATE)

    ms = _time_graph_of(run, reps, 2) / stack.layers
    bytes_ = (q.qlin_packed_bytes(stack.fmt, N, K, q.QLIN_PACK_GATE_UP) - 256) + 4 * stack.M * (K + N // 2)
    return ms, bytes_


def e2e_stack(stack, steps, warmup, pdl=True):
    """Same metric through the public API with host buffers: every step copies its inputs from
    pinned host memory, runs the stack, and reads its outputs back, all inside the timed region
    (one graph: H2D copy, the chain launch, D2H copy)."""
    hx = stack.xbuf.cpu().pin_memory()
    hy = torch.empty(stack.ybuf.shape, dtype=torch.float32).pin_memory()
    g = stack.capture(pdl, host_io=(hx, hy))
    ms = time_graph(g, steps, warmup)
    del g
    return ms, hx.numel() * 4, hy.numel() * 4


# ----------------------------------------------------------------------------- CPU baseline
def cpu_info():
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    return model, n


def oracle_rate(fmt, shapes, M, budget_s, threads, seed=7, xdt=torch.float32):
    """The fp64 oracle (as it stands) on a bounded sample: the 64 rows of a 64-row block of each
    (N, K) projection shape, in a random order, against M activation rows, repeated for budget_s seconds
    on `threads` host threads (the oracle's C calls release the GIL, so the threads run on separate
    cores).  Its cost per row depends on K only, so a 64-row block stands for all N rows.
    Returns (weight GB/s, GFLOP/s, rows, seconds)."""
    import oracle
    data = []
    for (N, K) in shapes:
        b, s, gs = synth.weights(fmt, 64, K, synth.gen(seed + K))
        x = synth.activations(M, K, synth.gen(seed + 1 + K), dtype=xdt).double().numpy()
        data.append((K, b.numpy(), None if s is None else s.numpy(), gs, x, oracle.row_bytes(fmt, K)))

    def work(tid):
        rng = np.random.default_rng(seed + tid)
        nb = fl = rows = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            for (K, b, s, gs, x, rb) in data:
                oracle.gemv(fmt, 64, K, b, x, scales=s, g=gs, rows=rng.permutation(64))
                nb += 64 * rb
                fl += 2 * M * K * 64
                rows += 64
        return nb, fl, rows, time.perf_counter() - t0

    if threads == 1:
        res = [work(0)]
    else:
        with ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(work, range(threads)))
    t = max(r[3] for r in res)
    return sum(r[0] for r in res) / t / 1e9, sum(r[1] for r in res) / t / 1e9, sum(r[2] for r in res), t


def cpu_baseline(fmt, shapes, M, unit="GB/s", budget_s=2.5, xdt=torch.float32, what=""):
    """cpu_baseline object: the oracle timed on all host cores and on one core."""
    model, ncores = cpu_info()
    g_all, f_all, rows_all, t_all = oracle_rate(fmt, shapes, M, budget_s, ncores, xdt=xdt)
    g_one, f_one, rows_one, t_one = oracle_rate(fmt, shapes, M, budget_s, 1, xdt=xdt)
    pick = (lambda g, f: g) if unit == "GB/s" else (lambda g, f: f / 1e3)  # TFLOP/s
    ks = "/".join(str(K) for _, K in shapes)
    return {"value": pick(g_all, f_all), "unit": unit, "cores": ncores, "kind": "oracle",
            "sample": (f"{rows_all} weight rows of the {what or 'workload'} projection shapes (K = {ks}) x M = {M} "
                       f"activation rows, fp64 oracle on {ncores} host threads for {t_all:.1f} s"),
            "single_thread": {"value": pick(g_one, f_one), "unit": unit, "cores": 1,
                              "sample": f"{rows_one} rows, one thread, {t_one:.1f} s"},
            "cpu_model": model}


# ----------------------------------------------------------------------------- other configs
def _graph_of(fn):
    """fn() (a sequence of launches) captured in one CUDA graph, after one eager warm-up run."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def _time_graph_of(fn, steps, warmup):
    """Capture fn() in one CUDA graph and time replays with events (ms per replay)."""
    g = _graph_of(fn)
    ms = time_graph(g, steps, warmup)
    del g
    return ms


def timed(fn, steps, warmup, min_s=0.3):
    """ms per replay of fn's graph and the clocks sampled meanwhile: `steps` replays between two
    events, repeated until at least min_s of device time has passed (so the clock sampler sees the
    region), after `warmup` untimed replays."""
    g = _graph_of(fn)
    for _ in range(max(warmup, 3)):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total_ms, n = 0.0, 0
    with ClockSampler(torch.cuda.current_device()) as clk:
        while total_ms < 1e3 * min_s:
            a.record()
            for _ in range(steps):
                g.replay()
            b.record()
            b.synchronize()
            total_ms += a.elapsed_time(b)
            n += steps
    del g
    return total_ms / n, clk.summary()


HBM_SPEC_GBS = 8000.0  # B200 HBM3e, NVIDIA's 8 TB/s figure (printed beside the measured copy peak)


def roofline_hbm(kernel, bytes_per_launch, us_per_launch, traffic=None):
    peak, src = peaks()
    gbs = bytes_per_launch / (us_per_launch * 1e-6) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": peak, "peak_source": f"{src} hbm_gbs (copy)",
            "unit": "GB/s", "frac": gbs / peak, "traffic": traffic, "spec_peak": HBM_SPEC_GBS,
            "frac_of_spec": gbs / HBM_SPEC_GBS,
            "algorithmic_bytes_per_launch": bytes_per_launch, "avg_launch_us": us_per_launch}


_PROBE = {}


def fp4_mma_probe(iters=8192):
    """The FP4 tensor path's MMA-only rate on this device, measured once per process outside every
    timed region: qlin_probe_fp4_mma (one CTA per SM, `iters` back-to-back M128 N256 K64
    mxf4nvf4 MMAs on fixed shared-memory operands), two warm-up launches, then one launch timed
    with CUDA events."""
    if not _PROBE:
        import gemm_dequant_gemv_q8_b200 as q
        cycles = torch.zeros(1024, dtype=torch.int64, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for _ in range(2):
            q.qlin_probe_fp4_mma(iters, cycles, status)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        ctas = q.qlin_probe_fp4_mma(iters, cycles, status)
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b)
        _PROBE.update(tflops=2.0 * 128 * 256 * 64 * iters * ctas / (ms * 1e-3) / 1e12,
                      cycles_per_mma=float(cycles[:ctas].max()) / iters, ctas=ctas, iters=iters,
                      status=int(status.item()))
    return _PROBE


def roofline_fp4(kernel, flop_per_launch, us_per_launch):
    peak, src, spec = fp4_peaks()
    tf = flop_per_launch / (us_per_launch * 1e-6) / 1e12
    try:
        pr = fp4_mma_probe()
    except Exception as e:  # the roofline line stands without the probe
        pr = {"error": f"{type(e).__name__}: {e}"}
    ok = pr.get("status") == 0 and bool(pr.get("tflops"))
    return {"bound": "tensor", "kernel": kernel, "achieved": tf, "peak": peak, "peak_source": src,
            "unit": "TFLOP/s", "frac": tf / peak, "traffic": None, "spec_peak": spec, "frac_of_spec": tf / spec,
            "probe_peak": pr["tflops"] if ok else None, "frac_of_probe": tf / pr["tflops"] if ok else None,
            "probe": {"what": "qlin_probe_fp4_mma: M128 N256 K64 mxf4nvf4 MMAs back to back, one CTA per SM, "
                              "fixed shared-memory operands", **pr},
            "algorithmic_flop_per_launch": flop_per_launch, "avg_launch_us": us_per_launch}


def cfg_q8_small(args, cpu=True):
    """Q8_0 GEMV, M = 1, K = 1024, N = 256: launch-latency bound; a graph of 1000 launches over
    distinct weight copies (278 MB, more than twice L2)."""
    import gemm_dequant_gemv_q8_b200 as q
    fmt, N, K, M, copies = q.QLIN_Q8_0, 256, 1024, 1, 1000
    packs = []
    for c in range(copies):
        b, s_, g = synth.weights(fmt, N, K, synth.gen(1000 + c, device="cuda"), device="cuda")
        packs.append(q.qlin_pack_weights(fmt, N, K, b, s_, g))
    x = synth.activations(M, K, synth.gen(1, device="cuda"), device="cuda")
    y = torch.empty(M, N, device="cuda")
    ws = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, N, K)) for _ in range(copies)]
    fn = lambda: [q.qlin_gemv(fmt, packs[c], N, K, x, y=y, ws=ws[c], flags=q.QLIN_FLAG_PDL) for c in range(copies)]
    ms, clk = timed(fn, 3, args.warmup)
    us = ms * 1e3 / copies
    bytes_ = (q.qlin_packed_bytes(fmt, N, K) - 256) + 4 * M * (K + N)
    e = {"workload": "Q8_0 GEMV M=1 K=1024 N=256 (launch-latency bound; graph of 1000 launches over distinct "
                     "weight copies, PDL)", "M": M, "value": bytes_ / (us * 1e-6) / 1e9, "unit": "GB/s",
         "us_per_launch": us, "gpu_launches_per_replay": copies,
         "roofline": roofline_hbm("gemv_kernel<Q8_0, M=1>", bytes_, us), "clocks": clk,
         "l2": "1000 distinct weight copies (278 MB) per replay, more than twice L2"}
    if cpu:
        e["cpu_baseline"] = cpu_baseline(fmt, [(N, K)], M, what="Q8_0 GEMV")
    return {"q8_0_gemv_m1": e}


def cfg_mlp(args, fmt_name="nvfp4", cpu=True):
    """27B-shaped MLP (gate_up 5120 -> 2 x 17408 + SiLU, down 17408 -> 5120), bf16 activations,
    M = 1 and 4.  Two layers with distinct weights (300 MB) per replay; the step is both layers as
    one GEMV chain with h in bf16 (the headline value), and also one qlin_gemv per projection."""
    import gemm_dequant_gemv_q8_b200 as q
    fmt = q.QLIN_NVFP4 if fmt_name == "nvfp4" else q.QLIN_MXFP4
    H, I, L = 5120, 17408, 2
    gu, dn = [], []
    for l in range(L):
        b, s_, g = synth.weights(fmt, 2 * I, H, synth.gen(3000 + l, device="cuda"), device="cuda")
        gu.append(q.qlin_pack_weights(fmt, 2 * I, H, b, s_, g, q.QLIN_PACK_GATE_UP))
        b, s_, g = synth.weights(fmt, H, I, synth.gen(3100 + l, device="cuda"), device="cuda")
        dn.append(q.qlin_pack_weights(fmt, H, I, b, s_, g))
        del b, s_
    wb = (q.qlin_packed_bytes(fmt, 2 * I, H, 1) - 256) + (q.qlin_packed_bytes(fmt, H, I) - 256)
    out = {}
    for M in (1, 4):
        x = synth.activations(M, H, synth.gen(3200, device="cuda"), dtype=torch.bfloat16, device="cuda")
        h = torch.empty(M, I, device="cuda")
        y = torch.empty(M, H, device="cuda")
        wsg = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, 2 * I, H)) for _ in range(L)]
        wsd = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, H, I)) for _ in range(L)]

        def fn():
            for l in range(L):
                q.qlin_gemv(fmt, gu[l], 2 * I, H, x, y=h, ws=wsg[l], flags=q.QLIN_EPI_SILU_GATE | q.QLIN_FLAG_PDL)
                q.qlin_gemv(fmt, dn[l], H, I, h, y=y, ws=wsd[l], flags=q.QLIN_FLAG_PDL)
        ms1 = _time_graph_of(fn, args.steps, args.warmup) / L
        bytes1 = wb + M * (2 * H + 4 * I + 4 * I + 4 * H)
        hb = [torch.empty(M, I, device="cuda", dtype=torch.bfloat16) for _ in range(L)]
        ops = []
        for l in range(L):
            ops.append(q.gemv_op(gu[l], 2 * I, H, x, hb[l], q.QLIN_EPI_SILU_GATE | q.QLIN_OUT_BF16))
            ops.append(q.gemv_op(dn[l], H, I, hb[l], y, q.QLIN_EPI_NONE, len(ops) - 1))
        cws = q.workspace(q.qlin_chain_workspace_bytes(fmt, M, ops))
        fn2 = lambda: q.qlin_gemv_chain(fmt, q.QLIN_BF16, M, ops, flags=q.QLIN_FLAG_PDL, ws=cws)
        ms, clk = timed(fn2, args.steps, args.warmup)
        bytes2 = wb + M * (2 * H + 2 * I + 2 * I + 4 * H)  # per layer; h in bf16
        gbs = bytes2 / (ms / L * 1e-3) / 1e9
        e = {"workload": f"{fmt_name.upper()} MLP shaped like a 27B model: gate_up 5120->2x17408 + SiLU, down "
                         f"17408->5120, bf16 x, M={M}; both of two layers' projections as one GEMV chain "
                         "(h in bf16), two layers with distinct weights per replay (300 MB)",
             "M": M, "value": gbs, "unit": "GB/s", "us_per_layer": ms / L * 1e3, "tokens_per_s": M / (ms / L * 1e-3),
             "launches_per_layer": {"us_per_layer": ms1 * 1e3, "gbs": bytes1 / (ms1 * 1e-3) / 1e9,
                                    "note": "one qlin_gemv per projection, fp32 h"},
             "roofline": roofline_hbm(f"chain_kernel<{fmt_name.upper()}, bf16 x, M={M}> (4 GEMVs: 2 layers)",
                                      L * bytes2, ms * 1e3),
             "clocks": clk}
        if cpu:
            e["cpu_baseline"] = cpu_baseline(fmt, [(2 * I, H), (H, I)], M, xdt=torch.bfloat16,
                                             what=f"{fmt_name.upper()} MLP")
        out[f"{fmt_name}_mlp_m{M}"] = e
    return out


def cfg_moe(args, cpu=True):
    """Q4_0 MoE expert layer shaped like an 8B-A1B model (hidden 2048, 32 experts of gate_up
    2048 -> 2 x 1792 and down 1792 -> 2048, top-4), M = 1 and 8 tokens with independent routing; a
    graph of 8 layers with distinct weights (1.6 GB), so one replay's selected experts exceed L2."""
    import gemm_dequant_gemv_q8_b200 as q
    fmt, E, H, I, k, L = q.QLIN_Q4_0, 32, 2048, 1792, 4, 8
    gu, dn = [], []
    for l in range(L):
        c = [synth.weights(fmt, 2 * I, H, synth.gen(4000 + 100 * l + e, device="cuda"), device="cuda") for e in range(E)]
        gu.append(q.pack_experts(fmt, E, 2 * I, H, c, q.QLIN_PACK_GATE_UP))
        c = [synth.weights(fmt, H, I, synth.gen(5000 + 100 * l + e, device="cuda"), device="cuda") for e in range(E)]
        dn.append(q.pack_experts(fmt, E, H, I, c))
        del c
    per_expert = (q.qlin_packed_bytes(fmt, 2 * I, H, 1) - 256) + (q.qlin_packed_bytes(fmt, H, I) - 256)
    out = {}
    for M in (1, 8):
        logits = [synth.router_logits(M, E, synth.gen(6000 + l, device="cuda"), device="cuda") for l in range(L)]
        x = synth.activations(M, H, synth.gen(6100, device="cuda"), device="cuda")
        ids = torch.empty(M, k, dtype=torch.int32, device="cuda")
        w = torch.empty(M, k, device="cuda")
        y = torch.empty(M, H, device="cuda")
        ws = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k)) for _ in range(L)]

        def fn():
            for l in range(L):
                q.qlin_moe_experts(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                                   topk_w=w, y=y, ws=ws[l], flags=q.QLIN_FLAG_PDL)
        ms, clk = timed(fn, args.steps, args.warmup)
        distinct = []
        for l in range(L):  # actual distinct experts per layer for these seeds
            q.qlin_moe_experts(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                               topk_w=w, y=y, ws=ws[l])
            distinct.append(len(set(ids.cpu().flatten().tolist())))
        nd = sum(distinct) / L
        bytes_ = nd * per_expert + M * (4 * H + 4 * H + 4 * E)
        us = ms / L * 1e3
        e = {"workload": "Q4_0 MoE expert layer shaped like an 8B-A1B model: hidden 2048, 32 experts gate_up "
                         f"2048->2x1792, down 1792->2048, top-4, M={M} tokens; a graph of 8 layers' launches "
                         "(distinct weights, 1.6 GB)", "M": M, "distinct_experts": nd,
             "value": bytes_ / (us * 1e-6) / 1e9, "unit": "GB/s", "us_per_layer": us,
             "roofline": roofline_hbm(f"moe_kernel<Q4_0, M={M}> (route + gate_up + SiLU + down + combine)", bytes_, us),
             "clocks": clk,
             "bytes": "selected experts' packed weights (the actual distinct count per layer) + x, y, logits"}
        if cpu:
            e["cpu_baseline"] = cpu_baseline(fmt, [(2 * I, H), (H, I)], M, what="MoE expert")
        out[f"q4_0_moe_m{M}"] = e
    del gu, dn
    return out


def cfg_moe_prefill(args, cpu=True):
    """NVFP4 / MXFP4 MoE expert layer of the 8B-A1B shape (hidden 2048, 32 experts of gate_up
    2048 -> 2 x 1792 and down 1792 -> 2048, top-4) over a prefill chunk of M = 512 (and 2048) bf16
    tokens on the tensor cores: route + sort, gather, two grouped GEMMs, combine.  Two layers with
    distinct weights alternate (each 198 MB of packed experts, above L2).  At 64 routed rows per
    expert on average the layer sits below the FP4 ridge point, so its roofline is HBM: every
    expert's packed weights once per layer, plus x, y and the logits."""
    import gemm_dequant_gemv_q8_b200 as q
    E, H, I, k, L = 32, 2048, 1792, 4, 2
    out = {}
    for fmt, fname in ((q.QLIN_NVFP4, "NVFP4"), (q.QLIN_MXFP4, "MXFP4")):
        gu, dn = [], []
        for l in range(L):
            c = [synth.weights(fmt, 2 * I, H, synth.gen(8000 + 100 * l + e, device="cuda"), device="cuda")
                 for e in range(E)]
            gu.append(q.pack_experts(fmt, E, 2 * I, H, c, q.QLIN_PACK_MMA | q.QLIN_PACK_GATE_UP))
            c = [synth.weights(fmt, H, I, synth.gen(8500 + 100 * l + e, device="cuda"), device="cuda")
                 for e in range(E)]
            dn.append(q.pack_experts(fmt, E, H, I, c, q.QLIN_PACK_MMA))
            del c
        per_expert = (q.qlin_packed_bytes(fmt, 2 * I, H, q.QLIN_PACK_MMA | q.QLIN_PACK_GATE_UP) - 256 +
                      q.qlin_packed_bytes(fmt, H, I, q.QLIN_PACK_MMA) - 256)
        for M in ((512, 2048) if fmt == q.QLIN_NVFP4 else (512,)):
            logits = [synth.router_logits(M, E, synth.gen(8900 + l, device="cuda"), device="cuda") for l in range(L)]
            x = synth.activations(M, H, synth.gen(8950, device="cuda"), dtype=torch.bfloat16, device="cuda")
            ids = torch.empty(M, k, dtype=torch.int32, device="cuda")
            w = torch.empty(M, k, device="cuda")
            y = torch.empty(M, H, device="cuda")
            ws = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, k)) for _ in range(L)]

            def fn():
                for l in range(L):
                    q.qlin_moe_prefill(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                                       topk_w=w, y=y, ws=ws[l])
            ms, clk = timed(fn, args.steps, args.warmup)
            distinct, rows_padded = [], []
            for l in range(L):  # the routing these seeds give: experts in use, padded sorted rows
                q.qlin_moe_prefill(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                                   topk_w=w, y=y, ws=ws[l])
                cnt = torch.bincount(ids.flatten().long(), minlength=E).cpu()
                distinct.append(int((cnt > 0).sum()))
                rows_padded.append(int(((cnt + 127) // 128 * 128).sum()))
            nd = sum(distinct) / L
            us = ms / L * 1e3
            flop = 2.0 * M * k * (2 * I * H + H * I)
            bytes_ = nd * per_expert + M * (2 * H + 4 * H + 4 * E)
            tf = flop / (us * 1e-6) / 1e12
            rl = roofline_hbm(f"moe prefill layer ({fname}: route, gather, grouped gate_up + SiLU, grouped down, "
                              "combine; 5 launches)", bytes_, us)
            rl["tensor_frac"] = tf / fp4_peaks()[0]
            e = {"workload": f"{fname} MoE expert layer of the 8B-A1B shape over a prefill chunk: hidden 2048, 32 "
                             f"experts gate_up 2048->2x1792, down 1792->2048, top-4, M={M} bf16 tokens; two layers' "
                             "weights alternate (198 MB each)", "M": M, "distinct_experts": nd,
                 "sorted_rows_padded": sum(rows_padded) / L, "us_per_layer": us, "tflops": tf,
                 "value": bytes_ / (us * 1e-6) / 1e9, "unit": "GB/s", "roofline": rl, "clocks": clk,
                 "bytes": "every routed expert's packed weights + x (bf16), y (fp32), logits",
                 "flop": "2 * M * top_k * (2I * H + H * I), padding rows excluded"}
            if cpu and M == 512:
                e["cpu_baseline"] = cpu_baseline(fmt, [(2 * I, H), (H, I)], M * k // E, xdt=torch.bfloat16,
                                                 what="MoE expert (the mean routed rows per expert)")
            out[f"{fname.lower()}_moe_prefill_m{M}"] = e
            del ws
        del gu, dn
        torch.cuda.empty_cache()
    return out


FP4_COPIES = 6  # packed FP4 copies of the K = 5120, N = 17408 matrix rotated by the chunk configs


def cfg_chunk(args, cpu=True, sweep=(1, 2, 4, 8, 16)):
    """NVFP4 prefill-chunk GEMM, K = 5120, N = 17408: M = 512 (tensor-bound) and 64 (HBM-bound),
    and an M sweep on the same matrix.  FP4_COPIES copies of the 50 MB packed matrix rotate, so one
    graph replay streams 300 MB, more than twice the 126 MB L2: no call finds its weights there."""
    import gemm_dequant_gemv_q8_b200 as q
    fmt, N, K = q.QLIN_NVFP4, 17408, 5120
    packs = []
    for c in range(FP4_COPIES):
        b, s_, g = synth.weights(fmt, N, K, synth.gen(7000 + c, device="cuda"), device="cuda")
        packs.append(q.qlin_pack_weights(fmt, N, K, b, s_, g, q.QLIN_PACK_MMA))
        del b, s_
    wbytes = q.qlin_packed_bytes(fmt, N, K, q.QLIN_PACK_MMA) - 256
    out, sw = {}, {}
    for M in (512, 64) + tuple(sweep):
        x = synth.activations(M, K, synth.gen(7100 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
        y = torch.empty(M, N, device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
        fn = lambda: [q.qlin_gemm_chunk(fmt, packs[c], N, K, x, y=y, ws=ws, flags=q.QLIN_FLAG_PDL)
                      for c in range(FP4_COPIES)]
        ms, clk = timed(fn, args.steps, args.warmup)
        us = ms / FP4_COPIES * 1e3
        flop = 2.0 * M * N * K
        bytes_ = wbytes + 2 * M * K + 4 * M * N
        tf, gbs = flop / (us * 1e-6) / 1e12, bytes_ / (us * 1e-6) / 1e9
        if M in (512, 64):
            kern = f"chunk_gemm_kernel<1> (activation quantization + tcgen05 mxf4nvf4 GEMM), M={M}"
            e = {"workload": f"NVFP4 prefill-chunk GEMM M={M} K=5120 N=17408, bf16 x, fp32 accumulate; one persistent "
                             f"launch; {FP4_COPIES} weight copies rotate (300 MB per replay, above twice L2)",
                 "M": M, "us_per_call": us,
                 "tflops": tf, "gbs": gbs, "clocks": clk}
            if M == 512:
                e.update(value=tf, unit="TFLOP/s", roofline=roofline_fp4(kern, flop, us))
                if cpu:
                    e["cpu_baseline"] = cpu_baseline(fmt, [(N, K)], M, unit="TFLOP/s", xdt=torch.bfloat16,
                                                     what="NVFP4 chunk")
            else:
                e.update(value=gbs, unit="GB/s", roofline=roofline_hbm(kern, bytes_, us))
                if cpu:
                    e["cpu_baseline"] = cpu_baseline(fmt, [(N, K)], M, xdt=torch.bfloat16, what="NVFP4 chunk")
            out[f"nvfp4_chunk_m{M}"] = e
        else:
            sw[str(M)] = {"us_per_call": us, "tflops": tf, "gbs": gbs, "hbm_frac": gbs / peaks()[0]}
    if sw:
        out["nvfp4_chunk_m_sweep"] = {"workload": "the same GEMM at small M (the GEMV regime on the chunk path)",
                                      "by_M": sw}
    # MXFP4 weights of the same shape on their own chunk path (MX-quantized activations, kind::mxf4).
    del packs
    mpacks = []
    for c in range(FP4_COPIES):
        b, s_, _ = synth.weights(q.QLIN_MXFP4, N, K, synth.gen(7300 + c, device="cuda"), device="cuda")
        mpacks.append(q.qlin_pack_weights(q.QLIN_MXFP4, N, K, b, s_, 1.0, q.QLIN_PACK_MMA))
        del b, s_
    mx = {}
    for M in (512, 64):
        x = synth.activations(M, K, synth.gen(7100 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
        y = torch.empty(M, N, device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, q.QLIN_MXFP4, M, N, K))
        fn = lambda: [q.qlin_gemm_chunk(q.QLIN_MXFP4, mpacks[c], N, K, x, y=y, ws=ws, flags=q.QLIN_FLAG_PDL)
                      for c in range(FP4_COPIES)]
        ms = _time_graph_of(fn, args.steps, args.warmup) / FP4_COPIES
        us = ms * 1e3
        tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
        mx[str(M)] = {"us_per_call": us, "tflops": tf, "fp4_frac": tf / fp4_peaks()[0],
                      "gbs": (wbytes + 2 * M * K + 4 * M * N) / (us * 1e-6) / 1e9}
    out["mxfp4_chunk"] = {"workload": "MXFP4 weights of the same shape (UE8M0 scales per 32): MX-quantized "
                                      "activations + tcgen05 kind::mxf4 GEMM in one launch", "by_M": mx}
    del mpacks
    # The bf16-operand path for the same NVFP4 weights (QLIN_PACK_MMA_BF16: exact e2m1 * e4m3 products
    # in bf16, x not quantized), tcgen05 kind::f16 on CTA pairs.
    bpacks = []
    for c in range(2):
        b, s_, g = synth.weights(fmt, N, K, synth.gen(7000 + c, device="cuda"), device="cuda")
        bpacks.append(q.qlin_pack_weights(fmt, N, K, b, s_, g, q.QLIN_PACK_MMA_BF16))
        del b, s_
    bpk, bsrc = bf16_peak()
    bp = {}
    for M in (512, 64):
        x = synth.activations(M, K, synth.gen(7100 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
        y = torch.empty(M, N, device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
        fl = q.QLIN_FLAG_PDL | q.QLIN_FLAG_BF16_COPY | q.QLIN_FLAG_CTA_PAIRS
        fn = lambda: [q.qlin_gemm_chunk(fmt, bpacks[c], N, K, x, y=y, ws=ws, flags=fl) for c in range(2)]
        ms = _time_graph_of(fn, args.steps, args.warmup) / 2
        us = ms * 1e3
        tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
        bp[str(M)] = {"us_per_call": us, "tflops": tf, "bf16_frac": tf / bpk, "bf16_peak": bpk,
                      "gbs": (N * K * 2 + 2 * M * K + 4 * M * N) / (us * 1e-6) / 1e9}
    out["nvfp4_chunk_bf16_path"] = {"workload": "the same NVFP4 weights through the bf16-operand path "
                                                "(QLIN_PACK_MMA_BF16 + QLIN_FLAG_BF16_COPY, CTA pairs): bf16 x not "
                                                "quantized, 2 B/weight", "by_M": bp, "bf16_peak_source": bsrc}
    return out


CONFIGS = {"q8_small": cfg_q8_small, "nvfp4_mlp": cfg_mlp, "moe": cfg_moe, "chunk": cfg_chunk,
           "moe_prefill": cfg_moe_prefill, "mxfp4_mlp": lambda a, cpu=True: cfg_mlp(a, "mxfp4", cpu)}


def run_config(name, args):
    """Measure one workload other than the default stack; one JSON line per entry."""
    import gemm_dequant_gemv_q8_b200 as q
    torch.cuda.set_device(0)
    entries = {}
    if name in CONFIGS:
        entries = CONFIGS[name](args, cpu=not args.no_cpu_baseline)
    elif name in ("q4_k_stack", "q6_k_stack"):
        # the default stack's shapes (every K a multiple of 256) in a GGUF K-quant, one chain per step
        fmt, fname, per256 = (q.QLIN_Q4_K, "Q4_K", 144) if name == "q4_k_stack" else (q.QLIN_Q6_K, "Q6_K", 210)
        stack = DenseStack(fmt, args.layers, mode="chain")
        ms, clk = timed(lambda: stack.step(True), args.steps, args.warmup)
        canon = sum(N * K * per256 // 256 for (_, N, K, _) in STACK) * args.layers
        entries[name] = dict(workload=f"{fname} dense decode layer stack, the Q4_0 stack's shapes ({args.layers} layers "
                             "of hidden 2560: qkv 2560->6144, o 4096->2560, gate_up 2560->2x9728 + SiLU, "
                             "down 9728->2560), one GEMV chain per step", M=1, ms_per_step=ms,
                             packed_weight_bytes=stack.weight_bytes, canonical_weight_bytes=canon,
                             value=stack.step_bytes / (ms * 1e-3) / 1e9, unit="GB/s", decode_tok_s=1e3 / ms,
                             roofline=roofline_hbm(f"chain_kernel<{fname}, M=1>", stack.step_bytes, ms * 1e3),
                             clocks=clk,
                             l2="inputs larger than L2: %.2f GB of packed weights per step" % (stack.weight_bytes / 1e9))
    elif name == "gguf_chunk":
        # GGUF prefill chunk: the bf16 copy of dequantized Q4_0 weights (QLIN_PACK_MMA) times bf16 x on
        # the tensor cores (kind::f16), at the NVFP4 chunk workload's shape
        fmt, N, K = q.QLIN_Q4_0, 17408, 5120
        packs = []
        for c in range(2):  # two copies (2 x 178 MB) so consecutive calls do not find the weights in L2
            b, _, _ = synth.weights(fmt, N, K, synth.gen(7100 + c, device="cuda"), device="cuda")
            packs.append(q.qlin_pack_weights(fmt, N, K, b, None, 1.0, q.QLIN_PACK_MMA))
            del b
        bpk, bsrc = bf16_peak()
        for M, pairs in ((512, True), (512, False), (64, False)):
            x = synth.activations(M, K, synth.gen(7200 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
            y = torch.empty(M, N, device="cuda")
            ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
            fl = q.QLIN_FLAG_PDL | (q.QLIN_FLAG_CTA_PAIRS if pairs else 0)
            fn = lambda: [q.qlin_gemm_chunk(fmt, packs[c], N, K, x, y=y, ws=ws, flags=fl) for c in range(2)]
            ms, clk = timed(fn, args.steps, args.warmup)
            us = ms / 2 * 1e3
            flop = 2.0 * M * N * K
            tf = flop / (us * 1e-6) / 1e12
            bytes_ = N * K * 2 + 2 * M * K + 4 * M * N
            tiling = "256 x 256 tiles on CTA pairs" if pairs else "128 x 256 tiles on single CTAs"
            entries[f"gguf_chunk_m{M}{'_pairs' if pairs else ''}"] = dict(
                workload=f"Q4_0 prefill-chunk GEMM M={M} K=5120 N=17408 (bf16 copy of the dequantized weights x bf16 "
                         f"activations, tcgen05 kind::f16, one launch, {tiling})", M=M, cta_pairs=pairs,
                us_per_call=us, value=tf, unit="TFLOP/s", gbs=bytes_ / (us * 1e-6) / 1e9,
                roofline={"bound": "tensor", "kernel": "chunk_bf16_kernel", "achieved": tf, "peak": bpk,
                          "peak_source": bsrc, "unit": "TFLOP/s", "frac": tf / bpk, "traffic": None,
                          "avg_launch_us": us},
                clocks=clk)
    for key, e in entries.items():
        e.update(metric=METRIC, config=name, entry=key, impl="qlin", n_gpus=1)
        print(json.dumps(e), flush=True)


# ----------------------------------------------------------------------------- small cases for ncu
def small_case(name, reps=3):
    """A few launches of one kernel on one layer, for ncu captures that end in seconds (the
    profiles under profiles/ name these commands): moe1 / moe8 = one Q4_0 MoE layer of the 8B-A1B
    shape at M = 1 / 8; moepf512 = one NVFP4 MoE prefill layer of that shape at M = 512 (five
    launches per call); mlp1 / mlp4 = one NVFP4 27B-shaped MLP as a two-op GEMV chain (h in bf16)
    at M = 1 / 4; chunk512 = the NVFP4 prefill-chunk GEMM (K 5120, N 17408) at M = 512."""
    import gemm_dequant_gemv_q8_b200 as q
    torch.cuda.set_device(0)
    if name.startswith("moe") and not name.startswith("moepf"):
        M = int(name[3:])
        fmt, E, H, I, k = q.QLIN_Q4_0, 32, 2048, 1792, 4
        c = [synth.weights(fmt, 2 * I, H, synth.gen(4000 + e, device="cuda"), device="cuda") for e in range(E)]
        gu = q.pack_experts(fmt, E, 2 * I, H, c, q.QLIN_PACK_GATE_UP)
        c = [synth.weights(fmt, H, I, synth.gen(5000 + e, device="cuda"), device="cuda") for e in range(E)]
        dn = q.pack_experts(fmt, E, H, I, c)
        del c
        logits = synth.router_logits(M, E, synth.gen(6000, device="cuda"), device="cuda")
        x = synth.activations(M, H, synth.gen(6100, device="cuda"), device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k))
        for _ in range(reps):
            q.qlin_moe_experts(fmt, gu, dn, E, H, I, k, x, router_logits=logits, ws=ws)
    elif name == "chunk512":
        fmt, N, K, M = q.QLIN_NVFP4, 17408, 5120, 512
        b, s_, g = synth.weights(fmt, N, K, synth.gen(7000, device="cuda"), device="cuda")
        pk = q.qlin_pack_weights(fmt, N, K, b, s_, g, q.QLIN_PACK_MMA)
        del b, s_
        x = synth.activations(M, K, synth.gen(7100 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
        y = torch.empty(M, N, device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
        for _ in range(reps):
            q.qlin_gemm_chunk(fmt, pk, N, K, x, y=y, ws=ws)
    elif name.startswith("moepf"):
        M = int(name[5:])
        fmt, E, H, I, k = q.QLIN_NVFP4, 32, 2048, 1792, 4
        c = [synth.weights(fmt, 2 * I, H, synth.gen(8000 + e, device="cuda"), device="cuda") for e in range(E)]
        gu = q.pack_experts(fmt, E, 2 * I, H, c, q.QLIN_PACK_MMA | q.QLIN_PACK_GATE_UP)
        c = [synth.weights(fmt, H, I, synth.gen(8500 + e, device="cuda"), device="cuda") for e in range(E)]
        dn = q.pack_experts(fmt, E, H, I, c, q.QLIN_PACK_MMA)
        del c
        logits = synth.router_logits(M, E, synth.gen(8900, device="cuda"), device="cuda")
        x = synth.activations(M, H, synth.gen(8950, device="cuda"), dtype=torch.bfloat16, device="cuda")
        ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE_PREFILL, fmt, M, H, I, E, k))
        for _ in range(reps):
            q.qlin_moe_prefill(fmt, gu, dn, E, H, I, k, x, router_logits=logits, ws=ws)
    elif name.startswith("mlp"):
        M = int(name[3:])
        fmt, H, I = q.QLIN_NVFP4, 5120, 17408
        b, s_, g = synth.weights(fmt, 2 * I, H, synth.gen(3000, device="cuda"), device="cuda")
        gu = q.qlin_pack_weights(fmt, 2 * I, H, b, s_, g, q.QLIN_PACK_GATE_UP)
        b, s_, g = synth.weights(fmt, H, I, synth.gen(3100, device="cuda"), device="cuda")
        dn = q.qlin_pack_weights(fmt, H, I, b, s_, g)
        del b, s_
        x = synth.activations(M, H, synth.gen(3200, device="cuda"), dtype=torch.bfloat16, device="cuda")
        hb = torch.empty(M, I, device="cuda", dtype=torch.bfloat16)
        y = torch.empty(M, H, device="cuda")
        ops = [q.gemv_op(gu, 2 * I, H, x, hb, q.QLIN_EPI_SILU_GATE | q.QLIN_OUT_BF16), q.gemv_op(dn, H, I, hb, y, 0, 0)]
        ws = q.workspace(q.qlin_chain_workspace_bytes(fmt, M, ops))
        for _ in range(reps):
            q.qlin_gemv_chain(fmt, q.QLIN_BF16, M, ops, ws=ws)
    else:
        raise ValueError(name)
    torch.cuda.synchronize()
    print(json.dumps({"small_case": name, "launches": reps}), flush=True)


# ----------------------------------------------------------------------------- reference arm
def reference_arm(args, workload, world):
    """The fp64 oracle as it stands on the host's cores: each step runs, on every host thread, 512
    random rows of each of the four projection shapes of the stack (row cost depends on K only)
    against one activation row.  The step time is measured (not extrapolated); value is weight
    GB/s, the unit of the GPU arm's value."""
    import oracle
    fmt = synth.Q4_0
    model, ncores = cpu_info()
    data = []
    for (name, N, K, epi) in STACK:
        b, s, gs = synth.weights(fmt, 64, K, synth.gen(11 + N))
        x = synth.activations(1, K, synth.gen(12 + K)).double().numpy()
        data.append((K, b.numpy(), gs, x, oracle.row_bytes(fmt, K)))
    rows_per_shape = 512

    def work(tid, step):
        rng = np.random.default_rng(1000 * step + tid)
        nb = 0
        for (K, b, gs, x, rb) in data:
            for _ in range(rows_per_shape // 64):
                oracle.gemv(fmt, 64, K, b, x, g=gs, rows=rng.permutation(64))
                nb += 64 * rb
        return nb

    with ThreadPoolExecutor(ncores) as ex:
        def step(i):
            return sum(ex.map(lambda t: work(t, i), range(ncores)))
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        nbytes = 0
        for i in range(args.steps):
            nbytes += step(args.warmup + i)
        dt = time.perf_counter() - t0
    gbs = nbytes / dt / 1e9
    ms = dt * 1e3 / args.steps
    stack_w = sum((N * K * 9 // 16) for (_, N, K, _) in STACK) * args.layers
    desc = (f"each step: {rows_per_shape} random weight rows of each of the four stack projection shapes "
            f"(K = 2560/4096/2560/9728) on each of {ncores} host threads, fp64 oracle ({nbytes // args.steps} "
            f"weight bytes per step; a full 36-layer token would be {stack_w} bytes)")
    return {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "decode_tok_s_equivalent": gbs * 1e9 / stack_w,
            "config": {"workload": workload, "format": "q4_0", "M": 1, "layers": args.layers},
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": ncores, "kind": "oracle", "sample": desc,
                             "cpu_model": model},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="qlin", choices=["qlin", "reference"])
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' entries")
    ap.add_argument("--mode", default="chain", choices=list(DenseStack.MODES),
                    help="how the stack step is launched (default: one persistent GEMV chain)")
    ap.add_argument("--dataflow", default="stated", choices=list(DenseStack.DATAFLOWS),
                    help="stated: independent inputs, down reads h; serial: every projection reads the "
                         "previous one's output (reported as an extra field either way)")
    ap.add_argument("--config", default="stack",
                    choices=["stack", "q8_small", "nvfp4_mlp", "mxfp4_mlp", "moe", "moe_prefill", "chunk", "q4_k_stack",
                             "q6_k_stack", "gguf_chunk"],
                    help="stack (default): the Q4_0 36-layer decode stack line; the others print their "
                         "entries alone")
    ap.add_argument("--small-case", choices=["moe1", "moe8", "mlp1", "mlp4", "moepf512", "chunk512"],
                    help="three launches of one layer's kernel (for ncu captures); prints no bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.small_case:
        small_case(args.small_case)
        return
    if args.config != "stack":
        run_config(args.config, args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    fmt = synth.Q4_0
    workload = (f"Q4_0 dense decode layer stack shaped like a 4B model, M=1: {args.layers} layers of "
                "hidden 2560; qkv 2560->6144 (q/k/v fused), o 4096->2560, gate_up 2560->2x9728 + SiLU, "
                "down 9728->2560")

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, workload, world)), flush=True)
        return

    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)

    stack = DenseStack(fmt, args.layers, mode=args.mode, dataflow=args.dataflow)
    graph = stack.capture(pdl=not args.no_pdl)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        graph.replay()
    barrier()
    with ClockSampler(local) as clk:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            graph.replay()
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b) / args.steps
    barrier()
    ms_max = max_over_ranks(ms, world)

    # The other dataflow on the same weights (device-timed, same launch mode).
    other_df = "serial" if args.dataflow == "stated" else "stated"
    other = DenseStack(fmt, args.layers, mode=args.mode, dataflow=other_df, share=stack)
    g2 = other.capture(pdl=not args.no_pdl)
    other_ms = time_graph(g2, args.steps, args.warmup)
    del g2
    other_ms = max_over_ranks(other_ms, world)

    if stack.chains:
        dom_ms, dom_bytes = time_chain_kernel(stack)
        dom_name = (f"chain_kernel<Q4_0, M=1> ({len(stack.chains[0][0])} GEMVs per launch, "
                    f"{len(stack.chains)} launches per step; timed in a graph without PDL)")
        traffic = recorded_traffic("chain_q4_0_m1") if (args.layers == LAYERS and args.mode == "chain") else None
    else:
        dom_ms, dom_bytes = time_dominant_kernel(stack)
        dom_name = "gemv_kernel<Q4_0, M=1, SiLU-gate> (gate_up 2560->19456)"
        traffic = None
    e2e_ms, h2d, d2h = e2e_stack(stack, args.steps, args.warmup, pdl=not args.no_pdl)
    e2e_ms = max_over_ranks(e2e_ms, world)
    del graph

    line = None
    if rank == 0:
        peak, peak_src = peaks()
        gbs = whole_job_gbs(stack.step_bytes, world, ms_max)
        rf = roofline_hbm(dom_name, dom_bytes, dom_ms * 1e3, traffic)
        line = {
            "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "decode_tok_s": world * 1e3 / ms_max,
            "hbm_frac": gbs / world / peak,
            "config": {"workload": workload, "format": "q4_0", "M": 1, "layers": args.layers,
                       "dataflow": args.dataflow,
                       "weight_bytes_per_step": stack.weight_bytes, "algorithmic_bytes_per_step": stack.step_bytes,
                       "launches_per_step": stack.launches_per_step, "mode": args.mode,
                       "cuda_graph": True, "pdl": not args.no_pdl,
                       "l2": "inputs larger than L2: %.2f GB of packed weights streamed per step (L2 126 MB)"
                             % (stack.weight_bytes / 1e9),
                       "parallelism": f"replicas{world}"},
            "roofline": rf,
            "e2e": {"value": whole_job_gbs(stack.step_bytes, world, e2e_ms), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            f"{other_df}_dataflow": {"value": whole_job_gbs(other.step_bytes, world, other_ms), "unit": "GB/s",
                                     "ms_per_step": other_ms, "mode": args.mode,
                                     "launches_per_step": other.launches_per_step,
                                     "decode_tok_s": 1e3 / other_ms},
            "gpu_launches": stack.launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(fmt, [(N, K) for (_, N, K, _) in STACK], 1, budget_s=4.0,
                                                what="stack")
    del stack, other
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        # The other workloads, each with its own value, roofline, clocks and CPU baseline.
        cfgs = {}
        for fn in (cfg_q8_small, cfg_mlp, cfg_moe, cfg_moe_prefill, cfg_chunk):
            try:
                cfgs.update(fn(args, cpu=not args.no_cpu_baseline))
            except Exception as ex:  # keep the headline line; record what failed
                cfgs[fn.__name__] = {"error": repr(ex)}
            torch.cuda.empty_cache()
        line["configs"] = cfgs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
