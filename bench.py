#!/usr/bin/env python3
"""Benchmark of the quantized decode-step linear layer on B200.

Default workload: a synthetic Q4_0 dense decode layer stack shaped like a 4B model at M = 1:
36 layers of hidden 2560, each with the projections q/k/v (2560 -> 4096/1024/1024, packed and
launched as one fused 6144-row GEMV), o (4096 -> 2560), gate_up (2560 -> 2 x 9728, fused SiLU gate)
and down (9728 -> 2560).  One step = one decode token through all 36 layers = 144 GEMV launches,
captured once in a CUDA graph (with programmatic dependent launch between the kernels) and
replayed.  Attention, norms, embeddings and the LM head are not part of the path and are not run.

Metric: quantized GEMV weight-stream GB/s (algorithmic bytes: packed codes + scales + activations
+ outputs, each once) and the equivalent decode tokens/s; JSON line on stdout (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlin|reference] [--config NAME]

--impl reference times the fp64 CPU oracle (the test reference) on a bounded sample of the same
workload; the oracle is used nowhere else in this file except the cpu_baseline leg.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

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


def time_chain_kernel(stack, reps=3):
    """Average duration of one chain launch, timed with CUDA events on the launching stream
    (eager launches, no graph); algorithmic bytes of the ops that launch covers."""
    q = stack.q
    st = torch.cuda.current_stream()

    def run():
        for ops, ws in stack.chains:
            q.qlin_gemv_chain(stack.fmt, q.QLIN_F32, stack.M, ops, ws=ws)

    run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        run()
    b.record(st)
    b.synchronize()
    ms = a.elapsed_time(b) / (reps * len(stack.chains))
    return ms, stack.step_bytes / len(stack.chains)


def time_dominant_kernel(stack, reps=3):
    """Average duration of the gate_up + SiLU GEMV launch (the largest per-launch share),
    timed with CUDA events on the launching stream, rotating over the layers' matrices
    (1 GB of weights at 36 layers, so every launch streams from HBM)."""
    q = stack.q
    name, N, K, epi = STACK[2]
    st = torch.cuda.current_stream()

    def run():
        for l in range(stack.layers):
            q.qlin_gemv(stack.fmt, stack.packed[l][2], N, K, stack.x[(l, 2)], y=stack.y[(l, 2)],
                        ws=stack.ws[l][2], flags=q.QLIN_EPI_SILU_GATE)

    run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(reps):
        run()
    b.record(st)
    b.synchronize()
    ms = a.elapsed_time(b) / (reps * stack.layers)
    bytes_ = (q.qlin_packed_bytes(stack.fmt, N, K, q.QLIN_PACK_GATE_UP) - 256) + 4 * stack.M * (K + N // 2)
    return ms, bytes_


def e2e_stack(stack, steps, warmup, pdl=True):
    """Same metric through the public API with host buffers: every step copies its inputs from
    pinned host memory, runs the stack, and reads its outputs back, all inside the timed region
    (one graph: H2D copy, 144 GEMV launches, D2H copy)."""
    hx = stack.xbuf.cpu().pin_memory()
    hy = torch.empty(stack.ybuf.shape, dtype=torch.float32).pin_memory()
    g = stack.capture(pdl, host_io=(hx, hy))
    ms = time_graph(g, steps, warmup)
    del g
    return ms, hx.numel() * 4, hy.numel() * 4


def cpu_baseline_stack(fmt, budget_s=12.0, seed=7):
    """The fp64 oracle on a bounded sample of the stack: rows of every projection shape, timed
    on the host; scaled to GB/s of weights processed.  Returns (GB/s, cores, description)."""
    import oracle
    rng = np.random.default_rng(seed)
    per_shape = []
    for (name, N, K, epi) in STACK:
        b, s, gs = synth.weights(fmt, 64, K, synth.gen(seed + N))
        x = synth.activations(1, K, synth.gen(seed + K)).double().numpy()
        per_shape.append((N, K, b.numpy(), None if s is None else s.numpy(), gs, x))
    # probe, then size the sample to the budget
    done_bytes, t_used, rows = 0, 0.0, 0
    t0 = time.perf_counter()
    while t_used < budget_s:
        for (N, K, b, s, gs, x) in per_shape:
            r = rng.integers(0, 64, 16)
            oracle.gemv(fmt, 64, K, b, x, scales=s, g=gs, rows=r)
            rowb = oracle.row_bytes(fmt, K)
            done_bytes += 16 * rowb
            rows += 16
        t_used = time.perf_counter() - t0
    gbs = done_bytes / t_used / 1e9
    desc = (f"{rows} weight rows of the four stack projection shapes (K = 2560/4096/2560/9728), "
            f"single-threaded fp64 oracle, {t_used:.1f} s")
    return gbs, 1, desc



# ----------------------------------------------------------------------------- other configs
def _time_graph_of(fn, steps, warmup):
    """Capture fn() (a sequence of launches) in one CUDA graph and time replays with events."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    ms = time_graph(g, steps, warmup)
    del g
    return ms


def run_config(name, args):
    """Measure one of the non-default workloads; one JSON line per (config, M)."""
    import gemm_dequant_gemv_q8_b200 as q
    torch.cuda.set_device(0)
    peak, peak_src = peaks()
    lines = []
    if name in ("q4_k_stack", "q6_k_stack"):
        # the default stack's shapes (every K a multiple of 256) in a GGUF K-quant, one chain per step
        fmt, fname, per256 = (q.QLIN_Q4_K, "Q4_K", 144) if name == "q4_k_stack" else (q.QLIN_Q6_K, "Q6_K", 210)
        stack = DenseStack(fmt, args.layers, mode="chain")
        graph = stack.capture(pdl=True)
        ms = time_graph(graph, args.steps, max(args.warmup, 3))
        del graph
        canon = sum(N * K * per256 // 256 for (_, N, K, _) in STACK) * args.layers
        lines.append(dict(workload=f"{fname} dense decode layer stack, the Q4_0 stack's shapes ({args.layers} layers "
                          "of hidden 2560: qkv 2560->6144, o 4096->2560, gate_up 2560->2x9728 + SiLU, "
                          "down 9728->2560), one GEMV chain per step", M=1, ms_per_step=ms,
                          packed_weight_bytes=stack.weight_bytes, canonical_weight_bytes=canon,
                          gbs=stack.step_bytes / (ms * 1e-3) / 1e9, decode_tok_s=1e3 / ms,
                          l2="inputs larger than L2: %.2f GB of packed weights per step" % (stack.weight_bytes / 1e9)))
    if name == "q8_small":
        fmt, N, K, M, copies = q.QLIN_Q8_0, 256, 1024, 1, 1000  # 278 MB of rotating copies > 2x L2
        packs = []
        for c in range(copies):
            b, s_, g = synth.weights(fmt, N, K, synth.gen(1000 + c, device="cuda"), device="cuda")
            packs.append(q.qlin_pack_weights(fmt, N, K, b, s_, g))
        x = synth.activations(M, K, synth.gen(1, device="cuda"), device="cuda")
        y = torch.empty(M, N, device="cuda")
        ws = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, N, K)) for _ in range(copies)]
        fn = lambda: [q.qlin_gemv(fmt, packs[c], N, K, x, y=y, ws=ws[c], flags=q.QLIN_FLAG_PDL) for c in range(copies)]
        ms = _time_graph_of(fn, max(3, args.steps // 4), args.warmup) / copies
        wb = q.qlin_packed_bytes(fmt, N, K) - 256
        bytes_ = wb + 4 * M * (K + N)
        lines.append(dict(workload="Q8_0 GEMV M=1 K=1024 N=256 (launch-latency bound; graph of 1000 "
                          "launches over distinct weight copies, PDL)", M=M, us_per_launch=ms * 1e3,
                          gbs=bytes_ / (ms * 1e-3) / 1e9))
    elif name in ("nvfp4_mlp", "mxfp4_mlp"):
        fmt, H, I = (q.QLIN_NVFP4 if name == "nvfp4_mlp" else q.QLIN_MXFP4), 5120, 17408
        fname = "NVFP4" if fmt == q.QLIN_NVFP4 else "MXFP4"
        for M in (1, 4):
            L = 2
            gu, dn, wsg, wsd = [], [], [], []
            for l in range(L):
                b, s_, g = synth.weights(fmt, 2 * I, H, synth.gen(3000 + l, device="cuda"), device="cuda")
                gu.append(q.qlin_pack_weights(fmt, 2 * I, H, b, s_, g, q.QLIN_PACK_GATE_UP))
                b, s_, g = synth.weights(fmt, H, I, synth.gen(3100 + l, device="cuda"), device="cuda")
                dn.append(q.qlin_pack_weights(fmt, H, I, b, s_, g))
                wsg.append(q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, 2 * I, H)))
                wsd.append(q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_GEMV, fmt, M, H, I)))
            x = synth.activations(M, H, synth.gen(3200, device="cuda"), dtype=torch.bfloat16, device="cuda")
            h = torch.empty(M, I, device="cuda")
            y = torch.empty(M, H, device="cuda")

            def fn():
                for l in range(L):
                    q.qlin_gemv(fmt, gu[l], 2 * I, H, x, y=h, ws=wsg[l], flags=q.QLIN_EPI_SILU_GATE | q.QLIN_FLAG_PDL)
                    q.qlin_gemv(fmt, dn[l], H, I, h, y=y, ws=wsd[l], flags=q.QLIN_FLAG_PDL)
            ms = _time_graph_of(fn, args.steps, args.warmup) / L
            wb = (q.qlin_packed_bytes(fmt, 2 * I, H, 1) - 256) + (q.qlin_packed_bytes(fmt, H, I) - 256)
            bytes_ = wb + M * (2 * H + 4 * I + 4 * I + 4 * H)
            lines.append(dict(workload=f"{fname} MLP shaped like a 27B model: gate_up 5120->2x17408 + SiLU, "
                              "down 17408->5120, bf16 activations; one qlin_gemv per projection (fp32 h)",
                              M=M, us_per_layer=ms * 1e3, gbs=bytes_ / (ms * 1e-3) / 1e9,
                              tokens_per_s=M / (ms * 1e-3)))
            # The same layers as one GEMV chain per step, h kept in bf16 (QLIN_OUT_BF16).
            hb = [torch.empty(M, I, device="cuda", dtype=torch.bfloat16) for _ in range(L)]
            ops = []
            for l in range(L):
                ops.append(q.gemv_op(gu[l], 2 * I, H, x, hb[l], q.QLIN_EPI_SILU_GATE | q.QLIN_OUT_BF16))
                ops.append(q.gemv_op(dn[l], H, I, hb[l], y, q.QLIN_EPI_NONE, len(ops) - 1))
            cws = q.workspace(q.qlin_chain_workspace_bytes(fmt, M, ops))
            fn2 = lambda: q.qlin_gemv_chain(fmt, q.QLIN_BF16, M, ops, flags=q.QLIN_FLAG_PDL, ws=cws)
            ms2 = _time_graph_of(fn2, args.steps, args.warmup) / L
            bytes2 = wb + M * (2 * H + 2 * I + 2 * I + 4 * H)
            lines.append(dict(workload=f"{fname} MLP shaped like a 27B model, as above; both layers as one "
                              "GEMV chain, h in bf16", M=M, us_per_layer=ms2 * 1e3,
                              gbs=bytes2 / (ms2 * 1e-3) / 1e9, tokens_per_s=M / (ms2 * 1e-3)))
            del gu, dn
    elif name == "moe":
        fmt, E, H, I, k = q.QLIN_Q4_0, 32, 2048, 1792, 4
        L = 8  # 8 layers (1.6 GB): one replay's selected experts (>= 8 x 25 MB) exceed L2
        canon_gu = [[synth.weights(fmt, 2 * I, H, synth.gen(4000 + 100 * l + e, device="cuda"), device="cuda")
                     for e in range(E)] for l in range(L)]
        gu = [q.pack_experts(fmt, E, 2 * I, H, c, q.QLIN_PACK_GATE_UP) for c in canon_gu]
        del canon_gu
        canon_dn = [[synth.weights(fmt, H, I, synth.gen(5000 + 100 * l + e, device="cuda"), device="cuda")
                     for e in range(E)] for l in range(L)]
        dn = [q.pack_experts(fmt, E, H, I, c) for c in canon_dn]
        del canon_dn
        per_expert = (q.qlin_packed_bytes(fmt, 2 * I, H, 1) - 256) + (q.qlin_packed_bytes(fmt, H, I) - 256)
        for M in (1, 8):
            logits = [synth.router_logits(M, E, synth.gen(6000 + l, device="cuda"), device="cuda") for l in range(L)]
            x = synth.activations(M, H, synth.gen(6100, device="cuda"), device="cuda")
            ids = torch.empty(M, k, dtype=torch.int32, device="cuda")
            w = torch.empty(M, k, device="cuda")
            y = torch.empty(M, H, device="cuda")
            ws = [q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_MOE, fmt, M, H, I, E, k)) for _ in range(L)]
            distinct = []

            def fn():
                for l in range(L):
                    q.qlin_moe_experts(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                                       topk_w=w, y=y, ws=ws[l], flags=q.QLIN_FLAG_PDL)
            ms = _time_graph_of(fn, args.steps, args.warmup) / L
            for l in range(L):  # actual distinct experts per layer for these seeds
                q.qlin_moe_experts(fmt, gu[l], dn[l], E, H, I, k, x, router_logits=logits[l], topk_ids=ids,
                                   topk_w=w, y=y, ws=ws[l])
                distinct.append(len(set(ids.cpu().flatten().tolist())))
            nd = sum(distinct) / L
            bytes_ = nd * per_expert + M * (4 * H + 4 * H + 4 * E)
            lines.append(dict(workload="Q4_0 MoE expert layer shaped like an 8B-A1B model: hidden 2048, 32 experts "
                              "gate_up 2048->2x1792, down 1792->2048, top-4; a graph of 8 layers' launches "
                              "(distinct weights)", M=M, distinct_experts=nd,
                              us_per_layer=ms * 1e3, gbs=bytes_ / (ms * 1e-3) / 1e9))
    if name == "gguf_chunk":
        # GGUF prefill chunk: the bf16 copy of dequantized Q4_0 weights (QLIN_PACK_MMA) times bf16 x on
        # the tensor cores (kind::f16), at the NVFP4 chunk workload's shape
        fmt, N, K = q.QLIN_Q4_0, 17408, 5120
        packs = []
        for c in range(2):  # two copies (2 x 178 MB) so consecutive calls do not find the weights in L2
            b, _, _ = synth.weights(fmt, N, K, synth.gen(7100 + c, device="cuda"), device="cuda")
            packs.append(q.qlin_pack_weights(fmt, N, K, b, None, 1.0, q.QLIN_PACK_MMA))
            del b
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                bf16_peak, bf16_src = float(json.load(f)["bf16_tflops"]), "measured bf16 burst (cuBLAS)"
        except Exception:
            bf16_peak, bf16_src = 1590.0, "fallback bf16"
        for M, pairs in ((512, True), (512, False), (64, False)):
            x = synth.activations(M, K, synth.gen(7200 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
            y = torch.empty(M, N, device="cuda")
            ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
            fl = q.QLIN_FLAG_PDL | (q.QLIN_FLAG_CTA_PAIRS if pairs else 0)
            fn = lambda: [q.qlin_gemm_chunk(fmt, packs[c], N, K, x, y=y, ws=ws, flags=fl) for c in range(2)]
            ms = _time_graph_of(fn, args.steps, args.warmup) / 2
            flop = 2.0 * M * N * K
            bytes_ = N * K * 2 + 2 * M * K + 4 * M * N
            tiling = "256 x 256 tiles on CTA pairs" if pairs else "128 x 256 tiles on single CTAs"
            lines.append(dict(workload=f"Q4_0 prefill-chunk GEMM M={M} K=5120 N=17408 (bf16 copy of the dequantized "
                              f"weights x bf16 activations, tcgen05 kind::f16, one launch, {tiling})", M=M,
                              cta_pairs=pairs, us_per_call=ms * 1e3,
                              tflops=flop / (ms * 1e-3) / 1e12, bf16_peak_tflops=bf16_peak, bf16_peak_source=bf16_src,
                              bf16_frac=flop / (ms * 1e-3) / 1e12 / bf16_peak, gbs=bytes_ / (ms * 1e-3) / 1e9))
    if name == "chunk":
        fmt, N, K = q.QLIN_NVFP4, 17408, 5120
        b, s_, g = synth.weights(fmt, N, K, synth.gen(7000, device="cuda"), device="cuda")
        packs = [q.qlin_pack_weights(fmt, N, K, b, s_, g, q.QLIN_PACK_MMA)]
        b2, s2, g2 = synth.weights(fmt, N, K, synth.gen(7001, device="cuda"), device="cuda")
        packs.append(q.qlin_pack_weights(fmt, N, K, b2, s2, g2, q.QLIN_PACK_MMA))  # 2 copies > L2 with y
        del b, s_, b2, s2
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                bf16 = float(json.load(f)["bf16_tflops"])
            fp4_peak, fp4_src = 4 * bf16, "measured bf16 burst x 4 (nominal fp4/bf16 ratio)"
        except Exception:
            fp4_peak, fp4_src = 4 * 1590.0, "fallback bf16 x 4"
        for M in (512, 64, 16, 8, 4, 2, 1):
            x = synth.activations(M, K, synth.gen(7100 + M, device="cuda"), dtype=torch.bfloat16, device="cuda")
            y = torch.empty(M, N, device="cuda")
            ws = q.workspace(q.qlin_workspace_bytes(q.QLIN_OP_CHUNK, fmt, M, N, K))
            fn = lambda: [q.qlin_gemm_chunk(fmt, packs[c], N, K, x, y=y, ws=ws, flags=q.QLIN_FLAG_PDL) for c in range(2)]
            ms = _time_graph_of(fn, args.steps, args.warmup) / 2
            flop = 2.0 * M * N * K
            bytes_ = (q.qlin_packed_bytes(fmt, N, K, q.QLIN_PACK_MMA) - 256) + 2 * M * K + 4 * M * N
            lines.append(dict(workload=f"NVFP4 prefill-chunk GEMM M={M} K=5120 N=17408 (activation quantization "
                              "+ tcgen05 block-scaled GEMM in one persistent launch)", M=M, us_per_call=ms * 1e3,
                              tflops=flop / (ms * 1e-3) / 1e12, fp4_peak_tflops=fp4_peak, fp4_peak_source=fp4_src,
                              fp4_frac=flop / (ms * 1e-3) / 1e12 / fp4_peak, gbs=bytes_ / (ms * 1e-3) / 1e9))
    for ln in lines:
        ln.update(metric=METRIC, unit="GB/s", value=ln["gbs"], hbm_frac=ln["gbs"] / peak,
                  peak=peak, peak_source=peak_src, config=name, impl="qlin", n_gpus=1)
        print(json.dumps(ln), flush=True)

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
    ap.add_argument("--mode", default="chain", choices=list(DenseStack.MODES),
                    help="how the stack step is launched (default: one persistent GEMV chain)")
    ap.add_argument("--dataflow", default="stated", choices=list(DenseStack.DATAFLOWS),
                    help="stated: independent inputs, down reads h; serial: every projection reads the "
                         "previous one's output (reported as an extra field either way)")
    ap.add_argument("--config", default="stack",
                    choices=["stack", "q8_small", "nvfp4_mlp", "mxfp4_mlp", "moe", "chunk", "q4_k_stack",
                             "q6_k_stack", "gguf_chunk"],
                    help="stack (default): the Q4_0 36-layer decode stack; the others print extra lines")
    args = ap.parse_args()
    if args.config != "stack":
        run_config(args.config, args)
        return
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    fmt = synth.Q4_0
    workload = (f"Q4_0 dense decode layer stack shaped like a 4B model, M=1: {args.layers} layers of "
                "hidden 2560; qkv 2560->6144 (q/k/v fused), o 4096->2560, gate_up 2560->2x9728 + SiLU, "
                "down 9728->2560")

    if args.impl == "reference":
        if rank != 0:
            return
        gbs, cores, desc = cpu_baseline_stack(fmt, budget_s=max(5.0, 2.0 * args.steps))
        stack_w = sum((N * K * 9 // 16) for (_, N, K, _) in STACK) * args.layers
        tok_s = gbs * 1e9 / stack_w
        line = {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 / tok_s, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference", "decode_tok_s": tok_s,
                "config": {"workload": workload, "format": "q4_0", "M": 1, "layers": args.layers},
                "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
                "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
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
                    f"{len(stack.chains)} launches per step)")
    else:
        dom_ms, dom_bytes = time_dominant_kernel(stack)
        dom_name = "gemv_kernel<Q4_0, M=1, SiLU-gate> (gate_up 2560->19456)"
    e2e_ms, h2d, d2h = e2e_stack(stack, args.steps, args.warmup, pdl=not args.no_pdl)
    e2e_ms = max_over_ranks(e2e_ms, world)
    del graph

    if rank == 0:
        peak, peak_src = peaks()
        gbs = whole_job_gbs(stack.step_bytes, world, ms_max)
        dom_gbs = dom_bytes / (dom_ms * 1e-3) / 1e9
        traffic = None  # the committed capture's estimate holds for the default 36-layer launch only
        try:
            if args.layers == LAYERS:
                with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
                    key = f"{args.mode}_q4_0_m1_bytes_per_launch" if stack.chains else "gate_up_q4_0_m1_bytes_per_launch"
                    traffic = json.load(f).get(key)
        except Exception:
            pass
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
            "roofline": {"bound": "hbm", "kernel": dom_name,
                         "achieved": dom_gbs, "peak": peak, "peak_source": f"{peak_src} hbm_gbs (copy)",
                         "unit": "GB/s", "frac": dom_gbs / peak, "traffic": traffic,
                         "algorithmic_bytes_per_launch": dom_bytes, "avg_launch_us": dom_ms * 1e3},
            "e2e": {"value": whole_job_gbs(stack.step_bytes, world, e2e_ms), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            f"{other_df}_dataflow": {"value": whole_job_gbs(other.step_bytes, world, other_ms), "unit": "GB/s",
                                     "ms_per_step": other_ms, "mode": args.mode,
                                     "launches_per_step": other.launches_per_step},
            "gpu_launches": stack.launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline and world == 1:
            cg, cores, desc = cpu_baseline_stack(fmt)
            line["cpu_baseline"] = {"value": cg, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
