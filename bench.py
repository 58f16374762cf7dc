#!/usr/bin/env python
"""Throughput of the block-scaled W8A8 linear layer (libbq) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bq|reference]
                    [--workload decode|prefill|fp8|moe|perchannel|mxfp8] [--no-sub]

Prints ONE JSON line.  The headline workload is the decode linear layer:
INT8, N = K = 4096, [128,128] weight blocks, token counts M in {1, 8, 32, 64};
one step = for each M, the dynamic 1x128 activation quantisation followed by
the block-scaled GEMM (bq_quant_act + bq_gemm, i.e. bq_linear).  Sixteen
weight copies rotate (268 MB > the 126 MB L2), so every GEMM streams its
weights from HBM.  `value` is whole-job algorithmic HBM bytes per second.
Sub-workloads (prefill INT8 4096x14336x4096, FP8 e4m3 2048x4096x14336, the
INT8 MoE layer T=4096, E=8, top-2 with the fused w13 + SiLU requantisation,
per-channel INT8 on the prefill shape, and the MXFP8 linear on the FP8
shape) report TOPS against the tensor roofline.

Multi-GPU: the layer shards over tokens with no exchange (replicas), so each
rank runs the same per-rank work ("scaling": "weak"); time is the max over
ranks of CUDA-event time.  `--impl reference` times the CPU oracle (the
plain C reference) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import bq_synth  # noqa: E402

METRIC = "block-scaled W8A8 GEMM TOPS & weight GB/s; % of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_traffic(kernel_source: str):
    """DRAM bytes per launch of the roofline kernel from the committed ncu
    record (profiles/roofline_traffic.json), or (None, why) when there is no
    record or the kernel source changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "block_scaled_w8a8_b200", "csrc", rec["source_file"])
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None, "no ncu record"
    if rec["source_file"] != kernel_source or rec["source_sha256"] != digest:
        return None, "kernel changed since the ncu capture"
    return float(rec["dram_bytes_per_launch"]), rec["capture"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

class Dist:
    """One process per GPU (torchrun env). Replicas only: ranks run the same
    workload on their own GPU with no data-path collective; the barrier and
    the max over ranks are the timing plumbing. NCCL on GPUs, gloo on CPU."""

    def __init__(self, n_gpus: int, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.n_gpus = n_gpus
        self.pg = None
        self.device = torch.device("cpu")
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                self.device = torch.device("cuda", self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                        device_id=self.device)
            else:
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)
            self.device = torch.device("cuda", 0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def whole_job_rate(world: int, steps: int, units_per_step: float, seconds: float) -> float:
    """Units all ranks processed per second: every rank runs `steps` steps of
    `units_per_step`, and `seconds` is the slowest rank's time (weak scaling)."""
    return world * steps * units_per_step / seconds


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"bq_clocks_{os.getpid()}_{gpu_index}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if not self.proc or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    mhz.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        # every sample taken while the timed region ran counts: a clock stuck
        # low must show in the median, not be filtered out
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "sm_min_mhz": min(mhz) if mhz else None, "samples": len(mhz),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def cdiv(a, b):
    return -(-a // b)


def timed_graph_steps(graphs, steps, warmup, stream, dist):
    """Replay graphs[i % len(graphs)] for warmup+steps; returns seconds of the
    timed steps (CUDA events, max over ranks)."""
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        graphs[(warmup + i) % len(graphs)].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    return dist.max(e0.elapsed_time(e1) / 1e3)


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()                       # warm (allocations, attributes)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def quant_weights(w, dtype, bq, bn=128, bk=128):
    q, s = bq.quant_weight(w, bn, bk, dtype)
    return q, s


# --------------------------------------------------------------------------
# workloads (CUDA path)
# --------------------------------------------------------------------------

def bench_decode(args, dist, bq, peaks, stream):
    N = K = 4096
    Ms = bq_synth.DECODE_MS
    NW = 16
    dev = torch.device("cuda", torch.cuda.current_device())
    Nb, Kb = cdiv(N, 128), cdiv(K, 128)
    ws_q, ws_s = [], []
    for i in range(NW):
        w = bq_synth.weights(N, K, 0.02, 100 + i, device=dev)
        q, s = quant_weights(w, bq.INT8, bq)
        ws_q.append(q)
        ws_s.append(s)
        del w
    xs = [bq_synth.activations(M, K, cfg.seed, cfg.n_outliers, cfg.outlier_scale, device=dev)
          for M, cfg in zip(Ms, bq_synth.DECODE)]
    outs = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for M in Ms]
    qa = [torch.empty(M, K, dtype=torch.uint8, device=dev) for M in Ms]
    sa = [torch.empty(Kb, M, dtype=torch.float32, device=dev) for M in Ms]
    gws = [bq.workspace(bq.gemm_workspace_size(M, N, K), dev) for M in Ms]
    torch.cuda.synchronize()

    lws = bq.workspace(max(bq.linear_workspace_size(M, N, K) for M in Ms), dev)

    def step(phase, quant=True, gemm=True):
        def run():
            for j, M in enumerate(Ms):
                wi = (4 * phase + j) % NW
                if quant and gemm:      # the public call: bq_linear
                    bq.linear(xs[j], ws_q[wi], ws_s[wi], 128, 128, bq.INT8, out=outs[j], ws=lws)
                elif quant:
                    bq.quant_act(xs[j], 128, bq.INT8, q=qa[j], s=sa[j])
                else:
                    bq.gemm(qa[j], sa[j], ws_q[wi], ws_s[wi], 128, 128, bq.INT8, out=outs[j],
                            ws=gws[j])
        return run

    phases = NW // len(Ms)
    graphs = [capture(step(p), stream) for p in range(phases)]
    gemm_graphs = [capture(step(p, quant=False), stream) for p in range(phases)]
    quant_graphs = [capture(step(p, gemm=False), stream) for p in range(phases)]

    gemm_bytes = sum(N * K + 4 * Nb * Kb + M * K + 4 * M * Kb + 2 * M * N for M in Ms)
    step_bytes = sum(N * K + 4 * Nb * Kb + 2 * M * K + 2 * M * N for M in Ms)
    with Clocks(torch.cuda.current_device()) as clk:
        t = timed_graph_steps(graphs, args.steps, args.warmup, stream, dist)
        t_gemm = timed_graph_steps(gemm_graphs, args.steps, args.warmup, stream, dist)
        t_quant = timed_graph_steps(quant_graphs, args.steps, args.warmup, stream, dist)
    clocks = clk.summary()

    # end to end through the public API with host buffers: H2D of the step's
    # activations from pinned memory, bq_linear, D2H of the outputs.  The four
    # layers are independent, so the copies run on their own streams: every
    # input goes up at the start of the step, each layer waits only for its
    # own, and each output comes back as soon as its layer is done.
    hx = [x.cpu().pin_memory() for x in xs]
    ho = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for M in Ms]
    dx = [torch.empty_like(x, device=dev) for x in xs]
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e(phase):
        def run():
            comp = torch.cuda.current_stream()
            start = torch.cuda.Event()
            start.record(comp)
            h2d_stream.wait_event(start)
            d2h_stream.wait_event(start)
            ready, done = [], []
            with torch.cuda.stream(h2d_stream):
                for j in range(len(Ms)):
                    dx[j].copy_(hx[j], non_blocking=True)
                    ready.append(torch.cuda.Event())
                    ready[j].record(h2d_stream)
            for j, M in enumerate(Ms):
                wi = (4 * phase + j) % NW
                comp.wait_event(ready[j])
                bq.linear(dx[j], ws_q[wi], ws_s[wi], 128, 128, bq.INT8, out=outs[j], ws=lws)
                done.append(torch.cuda.Event())
                done[j].record(comp)
            with torch.cuda.stream(d2h_stream):
                for j in range(len(Ms)):
                    d2h_stream.wait_event(done[j])
                    ho[j].copy_(outs[j], non_blocking=True)
            fin = torch.cuda.Event()
            fin.record(d2h_stream)
            comp.wait_event(fin)
        return run

    e2e_graphs = [capture(e2e(p), stream) for p in range(phases)]
    t_e2e = timed_graph_steps(e2e_graphs, args.steps, args.warmup, stream, dist)

    n = dist.world
    traffic, traffic_src = load_traffic("gemm_decode_cluster.cu")
    value = whole_job_rate(n, args.steps, step_bytes, t) / 1e9
    gemm_launch_s = t_gemm / (args.steps * len(Ms))
    achieved = gemm_bytes / len(Ms) / gemm_launch_s / 1e9
    res = {
        "value": value, "unit": "GB/s", "ms_per_step": 1e3 * t / args.steps,
        "roofline": {"bound": "hbm",
                     "kernel": "gemm_decode_cluster_kernel (block-scaled decode GEMM; four "
                               "launches per step, consecutive launches overlapped by "
                               "programmatic dependent launch)",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": gemm_bytes / len(Ms),
                     "avg_launch_us": 1e6 * gemm_launch_s},
        "quant_us_per_launch": 1e6 * t_quant / (args.steps * len(Ms)),
        "e2e": {"value": whole_job_rate(n, args.steps, step_bytes, t_e2e) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": sum(2 * M * K for M in Ms),
                "d2h_bytes_per_step": sum(2 * M * N for M in Ms)},
        "gpu_launches": args.steps * 2 * len(Ms),
        "clocks": clocks,
        "config": {"workload": "decode_int8_n4096_k4096_m1-8-32-64", "M": list(Ms), "N": N,
                   "K": K, "block": [128, 128], "act_group": 128,
                   "l2": "16 rotating weight copies (268 MB) > 126 MB L2",
                   "parallelism": f"replicas x{n}"},
        "dtype": "int8",
        "gemm_path": "auto",
    }
    del graphs, gemm_graphs, quant_graphs, e2e_graphs
    return res


def bench_linear_big(args, dist, bq, peaks, stream, cfg, n_rot):
    dev = torch.device("cuda", torch.cuda.current_device())
    M, N, K = cfg.M, cfg.N, cfg.K
    bn, bk = cfg.block_n, cfg.block_k
    mx = cfg.dtype == bq_synth.MXFP8
    wq, wsc = [], []
    for i in range(n_rot):
        w = bq_synth.weights(N, K, cfg.w_std, cfg.seed + 10 * i, device=dev)
        q, s = bq.mx_quant_weight(w) if mx else quant_weights(w, cfg.dtype, bq, bn, bk)
        wq.append(q)
        wsc.append(s)
        del w
    xs = [bq_synth.activations(M, K, cfg.seed + i, cfg.n_outliers, cfg.outlier_scale,
                               device=dev) for i in range(n_rot)]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    Kb = cdiv(K, bk)
    qa = torch.empty(M, K, dtype=torch.uint8, device=dev)
    if mx:
        sa = torch.empty(bq.mx_scale_bytes(M, K), dtype=torch.uint8, device=dev)
    else:
        sa = torch.empty(Kb, M, dtype=torch.float32, device=dev)
        gws = bq.workspace(bq.gemm_workspace_size(M, N, K, bn, bk, cfg.dtype), dev)
    torch.cuda.synchronize()

    def step(i, quant=True):
        def run():
            if mx:
                if quant:
                    bq.mx_quant_act(xs[i], q=qa, sf=sa)
                bq.mx_gemm(qa, sa, wq[i], wsc[i], out=out)
                return
            if quant:
                bq.quant_act(xs[i], bk, cfg.dtype, q=qa, s=sa)
            bq.gemm(qa, sa, wq[i], wsc[i], bn, bk, cfg.dtype, out=out, ws=gws)
        return run

    graphs = [capture(step(i), stream) for i in range(n_rot)]
    gemm_graphs = [capture(step(i, False), stream) for i in range(n_rot)]
    with Clocks(torch.cuda.current_device()) as clk:
        t = timed_graph_steps(graphs, args.steps, args.warmup, stream, dist)
        t_gemm = timed_graph_steps(gemm_graphs, args.steps, args.warmup, stream, dist)
    ops = 2.0 * M * N * K
    peak = 2.0 * peaks["bf16_tflops"]
    ach = ops / (t_gemm / args.steps) / 1e12
    del graphs, gemm_graphs
    return {"value": whole_job_rate(dist.world, args.steps, ops, t) / 1e12, "unit": "TOPS",
            "ms_per_step": 1e3 * t / args.steps,
            "roofline": {"bound": "tensor",
                         "kernel": ("tcgen05 mxf8f6f4.block_scale GEMM" if mx else
                                    "tcgen05 block-scaled GEMM"),
                         "achieved": ach, "peak": peak, "unit": "TFLOP/s" if cfg.dtype else
                         "TOPS", "frac": ach / peak, "traffic": None,
                         "peak_source": "2 x measured bf16 burst (8-bit dense = 2x bf16)",
                         "avg_launch_us": 1e6 * t_gemm / args.steps},
            "clocks": clk.summary(),
            "config": {"workload": cfg.name, "M": M, "N": N, "K": K, "block": [bn, bk],
                       "l2": f"{n_rot} rotating weight/activation copies"},
            "dtype": "mxfp8_e4m3" if mx else "fp8_e4m3" if cfg.dtype else "int8"}


def bench_tiny(args, dist, bq, stream):
    """Latency of the tiny block-wise INT8 linear layer (M = 16, N = 320,
    K = 200: partial blocks, the CUDA-core path since K = 200 is not a
    16-byte row), one bq_linear per call, 20 calls per graph replay."""
    cfg = bq_synth.TINY
    dev = torch.device("cuda", torch.cuda.current_device())
    w = bq_synth.weights(cfg.N, cfg.K, cfg.w_std, cfg.seed, device=dev)
    qw, sw = quant_weights(w, cfg.dtype, bq, cfg.block_n, cfg.block_k)
    x = bq_synth.activations(cfg.M, cfg.K, cfg.seed, cfg.n_outliers, cfg.outlier_scale,
                             device=dev)
    out = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device=dev)
    ws = bq.workspace(bq.linear_workspace_size(cfg.M, cfg.N, cfg.K), dev)
    calls = 20

    def run():
        for _ in range(calls):
            bq.linear(x, qw, sw, cfg.block_n, cfg.block_k, cfg.dtype, out=out, ws=ws)

    g = [capture(run, stream)]
    steps = max(3, args.steps // 4)
    t = timed_graph_steps(g, steps, args.warmup, stream, dist)
    del g
    return {"value": 1e6 * t / (steps * calls), "unit": "us", "higher_is_better": False,
            "config": {"workload": cfg.name, "M": cfg.M, "N": cfg.N, "K": cfg.K,
                       "block": [cfg.block_n, cfg.block_k]},
            "dtype": "int8", "note": "latency of one bq_linear call (quantiser + GEMM)"}


class MoeLayer:
    """The MoE layer of the block-int8 MoE workload (T tokens, E experts, top-k),
    device-resident: router logits, block-quantised w13 / w2, every
    intermediate, and run(parts) that enqueues the layer's library calls in
    order.  The full-size parity test drives the same object.  Every
    composition routes on the device ("route": softmax top-k of the logits).
    PARTS fuses the w13 GEMM with silu * up and its requantisation
    ("w13silu") and runs the w2 GEMM and the weighted combine as two calls;
    FUSED_COMBINE also puts the combine in the w2 epilogue ("w2comb": fp32
    atomic sums into token rows, then "fin" rounds them once to bf16);
    UNFUSED stores and re-reads every bf16 intermediate ("w13", "silu",
    "w2", "comb")."""

    PARTS = ("route", "perm", "gather", "w13silu", "w2", "comb")
    FUSED_COMBINE = ("route", "perm", "gather", "w13silu", "w2comb", "fin")
    UNFUSED = ("route", "perm", "gather", "w13", "silu", "w2", "comb")

    def __init__(self, bq, dev, cfg=None):
        cfg = cfg or bq_synth.MOE
        self.bq, self.cfg = bq, cfg
        T, H, I, E, topk = cfg.T, cfg.H, cfg.I, cfg.E, cfg.topk
        self.x = bq_synth.activations(T, H, cfg.seed, device=dev)
        self.logits = bq_synth.router_logits(T, E, cfg.seed).to(dev)
        self.ids_d = torch.empty(T, topk, dtype=torch.int32, device=dev)
        self.tw_d = torch.empty(T, topk, dtype=torch.float32, device=dev)
        self.q13 = torch.empty(E, 2 * I, H, dtype=torch.uint8, device=dev)
        self.s13 = torch.empty(E, 2 * cdiv(I, 128), cdiv(H, 128), dtype=torch.float32,
                               device=dev)
        self.q2 = torch.empty(E, H, I, dtype=torch.uint8, device=dev)
        self.s2 = torch.empty(E, cdiv(H, 128), cdiv(I, 128), dtype=torch.float32, device=dev)
        for e in range(E):
            w13 = self.w13_fp32(e, dev)
            for half in range(2):
                q, s = bq.quant_weight(w13[half * I:(half + 1) * I].contiguous(), 128, 128,
                                       cfg.dtype)
                self.q13[e, half * I:(half + 1) * I] = q
                self.s13[e, half * cdiv(I, 128):(half + 1) * cdiv(I, 128)] = s
            del w13
            q, s = bq.quant_weight(self.w2_fp32(e, dev), 128, 128, cfg.dtype)
            self.q2[e], self.s2[e] = q, s
        R = T * topk
        self.off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(R, dtype=torch.int32, device=dev)
        self.inv = torch.empty(R, dtype=torch.int32, device=dev)
        self.qa = torch.empty(R, H, dtype=torch.uint8, device=dev)
        self.sa = torch.empty(cdiv(H, 128), R, dtype=torch.float32, device=dev)
        self.y13 = torch.empty(R, 2 * I, dtype=torch.bfloat16, device=dev)
        self.qh = torch.empty(R, I, dtype=torch.uint8, device=dev)
        self.sh = torch.empty(cdiv(I, 128), R, dtype=torch.float32, device=dev)
        self.y2 = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        self.acc = torch.zeros(T, H, dtype=torch.float32, device=dev)   # "fin" re-zeroes it
        self.out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.ws = bq.workspace(bq.grouped_gemm_workspace_size(R, 2 * I, H, E), dev)
        torch.cuda.synchronize()

    def w13_fp32(self, e, dev):
        c = self.cfg
        return bq_synth.weights(2 * c.I, c.H, c.w_std, c.seed + 31 * e, device=dev)

    def w2_fp32(self, e, dev):
        c = self.cfg
        return bq_synth.weights(c.H, c.I, c.w_std, c.seed + 31 * e + 1, device=dev)

    def run(self, parts=PARTS):
        bq, c = self.bq, self.cfg
        L = bq.lib()
        st = torch.cuda.current_stream().cuda_stream
        if "route" in parts:
            bq.moe_route(self.logits, c.topk, ids=self.ids_d, weights=self.tw_d)
        if "perm" in parts:
            bq._check(L.bq_moe_permute(self.ids_d.data_ptr(), c.T, c.topk, c.E,
                                       self.off.data_ptr(), self.perm.data_ptr(),
                                       self.inv.data_ptr(), None, 0, st))
        if "gather" in parts:
            bq.moe_quant_gather(self.x, self.perm, c.topk, 128, c.dtype, q=self.qa, s=self.sa)
        if "w13" in parts:
            bq.grouped_gemm(self.qa, self.sa, self.off, self.q13, self.s13, 128, 128, c.I,
                            c.dtype, out=self.y13, ws=self.ws)
        if "silu" in parts:
            bq.moe_silu_mul_quant(self.y13, c.I, 128, c.dtype, q=self.qh, s=self.sh)
        if "w13silu" in parts:
            bq.grouped_gemm_silu_quant(self.qa, self.sa, self.off, self.q13, self.s13, c.dtype,
                                       q=self.qh, s=self.sh)
        if "w2" in parts:
            bq.grouped_gemm(self.qh, self.sh, self.off, self.q2, self.s2, 128, 128, 0, c.dtype,
                            out=self.y2, ws=self.ws)
        if "w2comb" in parts:
            bq.grouped_gemm_combine(self.qh, self.sh, self.off, self.q2, self.s2, self.perm,
                                    self.tw_d, self.acc, c.dtype)
        if "fin" in parts:
            bq.moe_combine_finish(self.acc, out=self.out)
        if "comb" in parts:
            bq.moe_combine(self.y2, self.inv, self.tw_d, out=self.out)


def bench_moe(args, dist, bq, peaks, stream):
    """The MoE layer in each composition the library offers (all compute the
    same layer: the fused SiLU epilogue is bit-identical to the unfused calls,
    the fused combine equal within its fp32-sum bound).  `value` is the
    fastest composition, the others are reported beside it; the roofline
    times that composition's two grouped GEMMs alone."""
    cfg = bq_synth.MOE
    dev = torch.device("cuda", torch.cuda.current_device())
    T, H, I, E, topk = cfg.T, cfg.H, cfg.I, cfg.E, cfg.topk
    R = T * topk
    moe = MoeLayer(bq, dev, cfg)
    comps = {"fused_w13": MoeLayer.PARTS, "unfused": MoeLayer.UNFUSED,
             "fused_w13_and_combine": MoeLayer.FUSED_COMBINE}
    gemms = {"fused_w13": ("w13silu", "w2"), "unfused": ("w13", "w2"),
             "fused_w13_and_combine": ("w13silu", "w2comb")}
    steps = max(3, args.steps // 4)
    times = {}
    with Clocks(torch.cuda.current_device()) as clk:
        for name, parts in comps.items():
            g = [capture(lambda parts=parts: moe.run(parts), stream)]
            times[name] = timed_graph_steps(g, steps, args.warmup, stream, dist)
            del g
        best = min(times, key=times.get)
        gg = [capture(lambda: moe.run(gemms[best]), stream)]
        t_g = timed_graph_steps(gg, steps, args.warmup, stream, dist)
        del gg
    t = times[best]
    ops = 2.0 * R * (2 * I) * H + 2.0 * R * H * I
    peak = 2.0 * peaks["bf16_tflops"]
    ach = ops / (t_g / steps) / 1e12
    return {"value": whole_job_rate(dist.world, steps, ops, t) / 1e12, "unit": "TOPS",
            "ms_per_step": 1e3 * t / steps, "steps": steps, "composition": best,
            "ms_per_step_by_composition": {k: 1e3 * v / steps for k, v in times.items()},
            "roofline": {"bound": "tensor",
                         "kernel": "tcgen05 grouped GEMMs of the timed composition: "
                                   + " + ".join(gemms[best]),
                         "achieved": ach, "peak": peak, "unit": "TOPS", "frac": ach / peak,
                         "traffic": None, "avg_pair_us": 1e6 * t_g / steps},
            "clocks": clk.summary(),
            "config": {"workload": cfg.name, "T": T, "H": H, "I": I, "E": E, "topk": topk,
                       "block": [128, 128], "routing": "device softmax top-2 of N(0,1) logits"},
            "dtype": "int8"}


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# --------------------------------------------------------------------------

class OracleDecode:
    """The decode workload on the CPU oracle: activation quantisation for
    M in {1, 8, 32, 64} and the block-scaled GEMM against the 4096 x 4096 INT8
    weight (the first of the GPU leg's rotating weights).  Inputs are prepared
    once; step() runs one whole decode step and returns its seconds."""

    def __init__(self, n_rows: int = 4096):
        import oracle
        self.oracle = oracle
        K = 4096
        w = bq_synth.weights(n_rows, K, 0.02, 100).numpy()
        self.qw, self.sw = oracle.quant_weight(w, 128, 128, oracle.INT8)
        self.xs = [bq_synth.bf16_bits(bq_synth.activations(M, K, c.seed, c.n_outliers,
                                                           c.outlier_scale))
                   for M, c in zip(bq_synth.DECODE_MS, bq_synth.DECODE)]
        Nb, Kb = cdiv(n_rows, 128), K // 128
        self.n_rows = n_rows
        self.bytes_per_step = sum(n_rows * K + 4 * Nb * Kb + 2 * M * K + 2 * M * n_rows
                                  for M in bq_synth.DECODE_MS)

    def step(self) -> float:
        o = self.oracle
        t0 = time.perf_counter()
        for xb in self.xs:
            qa, sa = o.quant_act(xb, 128, o.INT8)
            o.gemm(qa, sa, self.qw, self.sw, 128, 128, o.INT8)
        return time.perf_counter() - t0


def host_info():
    """Host cores and CPU model of the machine the CPU baseline runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count() or 1, "cpu_model": model}


def _timed_reps(step, seconds_target):
    first = step()
    reps = max(1, int(seconds_target / max(first, 1e-3)))
    return reps, sum(step() for _ in range(reps))


def cpu_baseline(seconds_target=8.0):
    """The decode workload on the oracle: single-threaded (the plain build) and
    on all host cores (the OpenMP build, rows split over threads)."""
    import oracle
    hi = host_info()
    od = OracleDecode()
    res = {}
    for threads in (1, hi["nproc"]):
        used = oracle.use_threads(threads)
        try:
            reps, dt = _timed_reps(od.step, seconds_target if threads == 1 else seconds_target / 2)
        finally:
            oracle.use_threads(1)
        res[threads] = {"value": reps * od.bytes_per_step / dt / 1e9, "unit": "GB/s",
                        "cores": used, "kind": "oracle",
                        "sample": f"{reps} whole decode steps (M in 1,8,32,64; N = K = 4096) "
                                  f"after one untimed step; C oracle on {used} thread(s); "
                                  f"{dt:.1f} s"}
    one, allc = res[1], res[hi["nproc"]]
    return dict(allc, single_thread=one, host=hi)


def cpu_baseline_linear(cfg, seconds_target=3.0):
    """A bounded sample of a big linear workload on the oracle (all host
    cores): the activation quantisation and the GEMM of a sample of token
    rows against a sample of weight rows over the whole K (the rate, ops per
    second, depends on neither count).  The weight rows are quantised off the
    clock, as the method does offline."""
    import oracle
    hi = host_info()
    threads = oracle.use_threads(hi["nproc"])
    try:
        mx = cfg.dtype == bq_synth.MXFP8
        n_rows = 256 if cfg.dtype == bq_synth.INT8 else 128
        w = bq_synth.weights(cfg.N, cfg.K, cfg.w_std, cfg.seed).numpy()[:n_rows]
        if mx:
            qw, sw = oracle.mx_quant(w.astype(np.float64))
        else:
            qw, sw = oracle.quant_weight(w, cfg.block_n, cfg.block_k, cfg.dtype)
        del w
        rows = max(2 * threads, 8)
        xb = bq_synth.bf16_bits(bq_synth.activations(rows, cfg.K, cfg.seed, cfg.n_outliers,
                                                     cfg.outlier_scale))

        def step():
            t0 = time.perf_counter()
            if mx:
                qa, sa = oracle.mx_quant(oracle.bf16_to_f64(xb))
                oracle.mx_gemm(qa, sa, qw, sw)
            else:
                qa, sa = oracle.quant_act(xb, cfg.block_k, cfg.dtype)
                oracle.gemm(qa, sa, qw, sw, cfg.block_n, cfg.block_k, cfg.dtype)
            return time.perf_counter() - t0

        reps, dt = _timed_reps(step, seconds_target)
    finally:
        oracle.use_threads(1)
    ops = 2.0 * rows * n_rows * cfg.K
    return {"value": reps * ops / dt / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "sample": f"{reps} x ({rows} of {cfg.M} token rows: quantisation + GEMM against "
                      f"{n_rows} of the {cfg.N} weight rows, K = {cfg.K}); C oracle on "
                      f"{threads} threads; {dt:.1f} s"}


def cpu_baseline_moe(seconds_target=4.0):
    """The MoE layer on the oracle, stage by stage, on a bounded sample: the
    permutation of all T x top-k pairs, then for expert 0 and a sample of
    its rows the w13 GEMM, silu * up with its requantisation, the w2 GEMM,
    and the weighted combine of the sampled tokens.  Each stage's rate is
    reported in its own unit; `value` is the layer's ops per second over the
    two grouped GEMMs' sampled rows."""
    import oracle
    cfg = bq_synth.MOE
    hi = host_info()
    threads = oracle.use_threads(hi["nproc"])
    try:
        T, H, I, E, topk = cfg.T, cfg.H, cfg.I, cfg.E, cfg.topk
        logits = bq_synth.router_logits(T, E, cfg.seed).numpy()
        t0 = time.perf_counter()
        ids, tw = oracle.moe_route(logits, topk)
        t_route = time.perf_counter() - t0
        rows = max(2 * threads, 8)
        # a sample of the expert's intermediate width: I2 gate rows, the
        # matching up rows, and the w2 columns they feed
        I2 = 256
        w13 = bq_synth.weights(2 * I, H, cfg.w_std, cfg.seed).numpy()
        w13 = np.concatenate([w13[:I2], w13[I:I + I2]])
        q13, s13 = oracle.quant_weight_gate_up(w13, I2, 128, 128, cfg.dtype)
        del w13
        w2 = np.ascontiguousarray(bq_synth.weights(H, I, cfg.w_std, cfg.seed + 1).numpy()[:, :I2])
        q2, s2 = oracle.quant_weight(w2, 128, 128, cfg.dtype)
        del w2
        I = I2
        xb = bq_synth.bf16_bits(bq_synth.activations(rows, H, cfg.seed))
        stages = {}

        def timed(fn):
            t0 = time.perf_counter()
            out = fn()
            return out, time.perf_counter() - t0

        stages["route"] = {"value": T / t_route / 1e6, "unit": "M tokens/s"}
        (_, _, _), t_perm = timed(lambda: oracle.moe_permute(ids, E))
        stages["permute"] = {"value": T * topk / t_perm / 1e6, "unit": "M pairs/s"}
        tot_gemm, tot_t = 0.0, 0.0
        for _ in range(max(1, int(seconds_target / 2))):
            (qa, sa), t_q = timed(lambda: oracle.quant_act(xb, 128, cfg.dtype))
            y13, t_13 = timed(lambda: oracle.gemm(qa, sa, q13, s13, 128, 128, cfg.dtype, seam=I))
            y13b = oracle.bf16_from_f64(y13)
            h, t_s = timed(lambda: oracle.silu_mul(y13b, I))
            (qh, sh), t_hq = timed(lambda: oracle.quant_act(h, 128, cfg.dtype))
            y2, t_2 = timed(lambda: oracle.gemm(qh, sh, q2, s2, 128, 128, cfg.dtype))
            y2b = oracle.bf16_from_f64(y2)
            inv = np.arange(rows, dtype=np.int32)
            _, t_c = timed(lambda: oracle.moe_combine(y2b, inv, np.full((rows // topk, topk),
                                                                        0.5, np.float32)))
            tot_gemm += 2.0 * rows * (2 * I) * H + 2.0 * rows * H * I
            tot_t += t_q + t_13 + t_s + t_hq + t_2 + t_c
        stages["w13_gemm"] = {"value": 2.0 * rows * 2 * I * H / t_13 / 1e12, "unit": "TOPS"}
        stages["silu_requant"] = {"value": rows * I / (t_s + t_hq) / 1e6, "unit": "M elem/s"}
        stages["w2_gemm"] = {"value": 2.0 * rows * H * I / t_2 / 1e12, "unit": "TOPS"}
        stages["combine"] = {"value": rows * H / t_c / 1e6, "unit": "M elem/s"}
    finally:
        oracle.use_threads(1)
    return {"value": tot_gemm / tot_t / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle",
            "stages": stages,
            "sample": f"routing of all {T} tokens; permute of all {T * topk} pairs; expert 0 with {rows} token rows and "
                      f"{I} of its {cfg.I} intermediate columns through quant, w13, silu*up + "
                      f"requant, w2 and combine; C oracle on {threads} threads; {tot_t:.1f} s"}


def cpu_baseline_tiny():
    """The tiny workload in full on the oracle, single-threaded: latency."""
    import oracle
    cfg = bq_synth.TINY
    w = bq_synth.weights(cfg.N, cfg.K, cfg.w_std, cfg.seed).numpy()
    qw, sw = oracle.quant_weight(w, cfg.block_n, cfg.block_k, cfg.dtype)
    xb = bq_synth.bf16_bits(bq_synth.activations(cfg.M, cfg.K, cfg.seed, cfg.n_outliers,
                                                 cfg.outlier_scale))

    def step():
        t0 = time.perf_counter()
        qa, sa = oracle.quant_act(xb, cfg.block_k, cfg.dtype)
        oracle.gemm(qa, sa, qw, sw, cfg.block_n, cfg.block_k, cfg.dtype)
        return time.perf_counter() - t0

    reps, dt = _timed_reps(step, 0.5)
    return {"value": 1e6 * dt / reps, "unit": "us", "cores": 1, "kind": "oracle",
            "sample": f"{reps} whole tiny layers (quantisation + GEMM), single-threaded"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    od = OracleDecode()
    for _ in range(args.warmup):
        od.step()
    tot_t = sum(od.step() for _ in range(args.steps))
    v = args.steps * od.bytes_per_step / tot_t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": "decode_int8_n4096_k4096_m1-8-32-64",
                       "M": list(bq_synth.DECODE_MS), "N": 4096, "K": 4096,
                       "block": [128, 128], "world_size": world},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "each step: one whole decode step (M in 1,8,32,64; "
                                       "N = K = 4096), single-threaded C oracle"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="bq", choices=["bq", "reference"])
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "prefill", "fp8", "moe", "perchannel", "mxfp8"])
    ap.add_argument("--no-sub", action="store_true", help="skip the sub-workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline leg")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        return run_reference(args)

    import block_scaled_w8a8_b200 as bq
    bq.lib()                         # fails loudly if the CUDA library is missing
    dist = Dist(args.gpus)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        subs = {}
        if args.workload == "decode":
            head = bench_decode(args, dist, bq, peaks, stream)
        elif args.workload == "prefill":
            head = bench_linear_big(args, dist, bq, peaks, stream, bq_synth.PREFILL, 3)
        elif args.workload == "fp8":
            head = bench_linear_big(args, dist, bq, peaks, stream, bq_synth.FP8_LINEAR, 3)
        elif args.workload == "perchannel":
            head = bench_linear_big(args, dist, bq, peaks, stream, bq_synth.PER_CHANNEL, 3)
        elif args.workload == "mxfp8":
            head = bench_linear_big(args, dist, bq, peaks, stream, bq_synth.MX_LINEAR, 3)
        else:
            head = bench_moe(args, dist, bq, peaks, stream)
        if not args.no_sub:
            for name in ("prefill", "fp8", "moe", "perchannel", "mxfp8"):
                if name == args.workload:
                    continue
                torch.cuda.empty_cache()
                if name == "prefill":
                    subs[name] = bench_linear_big(args, dist, bq, peaks, stream,
                                                  bq_synth.PREFILL, 3)
                elif name == "fp8":
                    subs[name] = bench_linear_big(args, dist, bq, peaks, stream,
                                                  bq_synth.FP8_LINEAR, 3)
                elif name == "perchannel":
                    subs[name] = bench_linear_big(args, dist, bq, peaks, stream,
                                                  bq_synth.PER_CHANNEL, 3)
                elif name == "mxfp8":
                    subs[name] = bench_linear_big(args, dist, bq, peaks, stream,
                                                  bq_synth.MX_LINEAR, 3)
                else:
                    subs[name] = bench_moe(args, dist, bq, peaks, stream)
        if not args.no_sub:
            torch.cuda.empty_cache()
            subs["tiny"] = bench_tiny(args, dist, bq, stream)
    bq.check_device_status()
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
        cpu = cpu_baseline()
        # the other workloads' oracle baselines (bounded samples, all host cores)
        big = {"prefill": bq_synth.PREFILL, "fp8": bq_synth.FP8_LINEAR,
               "perchannel": bq_synth.PER_CHANNEL, "mxfp8": bq_synth.MX_LINEAR}
        for name, sub in subs.items():
            if name in big:
                sub["cpu_baseline"] = cpu_baseline_linear(big[name])
            elif name == "moe":
                sub["cpu_baseline"] = cpu_baseline_moe()
            elif name == "tiny":
                sub["cpu_baseline"] = cpu_baseline_tiny()
    if dist.rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": head["unit"],
                "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
                "data": "synthetic (seeded Gaussian activations with outlier channels; "
                        "Gaussian weights block-quantised on the GPU)",
                "config": head["config"], "roofline": head["roofline"],
                "peaks_source": peak_src, "clocks": head["clocks"],
                "e2e": head.get("e2e"), "gpu_launches": head.get("gpu_launches"),
                "cpu_baseline": cpu, "workloads": subs}
        for k in ("quant_us_per_launch", "gemm_path"):
            if k in head:
                line[k] = head[k]
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
