#!/usr/bin/env python3
"""Benchmark of the 4-bit NF4 path on a Llama-7B-shaped stack.

One step = one pass of the whole hot path over the 224 linears of a 32-layer
Llama-7B-shaped stack (q/k/v/o 4096x4096, gate/up 11008x4096, down
4096x11008; bf16 weights ~ N(0, 0.02^2) resident in HBM).  For every linear,
in layer order:
  1. quantize the bf16 weight to NF4, blocksize 64, with double quantization;
  2. dequantize the packed weight back to bf16;
  3. prefill GEMM: X bf16 [2048, K] ~ N(0, 1) times the 4-bit weight;
  4. decode GEMV: x bf16 [1, K] ~ N(0, 1) times the 4-bit weight.
``value`` is the stack's packed 4-bit weight bytes per step divided by the
step time (GB/s), summed over ranks; per-row throughputs and roofline
fractions are reported under ``rows``.  Inputs (12.95 GB of bf16 weights) are
larger than L2, so no flush is needed between steps.

Multi-GPU: every rank runs its own replica of the stack (independent
problems, no collective on the data path); ``value`` counts all ranks.

``--impl reference`` times the CPU oracle (single thread) on a bounded sample
of the same workload instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "4-bit GEMV weight-GB/s & GEMM TFLOPS; quant/dequant GB/s; % of roofline"
WORKLOAD = ("llama7b-shaped stack, 32 layers x 7 linears (224): per linear "
            "quantize bf16->NF4 (bs 64, double quant) + dequantize->bf16 + "
            "prefill GEMM M=2048 + decode GEMV B=1")
GEMM_M = 2048
BS = 64

# DRAM bytes (read + write) per GEMM launch, averaged over the seven GEMMs of
# one layer, from one ncu capture (profiles/gemm4_dram_traffic_llama7b_layer.md).
# Reported only while the GEMM kernel's sources are the ones captured.
GEMM_TRAFFIC_BYTES = 37468818
GEMM_TRAFFIC_SOURCES = ("bit_blockwise_weight_nf4_b200/csrc/gemm.cu",
                        "bit_blockwise_weight_nf4_b200/csrc/common.cuh",
                        "bit_blockwise_weight_nf4_b200/csrc/sm100.cuh")
GEMM_TRAFFIC_SHA256 = "82bff8b020a3a34fcf3c9d310104139b8333349765e4ae10d819569003c77780"


def gemm_traffic():
    """Measured DRAM bytes per GEMM launch, or None when the kernel sources
    changed since the capture."""
    import hashlib
    h = hashlib.sha256()
    try:
        for p in GEMM_TRAFFIC_SOURCES:
            with open(os.path.join(ROOT, p), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return GEMM_TRAFFIC_BYTES if h.hexdigest() == GEMM_TRAFFIC_SHA256 else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32,
                    help="decoder layers in the stack (32 = the Llama-7B workload)")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one call at a time instead of "
                         "replaying them as one CUDA graph")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------- distributed
def dist_init():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        self.dev = device_index

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [c.strip() for c in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx.append(float(p[2]))
                except ValueError:
                    continue
                for name, val in zip(names, p[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


# ------------------------------------------------------------ workload
def stack_linears(n_layers):
    import synth
    return synth.llama7b_stack(n_layers)


def packed_bytes(N, K):
    nb = N * K // BS
    return N * K // 2 + nb + 4 * -(-nb // 256) + 4


def build_stack(n_layers, device):
    """Resident bf16 weights, their quantization states and the activations."""
    import torch
    import synth
    import bit_blockwise_weight_nf4_b200 as bnb4
    lins = stack_linears(n_layers)
    W, states = [], []
    for layer, lin in lins:
        idx = [l.name for l in synth.llama7b_layer()].index(lin.name)
        w = synth.weight_bf16(lin.N, lin.K, seed=synth.stack_weight_seed(layer, idx),
                              device=device)
        W.append(w.view(-1))
        states.append(bnb4.QuantState(lin.N * lin.K, BS, bnb4.NF4, True, device))
    X = {K: synth.activations_bf16(GEMM_M, K, seed=11 + K, device=device)
         for K in (synth.HIDDEN, synth.FFN)}
    x = {K: synth.activations_bf16(1, K, seed=13 + K, device=device)
         for K in (synth.HIDDEN, synth.FFN)}
    return lins, W, states, X, x


class Step:
    """All launches of one step on the current stream, with an event before
    and after every row so row times are measured inside the timed region."""

    ROWS = ("quantize", "dequantize", "gemm", "gemv")

    def __init__(self, lins, W, states, X, x, device):
        import torch
        import bit_blockwise_weight_nf4_b200 as bnb4
        self.bnb4 = bnb4
        self.lins, self.W, self.states, self.X, self.x = lins, W, states, X, x
        maxnk = max(l.N * l.K for _, l in lins)
        maxn = max(l.N for _, l in lins)
        self.deq = torch.empty(maxnk, dtype=torch.bfloat16, device=device)
        self.Y = torch.empty(GEMM_M * maxn, dtype=torch.bfloat16, device=device)
        self.y = [torch.empty(1, l.N, dtype=torch.bfloat16, device=device)
                  for _, l in lins]
        self.ws = bnb4.workspace_for(states[0])
        self.launches_per_step = 5 * len(lins)  # quantize is 2 kernels

    def new_events(self):
        """Timing events of one step; `external` makes a record captured in a
        CUDA graph a timed event-record node."""
        import torch
        return [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)]
                for _ in self.lins]

    def run(self, events=None):
        b = self.bnb4
        stream = b._stream()
        timed = events is not None
        for i, (_, lin) in enumerate(self.lins):
            st = self.states[i]
            ev = events[i] if timed else None
            if timed:
                ev[0].record()
            rc = b.bnb_quantize_4bit(self.W[i].data_ptr(), b.BF16, st.cstruct(),
                                     self.ws.data_ptr(), self.ws.numel(), stream)
            if timed:
                ev[1].record()
            rc |= b.bnb_dequantize_4bit(st.cstruct(), self.deq.data_ptr(), b.BF16, stream)
            if timed:
                ev[2].record()
            rc |= b.bnb_gemm_4bit(self.X[lin.K].data_ptr(), GEMM_M, lin.K, st.cstruct(),
                                  lin.N, self.Y.data_ptr(), stream)
            if timed:
                ev[3].record()
            rc |= b.bnb_gemv_4bit(self.x[lin.K].data_ptr(), 1, lin.K, st.cstruct(),
                                  lin.N, self.y[i].data_ptr(), stream)
            if timed:
                ev[4].record()
            if rc != 0:
                raise RuntimeError("launch failed on linear %d" % i)

    def row_times(self, events, t=None):
        """Seconds spent per row over the steps of `events` (after a
        synchronize), added to t."""
        t = t if t is not None else dict.fromkeys(self.ROWS, 0.0)
        for ev in events:
            for j, r in enumerate(self.ROWS):
                t[r] += ev[j].elapsed_time(ev[j + 1]) * 1e-3
        return t


def row_work(lins):
    """Algorithmic bytes / flops of one step per row."""
    q = dq = gv = gm = 0
    wb = 0
    for _, l in lins:
        n = l.N * l.K
        nb = n // BS
        ng = -(-nb // 256)
        state = n // 2 + nb + 4 * ng + 4
        q += 2 * n + state + 4 * nb            # read bf16, write state + fp32 absmax
        dq += state + 2 * n                   # read state, write bf16
        gv += state + 2 * l.K + 2 * l.N       # read state + x, write y
        gm += 2 * GEMM_M * l.N * l.K
        wb += n // 2
    return {"quantize": q, "dequantize": dq, "gemv": gv, "gemm": gm, "weight_bytes": wb}


# ------------------------------------------------------------ CPU oracle
def oracle_sample(budget_layers=1):
    """Time the single-threaded CPU oracle on layer 0's seven linears:
    quantize (bs 64, double quant) + dequantize to bf16 + GEMV B=1 in full,
    GEMM on 8 sampled rows of X extrapolated to 2048 rows.  Returns the
    4-bit weight GB/s of the full path and a description."""
    import numpy as np
    import oracle
    import synth
    lins = stack_linears(budget_layers)
    t_q = t_dq = t_gv = t_gm = 0.0
    wbytes = 0
    rows = 8
    for layer, lin in lins:
        idx = [l.name for l in synth.llama7b_layer()].index(lin.name)
        Wb = synth.bf16_bits(synth.weight_bf16(
            lin.N, lin.K, seed=synth.stack_weight_seed(layer, idx)).view(-1))
        t0 = time.perf_counter()
        st = oracle.quantize(Wb, BS, oracle.NF4, True)
        t1 = time.perf_counter()
        Wh = oracle.dequantize(st, oracle.BF16).reshape(lin.N, lin.K)
        t2 = time.perf_counter()
        x = synth.bf16_bits(synth.activations_bf16(1, lin.K, seed=13 + lin.K))
        oracle.linear_ref(x, Wh)
        t3 = time.perf_counter()
        X = synth.bf16_bits(synth.activations_bf16(rows, lin.K, seed=11 + lin.K))
        oracle.linear_ref(X, Wh)
        t4 = time.perf_counter()
        t_q += t1 - t0
        t_dq += t2 - t1
        t_gv += t3 - t2
        t_gm += (t4 - t3) * GEMM_M / rows
        wbytes += lin.N * lin.K // 2
    total = t_q + t_dq + t_gv + t_gm
    return {
        "value": wbytes / total / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
        "sample": ("layer 0 of the stack (7 linears, %.3f GB packed): quantize + "
                   "dequantize + GEMV B=1 timed in full, GEMM timed on %d of 2048 "
                   "rows and extrapolated; measured %.1f s, extrapolated %.1f s"
                   % (wbytes / 1e9, rows, t_q + t_dq + t_gv + t_gm * rows / GEMM_M,
                      total)),
        "rows_s": {"quantize": t_q, "dequantize": t_dq, "gemv": t_gv,
                   "gemm_extrapolated": t_gm},
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    samples = []
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up effects worth timing separately
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        samples.append(oracle_sample())
    wall = time.perf_counter() - t0
    v = statistics.median(s["value"] for s in samples)
    cb = dict(samples[0], value=v)
    cb.pop("rows_s", None)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32", "data": "synthetic",
        "config": {"workload": WORKLOAD + " (CPU oracle, bounded sample per step)"},
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import bit_blockwise_weight_nf4_b200 as bnb4
    bnb4.load()
    rank, world, local = dist_init()
    dev = torch.device("cuda", local)
    hbm, tf_burst, tf_sus, peak_src = load_peaks()

    lins, W, states, X, x = build_stack(args.layers, dev)
    step = Step(lins, W, states, X, x, dev)
    work = row_work(lins)
    torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step.run()
    torch.cuda.synchronize()
    if bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) != 0:
        raise RuntimeError("device error word set during warm-up")

    events = [step.new_events() for _ in range(args.steps)]
    graph = None
    if not args.eager:
        # the K timed steps (every launch and the per-row events) as one CUDA
        # graph: the same kernels on the same buffers, without per-call host
        # launch overhead between them
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(graph, stream=cap):
            for k in range(args.steps):
                step.run(events[k])
        torch.cuda.current_stream().wait_stream(cap)
        graph.replay()  # untimed: the graph's first launch
        torch.cuda.synchronize()
    clocks = ClockSampler(physical_gpu_index(local))
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    if graph is not None:
        graph.replay()
    else:
        for k in range(args.steps):
            step.run(events[k])
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    elapsed = t_start.elapsed_time(t_end) * 1e-3
    clk = clocks.stop()
    rows_t = None
    for ev in events:
        rows_t = step.row_times(ev, rows_t)
    rows_t = {k: v / args.steps for k, v in rows_t.items()}  # per step
    elapsed_max = max_over_ranks(elapsed, world)
    status = bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream)
    if status != 0:
        raise RuntimeError("device error word set: %s" % bnb4.bnb4_strerror(status))

    value = world * work["weight_bytes"] * args.steps / elapsed_max / 1e9
    n_gemm = len(lins)
    gemm_tflops = work["gemm"] / rows_t["gemm"] / 1e12
    rows = {
        "quantize": {"GB/s": work["quantize"] / rows_t["quantize"] / 1e9,
                     "frac_hbm": work["quantize"] / rows_t["quantize"] / 1e9 / hbm,
                     "ms": rows_t["quantize"] * 1e3},
        "dequantize": {"GB/s": work["dequantize"] / rows_t["dequantize"] / 1e9,
                       "frac_hbm": work["dequantize"] / rows_t["dequantize"] / 1e9 / hbm,
                       "ms": rows_t["dequantize"] * 1e3},
        "gemv_b1": {"weight_GB/s": work["weight_bytes"] / rows_t["gemv"] / 1e9,
                    "GB/s": work["gemv"] / rows_t["gemv"] / 1e9,
                    "frac_hbm": work["gemv"] / rows_t["gemv"] / 1e9 / hbm,
                    "ms": rows_t["gemv"] * 1e3},
        "gemm_m2048": {"TFLOP/s": gemm_tflops, "frac_bf16_sustained": gemm_tflops / tf_sus,
                       "frac_bf16_burst": gemm_tflops / tf_burst,
                       "ms": rows_t["gemm"] * 1e3},
    }
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": elapsed_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": args.layers, "linears": len(lins),
                   "weight_format": "nf4, blocksize 64, double quant",
                   "packed_weight_bytes": work["weight_bytes"],
                   "gemm_m": GEMM_M, "gemv_batch": 1,
                   "l2": "inputs larger than L2 (%.2f GB of bf16 weights), no flush"
                         % (sum(w.numel() * 2 for w in W) / 1e9),
                   "parallelism": "replicas x%d" % world,
                   "launch": "eager, one call per kernel" if args.eager
                             else "the timed steps replayed as one CUDA graph"},
        "roofline": {"bound": "tensor", "kernel": "gemm4 (fused dequant + tcgen05)",
                     "achieved": gemm_tflops, "peak": tf_sus, "unit": "TFLOP/s",
                     "frac": gemm_tflops / tf_sus, "traffic": gemm_traffic(),
                     "traffic_unit": "bytes per launch (dram read + write, ncu)",
                     "peak_source": "%s bf16 sustained (kernel inside a long step)"
                                    % peak_src,
                     "per_launch": "2*2048*N*K flops; %d launches per step" % n_gemm},
        "rows": rows,
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": clk,
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": tf_burst,
                  "bf16_tflops_sustained": tf_sus, "source": peak_src},
    }
    del graph
    if not args.no_e2e:
        line["e2e"] = run_e2e(step, W, X, x, lins, world, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample()
        cb.pop("rows_s", None)
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(step, W, X, x, lins, world, args):
    """Same step through the C ABI with the inputs in pinned HOST memory:
    every step copies the bf16 weights and activations host->device and reads
    the decode outputs back, all inside the timed region."""
    import torch
    host_W = [w.cpu().pin_memory() for w in W]
    host_X = {k: v.cpu().pin_memory() for k, v in X.items()}
    host_x = {k: v.cpu().pin_memory() for k, v in x.items()}
    host_y = [y.cpu().pin_memory() for y in step.y]
    h2d = sum(t.numel() * 2 for t in host_W) + sum(t.numel() * 2 for t in host_X.values()) \
        + sum(t.numel() * 2 for t in host_x.values())
    d2h = sum(t.numel() * 2 for t in host_y)
    k_e2e = max(1, min(args.steps, 3))

    def one():
        for d, h in zip(W, host_W):
            d.copy_(h, non_blocking=True)
        for k in X:
            X[k].copy_(host_X[k], non_blocking=True)
            x[k].copy_(host_x[k], non_blocking=True)
        step.run()
        for h, d in zip(host_y, step.y):
            h.copy_(d, non_blocking=True)

    one()
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(k_e2e):
        one()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    t = max_over_ranks(a.elapsed_time(b) * 1e-3, world)
    wbytes = sum(l.N * l.K // 2 for _, l in lins)
    return {"value": world * wbytes * k_e2e / t / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": k_e2e, "ms_per_step": t / k_e2e * 1e3}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
