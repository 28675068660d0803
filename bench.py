#!/usr/bin/env python3
"""Benchmark of the 4-bit NF4 / FP4 path: the five workloads of the method's
brief, each timed in isolation, inside one step.

One step runs, in this order, every row below; each row is a run of
back-to-back calls of one kind on buffers that no other row touches, so a
call never finds its inputs in L2 (every row's working set, and the 3.34 GB
stack pass between two steps, evicts the others):

  cfg1  NF4 round trip of an fp32 vector of 2^20 elements ~ N(0, 0.02^2)
        (seed 0), blocksize 64, double quant: quantize, then dequantize to
        fp32 (8 calls each, over 8 copies);
  cfg2  bf16 4096 x 4096 ~ N(0, 0.02^2) with 0.1% outliers x20, blocksize
        64, double quant: quantize and dequantize to bf16, NF4 and FP4
        (4 calls each, over 4 copies);
  cfg3  decode GEMV, bf16 x [B, K] ~ N(0, 1), B in {1, 8}, NF4 weights
        11008 x 4096 and 4096 x 11008 (4 calls each, over 4 weights);
  cfg4  prefill GEMM, bf16 X [2048, K] ~ N(0, 1), the three Llama-7B shapes,
        NF4 blocksize 64, NF4 blocksize 128 and FP4 blocksize 64;
  cfg5  the 32-layer Llama-7B-shaped stack (q/k/v/o 4096x4096, gate/up
        11008x4096, down 4096x11008; 6.48 B weights NF4-quantized with
        double quant at set-up): batch-1 GEMV through all 224 linears, as a
        decoder launches them (per layer: q/k/v in one grouped launch, o,
        gate/up in one grouped launch, down: 128 launches), and for
        comparison as 224 single calls and as two grouped calls (one per K).

``value`` is configuration 5's figure: the bytes of the stack's 4-bit
weights (codes, 8-bit scales and their scales, 3.341 GB) streamed per pass
of the per-layer launches, divided by the pass time (GB/s), summed over
ranks.  ``rows`` gives every
row's time per call, throughput and fraction of the measured peak; the
stack's quantization (set-up of configuration 5) is timed once as its own
row.  The timed steps replay as one CUDA graph with CUDA events around every
row.

Multi-GPU: every rank runs its own replica (independent problems, no
collective on the data path); ``value`` counts all ranks.

``--impl reference`` times the CPU oracle (single thread) on a bounded
sample of configuration 5 instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "4-bit GEMV weight-GB/s & GEMM TFLOPS; quant/dequant GB/s; % of roofline"
WORKLOAD = ("five configurations per step, each row isolated on its own buffers: "
            "cfg1 NF4 round trip fp32 2^20; cfg2 NF4/FP4 quantize+dequantize bf16 "
            "4096x4096 with outliers; cfg3 GEMV B=1,8 on 11008x4096 and 4096x11008; "
            "cfg4 GEMM M=2048 on the three Llama-7B shapes, NF4 bs64/bs128, FP4; "
            "cfg5 batch-1 GEMV through the 224 linears of a 32-layer "
            "Llama-7B-shaped NF4 stack, per-layer launches (value); plus the "
            "small-batch linear (16 and 64 token rows) on the three Llama-7B shapes")
GEMM_M = 2048
BS = 64
ROUNDTRIP_COPIES = 8
MATRIX_COPIES = 4
GEMV_WEIGHTS = 4
SMALL_BATCH_ROWS = (16, 64)  # token rows of the small-batch linear rows

# DRAM bytes (read + write) per launch of a kernel family, from one ncu
# capture each, with the sources hashed at capture time: a figure is
# reported only while the kernel's sources are the ones that were captured.
# integer-ALU operations per weight of the decode kernel's exact lookup: per
# 8 weights 16 byte permutes and 2 selector masks, and per 64-weight block
# table 8 permutes and 8 bf16 packs -- 2.25 + 0.25
ALU_OPS_PER_WEIGHT = 2.5

TRAFFIC = {
    # decode: DRAM bytes (read + write) over algorithmic bytes of cold
    # launches of both decode kernels -- the one-CTA-per-16-rows one on 11008
    # x 4096 (23.30 MB read, none written / 23.29 MB) and the persistent one
    # on the six K = 4096 linears of a layer (81.26 MB read + 2.09 MB written
    # / 81.27 MB); the family's traffic per launch is that ratio times its
    # algorithmic bytes per launch
    "gemv": {"ratio": (23.304448 + 0.0 + 81.260544 + 2.088448) / (23.290112 + 81.265152),
             "launch": "cold captures of both decode kernels (11008 x 4096 single; the "
                       "six K = 4096 linears of a layer in one persistent launch), scaled "
                       "by the algorithmic bytes per launch of the family",
             "sources": ("bit_blockwise_weight_nf4_b200/csrc/gemv.cu",
                         "bit_blockwise_weight_nf4_b200/csrc/gemv_direct.cu",
                         "bit_blockwise_weight_nf4_b200/csrc/l2warm.cuh",
                         "bit_blockwise_weight_nf4_b200/csrc/lut.cuh",
                         "bit_blockwise_weight_nf4_b200/csrc/common.cuh",
                         "bit_blockwise_weight_nf4_b200/csrc/sm100.cuh"),
             "sha256": "86e2dfca955d480d8ef1d629b19bd09c6d590179dbca7cb57a9c9e00583d0958"},
    "gemm": {"bytes": 46406315,
             "launch": "one prefill GEMM launch (M = 2048), averaged over the three "
                       "Llama-7B shapes",
             "sources": ("bit_blockwise_weight_nf4_b200/csrc/gemm.cu",
                         "bit_blockwise_weight_nf4_b200/csrc/common.cuh",
                         "bit_blockwise_weight_nf4_b200/csrc/sm100.cuh"),
             "sha256": "a4d455f160c1d22171a989b30e5f54ed374eecb17d3cbdd84bbbdd515bb19baf"},
}


def traffic_of(family):
    """Measured DRAM bytes per launch of `family`, or None when unmeasured or
    when its sources changed since the capture."""
    t = TRAFFIC.get(family)
    if t is None:
        return None
    h = hashlib.sha256()
    try:
        for p in t["sources"]:
            with open(os.path.join(ROOT, p), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return t if h.hexdigest() == t["sha256"] else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=32,
                    help="decoder layers of the configuration-5 stack (32 = Llama-7B)")
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
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]),
                "source": "measured"}
    except (OSError, KeyError, ValueError, TypeError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


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

    def __init__(self, device_index, interval_ms=50):
        self.proc = None
        self.path = None
        self.dev = device_index
        self.interval = interval_ms
        self.skip = 0  # lines written before the timed region

    def _lines(self):
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except OSError:
            return 0

    def ready(self, timeout_s=5.0):
        """Wait until the sampler writes (nvidia-smi can take a second to
        start), then mark where the timed region's samples begin."""
        if self.proc is None:
            return
        t0 = time.time()
        while self._lines() == 0 and time.time() - t0 < timeout_s and self.proc.poll() is None:
            time.sleep(0.02)
        self.skip = self._lines()

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", str(self.interval)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        with open(self.path) as f:
            for n, line in enumerate(f):
                if n < self.skip:
                    continue
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


def host_description():
    model = platform.processor() or "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


# ------------------------------------------------------- algorithmic work
def state_bytes(n, bs=BS, dq=True):
    """Bytes of a quantization state of n elements: packed codes, and the
    8-bit scales with their fp32 group scales and offset (double quant) or
    the fp32 absmax."""
    nb = -(-n // bs)
    if dq:
        return (n + 1) // 2 + nb + 4 * -(-nb // 256) + 4
    return (n + 1) // 2 + 4 * nb


def quantize_bytes(n, elt, bs=BS):
    """Algorithmic bytes of one quantize call: read the input, write the state."""
    return elt * n + state_bytes(n, bs)


def dequantize_bytes(n, elt_out, bs=BS):
    return state_bytes(n, bs) + elt_out * n


def gemv_bytes(N, K, B, bs=BS):
    return state_bytes(N * K, bs) + 2 * B * K + 2 * B * N


# ---------------------------------------------------------------- rows
class Call:
    """One C-ABI call: the entry point, its arguments (raw pointers) and
    the tensors those pointers point into, held for as long as the call may
    run; the stream is torch's current one at call time (the capture stream
    while a graph is being captured).  `launches`: how many times the call
    launches its row's kernels (a grouped decode call launches once per 32
    linears)."""

    def __init__(self, fn, *args, keep=(), launches=1):
        self.fn, self.args, self.keep, self.launches = fn, args, keep, launches

    def __call__(self):
        import bit_blockwise_weight_nf4_b200 as b
        return self.fn(*self.args, b._stream())


class Row:
    """A timed row: `calls` (C-ABI launches, each a zero-argument callable
    returning the status) run back to back on the current stream."""

    def __init__(self, name, cfg, family, bound, work, calls, kernels_per_call, **extra):
        self.name, self.cfg, self.family, self.bound = name, cfg, family, bound
        self.work = work                      # algorithmic bytes or flops per call
        self.calls = calls
        self.kpc = kernels_per_call
        self.extra = extra

    def run(self):
        for c in self.calls:
            rc = c()
            if rc != 0:
                raise RuntimeError("%s: launch failed with status %d" % (self.name, rc))


def build_rows(dev, n_layers):
    """Every row's inputs, resident on `dev`, and the calls that time it.
    Returns (rows, stack) where stack describes configuration 5."""
    import torch
    import synth
    import bit_blockwise_weight_nf4_b200 as b
    S = lambda: b._stream()
    rows = []

    def fresh(n, bs, qt):
        return b.QuantState(n, bs, qt, True, dev)

    # cfg1: NF4 round trip of a 2^20-element fp32 vector
    n1 = synth.ROUNDTRIP_N
    x1 = synth.normal_f32((n1,), seed=0, std=synth.WEIGHT_STD, device=dev)
    xs1 = [x1.clone() for _ in range(ROUNDTRIP_COPIES)]
    q1 = [fresh(n1, BS, b.NF4) for _ in xs1]
    d1 = [b.quantize_4bit(x, BS, b.NF4, True) for x in xs1]   # read by the dequantize row
    o1 = [torch.empty(n1, dtype=torch.float32, device=dev) for _ in xs1]
    ws = b.workspace_for(q1[0])
    wsn = ws.numel()

    def qcall(x, st, dt):
        return Call(b.bnb_quantize_4bit, x.data_ptr(), dt, st.cstruct(), ws.data_ptr(), wsn,
                    keep=(x, st, ws))

    def dcall(st, out, dt):
        return Call(b.bnb_dequantize_4bit, st.cstruct(), out.data_ptr(), dt, keep=(st, out))

    rows.append(Row("cfg1_quantize", "cfg1", "quantize", "hbm", quantize_bytes(n1, 4),
                    [qcall(x, s, b.F32) for x, s in zip(xs1, q1)], 2))
    rows.append(Row("cfg1_dequantize", "cfg1", "dequantize", "hbm", dequantize_bytes(n1, 4),
                    [dcall(s, o, b.F32) for s, o in zip(d1, o1)], 1))

    # cfg2: bf16 4096 x 4096 with outliers, NF4 and FP4
    R, C = synth.MATRIX_4096
    n2 = R * C
    w2 = synth.weight_bf16(R, C, seed=2, outlier_frac=synth.OUTLIER_FRAC, device=dev).view(-1)
    for qname, qt in (("nf4", b.NF4), ("fp4", b.FP4)):
        xs = [w2.clone() for _ in range(MATRIX_COPIES)]
        qs = [fresh(n2, BS, qt) for _ in xs]
        ds = [b.quantize_4bit(w2, BS, qt, True) for _ in xs]
        os_ = [torch.empty(n2, dtype=torch.bfloat16, device=dev) for _ in xs]
        rows.append(Row("cfg2_quantize_" + qname, "cfg2", "quantize", "hbm",
                        quantize_bytes(n2, 2), [qcall(x, s, b.BF16) for x, s in zip(xs, qs)], 2))
        rows.append(Row("cfg2_dequantize_" + qname, "cfg2", "dequantize", "hbm",
                        dequantize_bytes(n2, 2), [dcall(s, o, b.BF16) for s, o in zip(ds, os_)],
                        1))
    del w2

    # cfg3: decode GEMV
    def gemv_call(x, st, N, y):
        B, K = x.shape
        return Call(b.bnb_gemv_4bit, x.data_ptr(), B, K, st.cstruct(), N, y.data_ptr(),
                    keep=(x, st, y))

    for N, K in synth.GEMV_SHAPES:
        for Bt in synth.GEMV_BATCHES:
            x = synth.activations_bf16(Bt, K, seed=1, device=dev)
            sts = []
            for i in range(GEMV_WEIGHTS):
                w = synth.weight_bf16(N, K, seed=300 + 10 * Bt + i, device=dev)
                sts.append(b.quantize_4bit(w.view(-1), BS, b.NF4, True))
                del w
            y = torch.empty(Bt, N, dtype=torch.bfloat16, device=dev)
            rows.append(Row("cfg3_gemv_b%d_%dx%d" % (Bt, N, K), "cfg3", "gemv", "hbm",
                            gemv_bytes(N, K, Bt), [gemv_call(x, s, N, y) for s in sts], 1,
                            weight_bytes=N * K // 2))

    # the small-batch linear (16 and 64 token rows) on the three Llama-7B
    # shapes, through bnb_gemm_4bit: 16 rows run the decode kernel's 16-row
    # form, 64 the small-batch tcgen05 kernel
    for M in SMALL_BATCH_ROWS:
        for N, K in synth.GEMM_SHAPES:
            X = synth.activations_bf16(M, K, seed=2, device=dev)
            sts = []
            for i in range(GEMV_WEIGHTS):
                w = synth.weight_bf16(N, K, seed=500 + M + 10 * i + N // 1024, device=dev)
                sts.append(b.quantize_4bit(w.view(-1), BS, b.NF4, True))
                del w
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            rows.append(Row("f1_linear_m%d_%dx%d" % (M, N, K), "f1", "small", "hbm",
                            gemv_bytes(N, K, M),
                            [Call(b.bnb_gemm_4bit, X.data_ptr(), M, K, s.cstruct(), N,
                                  Y.data_ptr(), keep=(X, s, Y)) for s in sts], 1,
                            weight_bytes=N * K // 2))

    # cfg4: prefill GEMM
    def gemm_call(X, st, N, Y):
        M, K = X.shape
        return Call(b.bnb_gemm_4bit, X.data_ptr(), M, K, st.cstruct(), N, Y.data_ptr(),
                    keep=(X, st, Y))

    Xs = {K: synth.activations_bf16(GEMM_M, K, seed=1, device=dev)
          for K in (synth.HIDDEN, synth.FFN)}
    for vname, bs, qt in (("nf4_bs64", 64, b.NF4), ("nf4_bs128", 128, b.NF4),
                          ("fp4_bs64", 64, b.FP4)):
        for N, K in synth.GEMM_SHAPES:
            w = synth.weight_bf16(N, K, seed=400 + N + K, device=dev)
            st = b.quantize_4bit(w.view(-1), bs, qt, True)
            del w
            Y = torch.empty(GEMM_M, N, dtype=torch.bfloat16, device=dev)
            rows.append(Row("cfg4_gemm_%s_%dx%d" % (vname, N, K), "cfg4", "gemm", "tensor",
                            2 * GEMM_M * N * K, [gemm_call(Xs[K], st, N, Y)], 1))

    # cfg5: the Llama-7B-shaped stack, quantized at set-up (timed once)
    lins = synth.llama7b_stack(n_layers)
    names = [l.name for l in synth.llama7b_layer()]
    states = []
    qtime = 0.0
    qwork = 0
    for layer, lin in lins:
        w = synth.weight_bf16(lin.N, lin.K, seed=synth.stack_weight_seed(
            layer, names.index(lin.name)), device=dev).view(-1)
        st = fresh(lin.N * lin.K, BS, b.NF4)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        rc = b.bnb_quantize_4bit(w.data_ptr(), b.BF16, st.cstruct(), ws.data_ptr(), wsn, S())
        e1.record()
        if rc != 0:
            raise RuntimeError("stack quantize failed with status %d" % rc)
        torch.cuda.synchronize()
        qtime += e0.elapsed_time(e1) * 1e-3
        qwork += quantize_bytes(lin.N * lin.K, 2)
        states.append(st)
        del w
    xk = {K: synth.activations_bf16(1, K, seed=1, device=dev) for K in (synth.HIDDEN, synth.FFN)}
    # every linear's output is a view of one buffer, so a pass's results
    # read back to the host in one copy
    y_all = torch.empty(sum(lin.N for _, lin in lins), dtype=torch.bfloat16, device=dev)
    ys, o = [], 0
    for _, lin in lins:
        ys.append(y_all[o:o + lin.N].view(1, lin.N))
        o += lin.N
    stack_state = sum(state_bytes(lin.N * lin.K) for _, lin in lins)
    pass_bytes = sum(gemv_bytes(lin.N, lin.K, 1) for _, lin in lins)
    pass_weights = sum(lin.N * lin.K // 2 for _, lin in lins)

    def group_call(idx):
        probs = (b.GemvProblem * len(idx))()
        for j, i in enumerate(idx):
            lin = lins[i][1]
            probs[j] = b.GemvProblem(xk[lin.K].data_ptr(), states[i].cstruct(), lin.K, lin.N,
                                     None, ys[i].data_ptr())
        return Call(b.bnb_gemv_4bit_grouped, probs, 1, b.BF16,
                    keep=[states[i] for i in idx] + [ys[i] for i in idx] + list(xk.values()),
                    launches=(len(idx) + 31) // 32)

    # the decoder's natural launches per layer: q/k/v (one input), o,
    # gate/up (one input), down
    layer_groups = []
    for L in range(n_layers):
        base = 7 * L
        layer_groups += [[base, base + 1, base + 2], [base + 3], [base + 4, base + 5],
                         [base + 6]]

    def pass_row(name, calls):
        return Row(name, "cfg5", "gemv", "hbm", pass_bytes / len(calls), calls, 1,
                   weight_bytes=pass_weights / len(calls))

    stack_row = pass_row("cfg5_gemv_stack_layer_groups", [group_call(g) for g in layer_groups])
    rows.append(stack_row)
    rows.append(pass_row("cfg5_gemv_stack_single_calls",
                         [gemv_call(xk[lin.K], st, lin.N, y)
                          for (_, lin), st, y in zip(lins, states, ys)]))
    # the whole list in as few calls as the one-K rule allows: every linear
    # with K = 4096 in one call, every K = 11008 one in another
    by_k = {}
    for i, (_, lin) in enumerate(lins):
        by_k.setdefault(lin.K, []).append(i)
    rows.append(pass_row("cfg5_gemv_stack_by_k", [group_call(ix) for ix in by_k.values()]))
    stack = {"lins": lins, "states": states, "x": xk, "y": ys, "y_all": y_all,
             "state_bytes": stack_state,
             "row": stack_row, "groups": layer_groups, "quantize_s": qtime,
             "quantize_bytes": qwork}
    return rows, stack


class Step:
    """The rows of one step, with an event at every row boundary."""

    def __init__(self, rows):
        self.rows = rows

    def new_events(self):
        import torch
        return [torch.cuda.Event(enable_timing=True, external=True)
                for _ in range(len(self.rows) + 1)]

    def run(self, events=None):
        for i, r in enumerate(self.rows):
            if events is not None:
                events[i].record()
            r.run()
        if events is not None:
            events[-1].record()

    def kernels(self):
        return sum(r.kpc * sum(c.launches for c in r.calls) for r in self.rows)


# ------------------------------------------------------------ CPU oracle
def _oracle_stack_linear(layer, lin, names):
    """(state bytes, seconds) of the oracle's GEMV of one stack linear:
    dequantize to bf16 and the fp64 dot products, from the oracle's own
    quantization (not timed)."""
    import oracle
    import synth
    Wb = synth.bf16_bits(synth.weight_bf16(
        lin.N, lin.K, seed=synth.stack_weight_seed(layer, names.index(lin.name))).view(-1))
    st = oracle.quantize(Wb, BS, oracle.NF4, True)
    x = synth.bf16_bits(synth.activations_bf16(1, lin.K, seed=1))
    t0 = time.perf_counter()
    Wh = oracle.dequantize(st, oracle.BF16).reshape(lin.N, lin.K)
    oracle.linear_ref(x, Wh)
    return state_bytes(lin.N * lin.K), time.perf_counter() - t0


def oracle_baseline():
    """The single-threaded CPU oracle timed on bounded samples of every
    configuration; `value` is configuration 5's figure (state GB/s of the
    GEMV pass) from layers 0 and 31, extrapolated x16."""
    import oracle
    import synth
    per = {}
    t0 = time.perf_counter()
    # cfg1 in full
    x1 = synth.normal_f32((synth.ROUNDTRIP_N,), seed=0, std=synth.WEIGHT_STD).numpy()
    a = time.perf_counter()
    st = oracle.quantize(x1, BS, oracle.NF4, True)
    b_ = time.perf_counter()
    oracle.dequantize(st, oracle.F32)
    c = time.perf_counter()
    per["cfg1_quantize_GB/s"] = quantize_bytes(x1.size, 4) / (b_ - a) / 1e9
    per["cfg1_dequantize_GB/s"] = dequantize_bytes(x1.size, 4) / (c - b_) / 1e9
    # cfg2 in full, NF4
    R, C = synth.MATRIX_4096
    w2 = synth.bf16_bits(synth.weight_bf16(R, C, seed=2, outlier_frac=synth.OUTLIER_FRAC)
                         .view(-1))
    a = time.perf_counter()
    st2 = oracle.quantize(w2, BS, oracle.NF4, True)
    b_ = time.perf_counter()
    oracle.dequantize(st2, oracle.BF16)
    c = time.perf_counter()
    per["cfg2_quantize_nf4_GB/s"] = quantize_bytes(R * C, 2) / (b_ - a) / 1e9
    per["cfg2_dequantize_nf4_GB/s"] = dequantize_bytes(R * C, 2) / (c - b_) / 1e9
    # cfg3: B = 8 on 11008 x 4096 in full (dequantize + fp64 dot products)
    N, K = synth.GEMV_SHAPES[0]
    wb = synth.bf16_bits(synth.weight_bf16(N, K, seed=300).view(-1))
    st3 = oracle.quantize(wb, BS, oracle.NF4, True)
    x8 = synth.bf16_bits(synth.activations_bf16(8, K, seed=1))
    a = time.perf_counter()
    Wh = oracle.dequantize(st3, oracle.BF16).reshape(N, K)
    oracle.linear_ref(x8, Wh)
    per["cfg3_gemv_b8_%dx%d_GB/s" % (N, K)] = gemv_bytes(N, K, 8) / (time.perf_counter() - a) / 1e9
    # cfg4: 8 of 2048 rows of the 4096 x 4096 GEMM, extrapolated
    X = synth.bf16_bits(synth.activations_bf16(8, K, seed=1))
    Wq = Wh[:synth.HIDDEN]
    a = time.perf_counter()
    oracle.linear_ref(X, Wq)
    t8 = time.perf_counter() - a
    per["cfg4_gemm_4096x4096_TFLOP/s_extrapolated"] = \
        2 * GEMM_M * synth.HIDDEN * K / (t8 * GEMM_M / 8) / 1e12
    # cfg5: layers 0 and 31, extrapolated x16
    names = [l.name for l in synth.llama7b_layer()]
    sb = st_s = 0.0
    for layer in (0, synth.N_LAYERS - 1):
        for lin in synth.llama7b_layer():
            nb, s = _oracle_stack_linear(layer, lin, names)
            sb += nb
            st_s += s
    v = sb / st_s / 1e9
    wall = time.perf_counter() - t0
    return dict({
        "value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
        "sample": ("configuration 5 (GEMV pass, bytes of the 4-bit weight state per "
                   "second): the oracle's dequantize + fp64 dot products on layers 0 and 31 "
                   "(14 linears, %.3f GB), extrapolated x16; also cfg1 and cfg2 (NF4) in "
                   "full, cfg3 B=8 on 11008x4096 in full, cfg4 on 8 of 2048 rows "
                   "(extrapolated); %.1f s of CPU work in all" % (sb / 1e9, wall)),
        "per_config": per,
    }, **host_description())


def arm_config(args, world, stack_state_bytes):
    """The `config` of both arms' lines (the reference arm times the same
    metric, configuration 5's state bytes per second, on a sample)."""
    return {"workload": WORKLOAD, "layers": args.layers,
            "value": "configuration 5: 4-bit weight state bytes of the stack "
                     "(codes + 8-bit scales + group scales, %.3f GB) per GEMV pass "
                     "time, 4 launches per layer (q/k/v grouped, o, gate/up grouped, "
                     "down)" % (stack_state_bytes / 1e9),
            "weight_format": "nf4 unless named, blocksize 64 unless named, double quant",
            "l2": "no flush: every row runs on its own buffers, each call on a "
                  "different copy, and the 3.34 GB stack pass evicts L2 between steps",
            "parallelism": "replicas x%d" % world,
            "launch": "eager, one call per kernel" if args.eager
                      else "the timed steps replayed as one CUDA graph"}


def run_reference(args):
    """The oracle as the reference arm: each step is one linear of layers 0
    and 31 of the configuration-5 stack (dequantize + fp64 dot products),
    cycling; value = state bytes per second over the steps."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import synth
    names = [l.name for l in synth.llama7b_layer()]
    sample = [(layer, lin) for layer in (0, synth.N_LAYERS - 1)
              for lin in synth.llama7b_layer()]
    for i in range(args.warmup):
        _oracle_stack_linear(*sample[i % len(sample)], names)
    tot_b = tot_s = 0.0
    t0 = time.perf_counter()
    for i in range(max(1, args.steps)):
        nb, s = _oracle_stack_linear(*sample[i % len(sample)], names)
        tot_b += nb
        tot_s += s
    wall = time.perf_counter() - t0
    v = tot_b / tot_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(args, world, sum(state_bytes(lin.N * lin.K)
                                              for lin in synth.llama7b_layer()) * args.layers),
        "cpu_baseline": dict({"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                              "sample": "configuration 5 through the CPU oracle "
                                        "(dequantize + fp64 dot products): one linear of "
                                        "layers 0 / 31 per step, cycling (%d steps)"
                                        % max(1, args.steps)},
                             **host_description()),
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
    peaks = load_peaks()

    rows, stack = build_rows(dev, args.layers)
    step = Step(rows)
    torch.cuda.synchronize()

    warm = max(3, args.warmup)
    for _ in range(warm):
        step.run()
    torch.cuda.synchronize()
    if bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream) != 0:
        raise RuntimeError("device error word set during warm-up")

    events = [step.new_events() for _ in range(args.steps)]
    graph = None
    if not args.eager:
        # the K timed steps (every launch and the row events) as one CUDA
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
    clocks.ready()
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
    status = bnb4.bnb4_device_status(torch.cuda.current_stream().cuda_stream)
    if status != 0:
        raise RuntimeError("device error word set: %s" % bnb4.bnb4_strerror(status))

    # seconds per call of every row, averaged over the timed steps
    per_call = {}
    for i, r in enumerate(rows):
        t = sum(ev[i].elapsed_time(ev[i + 1]) for ev in events) * 1e-3 / args.steps
        per_call[r.name] = t / len(r.calls)
    srow = stack["row"]
    t_pass = max_over_ranks(per_call[srow.name] * len(srow.calls), world)
    elapsed_max = max_over_ranks(elapsed, world)
    value = world * stack["state_bytes"] / t_pass / 1e9

    # burst peaks for rows timed at boost clocks, sustained below them
    burst = clk is None or clk["sm_mhz"] >= 0.9 * clk["sm_max_mhz"]
    tf_peak = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    tf_kind = "bf16 burst" if burst else "bf16 sustained"
    out_rows = {}
    for r in rows:
        t = per_call[r.name]
        d = {"config": r.cfg, "kernel_family": r.family, "calls_per_step": len(r.calls),
             "us_per_call": t * 1e6}
        if r.bound == "tensor":
            a = r.work / t / 1e12
            d.update({"TFLOP/s": a, "frac_bf16_burst": a / peaks["bf16_tflops"],
                      "frac_bf16_sustained": a / peaks["bf16_tflops_sustained"]})
        else:
            a = r.work / t / 1e9
            d.update({"GB/s": a, "frac_hbm": a / peaks["hbm_gbs"]})
            if "weight_bytes" in r.extra:
                d["weight_GB/s"] = r.extra["weight_bytes"] / t / 1e9
        out_rows[r.name] = d
    for r in rows:
        if r.cfg == "cfg5":
            t = per_call[r.name] * len(r.calls)
            out_rows[r.name].update({
                "ms_per_pass": t * 1e3,
                "launches_per_pass": sum(c.launches for c in r.calls),
                "state_GB/s": stack["state_bytes"] / t / 1e9,
                "state_bytes_per_pass": stack["state_bytes"],
                "target_ms_at_70pct_hbm":
                    stack["state_bytes"] / (0.7 * peaks["hbm_gbs"] * 1e9) * 1e3})
    out_rows["cfg5_quantize_stack_setup"] = {
        "config": "cfg5", "kernel_family": "quantize", "calls": len(stack["lins"]),
        "note": "set-up of configuration 5, timed once call by call (not in the step)",
        "GB/s": stack["quantize_bytes"] / stack["quantize_s"] / 1e9,
        "frac_hbm": stack["quantize_bytes"] / stack["quantize_s"] / 1e9 / peaks["hbm_gbs"],
        "ms": stack["quantize_s"] * 1e3}

    # the kernel family with the most time per step
    fam = {}
    for r in rows:
        f = fam.setdefault(r.family, {"s": 0.0, "work": 0.0, "launches": 0, "bound": r.bound})
        f["s"] += per_call[r.name] * len(r.calls)
        f["work"] += r.work * len(r.calls)
        f["launches"] += r.kpc * sum(c.launches for c in r.calls)
    dom_name = max(fam, key=lambda k: fam[k]["s"])
    dom = fam[dom_name]
    tr = traffic_of(dom_name)
    if dom["bound"] == "tensor":
        ach, peak, unit = dom["work"] / dom["s"] / 1e12, tf_peak, "TFLOP/s"
        psrc = "%s %s" % (peaks["source"], tf_kind)
    else:
        ach, peak, unit = dom["work"] / dom["s"] / 1e9, peaks["hbm_gbs"], "GB/s"
        psrc = "%s HBM copy bandwidth" % peaks["source"]
    roofline = {
        "bound": dom["bound"], "kernel": dom_name, "achieved": ach, "peak": peak,
        "unit": unit, "frac": ach / peak,
        "traffic": (tr["bytes"] if "bytes" in tr else tr["ratio"] * dom["work"] / dom["launches"])
                   if tr else None,
        "traffic_launch": tr["launch"] if tr else None,
        "peak_source": psrc,
        "per_launch": "algorithmic work of the %d launches per step of this family "
                      "over their summed event time" % dom["launches"],
        "share_of_step": dom["s"] / (elapsed_max / args.steps),
    }
    if dom_name == "gemv":
        # the decode kernel's own bound: the integer ALU pipe of its exact
        # table lookup (16 byte permutes + 2 logic ops per 8 weights, and one
        # permute + one pack per 8 weights for the per-block tables), 16
        # lanes per cycle per SM sub-partition
        weights = sum(2.0 * r.extra["weight_bytes"] * len(r.calls)
                      for r in rows if r.family == "gemv" and "weight_bytes" in r.extra)
        s_w = sum(per_call[r.name] * len(r.calls)
                  for r in rows if r.family == "gemv" and "weight_bytes" in r.extra)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = clk["sm_max_mhz"] if clk else 1965.0
        alu_peak = sms * 4 * 16 * mhz * 1e6 / 1e12
        alu_ach = weights * ALU_OPS_PER_WEIGHT / s_w / 1e12
        roofline["alu"] = {"achieved": alu_ach, "peak": alu_peak, "unit": "T lane-op/s",
                           "frac": alu_ach / alu_peak, "ops_per_weight": ALU_OPS_PER_WEIGHT,
                           "peak_source": "%d SMs x 4 sub-partitions x 16 ALU lanes x %.0f MHz"
                                          % (sms, mhz)}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": warm,
        "ms_per_step": elapsed_max / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": arm_config(args, world, stack["state_bytes"]),
        "roofline": roofline,
        "rows": out_rows,
        "gpu_launches": step.kernels() * args.steps,
        "clocks": clk,
        "peaks": peaks,
    }
    del graph
    if not args.no_e2e:
        line["e2e"] = run_e2e(stack, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(stack, world, steps=10):
    """Configuration 5 end to end through the C ABI, eager, with the
    activations coming from page-locked HOST memory and every output read
    back: per step, copy x in, make the pass's 128 bnb_gemv_4bit_grouped
    calls (their descriptors built once, as a C caller would keep them),
    copy the 224 outputs (one buffer) out -- all inside the timed region."""
    import torch
    xs = stack["x"]
    host_x = {k: v.cpu().pin_memory() for k, v in xs.items()}
    host_y = stack["y_all"].cpu().pin_memory()
    h2d = sum(t.numel() * 2 for t in host_x.values())
    d2h = host_y.numel() * 2
    calls = stack["row"].calls  # the timed pass's launches (q/k/v, o, gate/up, down)

    def one():
        for k in xs:
            xs[k].copy_(host_x[k], non_blocking=True)
        for c in calls:
            rc = c()
            if rc != 0:
                raise RuntimeError("bnb_gemv_4bit_grouped failed with status %d" % rc)
        host_y.copy_(stack["y_all"], non_blocking=True)

    one()
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        one()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    t = max_over_ranks(a.elapsed_time(b) * 1e-3, world)
    return {"value": world * stack["state_bytes"] * steps / t / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps, "ms_per_step": t / steps * 1e3,
            "path": "bnb_gemv_4bit_grouped (C ABI through its Python binding), 4 calls per "
                    "layer as in the timed pass, eager; x in from page-locked host memory, "
                    "the 224 outputs out in one copy"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
