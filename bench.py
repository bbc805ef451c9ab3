"""Throughput of the SmoothQuant W8A8 linear path on B200.

A step is one pass of the whole path over one batch: per-input-channel
activation absmax (calibration) -> smoothing factor and weight column absmax
-> SSZ int8 weight quantization of the smoothed weight -> per-token int8
activation quantization -> INT8 GEMM with fused dequant.  On one GPU the step
is captured once as a CUDA graph and replayed.  Inputs are seeded
synthetic LLM-shaped data resident in HBM; L2 is flushed (a 512 MB write,
then a 384 MB read that writes the dirty lines back) before every timed step,
outside the timed events.  Default workload: the MLP up-projection
8192 x 4096 -> 11008 (the largest single-GPU linear; compute-bound GEMM).

value  = the W8A8 linear's INT8 TOPS: 2*M*N*K int8 ops per step, over all
         ranks, divided by the device time of the per-inference part of each
         step (per-token activation quantization + GEMM with dequant; max over
         ranks).  The once-per-weight part (calibration, smoothing, SSZ) runs
         inside every timed step too and is reported beside it in GB/s and as
         a fraction of its roofline (`weight_path`); `ms_per_step` is the whole
         step, `path` gives its TOPS.
e2e    = the same metric through the C ABI with the activations copied from
         pinned host memory every step and the output copied back (copies
         timed), the quantized weights resident on the device.

Multi-GPU (torchrun): data parallel, each rank a replica of the layer with its
own batch of tokens (weak scaling).  The calibration statistic, the [K]
activation absmax, is all-reduced with MAX over NCCL so all replicas derive
the same smoothing factor; the SSZ search is split by output channel (each
rank searches N/G channels) and its codes, scales and rounds are
all-gathered, so every replica holds the same quantized weight without
repeating the search.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "mlp_up_8192x4096x11008"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--eager", action="store_true",
                   help="launch every call of a timed step from Python (default on one GPU: the step is "
                        "captured once as a CUDA graph and replayed)")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--no-next-rows", action="store_true",
                   help="skip the per-kernel timings of the rows beyond the five-step path")
    p.add_argument("--record-traffic", metavar="NCU_CSV",
                   help="read an ncu --csv capture (gpu__time_duration.sum, dram__bytes_read.sum, "
                        "dram__bytes_write.sum) of this workload and write profiles/dram_traffic.json")
    p.add_argument("--decode-launches", action="store_true",
                   help="only launch the 16 x 8192 -> 28672 decode GEMMs on random codes, three with int8 "
                        "weights then three with packed int4 weights, and exit (the workload of the decode "
                        "kernel's ncu capture)")
    p.add_argument("--next-row-launches", action="store_true",
                   help="only launch, on the MLP up-projection inputs (8192 x 4096 -> 11008, seed 0), the "
                        "asymmetric SSZ twice, then the int4 SSZ, packing and three W4A8 GEMMs, and exit (the "
                        "workload of those kernels' ncu captures)")
    p.add_argument("--gemm-sweep", choices=["time", "launch"],
                   help="time: w8a8_gemm_dequant over a sweep of K and M at N = 1024 and the two prefill "
                        "shapes, 20 back-to-back launches per CUDA-graph replay, beside torch._int_mm "
                        "(cuBLASLt, int32 out) as the library ceiling, one JSON line a shape; launch: only "
                        "launch w8a8_gemm_dequant twice a shape (the launch list's workload); then exit")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


B200_SMS = 148
FP32_LANES_PER_SM = 128
NOMINAL_SM_MHZ = 1965.0
SSZ_OPS_PER_ELEMENT_ROUND = 10  # codes, residual, clamp, compare and sums per element and round


def algorithmic_work_mnk(M, K, N, xb, yb, bits=8):
    """Bytes (or int8 ops) each kernel must move (or do) per launch."""
    return {
        "calib_absmax": {"bytes": xb * M * K + 4 * K},
        "smooth_fold": {"bytes": xb * N * K + 3 * 4 * K},
        "ssz_quant_weight": {"bytes": xb * N * K + N * K + 4 * K + 4 * N + 8 * N + 4 * N},
        # int4 weights: the codes packed two per byte (N K read, N K / 2 written)
        "sq_pack_int4": {"bytes": N * K + N * K // 2 if bits == 4 else 0},
        "quant_act_per_token": {"bytes": xb * M * K + M * K + 4 * K + 4 * M},
        # int4: the W4A8 GEMM reads the weight codes packed
        "w8a8_gemm_dequant": {"ops": 2 * M * N * K,
                              "bytes": M * K + (N * K if bits == 8 else N * K // 2) + 4 * M + 4 * N + yb * M * N},
    }


def algorithmic_work(cfg):
    xb = 2 if cfg.in_dtype == "bf16" else 4
    yb = 2 if cfg.out_dtype == "bf16" else 4
    return algorithmic_work_mnk(cfg.M, cfg.K, cfg.N, xb, yb, cfg.bits)


# every source a step's kernels are compiled from (besides common.cuh)
KERNEL_SOURCES = {
    "calib_absmax": ("smooth.cu",), "smooth_fold": ("smooth.cu",), "ssz_quant_weight": ("ssz.cu", "dd.cuh"),
    "sq_pack_int4": ("gemm.cu",), "quant_act_per_token": ("quant_act.cu",),
    "w8a8_gemm_dequant": ("gemm.cu", "gemm_decode.cuh"),
}


def source_sha(files):
    h = hashlib.sha256()
    for f in (*files, "common.cuh"):
        with open(os.path.join(ROOT, "w8a8_linear_layers_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dram_traffic(step_name, workload):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since it was captured."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(step_name)
    if not e or e.get("src_sha") != source_sha(KERNEL_SOURCES[step_name]):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.result = None
        if self.proc is None:
            return
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if sm:
            self.result = {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                           "samples": len(sm)}


# ------------------------------------------------------------------ our arm
NAMES = ["calib_absmax", "smooth_fold", "ssz_quant_weight", "sq_pack_int4", "quant_act_per_token",
         "w8a8_gemm_dequant"]
WEIGHT_PATH = ("calib_absmax", "smooth_fold", "ssz_quant_weight", "sq_pack_int4")  # once per weight
LINEAR = ("quant_act_per_token", "w8a8_gemm_dequant")  # every inference
NW = len(WEIGHT_PATH) + 1  # weight-path events per linear
GPT_WORKLOAD = "gpt345m_8x1024"


class Problem:
    """One linear layer of the workload with its device buffers."""

    def __init__(self, torch, x, wt, alpha, bits, max_iters, ydt):
        dev = x.device
        M, K = x.shape
        N = wt.shape[0]
        self.x, self.wt, self.alpha, self.bits, self.max_iters = x, wt, alpha, bits, max_iters
        self.M, self.K, self.N = M, K, N
        f32 = dict(device=dev, dtype=torch.float32)
        self.ax, self.aw, self.s, self.inv = (torch.empty(K, **f32) for _ in range(4))
        self.qw = torch.empty(N, K, device=dev, dtype=torch.int8)
        self.sw = torch.empty(N, **f32)
        self.qw4 = torch.empty(N, K // 2, device=dev, dtype=torch.uint8) if bits == 4 else None
        self.iters = torch.empty(N, device=dev, dtype=torch.int32)  # SSZ rounds per channel (ALU work)
        self.qx = torch.empty(M, K, device=dev, dtype=torch.int8)
        self.sx = torch.empty(M, **f32)
        self.y = torch.empty(M, N, device=dev, dtype=ydt)


def make_problems(args, torch, rank, dev):
    """The workload's linears on this rank: each replica draws its own tokens
    (seed = rank) and the same weights."""
    import synthetic
    if args.workload == GPT_WORKLOAD:
        from synthetic import gpt
        weights = gpt.make_weights(0, dev)
        cap = {}
        gpt.forward(weights, gpt.make_tokens(rank), capture=cap)
        return [Problem(torch, cap[k], weights[k], 0.5, 8, 20, torch.bfloat16) for k in sorted(cap)]
    cfg = synthetic.CONFIGS[args.workload]
    x_cpu, w_cpu = synthetic.make_linear(cfg, seed=0)
    if rank > 0:
        x_cpu, _ = synthetic.make_linear(cfg, seed=rank)
    ydt = torch.bfloat16 if cfg.out_dtype == "bf16" else torch.float32
    return [Problem(torch, x_cpu.to(dev), w_cpu.to(dev), cfg.alpha, cfg.bits, cfg.max_iters, ydt)]


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import w8a8_linear_layers_b200 as w
    from w8a8_linear_layers_b200 import distributed as wdist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    probs = make_problems(args, torch, rank, dev)
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()

    def forward(p, xin, evs=None, base=0):
        """The per-inference part: per-token codes, then the GEMM (with evs:
        an event before, between and after, for the per-kernel split)."""
        if evs is not None:
            evs[base].record()
        w.quant_act_per_token(xin, p.inv, p.qx, p.sx)
        if evs is not None:
            evs[base + 1].record()
        if p.bits == 8:
            w.w8a8_gemm_dequant(p.qx, p.sx, p.qw, p.sw, p.y)
        else:
            w.w4a8_gemm_dequant(p.qx, p.sx, p.qw4, p.sw, p.y)
        if evs is not None:
            evs[base + 2].record()

    def weight_path(p, evs=None, base=0):
        """The once-per-weight part of one linear; with evs, an event before
        each kernel (WEIGHT_PATH order) and one after the last, on the
        current stream (the launching one, or a graph's capture stream)."""
        def mark(i):
            if evs is not None:
                evs[base + i].record()
        mark(0)
        w.sq_calib_absmax(p.x, p.ax)
        mark(1)
        wdist.allreduce_calibration(p.ax)
        w.sq_smooth_fold(p.ax, p.wt, p.alpha, p.aw, p.s, p.inv)
        mark(2)
        if world > 1:  # each rank searches its block of output channels, then all-gather
            wdist.ssz_quant_weight_sharded(p.wt, p.s, p.bits, p.max_iters, p.qw, p.sw, p.iters)
        else:
            w.ssz_quant_weight(p.wt, p.s, p.bits, p.max_iters, p.qw, p.sw, iters_out=p.iters)
        mark(3)
        if p.bits == 4:  # int4 weights: packed two per byte for the W4A8 GEMM
            w.sq_pack_int4(p.qw, p.qw4)
            mark(4)  # int8 records no packing event: an empty pair would time only the gap

    nw_ev = NW * len(probs)  # events of the weight path; then two around the linears

    def step(evs=None):
        """One pass of the whole path over every linear: the once-per-weight
        part of each (its kernels bracketed by events), then the per-inference
        part of each, back to back with events only around the block (an
        event node between two kernels adds its own latency and keeps the
        next kernel from starting early, so the linears' time is taken
        without them; the per-kernel split comes from instrumented replays)."""
        for i, p in enumerate(probs):
            weight_path(p, evs, NW * i)
        if evs is not None:
            evs[nw_ev].record()
        for p in probs:
            forward(p, p.x)
        if evs is not None:
            evs[nw_ev + 1].record()

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if w.device_fault() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during warm-up")

    # One GPU: the step is captured once as a CUDA graph (its events
    # included) and replayed every timed step, so that the host's
    # launch of some 5 calls per linear never holds the GPU back.  Several
    # ranks launch eagerly (no collective is captured).
    graph = None
    if world == 1 and not args.eager:
        gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nw_ev + 2)]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(gev)
        flush()
        graph.replay()  # untimed
        torch.cuda.synchronize()

    def elapsed(e):
        """Per linear j: {weight-path kernel: ms} from a step's events (int8
        weights: no packing event), and the per-inference block's ms."""
        out = []
        for j, p in enumerate(probs):
            b = NW * j
            t = {n: e[b + i].elapsed_time(e[b + i + 1]) for i, n in enumerate(WEIGHT_PATH[:3])}
            t["sq_pack_int4"] = e[b + 3].elapsed_time(e[b + 4]) if p.bits == 4 else 0.0
            out.append(t)
        return out, e[nw_ev].elapsed_time(e[nw_ev + 1])

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nw_ev + 2)] for _ in range(args.steps)]
    per_step = []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush()                # L2 flush, outside the timed events
            if graph is not None:
                graph.replay()
                torch.cuda.synchronize()  # this step's events, before the next replay records them again
                per_step.append(elapsed(gev))
            else:
                step(evs[i])
        torch.cuda.synchronize()
        wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    if graph is None:
        per_step = [elapsed(e) for e in evs]
    step_ms = [sum(sum(t.values()) for t in st) + blk for st, blk in per_step]
    linear_step_ms = [blk for _, blk in per_step]
    total_ms = wdist.max_over_ranks(sum(step_ms), device=dev)
    linear_ms = wdist.max_over_ranks(sum(linear_step_ms), device=dev)
    if w.device_fault() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait during timing")

    # ---- outside the timed region: the per-inference block again, (a) with
    # an event before, between and after the two kernels of every linear (the
    # per-kernel split; each time then carries an event node's latency), and
    # (b) with events only around each group of linears of one shape (the
    # per-shape linear time, as in the timed block)
    groups = {}
    for j, p in enumerate(probs):
        groups.setdefault((p.M, p.K, p.N), []).append(j)
    iev = [torch.cuda.Event(enable_timing=True, external=graph is not None) for _ in range(3 * len(probs))]
    gev2 = [torch.cuda.Event(enable_timing=True, external=graph is not None) for _ in range(2 * len(groups))]

    def inst_split():
        for j, p in enumerate(probs):
            forward(p, p.x, iev, 3 * j)

    def inst_groups():
        for g, idx in enumerate(groups.values()):
            gev2[2 * g].record()
            for j in idx:
                forward(probs[j], probs[j].x)
            gev2[2 * g + 1].record()

    reps = max(3, min(args.steps, 10))
    split = [[0.0, 0.0] for _ in probs]
    grp_ms = [0.0] * len(groups)
    for fn, sink in ((inst_split, "split"), (inst_groups, "groups")):
        g2 = None
        if graph is not None:
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                fn()
        for r in range(reps + 1):
            flush()
            if g2 is not None:
                g2.replay()
            else:
                fn()
            torch.cuda.synchronize()
            if r == 0:
                continue  # warm-up replay
            if sink == "split":
                for j in range(len(probs)):
                    split[j][0] += iev[3 * j].elapsed_time(iev[3 * j + 1]) / reps
                    split[j][1] += iev[3 * j + 1].elapsed_time(iev[3 * j + 2]) / reps
            else:
                for g in range(len(groups)):
                    grp_ms[g] += gev2[2 * g].elapsed_time(gev2[2 * g + 1]) / reps
        del g2
    # per kernel (summed over the linears, mean over steps) and per linear and kernel
    kern_ms = {n: statistics.mean(sum(t[n] for t in st) for st, _ in per_step) for n in WEIGHT_PATH}
    kern_ms["quant_act_per_token"] = sum(a for a, _ in split)
    kern_ms["w8a8_gemm_dequant"] = sum(b for _, b in split)
    lin_ms = [[statistics.mean(st[j][n] for st, _ in per_step) for n in WEIGHT_PATH] + split[j]
              for j in range(len(probs))]
    shape_ms = {"%dx%d->%d" % k: grp_ms[g] / len(idx) for g, (k, idx) in enumerate(groups.items())}

    ops_per_step = sum(2.0 * p.M * p.N * p.K for p in probs)
    value = ops_per_step * world * args.steps / (linear_ms * 1e-3) / 1e12
    path_value = ops_per_step * world * args.steps / (total_ms * 1e-3) / 1e12

    next_rows = (time_next_rows(args, w, torch, probs, flush, stream)
                 if world == 1 and not args.no_next_rows else None)

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, w, wdist, torch, probs, forward, flush, stream, ops_per_step, world)
    del graph
    return finish(args, world, probs, kern_ms, total_ms, linear_ms, value, path_value, e2e, clk, wall1 - wall0,
                  next_rows, launch="eager" if world > 1 or args.eager else "cuda_graph", lin_ms=lin_ms,
                  shape_ms=shape_ms)


class L2Flush:
    """Evicts the inputs from L2 (126 MB) before a timed region: a 512 MB
    write, then a 384 MB read, so that the lines the write left dirty are
    written back here and not by the timed kernels."""

    def __init__(self, torch, dev):
        self.wbuf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.rbuf = torch.ones(384 << 20, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.wbuf.zero_()
        self.rbuf.max()


def time_next_rows(args, w, torch, probs, flush, stream, reps=50):
    """Kernels of the rows built beyond the five-step path, timed one launch
    at a time like the path's kernels (L2 flushed before each, outside the
    events), on the first linear of the workload:
    - quant_act_static: codes at a static per-tensor scale (range calibrated
      beforehand on the same activations);
    - sq_layernorm_quant: LayerNorm, smoothing and per-token codes in one
      pass (unfused_bytes: what a separate LayerNorm output would add);
    - ssz_quant_weight_asym, quant_act_per_token_rowsum and
      w8a8_gemm_dequant_asym: the asymmetric int8 weight path;
    - sq_pack_int4 and w4a8_gemm_dequant (packed int4 weights) against
      w8a8_gemm_dequant on the 16 x 8192 -> 28672 decode shape;
    - that decode linear's forward, eager and as a CUDA graph replay.
    Per-launch times include the launch gap that in-step events hide."""
    p = probs[0]
    peaks, _ = load_peaks()
    out = {}
    rng = torch.empty(1, device=p.x.device)
    w.sq_static_range_update(p.ax, p.inv, rng, first=True)

    def timed(fn):
        ts = []
        for i in range(reps + 3):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        return statistics.mean(ts)

    ms = timed(lambda: w.quant_act_static(p.x, p.inv, rng, p.qx, p.sx))
    nbytes = p.x.element_size() * p.M * p.K + p.M * p.K + 4 * p.K + 4 * p.M + 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    out["quant_act_static"] = {"us": round(ms * 1e3, 2), "bound": "hbm", "achieved": round(gbs, 1),
                               "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                               "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic": {"bytes": nbytes},
                               "shape": [p.M, p.K]}

    # activation quantization fused upstream: LayerNorm + smoothing + codes
    # in one pass over the layer input (the X of this linear serves as h)
    g_ln = torch.ones(p.K, device=p.x.device)
    b_ln = torch.zeros(p.K, device=p.x.device)
    ms = timed(lambda: w.sq_layernorm_quant(p.x, g_ln, b_ln, 1e-5, p.inv, p.qx, p.sx))
    nbytes = p.x.element_size() * p.M * p.K + p.M * p.K + 12 * p.K + 4 * p.M
    gbs = nbytes / (ms * 1e-3) / 1e9
    out["sq_layernorm_quant"] = {"us": round(ms * 1e3, 2), "bound": "hbm", "achieved": round(gbs, 1),
                                 "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                                 "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic": {"bytes": nbytes},
                                 "shape": [p.M, p.K],
                                 "unfused_bytes": 2 * p.x.element_size() * p.M * p.K + nbytes}

    # asymmetric int8 weights: SSZ over (scale, offset), per-token codes with
    # row sums, GEMM with the offset dequant
    dev = p.x.device
    qa, sa, ow = torch.empty_like(p.qw), torch.empty_like(p.sw), torch.empty(p.N, device=dev)
    its = torch.empty(p.N, device=dev, dtype=torch.int32)
    rs = torch.empty(p.M, device=dev, dtype=torch.int32)
    ms = timed(lambda: w.ssz_quant_weight_asym(p.wt, p.s, p.max_iters, qa, sa, ow, iters_out=its))
    iters = float(its.double().mean().item())
    ops = SSZ_OPS_PER_ELEMENT_ROUND * p.N * p.K * (1.0 + iters)
    sm_mhz = NOMINAL_SM_MHZ
    alu_peak = B200_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6 / 1e12
    ach = ops / (ms * 1e-3) / 1e12
    out["ssz_quant_weight_asym"] = {"us": round(ms * 1e3, 2), "bound": "alu", "achieved": round(ach, 2),
                                    "peak": round(alu_peak, 2), "unit": "Tops/s", "frac": round(ach / alu_peak, 4),
                                    "mean_iters": round(iters, 3), "peak_clock_mhz": sm_mhz,
                                    "shape": [p.N, p.K]}
    ms = timed(lambda: w.quant_act_per_token_rowsum(p.x, p.inv, p.qx, p.sx, rs))
    nbytes = p.x.element_size() * p.M * p.K + p.M * p.K + 4 * p.K + 8 * p.M
    gbs = nbytes / (ms * 1e-3) / 1e9
    out["quant_act_per_token_rowsum"] = {"us": round(ms * 1e3, 2), "bound": "hbm", "achieved": round(gbs, 1),
                                         "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                                         "frac": round(gbs / peaks["hbm_gbs"], 4), "shape": [p.M, p.K]}
    if p.bits == 8:
        ms = timed(lambda: w.w8a8_gemm_dequant_asym(p.qx, p.sx, rs, qa, sa, ow, p.y))
        tops = 2.0 * p.M * p.N * p.K / (ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"] * INT8_OVER_BF16
        out["w8a8_gemm_dequant_asym"] = {"us": round(ms * 1e3, 2), "bound": "tensor", "achieved": round(tops, 1),
                                         "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(tops / peak, 4),
                                         "shape": [p.M, p.N, p.K]}

    # packed int4 weights on the decode shape (16 tokens, 8192 -> 28672),
    # where the GEMM is bound by the weight bytes: W4A8 against W8A8 on the
    # same codes (random codes, the kernels' speed does not depend on them)
    Md, Kd, Nd = 16, 8192, 28672
    g = torch.Generator(device=dev).manual_seed(0)
    qxd = torch.randint(-127, 128, (Md, Kd), device=dev, dtype=torch.int8, generator=g)
    q4 = torch.randint(-7, 8, (Nd, Kd), device=dev, dtype=torch.int8, generator=g)
    sxd = torch.rand(Md, device=dev, generator=g) * 1e-2
    swd = torch.rand(Nd, device=dev, generator=g) * 1e-2
    packed = torch.empty(Nd, Kd // 2, device=dev, dtype=torch.uint8)
    w.sq_pack_int4(q4, packed)
    yd = torch.empty(Md, Nd, device=dev, dtype=torch.bfloat16)
    for name, fn, wbytes in (("w8a8_gemm_dequant_decode", lambda: w.w8a8_gemm_dequant(qxd, sxd, q4, swd, yd), Nd * Kd),
                             ("w4a8_gemm_dequant_decode", lambda: w.w4a8_gemm_dequant(qxd, sxd, packed, swd, yd),
                              Nd * Kd // 2)):
        ms = timed(fn)
        nbytes = Md * Kd + wbytes + 2 * Md * Nd + 4 * Md + 4 * Nd
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"us": round(ms * 1e3, 2), "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "algorithmic": {"bytes": nbytes, "ops": 2 * Md * Nd * Kd}, "shape": [Md, Nd, Kd]}
    # the decode linear's forward (per-token codes, then the GEMM) issued
    # from Python call by call, and the same two kernels replayed as one
    # CUDA graph (W8A8Linear.graphed); weights set from the codes above
    xd = torch.randn(Md, Kd, device=dev, dtype=torch.bfloat16, generator=g)
    for kind in ("sym8", "int4"):
        lin = w.W8A8Linear(torch.empty(Nd, Kd, device=dev, dtype=torch.bfloat16), weights=kind)
        lin.inv_s.fill_(1.0)
        lin.sw.copy_(swd)
        if kind == "int4":
            lin.qw4.copy_(packed)
        else:
            lin.qw.copy_(q4)
        gl = lin.graphed(Md)
        gl.x.copy_(xd)
        ms_e = timed(lambda: lin.forward(xd, yd))
        ms_g = timed(gl.replay)
        out["decode_forward_" + kind] = {"eager_us": round(ms_e * 1e3, 2), "graph_us": round(ms_g * 1e3, 2),
                                         "kernels": 2, "shape": [Md, Nd, Kd]}
        del lin, gl
    ms = timed(lambda: w.sq_pack_int4(q4, packed))
    nbytes = Nd * Kd + Nd * Kd // 2
    gbs = nbytes / (ms * 1e-3) / 1e9
    out["sq_pack_int4"] = {"us": round(ms * 1e3, 2), "bound": "hbm", "achieved": round(gbs, 1),
                           "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                           "shape": [Nd, Kd]}
    del q4, packed, qxd, yd
    return out


E2E_CHUNK_ROWS = 2048  # at most this many rows a transfer unit (a linear's tokens are cut into chunks)
E2E_CHUNKS = 4         # at least this many chunks a linear where its rows allow (256 rows a chunk at least)
E2E_SLOTS = 3          # device buffers in rotation: one filling, one computing, one draining


def e2e_chunk_rows(M):
    """Rows of an end-to-end transfer chunk for linears of up to M tokens."""
    return max(256, min(E2E_CHUNK_ROWS, -(-M // E2E_CHUNKS)))


def run_e2e(args, w, wdist, torch, probs, forward, flush, stream, ops_per_step, world):
    """The per-inference linears end to end: every step copies the
    activations from pinned host memory, quantizes them, runs the GEMM and
    copies the output back, all inside the timed events; the quantized
    weights (the layers' parameters) stay resident on the device.  The
    library's HostStreamer cuts the tokens into chunks (M / E2E_CHUNKS rows,
    within [256, E2E_CHUNK_ROWS]) whose copy in, codes + GEMM and copy out
    overlap on three streams through E2E_SLOTS device buffers."""
    hosts = [(p.x.cpu().pin_memory(), torch.empty_like(p.y, device="cpu").pin_memory()) for p in probs]
    dev = probs[0].x.device
    R = e2e_chunk_rows(max(p.M for p in probs))
    streamer = w.HostStreamer(dev, R, max(p.K for p in probs), max(p.N for p in probs), probs[0].x.dtype,
                              probs[0].y.dtype, slots=E2E_SLOTS)

    def chunk_fn(p):
        def fn(x, qx, sx, y):
            w.quant_act_per_token(x, p.inv, qx, sx)
            if p.bits == 8:
                w.w8a8_gemm_dequant(qx, sx, p.qw, p.sw, y)
            else:
                w.w4a8_gemm_dequant(qx, sx, p.qw4, p.sw, y)
        return fn

    jobs = [(xh, yh, chunk_fn(p)) for p, (xh, yh) in zip(probs, hosts)]
    e2e_ms = []
    for i in range(args.warmup + args.e2e_steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        streamer.run(jobs, stream)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    # the chunked pipeline must reproduce the resident path's output
    for p, (xh, yh) in zip(probs, hosts):
        forward(p, p.x)
        if not torch.equal(yh, p.y.cpu()):
            raise RuntimeError("the chunked end-to-end output differs from the resident path's")
    e2e_total = wdist.max_over_ranks(sum(e2e_ms), device=dev)
    e2e_value = ops_per_step * world * len(e2e_ms) / (e2e_total * 1e-3) / 1e12
    h2d = sum(p.x.numel() * p.x.element_size() for p in probs)
    d2h = sum(p.y.numel() * p.y.element_size() for p in probs)
    return {"value": round(e2e_value, 3), "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(e2e_total / len(e2e_ms), 4), "chunk_rows": R,
            "what": "activations copied host->device from pinned memory, per-token quantization, GEMM + dequant, "
                    "output copied device->host, every step, in chunks of %d tokens whose copies in, compute and "
                    "copies out overlap on three streams (HostStreamer); quantized weights resident" % R}


def per_shape_table(probs, lin_ms, peaks, shape_ms=None):
    """Workloads of several linears: per distinct (M, K, N) the number of
    linears, the mean time of each kernel (the activation quantization and
    the GEMM each from events around it, which add an event node's
    latency), the GEMM's TOPS and the linear's (activation quantization +
    GEMM, from events around the shape's group of linears run back to back,
    as in the timed block)."""
    groups = {}
    for p, ms in zip(probs, lin_ms):
        groups.setdefault((p.M, p.K, p.N), []).append(ms)
    out = {}
    peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    for (M, K, N), rows in groups.items():
        mean = [statistics.mean(r[i] for r in rows) for i in range(len(NAMES))]
        gemm_ms = mean[NAMES.index("w8a8_gemm_dequant")]
        lin = gemm_ms + mean[NAMES.index("quant_act_per_token")]
        if shape_ms:
            lin = shape_ms["%dx%d->%d" % (M, K, N)]
        tops = 2.0 * M * N * K / (gemm_ms * 1e-3) / 1e12
        out["%dx%d->%d" % (M, K, N)] = {
            "linears": len(rows), "us": {n: round(m * 1e3, 2) for n, m in zip(NAMES, mean)},
            "gemm_tops": round(tops, 1), "gemm_frac": round(tops / peak, 4),
            "linear_tops": round(2.0 * M * N * K / (lin * 1e-3) / 1e12, 1)}
    return out


def finish(args, world, probs, kern_ms, total_ms, linear_ms, value, path_value, e2e, clk, wall_s, next_rows=None,
           launch="eager", lin_ms=None, shape_ms=None):
    names = [n for n in NAMES if n != "sq_pack_int4" or any(p.bits == 4 for p in probs)]
    # ---- rooflines per kernel (algorithmic work summed over the workload's linears)
    peaks, src = load_peaks()
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    work = {n: {} for n in names}
    for p in probs:
        for n, v in algorithmic_work_mnk(p.M, p.K, p.N, p.x.element_size(), p.y.element_size(), p.bits).items():
            if n not in work:
                continue
            for key, val in v.items():
                work[n][key] = work[n].get(key, 0) + val
    # SSZ is bound by its search rounds, not by HBM: ALU work = c N K (1 + iters)
    # operations (c = 10 per element and round), against every FP32 lane of
    # every SM at the SM clock sampled during the timed region
    iters = sum(float(p.iters.double().sum().item()) for p in probs) / sum(p.N for p in probs)
    ssz_ops = sum(SSZ_OPS_PER_ELEMENT_ROUND * p.N * p.K * (1.0 + float(p.iters.double().mean().item()))
                  for p in probs)
    sm_mhz = (clk.result or {}).get("sm_mhz") or NOMINAL_SM_MHZ
    alu_peak = B200_SMS * FP32_LANES_PER_SM * sm_mhz * 1e6 / 1e12  # T ops/s
    kernels = {}
    for n in names:
        t_s = kern_ms[n] * 1e-3
        entry = {"us": round(kern_ms[n] * 1e3, 2)}
        if n == "ssz_quant_weight":
            ach = ssz_ops / t_s / 1e12
            hbm = work[n]["bytes"] / t_s / 1e9
            entry.update(bound="alu", achieved=round(ach, 2), peak=round(alu_peak, 2), unit="Tops/s",
                         frac=round(ach / alu_peak, 4), mean_iters=round(iters, 3),
                         hbm={"achieved": round(hbm, 1), "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
                              "frac": round(hbm / peaks["hbm_gbs"], 4)})
            work[n] = dict(work[n], ops=ssz_ops)
        elif "ops" in work[n] and (work[n]["ops"] / max(work[n]["bytes"], 1)
                                   >= int8_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)):
            # at or above the ridge point: bound by the tensor cores
            ach = work[n]["ops"] / t_s / 1e12
            entry.update(bound="tensor", achieved=round(ach, 1), peak=round(int8_peak, 1), unit="TFLOP/s",
                         frac=round(ach / int8_peak, 4))
        else:
            ach = work[n]["bytes"] / t_s / 1e9
            peak = peaks["hbm_gbs"]
            entry.update(bound="hbm", achieved=round(ach, 1), peak=round(peak, 1), unit="GB/s",
                         frac=round(ach / peak, 4))
        entry["algorithmic"] = work[n]
        entry["traffic"] = dram_traffic(n, args.workload)
        kernels[n] = entry
    dom = max(names, key=lambda n: kern_ms[n])
    roof = {k: kernels[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roof["kernel"] = dom
    roof["peak_source"] = {"tensor": "%s (bf16 burst x2 for int8)" % src, "hbm": "%s (hbm copy)" % src,
                           "alu": "derived: %d SMs x %d FP32 lanes x sampled SM clock" % (B200_SMS, FP32_LANES_PER_SM)
                           }[roof["bound"]]

    p0 = probs[0]
    launches_per_step = {"calib_absmax": 1, "smooth_fold": 2, "ssz_quant_weight": 1, "sq_pack_int4": int(p0.bits == 4),
                         "quant_act_per_token": 1, "w8a8_gemm_dequant": 1}
    M, K, N = p0.M, p0.K, p0.N
    lin_step = linear_ms / args.steps
    result = {
        "metric": "W8A8 linear INT8 TOPS (% of peak); quant/SSZ GB/s (% of HBM) on 1 B200",
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8 codes, int32 acc, %s in/out, fp32 scales" % ("bf16" if p0.x.element_size() == 2 else "f32"),
        "data": "synthetic (seeded LLM-shaped activations with outlier channels, N(0,std) weights)",
        "config": {"workload": args.workload, "linears": len(probs), "M_tokens_per_gpu": M, "K": K, "N": N,
                   "alpha": p0.alpha, "weight_bits": p0.bits, "ssz_max_iters": p0.max_iters,
                   "parallelism": ("dp%d (replicas; MAX all-reduce of the calibration absmax; SSZ split by output "
                                   "channel and all-gathered)" % world),
                   "l2": "flushed (512 MB write, then 384 MB read) before every timed step, outside the timed events",
                   "launch": {"cuda_graph": "each timed step one CUDA graph replay (captured once, events "
                                            "inside it)",
                              "eager": "every call of a timed step launched from Python"}[launch]},
        "value_definition": ("2*M*N*K int8 ops over the device time of the per-inference linears (per-token "
                             "activation quantization + GEMM with fused dequant), run back to back inside each "
                             "timed step with events only around them; every timed step first runs the "
                             "once-per-weight path of every linear (calibration, smoothing, SSZ, each kernel "
                             "between events), whose time is in ms_per_step and whose throughput is in "
                             "weight_path.  The activation-quantization and GEMM entries of kernels come from "
                             "replays of the linears outside the timed region with an event around each kernel "
                             "(each carries an event node's latency)"),
        "linear": {"ms_per_step": round(lin_step, 4), "tops": round(value, 2), "peak": round(int8_peak, 1),
                   "frac": round(value / int8_peak, 4), "kernels": list(LINEAR)},
        "path": {"ms_per_step": round(total_ms / args.steps, 4), "tops": round(path_value, 2),
                 "what": "the whole path per step: calibration, smoothing, SSZ, activation quantization, GEMM"},
        "weight_path": {n: kernels[n] for n in names if n in WEIGHT_PATH},
        "roofline": roof,
        "kernels": kernels,
        "e2e": e2e,
        "gpu_launches": sum(launches_per_step.values()) * len(probs) * args.steps,
        "clocks": clk.result,
        "wall_s_timed_region": round(wall_s, 3),
    }
    if lin_ms is not None and len(probs) > 1:
        result["per_shape"] = per_shape_table(probs, lin_ms, peaks, shape_ms)
    if next_rows:
        result["next_rows"] = next_rows
    return result


# ------------------------------------------------------------------ oracle arm
def oracle_linear_times(x, wt, alpha, bits, max_iters, frac=1.0):
    """Time the CPU oracle on one linear (x [M,K], wt [N,K] fp32 numpy).
    frac < 1 runs the SSZ search, the activation quantization and the
    GEMM+dequant on that fraction of their rows (rows are independent in all
    three) and scales their times back up; the calibration and weight-absmax
    passes always run in full.  Returns (per-stage seconds scaled to the full
    linear, description, per-stage seconds actually spent)."""
    import oracle
    M, K = x.shape
    N = wt.shape[0]
    t, spent = {}, {}
    t0 = time.perf_counter()
    ax = oracle.calib_absmax(x)
    t["calib_absmax"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    aw = oracle.weight_col_absmax(wt)
    s, inv_s = oracle.smooth_factor(ax, aw, alpha)
    t["smooth_fold"] = time.perf_counter() - t0
    n_s = max(1, min(N, int(round(N * frac))))
    m_s = max(1, min(M, int(round(M * frac))))
    t0 = time.perf_counter()
    wq = oracle.ssz_quant_weight(wt[:n_s], bits=bits, max_iters=max_iters, s=s)
    spent["ssz_quant_weight"] = time.perf_counter() - t0
    t["ssz_quant_weight"] = spent["ssz_quant_weight"] * N / n_s
    t0 = time.perf_counter()
    qx, sx = oracle.quant_act_per_token(x[:m_s], inv_s)
    spent["quant_act_per_token"] = time.perf_counter() - t0
    t["quant_act_per_token"] = spent["quant_act_per_token"] * M / m_s
    t0 = time.perf_counter()
    acc = oracle.gemm_i8(qx, wq["q"])
    oracle.dequant(acc, sx, wq["scale"])
    spent["w8a8_gemm_dequant"] = time.perf_counter() - t0
    t["w8a8_gemm_dequant"] = spent["w8a8_gemm_dequant"] * (M * N) / (m_s * n_s)
    spent["calib_absmax"], spent["smooth_fold"] = t["calib_absmax"], t["smooth_fold"]
    if frac >= 1.0:
        sample = "whole linear (%d tokens x %d -> %d)" % (M, K, N)
    else:
        sample = ("%d tokens x %d -> %d: calibration and weight absmax in full; SSZ on %d of %d channels, "
                  "activation quantization on %d of %d tokens, GEMM+dequant on their %dx%d block; each scaled "
                  "to the full linear" % (M, K, N, n_s, N, m_s, M, m_s, n_s))
    return t, sample, spent


_INPUTS = {}


def _oracle_inputs(cfg):
    import synthetic
    if cfg.name not in _INPUTS:
        x, wt = synthetic.make_linear(cfg, seed=0)
        _INPUTS[cfg.name] = (x.float().numpy(), wt.float().numpy())
    return _INPUTS[cfg.name]


def _gpt_sample_inputs():
    """Layer 0 of the GPT-345M-shaped harness on the CPU over one of the 8
    sequences (1024 tokens): the four linears' inputs and weights."""
    if GPT_WORKLOAD not in _INPUTS:
        import torch
        from synthetic import gpt
        weights = gpt.make_weights(0, "cpu")
        cap = {}
        gpt.forward(weights, gpt.make_tokens(0)[:1], capture=cap, layers=1)
        _INPUTS[GPT_WORKLOAD] = [(cap[(0, n)].float().numpy(), weights[(0, n)].float().numpy()) for n in gpt.LINEARS]
        del weights, torch
    return _INPUTS[GPT_WORKLOAD]


def oracle_workload(workload, frac=1.0):
    """The oracle on one step of a workload: (int8 ops per step, per-stage
    seconds scaled to the full step, sample description, per-stage seconds
    actually spent).  The GPT-345M
    workload is sampled as layer 0 over one sequence, its token-proportional
    stages (calibration, activation quantization, GEMM) scaled by 8 to the
    8 x 1024 batch and every stage by the 24 layers."""
    import synthetic
    if workload == GPT_WORKLOAD:
        from synthetic import gpt
        tot, descs, spent = {}, [], {}
        for x, wt in _gpt_sample_inputs():
            t, d, sp = oracle_linear_times(x, wt, 0.5, 8, 20, frac)
            for k, v in sp.items():
                spent[k] = spent.get(k, 0.0) + v
            for k, v in t.items():
                per_token = k in ("calib_absmax", "quant_act_per_token", "w8a8_gemm_dequant")
                tot[k] = tot.get(k, 0.0) + v * gpt.LAYERS * (gpt.BATCH if per_token else 1)
            descs.append(d)
        sample = ("layer 0 of the GPT-345M-shaped harness over 1 of 8 sequences (" + "; ".join(descs) +
                  "); token-proportional stages x8, all stages x24 layers")
        return gpt.flops_per_pass(), tot, sample, spent
    cfg = synthetic.CONFIGS[workload]
    x, wt = _oracle_inputs(cfg)
    t, sample, spent = oracle_linear_times(x, wt, cfg.alpha, cfg.bits, cfg.max_iters, frac)
    return 2.0 * cfg.M * cfg.N * cfg.K, t, sample, spent


def oracle_metric(ops, t):
    """(linear TOPS, whole-path TOPS) of the oracle's per-stage seconds."""
    lin = t["quant_act_per_token"] + t["w8a8_gemm_dequant"]
    return ops / lin / 1e12, ops / sum(t.values()) / 1e12


def oracle_frac(workload, seconds):
    """The sample fraction that makes one oracle step take about `seconds`:
    a 1/64 probe, then fixed + (SSZ + act) f + GEMM f^2 = seconds (the GEMM
    runs on an f M x f N block, the row-sampled stages on f of their rows)."""
    f0 = 1.0 / 64
    _, _, _, t = oracle_workload(workload, frac=f0)  # seconds spent on the probe
    c = t["calib_absmax"] + t["smooth_fold"] - seconds  # always run in full
    b = (t["ssz_quant_weight"] + t["quant_act_per_token"]) / f0
    a = t["w8a8_gemm_dequant"] / (f0 * f0)
    f = (-b + (b * b - 4 * a * c) ** 0.5) / (2 * a) if a > 0 else -c / max(b, 1e-9)
    return min(1.0, max(1.0 / 1024, f))


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(workload):
    """The oracle as it stands on the host cores, one step of the workload
    sampled to about 15 s, in the bench's metric."""
    frac = oracle_frac(workload, 15.0)
    ops, t, sample, _ = oracle_workload(workload, frac)
    lin, path = oracle_metric(ops, t)
    return {"value": round(lin, 6), "unit": "TOPS", "cores": cores(), "kind": "oracle", "sample": sample,
            "path_tops": round(path, 6), "seconds_per_step": round(sum(t.values()), 3),
            "stage_seconds": {k: round(v, 3) for k, v in t.items()}}


def run_reference(args, rank):
    """The oracle as it stands, timed on the host cores in the bench's
    metric.  Each step is a sample of the workload sized so that warm-up +
    steps take about two minutes; its times are scaled to one full step."""
    if rank != 0:
        return None
    frac = oracle_frac(args.workload, 120.0 / max(1, args.warmup + args.steps))
    steps = []
    for _ in range(args.warmup + args.steps):
        ops, t, sample, _ = oracle_workload(args.workload, frac)
        steps.append(t)
    timed = steps[args.warmup:]
    tot = {k: sum(t[k] for t in timed) for k in timed[0]}
    lin, path = oracle_metric(ops * len(timed), tot)
    return {
        "impl": "reference",
        "metric": "W8A8 linear INT8 TOPS (% of peak); quant/SSZ GB/s (% of HBM) on 1 B200",
        "value": lin, "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(tot.values()) / len(timed), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8 codes, int32 acc, fp32 decisions, fp64 sums (CPU)",
        "data": "synthetic", "config": {"workload": args.workload},
        "value_definition": "2*M*N*K over the oracle's activation quantization + GEMM+dequant time",
        "path": {"tops": path},
        "cpu_baseline": {"value": lin, "unit": "TOPS", "cores": cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": lin, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# kernel name prefix in an ncu capture -> step of the path
NCU_KERNELS = [("col_absmax_kernel", None), ("smooth_factor_kernel", "smooth_fold"), ("ssz_kernel", "ssz_quant_weight"),
               ("quant_act_kernel", "quant_act_per_token"), ("w8a8_gemm_kernel", "w8a8_gemm_dequant"),
               ("w8a8_gemm_pair_kernel", "w8a8_gemm_dequant")]


def record_traffic(csv_path, workload):
    """DRAM bytes per launch of each kernel from an ncu capture of this
    bench's workload (all its kernels, or some of them: the others keep their
    earlier records); written with the hash of each kernel's source so the
    numbers are dropped once the kernel changes."""
    import csv
    import collections
    rows = [r for r in csv.reader(open(csv_path)) if r]
    hdr = next(r for r in rows if r[0] == "ID")
    per = collections.defaultdict(lambda: collections.defaultdict(dict))
    for r in rows[rows.index(hdr) + 1:]:
        if len(r) != len(hdr):
            continue
        d = dict(zip(hdr, r))
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "nsecond": 1e-9, "usecond": 1e-6,
                 "msecond": 1e-3}.get(d["Metric Unit"], 1.0)
        per[d["Kernel Name"]][d["ID"]][d["Metric Name"]] = float(d["Metric Value"].replace(",", "")) * scale
    # launches in ID order; a step launches col_absmax twice (X, then W),
    # smooth_factor, ssz, quant_act, gemm
    launches = []
    for kname, ls in per.items():
        for lid, v in ls.items():
            launches.append((int(lid), kname, v))
    launches.sort()
    acc = collections.defaultdict(list)
    n_col = 0
    for _, kname, v in launches:
        if "dram__bytes_read.sum" not in v:
            continue
        t = v["dram__bytes_read.sum"] + v.get("dram__bytes_write.sum", 0.0)
        if "col_absmax_kernel" in kname:
            acc["calib_absmax" if n_col % 2 == 0 else "smooth_fold"].append(t)
            n_col += 1
            continue
        for prefix, step in NCU_KERNELS:
            if step and prefix in kname:
                if step == "smooth_fold" and acc["smooth_fold"]:
                    acc["smooth_fold"][-1] += t  # same step as the preceding W absmax
                else:
                    acc[step].append(t)
    out = {}
    for step, ts in acc.items():
        if ts:
            out[step] = {"bytes_per_launch": int(sum(ts) / len(ts)), "launches": len(ts),
                         "src_sha": source_sha(KERNEL_SOURCES[step])}
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    allw = json.load(open(path)) if os.path.exists(path) else {}
    allw.setdefault(workload, {}).update(out)  # a capture of some kernels keeps the others' records
    with open(path, "w") as f:
        json.dump(allw, f, indent=1, sort_keys=True)
    print(json.dumps(out, indent=1))


def decode_launches():
    """Three w8a8_gemm_dequant then three w4a8_gemm_dequant launches on the
    16 x 8192 -> 28672 decode shape (random codes in the int4 range, seed 0),
    for an ncu capture of the few-token GEMM kernel."""
    import torch

    import w8a8_linear_layers_b200 as w
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(0)
    M, N, K = 16, 28672, 8192
    qx = torch.randint(-127, 128, (M, K), device=dev, dtype=torch.int8, generator=g)
    qw = torch.randint(-7, 8, (N, K), device=dev, dtype=torch.int8, generator=g)
    sx = torch.rand(M, device=dev, generator=g) * 1e-2
    sw = torch.rand(N, device=dev, generator=g) * 1e-2
    packed = torch.empty(N, K // 2, device=dev, dtype=torch.uint8)
    w.sq_pack_int4(qw, packed)
    y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
    for _ in range(3):
        w.w8a8_gemm_dequant(qx, sx, qw, sw, y)
    for _ in range(3):
        w.w4a8_gemm_dequant(qx, sx, packed, sw, y)
    torch.cuda.synchronize()
    if w.device_fault() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait")


GEMM_SWEEP = ([(8192, k, 1024) for k in (128, 256, 512, 1024, 2048, 4096, 8192)]
              + [(m, 1024, 1024) for m in (512, 2048, 4096, 6144, 10240, 16384, 32768)]
              + [(2048, 4096, 4096), (8192, 4096, 1024)])


def gemm_sweep(mode, rep=20, replays=8):
    """The int8 GEMM + dequant alone on random codes (seed 0) of each
    GEMM_SWEEP shape (M, K, N).  Back-to-back launches in one CUDA graph
    show the per-launch cost a chain of linears pays (launch, prologue,
    pipeline fill, final epilogue) beside the main loop's; torch._int_mm
    beside it is the library's int8 GEMM (no dequant, int32 out), a
    ceiling for comparison only."""
    import torch

    import w8a8_linear_layers_b200 as w
    dev = "cuda"
    for M, K, N in GEMM_SWEEP:
        g = torch.Generator(device=dev).manual_seed(0)
        qx = torch.randint(-127, 128, (M, K), device=dev, dtype=torch.int8, generator=g)
        qw = torch.randint(-127, 128, (N, K), device=dev, dtype=torch.int8, generator=g)
        sx = torch.rand(M, device=dev, generator=g) * 1e-2
        sw = torch.rand(N, device=dev, generator=g) * 1e-2
        y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        if mode == "launch":
            for _ in range(2):
                w.w8a8_gemm_dequant(qx, sx, qw, sw, y)
            torch.cuda.synchronize()
            continue
        line = dict(M=M, K=K, N=N)
        for name, fn in (("w8a8_gemm_dequant", lambda: w.w8a8_gemm_dequant(qx, sx, qw, sw, y)),
                         ("library_int_mm", lambda: torch._int_mm(qx, qw.t()))):
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                for _ in range(3):
                    fn()
            torch.cuda.current_stream().wait_stream(s)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(rep):
                    fn()
            ts = []
            for _ in range(replays):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                e0.record()
                graph.replay()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3 / rep)
            del graph
            us = sorted(ts)[len(ts) // 2]
            line[name] = dict(us=round(us, 2), tops=round(2.0 * M * N * K / us / 1e6, 1))
        print(json.dumps(line), flush=True)
    if w.device_fault() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait")


def next_row_launches():
    """The asymmetric SSZ (twice), then the int4 SSZ, its packing and three
    W4A8 GEMMs on the 8192 x 4096 -> 11008 MLP up-projection inputs (seed 0,
    alpha 0.8, 20 rounds), for ncu captures of those kernels."""
    import torch

    import synthetic
    import w8a8_linear_layers_b200 as w
    cfg = synthetic.CONFIGS[DEFAULT_WORKLOAD]
    x_cpu, w_cpu = synthetic.make_linear(cfg, seed=0)
    x, wt = x_cpu.cuda(), w_cpu.cuda()
    M, K = x.shape
    N = wt.shape[0]
    f32 = dict(device="cuda", dtype=torch.float32)
    ax, aw, s, inv_s = (torch.empty(K, **f32) for _ in range(4))
    w.sq_calib_absmax(x, ax)
    w.sq_smooth_fold(ax, wt, cfg.alpha, aw, s, inv_s)
    q = torch.empty(N, K, device="cuda", dtype=torch.int8)
    sw, ow = torch.empty(N, **f32), torch.empty(N, **f32)
    for _ in range(2):
        w.ssz_quant_weight_asym(wt, s, 20, q, sw, ow)
    w.ssz_quant_weight(wt, s, 4, 20, q, sw)
    packed = torch.empty(N, K // 2, device="cuda", dtype=torch.uint8)
    w.sq_pack_int4(q, packed)
    qx = torch.empty(M, K, device="cuda", dtype=torch.int8)
    sx = torch.empty(M, **f32)
    w.quant_act_per_token(x, inv_s, qx, sx)
    y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    for _ in range(3):
        w.w4a8_gemm_dequant(qx, sx, packed, sw, y)
    torch.cuda.synchronize()
    if w.device_fault() != 0:
        raise RuntimeError("a kernel gave up on a bounded wait")


def main():
    args = parse()
    if args.next_row_launches:
        next_row_launches()
        return
    if args.gemm_sweep:
        gemm_sweep(args.gemm_sweep)
        return
    if args.decode_launches:
        decode_launches()
        return
    if args.record_traffic:
        record_traffic(args.record_traffic, args.workload)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores()))
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.workload)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
