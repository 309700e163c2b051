#!/usr/bin/env python
"""Benchmark of the MXFP4 W4A4 linear layer on B200: quantize activations + block-scaled GEMM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mxq|reference] [--workload NAME]

One step = one mxq_linear call over one batch of the prefill gate+up problem
(A [8192, 5120] bf16 -> MXFP4 CEIL per token, W [34816, 5120] pre-quantized MXFP4 EVEN, bf16 out):
dynamic activation quantization (block amax, scale, encode, pack, swizzled scales) and the
tcgen05 GEMM with its bf16 epilogue.  The metric is 2*M*N*K / step time, in TFLOP/s.

Per rank the working set (A 84 MB + W 95 MB read, 570 MB written per step) is larger than the
126 MB L2, so no separate L2 flush is done between steps; workloads smaller than the L2 (decode)
rotate through copies of the weights instead.  Under torchrun every rank runs its own
copy of the problem (weak scaling, no collective on the data path); the timed region is bracketed
by a barrier + synchronize and the max over ranks is reported.

`--impl reference` times the scalar CPU oracle (quantize + fp64 GEMM) on a bounded sample of the
same problem on the host cores, in the same unit.
"""
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

from nvfp4_block_scaled_mx_b200 import synth  # noqa: E402

METRIC = "MXFP4 W4A4 linear TFLOPS (act-quant+GEMM) and quantize GB/s vs B200 peaks"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
FP4_PER_BF16 = 4.0   # nominal dense fp4 : bf16 tensor throughput (9 : 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0
# algorithmic bytes per element of the quantizer: 2 B read + elements written + scale bytes
QUANT_BYTES_PER_ELEM = {"mxfp4": 2.0 + 0.5 + 1 / 32, "nvfp4": 2.0 + 0.5 + 1 / 16, "mxfp8": 2.0 + 1.0 + 1 / 32}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mxq", choices=["mxq", "reference"])
    ap.add_argument("--workload", default="prefill_gate_up")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-others", action="store_true", help="skip the informational other-problem timings")
    ap.add_argument("--M", type=int, default=None, help="override the workload's M (profiling runs)")
    ap.add_argument("--N", type=int, default=None, help="override the workload's N (profiling runs)")
    ap.add_argument("--op", default="linear",
                    choices=["linear", "w4a16", "quantize", "fake_quantize", "scaled_mm"],
                    help="time one kernel alone on the workload's shape and print its own JSON line, not the "
                         "benchmark line (profiling runs): w4a16 = the weight-only GEMM; quantize / "
                         "fake_quantize = the activation quantizer / fake quantizer on A [M, K]; scaled_mm = "
                         "the block-scaled GEMM beside torch's cuBLASLt scaled_mm on the same bytes (context)")
    ap.add_argument("--fmt", default="mxfp4", choices=["mxfp4", "nvfp4", "mxfp8"],
                    help="format of --op w4a16 (weights; mxfp4 or nvfp4), quantize and fake_quantize")
    ap.add_argument("--rule", default="ceil", choices=["even", "ceil"], help="MX scale rule of --op quantize / "
                    "fake_quantize")
    return ap.parse_args()


def peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def sustained_bf16_tflops():
    """The measured bf16 GEMM rate in a seconds-long loop under the power cap (None if unknown)."""
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as fh:
            v = json.load(fh).get("bf16_tflops_sustained")
        return float(v) if v else None
    return None


def traffic_for(key):
    if os.path.exists(TRAFFIC_PATH):
        with open(TRAFFIC_PATH) as fh:
            return json.load(fh).get(key)
    return None


# ---------------------------------------------------------------- distributed plumbing

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device):
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_weak(per_rank_units, world):
    """Whole-job units: every rank processes the same per-rank amount (weak scaling)."""
    return per_rank_units * world


# ---------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        num = lambda v: float(v) if v.strip().replace(".", "").isdigit() else None
        smp = [(num(r[1]), num(r[3])) for r in rows]
        smp = [(c, w) for c, w in smp if c is not None and w is not None]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        # the samples under load (power draw at least half the window's maximum); the idle moments
        # before and after the timed region run at the top clock and would hide a power-capped clock
        top = max((w for _, w in smp), default=0.0)
        load = [c for c, w in smp if w >= 0.5 * top]
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": top if smp else None}


# ---------------------------------------------------------------- the mxq arm

def time_loop(fn, iters, stream):
    """Average device time of fn() over iters launches, CUDA events on `stream`."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(iters):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / iters / 1e3


def l2_flush_buffer(device):
    """512 MB for time_flushed: a 256 MB half that is written and a 256 MB half that is read."""
    return torch.zeros(512 << 20, dtype=torch.uint8, device=device)


def time_flushed(fn, iters, stream, flush):
    """Median device time of fn() with the L2 flushed before each launch: a 256 MB write (twice the
    126 MB L2), then a 256 MB read of other memory, which writes the flush's dirty lines back to HBM
    before the timed launch starts, so that the launch meets a cold, clean L2."""
    half = flush.numel() // 2
    ts = []
    for _ in range(iters):
        flush[:half].zero_()
        flush[half:].view(torch.int32).sum()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        fn()
        end.record(stream)
        end.synchronize()
        ts.append(start.elapsed_time(end) / 1e3)
    return sorted(ts)[len(ts) // 2]


def run_mxq(args, world, rank, local):
    from nvfp4_block_scaled_mx_b200 import mxq
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl mxq needs a CUDA device (there is no CPU fallback)")
    dev = torch.device("cuda", local)
    cfg = synth.CONFIGS[args.workload]
    M = args.M or cfg["M"]
    N = args.N or cfg["N"]
    K, fmt = cfg["K"], cfg["fmt"]
    workload = args.workload if (M, N) == (cfg["M"], cfg["N"]) else "%s(M=%d,N=%d)" % (args.workload, M, N)
    stream = torch.cuda.current_stream(dev)
    hbm_gbs, bf16_tflops, peak_src = peaks()

    A, W = synth.make_inputs(args.workload, device=dev, M=M, N=N)
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        g_a, _ = mxq.global_scale(A)
    W_q, W_sf = mxq.quantize(W, fmt, cfg["w_rule"], global_scale=g_w, layout=mxq.SF_SWIZZLED)
    ws = torch.empty(mxq.mxq_linear_workspace_size(M, K, mxq.FMT[fmt]), dtype=torch.uint8, device=dev)
    out_dtype = torch.float32 if cfg["out"] == "fp32" else torch.bfloat16
    out = torch.empty(M, N, dtype=out_dtype, device=dev)
    flops = 2.0 * M * N * K
    # a working set smaller than the L2: consecutive steps read different copies of the larger
    # operand (together more than twice the L2) -- the weights at decode, as consecutive layers of a
    # model do (the activations stay L2-resident, as a previous layer leaves them), the bf16
    # activations of a few-column layer -- so that every step streams it from HBM
    L2_BYTES = 126 << 20
    wbytes = W_q.numel() + W_sf.numel()
    abytes = A.numel() * A.element_size()
    working = wbytes + abytes + out.numel() * out.element_size()
    rotate_a = working <= L2_BYTES and abytes > wbytes
    copies = 1 if working > L2_BYTES else -(-2 * L2_BYTES // (abytes if rotate_a else wbytes))
    wset = [(W_q, W_sf)] + ([] if rotate_a else [(W_q.clone(), W_sf.clone()) for _ in range(copies - 1)])
    aset = [A] + ([A.clone() for _ in range(copies - 1)] if rotate_a else [])
    if copies == 1:
        l2_note = "working set > 126 MB L2, no flush"
    elif rotate_a:
        l2_note = ("bf16 activations rotate through %d copies (%.0f MB > 2 x L2) between steps; weights "
                   "L2-resident" % (copies, copies * abytes / 1e6))
    else:
        l2_note = ("weights rotate through %d copies (%.0f MB > 2 x L2) between steps; activations L2-resident" % (
            copies, copies * wbytes / 1e6))
    it = [0]

    def operands(i):
        return aset[i % len(aset)], wset[i % len(wset)]

    def step():
        x, (wq, wsf) = operands(it[0])
        it[0] += 1
        mxq.linear(x, wq, wsf, N, fmt, act_rule=cfg["a_rule"], out_dtype=out_dtype, g_W=g_w, g_A=g_a,
                   workspace=ws, out=out, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    mxq.mxq_device_status(reset=True)

    timing = "eager calls through the binding"

    def run_steps(n):
        for _ in range(n):
            step()

    one_launch = mxq.linear_kernel_count(M, N, K, fmt) == 1
    if one_launch:
        # one launch per call (few tokens, or few columns): a call is microseconds of GPU work, not
        # much more than the host needs to launch it through the Python binding (about 12 us) or to
        # replay a one-call CUDA graph (about 2.5 us of launch gap per replay), so the steps run from
        # CUDA graphs of consecutive calls, each call on the next operand copy, as serving replays
        # one graph over a step's layers; every step is still one full call (its operands from HBM,
        # its activations quantized, its output stored)
        gs = torch.cuda.Stream(device=dev)
        torch.cuda.synchronize()

        def capture(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gs):
                for i in range(n):
                    x, (wq, wsf) = operands(i)
                    mxq.linear(x, wq, wsf, N, fmt, act_rule=cfg["a_rule"], out_dtype=out_dtype, g_W=g_w, g_A=g_a,
                               workspace=ws, out=out)
            return g

        per_graph = copies * -(-16 // copies)  # a whole number of weight-copy rotations, at least 16 calls
        graphs = {per_graph: capture(per_graph)}

        def run_steps(n):
            # exactly n calls: whole graphs of per_graph calls, then one graph of the remainder
            for _ in range(n // per_graph):
                graphs[per_graph].replay()
            r = n % per_graph
            if r:
                if r not in graphs:
                    graphs[r] = capture(r)
                graphs[r].replay()

        run_steps(max(3, args.warmup))
        run_steps(args.steps % per_graph)  # capture the remainder graph outside the timed region
        torch.cuda.synchronize()
        timing = ("CUDA graphs of %d consecutive calls (each on the next operand copy), %d steps in all; the host "
                  "launch cost stays outside the measurement" % (per_graph, args.steps))

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        start.record(stream)
        run_steps(args.steps)
        end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    elapsed = start.elapsed_time(end) / 1e3
    status = mxq.mxq_device_status(reset=True)
    if status != 0:
        raise SystemExit("a kernel reported a bounded-wait timeout (status 0x%x)" % status)
    elapsed_max = max_over_ranks(elapsed, world, dev)
    value = aggregate_weak(flops * args.steps, world) / elapsed_max / 1e12

    # dominant kernel timed alone: the GEMM on the step's own quantized activations
    a_q = ws[: M * K // 2].view(M, K // 2) if fmt != "mxfp8" else ws[: M * K].view(M, K)
    qbytes = a_q.numel()
    a_sf = ws[(qbytes + 255) // 256 * 256:]
    gemm_s = time_loop(lambda: mxq.gemm(a_q, a_sf, W_q, W_sf, M, N, K, fmt, out_dtype=out_dtype, g_A=g_a, g_B=g_w,
                                        out=out, stream=stream), max(10, args.steps // 4), stream)
    # the quantizers are timed one launch at a time with the 126 MB L2 flushed before each
    flush = l2_flush_buffer(dev)
    quant_s = time_flushed(lambda: mxq.quantize(A, fmt, cfg["a_rule"], global_scale=g_a, layout=mxq.SF_SWIZZLED,
                                                q_out=a_q, sf_out=a_sf, stream=stream), 20, stream, flush)
    tensor_peak = bf16_tflops * (FP8_PER_BF16 if fmt == "mxfp8" else FP4_PER_BF16)
    gemm_tflops = flops / gemm_s / 1e12
    kind = {"mxfp4": "mxf4", "nvfp4": "mxf4nvf4", "mxfp8": "mxf8f6f4"}[fmt]
    roofline = {"bound": "tensor", "kernel": ("gemm_pair_kernel (tcgen05 cta_group::2 kind::%s)" if M > 128 else
                                              "gemm_kernel (tcgen05 kind::%s)") % kind,
                "achieved": round(gemm_tflops, 1), "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
                "frac": round(gemm_tflops / tensor_peak, 4),
                "peak_source": "%s bf16 %.1f TFLOP/s x %g nominal %s:bf16 ratio" % (
                    peak_src, bf16_tflops, FP4_PER_BF16 if fmt != "mxfp8" else FP8_PER_BF16, fmt),
                "frac_of_datasheet": round(gemm_tflops / (9000.0 if fmt != "mxfp8" else 4500.0), 4),
                "frac_of_sustained_peak": (round(gemm_tflops / (sustained_bf16_tflops() * (FP8_PER_BF16 if fmt == "mxfp8"
                                                                                           else FP4_PER_BF16)), 4)
                                           if sustained_bf16_tflops() else None),
                "traffic": traffic_for("gemm_%s_%s" % (fmt, workload)),
                "algorithmic_flops_per_launch": flops, "ms_per_launch": round(gemm_s * 1e3, 4)}
    if M <= 128 or one_launch:
        # few tokens or few columns: the layer streams its weights (few tokens) or its bf16 activations
        # (few columns) once and is HBM-bound.  Timed with the L2 flushed before each launch, as the
        # linear call itself when that is one launch (the GEMM quantizing its own activations: bf16
        # rows in), else as the GEMM on quantized activations
        if one_launch:
            # one launch per step: its average duration is the timed region's per step, with the
            # weights streamed from HBM (rotating copies) or a working set larger than the L2
            lin_cold = time_flushed(lambda: mxq.linear(A, W_q, W_sf, N, fmt, act_rule=cfg["a_rule"], out_dtype=out_dtype,
                                                       g_W=g_w, g_A=g_a, workspace=ws, out=out, stream=stream),
                                    20, stream, flush)
            lin_s = elapsed / args.steps
            gbytes = W_q.numel() + W_sf.numel() + 2 * M * K + out.numel() * out.element_size()
            kname = ("gemm_decode_kernel (tcgen05 kind::%s, few tokens, activations quantized in the kernel)" if M <= 32
                     else "gemm_rowq_kernel (tcgen05 kind::%s, few columns, activations quantized in the kernel)") % kind
        else:
            lin_cold = time_flushed(lambda: mxq.gemm(a_q, a_sf, W_q, W_sf, M, N, K, fmt, out_dtype=out_dtype, g_A=g_a,
                                                     g_B=g_w, out=out, stream=stream), 20, stream, flush)
            lin_s = lin_cold
            gbytes = W_q.numel() + W_sf.numel() + a_q.numel() + a_sf.numel() + out.numel() * out.element_size()
            kname = "gemm_splitk_kernel / gemm_kernel (tcgen05 kind::%s, few tokens)" % kind
        roofline = {"bound": "hbm", "kernel": kname,
                    "achieved": round(gbytes / lin_s / 1e9, 1), "peak": round(hbm_gbs, 1), "unit": "GB/s",
                    "frac": round(gbytes / lin_s / 1e9 / hbm_gbs, 4), "peak_source": "%s HBM copy" % peak_src,
                    "traffic": traffic_for("linear_%s_%s" % (fmt, workload)) if one_launch else None,
                    "algorithmic_bytes_per_launch": gbytes, "ms_per_launch": round(lin_s * 1e3, 4),
                    "l2": ("average launch over the timed region (%s)" % l2_note if one_launch else
                           "flushed per launch (the launch latency is inside the time)"),
                    "ms_single_launch_l2_flushed": round(lin_cold * 1e3, 4)}
    qb = QUANT_BYTES_PER_ELEM[fmt] * M * K
    quant = {"workload": "activation quantize %dx%d %s %s" % (M, K, fmt, cfg["a_rule"]),
             "gbs": round(qb / quant_s / 1e9, 1), "frac": round(qb / quant_s / 1e9 / hbm_gbs, 4),
             "peak_gbs": hbm_gbs, "ms": round(quant_s * 1e3, 4), "algorithmic_bytes": qb, "l2": "flushed per launch"}
    fq_out = torch.empty_like(A)
    fq_s = time_flushed(lambda: mxq.fake_quantize(A, fmt, cfg["a_rule"], global_scale=g_a, out=fq_out, stream=stream),
                        20, stream, flush)
    fake_quant = {"workload": "fake quantize (quantize-dequantize to bf16) %dx%d %s %s" % (M, K, fmt, cfg["a_rule"]),
                  "gbs": round(4.0 * M * K / fq_s / 1e9, 1), "frac": round(4.0 * M * K / fq_s / 1e9 / hbm_gbs, 4),
                  "ms": round(fq_s * 1e3, 4), "algorithmic_bytes_per_elem": 4.0, "l2": "flushed per launch"}
    del fq_out

    # weight (RTN, EVEN) quantizer on the 451 MB weight tensor
    wq_s = time_flushed(lambda: mxq.quantize(W, fmt, cfg["w_rule"], global_scale=g_w, layout=mxq.SF_SWIZZLED,
                                             q_out=W_q, sf_out=W_sf, stream=stream), 10, stream, flush)
    del flush
    wb = QUANT_BYTES_PER_ELEM[fmt] * N * K
    quant_w = {"workload": "weight quantize %dx%d %s %s" % (N, K, fmt, cfg["w_rule"]),
               "gbs": round(wb / wq_s / 1e9, 1), "frac": round(wb / wq_s / 1e9 / hbm_gbs, 4), "peak_gbs": hbm_gbs,
               "ms": round(wq_s * 1e3, 4)}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(lambda a, o, st: mxq.linear(a, W_q, W_sf, N, fmt, act_rule=cfg["a_rule"], out_dtype=out_dtype,
                                                  g_W=g_w, g_A=g_a, workspace=ws, out=o, stream=st),
                      A, out, flops, args, world, dev)
    # full-size bf16 inputs for the oracle quantizer timing of the CPU baseline (rank 0, N = 1)
    host_inputs = (A.cpu(), W.cpu()) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else (None, None)
    others = None
    if not args.no_others and world == 1:
        del A, W, W_q, W_sf, ws, out
        torch.cuda.empty_cache()
        others = other_workloads(stream, bf16_tflops)

    res = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(elapsed_max / args.steps * 1e3, 4), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "e2m1xe2m1->f32 (bf16 out)" if fmt != "mxfp8" else
           "e4m3xe4m3->f32 (bf16 out)", "data": "synthetic (seeded, random-init weights)",
           "config": {"workload": workload, "M": M, "N": N, "K": K, "fmt": fmt, "act_rule": cfg["a_rule"],
                      "weight_rule": cfg["w_rule"], "out": cfg["out"], "l2": l2_note, "timing": timing,
                      "parallelism": "replicas x%d (no collective)" % world},
           "gpu_launches": mxq.linear_kernel_count(M, N, K, fmt) * args.steps, "roofline": roofline, "quantize": quant, "quantize_weight": quant_w,
           "fake_quantize": fake_quant,
           "clocks": clk.summary(), "e2e": e2e, "other_workloads": others}
    return res, host_inputs


def other_workloads(stream, bf16_tflops):
    """mxq_linear on the remaining problems (decode, NVFP4 down-proj, MXFP8 attention, lm_head, N = 96)
    and the weight-only GEMM on the prefill and decode shapes: device-resident inputs, CUDA events,
    informational (the headline is the prefill problem)."""
    from nvfp4_block_scaled_mx_b200 import mxq
    res = {}
    for name in ["decode", "down_nvfp4", "attn_mxfp8", "lm_head", "in_proj_ba"]:
        cfg = synth.CONFIGS[name]
        M, N, K, fmt = cfg["M"], cfg["N"], cfg["K"], cfg["fmt"]
        A, W = synth.make_inputs(name, device="cuda")
        g_w = g_a = None
        if fmt == "nvfp4":
            g_w, _ = mxq.global_scale(W)
            g_a, _ = mxq.global_scale(A)
        W_q, W_sf = mxq.quantize(W, fmt, cfg["w_rule"], global_scale=g_w)
        del W
        ws = torch.empty(mxq.mxq_linear_workspace_size(M, K, mxq.FMT[fmt]), dtype=torch.uint8, device="cuda")
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        f = lambda: mxq.linear(A, W_q, W_sf, N, fmt, act_rule=cfg["a_rule"], g_W=g_w, g_A=g_a, workspace=ws, out=out,
                               stream=stream)
        qr = {}
        if name == "down_nvfp4":
            # NVFP4 running-max observer quantizer on the 365 MB activation tensor, timed before the
            # GEMM loop: right after a few hundred milliseconds of dense NVFP4 GEMM the SM clock is
            # still power-capped (about 1.45 GHz), which costs this quantizer's per-block divisions
            # about 12 %
            st_in = torch.tensor([float(mxq.global_scale(A)[1].item())], dtype=torch.float32, device="cuda")
            st_out = torch.empty(1, dtype=torch.float32, device="cuda")
            q, sf = mxq.quantize_running(A, st_in, st_out)
            flush = l2_flush_buffer("cuda")
            tq = time_flushed(lambda: mxq.quantize_running(A, st_in, st_out, q_out=q, sf_out=sf, stream=stream), 10,
                              stream, flush)
            qr["quantize_running_gbs"] = round(QUANT_BYTES_PER_ELEM["nvfp4"] * M * K / tq / 1e9, 1)
            # the plain NVFP4 activation quantizer (static global scale) on the same tensor
            tq = time_flushed(lambda: mxq.quantize(A, "nvfp4", global_scale=g_a, q_out=q, sf_out=sf, stream=stream), 10,
                              stream, flush)
            qr["quantize_gbs"] = round(QUANT_BYTES_PER_ELEM["nvfp4"] * M * K / tq / 1e9, 1)
            qr["quantize_frac_of_measured_hbm"] = round(qr["quantize_gbs"] / peaks()[0], 4)
            qr["quantize_l2"] = "flushed per launch, timed before the GEMM loop"
            del q, sf, flush
        for _ in range(3):
            f()
        calls = 1
        if M <= 32:  # few tokens: graphs of 16 calls, as for the decode bench (host launch cost outside)
            calls = 16
            gs = torch.cuda.Stream()
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=gs):
                for _ in range(calls):
                    mxq.linear(A, W_q, W_sf, N, fmt, act_rule=cfg["a_rule"], g_W=g_w, g_A=g_a, workspace=ws, out=out)
            f = gr.replay
            for _ in range(3):
                f()
        iters = 200 if M * N < 1e8 else 30
        t = time_loop(f, max(1, iters // calls), stream) / calls
        peak = bf16_tflops * (FP8_PER_BF16 if fmt == "mxfp8" else FP4_PER_BF16)
        r = {"M": M, "N": N, "K": K, "fmt": fmt, "ms": round(t * 1e3, 4), "tflops": round(2.0 * M * N * K / t / 1e12, 1),
             "frac_of_measured_peak": round(2.0 * M * N * K / t / 1e12 / peak, 4)}
        if name == "decode":  # weight-stream bound: codes + scales of W per call
            wbytes = W_q.numel() + W_sf.numel()
            r["weight_gbs"] = round(wbytes / t / 1e9, 1)
            r["l2"] = ("CUDA graphs of 16 calls on one weight copy (L2-resident); --workload decode streams them from "
                       "HBM")
        if name == "in_proj_ba":
            r["l2"] = ("back-to-back eager calls on one activation tensor (84 MB, partly L2-resident); --workload "
                       "in_proj_ba streams rotating copies from HBM")
        r.update(qr)
        res[name] = r
        del A, W_q, W_sf, ws, out
        torch.cuda.empty_cache()
    # weight-only (W4A16): bf16 activations times the same MXFP4 weights, on the prefill gate+up and
    # decode shapes; tensor-bound against the measured bf16 peak at prefill, weight-stream-bound at decode
    for name in ["prefill_gate_up", "decode"]:
        cfg = synth.CONFIGS[name]
        M, N, K = cfg["M"], cfg["N"], cfg["K"]
        A, W = synth.make_inputs(name, device="cuda")
        W_q, W_sf = mxq.quantize(W, "mxfp4", "even")
        del W
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        f = lambda: mxq.gemm_w4a16(A, W_q, W_sf, N, "mxfp4", out=out, stream=stream)
        for _ in range(3):
            f()
        calls = 1
        if M <= 32:  # few tokens: graphs of 16 calls (host launch cost outside)
            calls = 16
            gs = torch.cuda.Stream()
            torch.cuda.synchronize()
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=gs):
                for _ in range(calls):
                    mxq.gemm_w4a16(A, W_q, W_sf, N, "mxfp4", out=out)
            f = gr.replay
            for _ in range(3):
                f()
        t = time_loop(f, max(1, (200 if M * N < 1e8 else 10) // calls), stream) / calls
        r = {"M": M, "N": N, "K": K, "fmt": "mxfp4 weights, bf16 activations", "ms": round(t * 1e3, 4),
             "tflops": round(2.0 * M * N * K / t / 1e12, 1),
             "frac_of_measured_bf16": round(2.0 * M * N * K / t / 1e12 / bf16_tflops, 4)}
        if name == "decode":
            r["weight_gbs"] = round((W_q.numel() + W_sf.numel()) / t / 1e9, 1)
            r["l2"] = "CUDA graphs of 16 calls on one weight copy (L2-resident)"
        res["w4a16_" + name] = r
        del A, W_q, W_sf, out
        torch.cuda.empty_cache()
    return res


def run_e2e(linear_into, A, out, flops, args, world, dev):
    """The same step through host buffers: every step copies its activations in from pinned host
    memory and its bf16 output back to pinned host memory.  Consecutive steps are pipelined on
    three streams (upload of step i+1 and download of step i-1 overlap the linear of step i) with
    two device buffers each way; the timed region runs from the first upload to the last download."""
    iters = max(4, min(24, args.steps // 10))
    A_h = [torch.empty(A.shape, dtype=A.dtype, pin_memory=True) for _ in range(2)]
    for h in A_h:
        h.copy_(A)
    out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    A_d = [A, torch.empty_like(A)]
    out_d = [out, torch.empty_like(out)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_ready = [ev(), ev()]
    comp_done = [ev(), ev()]
    out_done = [ev(), ev()]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(comp_done[b])     # A_d[b] is free once step i-2 computed
            with torch.cuda.stream(s_in):
                A_d[b].copy_(A_h[b], non_blocking=True)
            in_ready[b].record(s_in)
            s_comp.wait_event(in_ready[b])
            if i >= 2:
                s_comp.wait_event(out_done[b])    # out_d[b] is free once step i-2 downloaded
            linear_into(A_d[b], out_d[b], s_comp)
            comp_done[b].record(s_comp)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                out_h[b].copy_(out_d[b], non_blocking=True)
            out_done[b].record(s_out)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    start.record(s_in)
    run(iters)
    end.record(s_out)
    torch.cuda.synchronize()
    t = start.elapsed_time(end) / 1e3 / iters
    t = max_over_ranks(t, world, dev)
    return {"value": round(aggregate_weak(flops, world) / t / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": A.numel() * A.element_size(), "d2h_bytes_per_step": out.numel() * out.element_size(),
            "ms_per_step": round(t * 1e3, 3), "pipelined": "upload / linear / download overlapped across steps"}


# ---------------------------------------------------------------- the oracle (CPU) arm

def oracle_sample(workload, rows, cols, seed=0):
    """Inputs of a bounded CPU sample: `rows` activation rows and `cols` weight rows of the problem."""
    cfg = synth.CONFIGS[workload]
    gen = synth.make_generator(1000 * cfg["seed"] + 7 + seed)
    A = synth.draw_matrix(rows, cfg["K"], cfg["a"], gen)
    W = synth.draw_matrix(cols, cfg["K"], cfg["w"], gen)
    return cfg, A, W


def oracle_step(orc, cfg, A, Wq, Wsf, gW, threads=1):
    fmts = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4, "mxfp8": orc.MXFP8}
    rules = {"even": orc.EVEN, "ceil": orc.CEIL}
    f = fmts[cfg["fmt"]]
    gA = 1.0
    if cfg["fmt"] == "nvfp4":
        gA, _ = orc.global_scale(A)
    Aq, Asf = orc.quantize(A, f, rules[cfg["a_rule"]], g=float(gA), threads=threads)
    orc.gemm(Aq, Asf, Wq, Wsf, A.shape[0], Wq.shape[0], cfg["K"], f, gA=float(gA), gB=float(gW), threads=threads)


def cpu_baseline(workload, A_full=None, W_full=None, rows=128, cols=4096):
    """The oracle as it stands, timed on this host's cores: the linear step (quantize a sample of
    activation rows + fp64 GEMM against a sample of quantized weight rows) on one thread and on every
    usable CPU (one POSIX thread per range of output columns), and the oracle quantizer's GB/s over
    the full activation and weight tensors of the workload (all CPUs; activations also on one
    thread).  About 10-30 s of CPU work on a many-core host."""
    import oracle as orc
    orc.build()
    cfg, A, W = oracle_sample(workload, rows, cols)
    fmts = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4, "mxfp8": orc.MXFP8}
    rules = {"even": orc.EVEN, "ceil": orc.CEIL}
    f = fmts[cfg["fmt"]]
    usable, online = orc.cpus_usable(), orc.cpus_online()
    gW = 1.0
    if cfg["fmt"] == "nvfp4":
        gW, _ = orc.global_scale(W)
    Wq, Wsf = orc.quantize(W, f, rules[cfg["w_rule"]], g=float(gW), threads=usable)
    flops = 2.0 * rows * cols * cfg["K"]
    rates = {}
    for threads in (1, usable):
        t0 = time.perf_counter()
        oracle_step(orc, cfg, A, Wq, Wsf, gW, threads=threads)
        dt = time.perf_counter() - t0
        rates[threads] = (flops / dt / 1e12, dt)
    res = {"value": rates[usable][0], "unit": "TFLOP/s", "cores": usable, "host_cpus_online": online,
           "kind": "oracle",
           "sample": "%d activation rows x %d weight rows x K=%d of %s: %s quantize of the rows + fp64 GEMM, "
                     "scalar C on %d threads (%.2f s); host has %d online CPUs, %d usable" % (
                         rows, cols, cfg["K"], workload, cfg["a_rule"].upper(), usable, rates[usable][1], online,
                         usable),
           "single_thread": {"value": rates[1][0], "unit": "TFLOP/s", "cores": 1, "seconds": round(rates[1][1], 2)}}
    qres = {}
    bpe = QUANT_BYTES_PER_ELEM[cfg["fmt"]]
    for which, x, rule, thread_counts in (("activations", A_full, cfg["a_rule"], (1, usable)),
                                          ("weights", W_full, cfg["w_rule"], (usable,))):
        if x is None:
            continue
        g = float(orc.global_scale(x)[0]) if cfg["fmt"] == "nvfp4" else 1.0
        r = {"shape": list(x.shape), "rule": rule}
        for threads in thread_counts:
            t0 = time.perf_counter()
            orc.quantize(x, f, rules[rule], g=g, threads=threads)
            dt = time.perf_counter() - t0
            r["gbs_%s" % ("1_thread" if threads == 1 else "%d_threads" % threads)] = round(bpe * x.numel() / dt / 1e9, 3)
        qres[which] = r
    if qres:
        res["quantize_full_tensors"] = qres
    return res


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle as orc
    orc.build()
    threads = orc.cpus_usable()
    rows, cols = 8, 512
    cfg, A, W = oracle_sample(args.workload, rows, cols)
    fmts = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4, "mxfp8": orc.MXFP8}
    rules = {"even": orc.EVEN, "ceil": orc.CEIL}
    gW = 1.0
    if cfg["fmt"] == "nvfp4":
        gW, _ = orc.global_scale(W)
    Wq, Wsf = orc.quantize(W, fmts[cfg["fmt"]], rules[cfg["w_rule"]], g=float(gW), threads=threads)
    for _ in range(max(1, args.warmup)):
        oracle_step(orc, cfg, A, Wq, Wsf, gW, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(orc, cfg, A, Wq, Wsf, gW, threads=threads)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * cols * cfg["K"]
    value = flops * args.steps / dt / 1e12
    sample = ("per step %d activation rows x %d weight rows x K=%d of %s (quantize rows + fp64 GEMM), "
              "scalar C oracle on %d threads (host: %d online CPUs)" % (rows, cols, cfg["K"], args.workload, threads,
                                                                        orc.cpus_online()))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": args.workload, "M": cfg["M"], "N": cfg["N"],
                                                     "K": cfg["K"], "fmt": cfg["fmt"]},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_w4a16_op(args):
    """Weight-only GEMM alone: bf16 activations of the workload's shape times its weights quantized
    to --fmt, timed warm (back-to-back launches) and with the L2 flushed before each launch."""
    from nvfp4_block_scaled_mx_b200 import mxq
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --op w4a16 needs a CUDA device (there is no CPU fallback)")
    if args.fmt not in ("mxfp4", "nvfp4"):
        raise SystemExit("bench.py --op w4a16 takes --fmt mxfp4 or nvfp4 (4-bit weights)")
    cfg = synth.CONFIGS[args.workload]
    M, N, K = args.M or cfg["M"], args.N or cfg["N"], cfg["K"]
    A = synth.random_bf16((M, K), 71, device="cuda")
    W = synth.random_bf16((N, K), 72, std=0.02, device="cuda")
    g_w = mxq.global_scale(W)[0] if args.fmt == "nvfp4" else None
    W_q, W_sf = mxq.quantize(W, args.fmt, "even", global_scale=g_w)
    del W
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    f = lambda: mxq.gemm_w4a16(A, W_q, W_sf, N, args.fmt, g_W=g_w, out=out, stream=stream)
    for _ in range(max(3, args.warmup)):
        f()
    warm = time_loop(f, args.steps, stream)
    flush = l2_flush_buffer("cuda")
    cold = time_flushed(f, max(3, args.steps), stream, flush)
    wbytes = W_q.numel() + W_sf.numel()
    return {"op": "w4a16", "workload": args.workload, "M": M, "N": N, "K": K, "fmt": args.fmt,
            "warm_ms": round(warm * 1e3, 4), "l2_flushed_ms": round(cold * 1e3, 4),
            "tflops_warm": round(2.0 * M * N * K / warm / 1e12, 1),
            "weight_gbs_l2_flushed": round(wbytes / cold / 1e9, 1)}


def run_quantize_op(args):
    """The activation quantizer (or fake quantizer) alone on A [M, K] of the workload (N(0,1) bf16),
    timed with the L2 flushed before each launch, against the measured HBM bandwidth."""
    from nvfp4_block_scaled_mx_b200 import mxq
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --op %s needs a CUDA device (there is no CPU fallback)" % args.op)
    cfg = synth.CONFIGS[args.workload]
    M, K = args.M or cfg["M"], cfg["K"]
    A = synth.random_bf16((M, K), 73, device="cuda")
    g = mxq.global_scale(A)[0] if args.fmt == "nvfp4" else None
    rule = "even" if args.fmt == "nvfp4" else args.rule
    stream = torch.cuda.current_stream()
    if args.op == "quantize":
        q, sf = mxq.quantize(A, args.fmt, rule, global_scale=g, stream=stream)
        f = lambda: mxq.quantize(A, args.fmt, rule, global_scale=g, q_out=q, sf_out=sf, stream=stream)
        bpe = QUANT_BYTES_PER_ELEM[args.fmt]
    else:
        y = torch.empty_like(A)
        f = lambda: mxq.fake_quantize(A, args.fmt, rule, global_scale=g, out=y, stream=stream)
        bpe = 4.0
    for _ in range(max(3, args.warmup)):
        f()
    flush = l2_flush_buffer("cuda")
    t = time_flushed(f, max(3, args.steps), stream, flush)
    hbm = peaks()[0]
    return {"op": args.op, "M": M, "K": K, "fmt": args.fmt, "rule": rule, "ms": round(t * 1e3, 4),
            "gbs": round(bpe * M * K / t / 1e9, 1), "frac_of_measured_hbm": round(bpe * M * K / t / 1e9 / hbm, 4),
            "algorithmic_bytes_per_elem": bpe, "l2": "flushed per launch"}


def run_scaled_mm_op(args):
    """Context, not a product path: the workload's block-scaled GEMM (activations and weights quantized
    by this library) timed beside torch.nn.functional.scaled_mm, which runs cuBLASLt's block-scaled
    GEMM on the same code and swizzled-scale bytes.  Back-to-back launches, CUDA events.  Also the
    largest difference of the two outputs relative to the largest output (0 when they agree bit for
    bit; NVFP4 differs by where the global scales are applied)."""
    import torch.nn.functional as F
    from nvfp4_block_scaled_mx_b200 import mxq
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --op scaled_mm needs a CUDA device")
    cfg = synth.CONFIGS[args.workload]
    M, N, K, fmt = cfg["M"], cfg["N"], cfg["K"], cfg["fmt"]
    A, W = synth.make_inputs(args.workload, device="cuda")
    g_a = g_w = None
    if fmt == "nvfp4":
        g_w, g_a = mxq.global_scale(W)[0], mxq.global_scale(A)[0]
    Aq, Asf = mxq.quantize(A, fmt, cfg["a_rule"], global_scale=g_a)
    Wq, Wsf = mxq.quantize(W, fmt, cfg["w_rule"], global_scale=g_w)
    del A, W
    stream = torch.cuda.current_stream()
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ours = lambda: mxq.gemm(Aq, Asf, Wq, Wsf, M, N, K, fmt, g_A=g_a, g_B=g_w, out=out, stream=stream)
    elem = torch.float8_e4m3fn if fmt == "mxfp8" else torch.float4_e2m1fn_x2
    sdt = torch.float8_e4m3fn if fmt == "nvfp4" else torch.float8_e8m0fnu
    rec = F.ScalingType.BlockWise1x16 if fmt == "nvfp4" else F.ScalingType.BlockWise1x32
    sw = F.SwizzleType.SWIZZLE_32_4_4
    lib = lambda: F.scaled_mm(Aq.view(elem), Wq.view(elem).t(), Asf.view(sdt), rec, Wsf.view(sdt), rec,
                              swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16)
    for _ in range(max(3, args.warmup)):
        ours()
    t_ours = time_loop(ours, args.steps, stream)
    ref = lib()
    for _ in range(max(3, args.warmup)):
        lib()
    t_lib = time_loop(lib, args.steps, stream)
    ours()
    torch.cuda.synchronize()
    r = ref.float() * (g_a * g_w) if fmt == "nvfp4" else ref.float()
    flops = 2.0 * M * N * K
    return {"op": "scaled_mm", "workload": args.workload, "M": M, "N": N, "K": K, "fmt": fmt,
            "mxq_ms": round(t_ours * 1e3, 4), "mxq_tflops": round(flops / t_ours / 1e12, 1),
            "scaled_mm_ms": round(t_lib * 1e3, 4), "scaled_mm_tflops": round(flops / t_lib / 1e12, 1),
            "max_rel_diff": float((out.float() - r).abs().max() / r.abs().max())}


def main():
    args = parse()
    if args.op == "scaled_mm":
        print(json.dumps(run_scaled_mm_op(args)), flush=True)
        return
    if args.op == "w4a16":
        print(json.dumps(run_w4a16_op(args)), flush=True)
        return
    if args.op in ("quantize", "fake_quantize"):
        print(json.dumps(run_quantize_op(args)), flush=True)
        return
    world, rank, local = dist_init()
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res, host_inputs = run_mxq(args, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(args.workload, *host_inputs)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
