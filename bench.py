"""Benchmark of the NVFP4 linear layer (fprop + dgrad + wgrad with every quantize, RHT and
transpose kernel) at T=8192 tokens, d=5120 in-features, n=20480 out-features on B200s.

One step = nvfp4_linear_fwd (16x16 weight quantization + both activation forms + fprop GEMM)
followed by nvfp4_linear_bwd (both SR gradient forms + dgrad GEMM + wgrad GEMM), on synthetic
inputs resident in HBM.  value = 3 * 2 * T * d * n / step time (TFLOPS), whole job.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
N > 1 runs under torch.distributed.run (one rank per GPU, NCCL); each rank runs the full layer
on its own batch (weak scaling).  --impl reference times the CPU oracle on this host.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "NVFP4 linear fwd+bwd TFLOPS at 8192x5120x20480; quantize HBM GB/s"
T_TOK, D_IN, D_OUT = 8192, 5120, 20480
FLOP_STEP = 3 * 2 * T_TOK * D_IN * D_OUT
FLOP_GEMM = 2 * T_TOK * D_IN * D_OUT
# algorithmic bytes of one two-pass dual quantize call per input element:
# 2 B read (amax) + 2 B read (quantize) + 2 forms x (0.5 B codes + 1/16 B scales)
Q_BYTES_PER_ELEM = 2 + 2 + 2 * (0.5 + 1 / 16)
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FP4_OVER_BF16 = 4.0   # nominal dense FP4 / BF16 tensor throughput ratio on B200 (9 / 2.25 PFLOP/s)
FP4_DENSE_DATASHEET_TFLOPS = 9000.0
# tcgen05 block-scaled FP4 instruction rate: 16384 dense FP4 FMA per clock per SM (measured on
# this GPU: four 128x256x64 MMAs take 512 cycles), 148 SMs
FP4_FLOP_PER_CLK = 2 * 16384 * 148
# DRAM bytes (read + write) per GEMM launch, the mean over the fprop, dgrad and wgrad launches
# of one ncu capture of the SM-pair GEMM at this layer's shapes, valid for the GEMM sources it was
# taken on only (the kernel file and the device header it includes): reported as null once they
# no longer hash to those sources.
GEMM_SRCS = [os.path.join(ROOT, "nvfp4_bit_quantized_02_b200", "csrc", f) for f in ("gemm_sm100.cu", "nvfp4_device.cuh")]
GEMM_TRAFFIC = {"sha256": "2d68f32034fdb4cd69f13713f8e15c3a40a64b119d1956d1ee305df8c54f9192",
                "bytes_per_launch": 478.2e6}


def gemm_src_hash():
    h = hashlib.sha256()
    for path in GEMM_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_traffic():
    try:
        h = gemm_src_hash()
    except OSError:
        return None
    return GEMM_TRAFFIC["bytes_per_launch"] if h == GEMM_TRAFFIC["sha256"] else None


def load_peaks():
    """The measured peaks of this machine's B200s, else the earlier measurement used as fallback
    (per key: a missing or malformed entry falls back alone, and the basis says so)."""
    fallback = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
    except (OSError, ValueError):
        return fallback, "fallback"
    out, kind = {}, "measured"
    for k, v in fallback.items():
        x = p.get(k) if isinstance(p, dict) else None
        if isinstance(x, (int, float)) and not isinstance(x, bool) and x > 0:
            out[k] = float(x)
        else:
            out[k], kind = v, "measured (fallback for missing entries)"
    return out, kind


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path:
                try:
                    os.remove(self.path)
                except OSError:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        smax = max(int(r[2]) for r in rows)
        loaded = [r for r in rows if float(r[3] or 0) > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(int(r[1]) for r in loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded), "sm_mhz_min": min(sm)}


def linear_config(world: int = 1) -> dict:
    """The workload of the default line (both arms report it)."""
    return {"workload": "NVFP4 linear fwd+bwd: fprop 8192x20480x5120, dgrad 8192x5120x20480, "
                        "wgrad 20480x5120x8192, W 16x16 quantized every step",
            "parallelism": f"dp{world}" + (" (amax all-reduce between quantize passes, dW reduce-scatter "
                                           "overlapping dgrad)" if world > 1 else ""),
            "tokens": T_TOK, "d_in": D_IN, "d_out": D_OUT, "rht": "16-point, wgrad operands",
            "sr": "Philox4x32-10, dY both forms",
            "l2": "256 MiB buffer written between timed steps (outside the events); inputs 629 MB > L2"}


# ---------------------------------------------------------------------------------------
# cross-rank aggregation (weak scaling: every rank runs the whole layer on its own batch)
# ---------------------------------------------------------------------------------------
def reduce_max(x: float, dist, device) -> float:
    """The maximum of x over all ranks (x itself on one rank)."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_tflops(world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank did one layer step in the slowest rank's step time."""
    return world * FLOP_STEP / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------------------
def make_inputs(device):
    import synth
    x = synth.activations(T_TOK, D_IN, seed=0, outlier_frac=0.001)
    w = synth.weights(D_OUT, D_IN, seed=1)
    dy = synth.grad_output(T_TOK, D_OUT, seed=2)
    return x, w, dy


def run_ours(args, rank, world, local_rank):
    import nvfp4_bit_quantized_02_b200 as nv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = torch.distributed if world > 1 else None
    x_h, w_h, dy_h = make_inputs(dev)
    x, w, dy = x_h.to(dev), w_h.to(dev), dy_h.to(dev)
    ctx = nv.LinearContext(T_TOK, D_IN, D_OUT, rht_seed=0, device=dev)
    y = torch.empty((T_TOK, D_OUT), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((T_TOK, D_IN), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((D_OUT, D_IN), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2

    # The step as a user runs it: the two public entry points of the linear layer.  Over N > 1
    # ranks each rank holds its own 8192 tokens of an N x 8192-token batch and the step is the
    # data-parallel one: the amax of X and dY all-reduced between the quantize passes (every
    # rank's forms are its slice of the whole batch's), and the dW partial sums reduce-scattered
    # over NCCL while the dgrad GEMM runs.
    dp = nv.DPLinear(T_TOK, D_IN, D_OUT, rht_seed=0, device=dev) if world > 1 else None

    def step(sr_seed):
        if dp is None:
            nv.nvfp4_linear_fwd(ctx, x, w, y)
            nv.nvfp4_linear_bwd(ctx, dy, sr_seed, dx, dw)
        else:
            dp.fwd(x, w, y)
            dp.bwd(dy, sr_seed, dx)

    # The same step as the sequence of public calls that nvfp4_linear_fwd / nvfp4_linear_bwd
    # make, with an event between calls: the per-kernel fields (roofline, quantize, per-GEMM).
    def step_calls(sr_seed, ev):
        ev[0].record()
        nv.nvfp4_quantize_dual(x, mode=nv.RNE, rht_seed=0, out_row=ctx.xq, out_col=ctx.xq_rht, ws=ctx.ws)
        ev[1].record()
        nv.nvfp4_quantize_weight(w, out=ctx.wq, out_t=ctx.wqt, ws=ctx.ws)
        ev[2].record()
        nv.nvfp4_gemm(ctx.xq, ctx.wq, out=y, ws=ctx.ws)
        ev[3].record()
        nv.nvfp4_quantize_dual(dy, mode=nv.SR, rht_seed=0, sr_seed=sr_seed, stream_row=nv.STREAM_DGRAD,
                               stream_col=nv.STREAM_WGRAD, out_row=ctx.dyq, out_col=ctx.dyq_rht, ws=ctx.ws)
        ev[4].record()
        nv.nvfp4_gemm(ctx.dyq, ctx.wqt, out=dx, ws=ctx.ws)
        ev[5].record()
        nv.nvfp4_gemm(ctx.dyq_rht, ctx.xq_rht, out=dw, ws=ctx.ws)
        ev[6].record()

    launches_per_step = 2 + 2 + 1 + 2 + 1 + 1   # amax+tile (X), amax+tile (W), fprop, amax+tile (dY), dgrad, wgrad

    for i in range(args.warmup):
        step(1000 + i)
    torch.cuda.synchronize()
    status = nv.nvfp4_poll(ctx.ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for k in range(args.steps):
            flush.fill_(k & 0xFF)                  # evict L2 between steps (outside the events)
            events[k][0].record()
            step(k)
            events[k][1].record()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    status = nv.nvfp4_poll(ctx.ws)
    if status != 0:
        raise RuntimeError(f"device status {status} during timing")
    ms_per_step = reduce_max(sum(a.elapsed_time(b) for a, b in events), dist, dev) / args.steps

    # per-call breakdown (same inputs, same L2 flush between steps)
    cev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        step_calls(k, cev[k])
    torch.cuda.synchronize()
    if nv.nvfp4_poll(ctx.ws) != 0:
        raise RuntimeError("device status during the per-call breakdown")
    seg = [[cev[k][i].elapsed_time(cev[k][i + 1]) for i in range(6)] for k in range(args.steps)]
    calls_ms_per_step = statistics.mean(sum(s_) for s_ in seg)

    # the step with the weight's forms cached (quantized once, as between optimizer steps with
    # gradient accumulation): nvfp4_linear_fwd skips the weight's quantize
    cached_w = None
    if dp is None:
        ctx.w_cached = True
        cev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            cev2[k][0].record()
            step(k)
            cev2[k][1].record()
        torch.cuda.synchronize()
        ctx.w_cached = False
        if nv.nvfp4_poll(ctx.ws) != 0:
            raise RuntimeError("device status during the cached-weight steps")
        cms = statistics.mean(a.elapsed_time(b) for a, b in cev2)
        cached_w = {"value": job_tflops(world, cms), "unit": "TFLOPS", "ms_per_step": cms,
                    "workload": "the same layer step with the weight's 16x16 forms cached (no weight quantize)"}

    gemm_ms = [s_[i] for s_ in seg for i in (2, 4, 5)]
    q_ms = sum(s_[0] + s_[1] + s_[3] for s_ in seg)
    q_bytes = args.steps * Q_BYTES_PER_ELEM * (D_OUT * D_IN + T_TOK * D_IN + T_TOK * D_OUT)
    peaks, peak_kind = load_peaks()
    gemm_avg_ms = statistics.mean(gemm_ms)
    achieved = FLOP_GEMM / (gemm_avg_ms * 1e-3) / 1e12
    # each GEMM launch is timed alone (a third of a ~2 ms step): the burst bf16 figure is its basis
    peak_tensor = FP4_OVER_BF16 * peaks["bf16_tflops"]
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9

    # ---- end to end through the public API from pinned host buffers ---------------------
    e2e = None
    if args.e2e_steps > 0:
        hx, hw, hdy = (t.pin_memory() for t in (x_h, w_h, dy_h))
        hy = torch.empty((T_TOK, D_OUT), dtype=torch.bfloat16).pin_memory()
        hdx = torch.empty((T_TOK, D_IN), dtype=torch.bfloat16).pin_memory()
        dw_dev = dw if dp is None else dp.dw          # over N > 1 ranks: this rank's rows of the batch's dW
        hdw = torch.empty(tuple(dw_dev.shape), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hx, hw, hdy))
        d2h = sum(t.numel() * t.element_size() for t in (hy, hdx, hdw))

        # Host-to-device copies, compute and device-to-host copies on three streams, ordered by
        # events so the two copy directions (PCIe is full duplex) overlap each other and the
        # compute.  The inputs alternate between two device copies, so step k's uploads need
        # only wait for step k-2's compute to finish reading its copy; step k's forward waits
        # for its x and w and for step k-1's read-back of y; its backward for its dy and for
        # step k-1's read-back of dx and dw; each read-back waits for its result.
        comp = torch.cuda.current_stream(dev)
        up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        evt = lambda: torch.cuda.Event()  # noqa: E731
        ins = [(x, w, dy), tuple(torch.empty_like(t) for t in (x, w, dy))]
        prev = {"bwd": [None, None], "y_read": None, "dxdw_read": None, "k": 0}

        def e2e_step(seed):
            slot = prev["k"] & 1
            prev["k"] += 1
            x, w, dy = ins[slot]
            with torch.cuda.stream(up_s):
                if prev["bwd"][slot] is not None:
                    up_s.wait_event(prev["bwd"][slot])
                x.copy_(hx, non_blocking=True)
                w.copy_(hw, non_blocking=True)
                xw_in = evt()
                xw_in.record(up_s)
                dy.copy_(hdy, non_blocking=True)
                dy_in = evt()
                dy_in.record(up_s)
            comp.wait_event(xw_in)
            if prev["y_read"] is not None:
                comp.wait_event(prev["y_read"])
            if dp is None:
                nv.nvfp4_linear_fwd(ctx, x, w, y)
            else:
                dp.fwd(x, w, y)
            y_done = evt()
            y_done.record(comp)
            comp.wait_event(dy_in)
            if prev["dxdw_read"] is not None:
                comp.wait_event(prev["dxdw_read"])
            if dp is None:
                nv.nvfp4_linear_bwd(ctx, dy, seed, dx, dw)
            else:
                dp.bwd(dy, seed, dx)
            bwd_done = evt()
            bwd_done.record(comp)
            with torch.cuda.stream(down_s):
                down_s.wait_event(y_done)
                hy.copy_(y, non_blocking=True)
                y_read = evt()
                y_read.record(down_s)
                down_s.wait_event(bwd_done)
                hdx.copy_(dx, non_blocking=True)
                hdw.copy_(dw_dev, non_blocking=True)
                dxdw_read = evt()
                dxdw_read.record(down_s)
            prev["bwd"][slot] = bwd_done
            prev.update(y_read=y_read, dxdw_read=dxdw_read)

        e2e_step(0)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        up_s.wait_event(e0)                      # the first upload starts inside the timed region
        for k in range(args.e2e_steps):
            e2e_step(k)
        comp.wait_event(prev["dxdw_read"])      # the last read-back ends the timed region
        comp.wait_event(prev["y_read"])
        e1.record(comp)
        torch.cuda.synchronize()
        # the read-backs hold the last step's results
        if not (torch.equal(hy, y.cpu()) and torch.equal(hdx, dx.cpu()) and torch.equal(hdw, dw_dev.cpu())):
            raise RuntimeError("end-to-end read-back differs from the device results")
        e2e_ms = reduce_max(e0.elapsed_time(e1), dist, dev) / args.e2e_steps
        e2e = {"value": job_tflops(world, e2e_ms), "unit": "TFLOPS", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "path": "pinned host X, W, dY -> nvfp4_linear_fwd/bwd (N > 1: the data-parallel step) -> pinned "
                       "host Y, dX, dW (N > 1: this rank's rows); uploads, compute and read-backs on three "
                       "event-ordered streams, the inputs alternating between two device copies"}

    ffn = ffn_fields(args, world, dev, dist, flush) if args.ffn else None
    variants = variant_fields(args, dev, flush, x, w, dy) if args.variants else None
    if rank != 0:
        return None
    clocks = clk.summary()
    inst_peak = FP4_FLOP_PER_CLK * clocks["sm_mhz"] * 1e6 / 1e12 if clocks.get("sm_mhz") else None
    line = {
        "metric": METRIC,
        "value": job_tflops(world, ms_per_step),
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3/16, fp32 scale) operands, fp32 accumulate",
        "data": "synthetic (seeded N(0,1) X with 0.1% x50 outlier channels, N(0,0.02) W, N(0,1e-4) dY; bf16)",
        "config": linear_config(world),
        "roofline": {"bound": "tensor", "kernel": "gemm_nvf4_2sm_kernel", "achieved": achieved,
                     "peak": peak_tensor, "unit": "TFLOP/s", "frac": achieved / peak_tensor,
                     "traffic": gemm_traffic(),
                     "peak_basis": f"{FP4_OVER_BF16:g} x {peak_kind} burst bf16 ({peaks['bf16_tflops']} TF/s)",
                     "frac_of_9pf_datasheet": achieved / FP4_DENSE_DATASHEET_TFLOPS,
                     "frac_of_instruction_rate_at_clock": achieved / inst_peak if inst_peak else None,
                     "per_launch_flop": FLOP_GEMM, "avg_launch_ms": gemm_avg_ms},
        "quantize": {"gbs": q_gbs, "unit": "GB/s", "peak_hbm_gbs": peaks["hbm_gbs"], "frac": q_gbs / peaks["hbm_gbs"],
                     "frac_of_8000_gbs": q_gbs / 8000.0,
                     "bound": {"X": "instruction issue (64 % issue-active; ALU and FMA pipes ~50 %)",
                               "W": "ALU pipe (61 %): 16x16 tile maxima and widening",
                               "dY": "heavy FMA pipe (65 %: Philox products, f32x2 SR arithmetic) with the ALU (55 %)"},
                     "bytes_per_elem": Q_BYTES_PER_ELEM, "peak_basis": peak_kind,
                     "per_call_ms": {"X": statistics.mean(s_[0] for s_ in seg), "W": statistics.mean(s_[1] for s_ in seg),
                                     "dY": statistics.mean(s_[3] for s_ in seg)},
                     "per_call_gbs": {
                         "X": Q_BYTES_PER_ELEM * T_TOK * D_IN / statistics.mean(s_[0] for s_ in seg) / 1e6,
                         "W": Q_BYTES_PER_ELEM * D_OUT * D_IN / statistics.mean(s_[1] for s_ in seg) / 1e6,
                         "dY": Q_BYTES_PER_ELEM * T_TOK * D_OUT / statistics.mean(s_[3] for s_ in seg) / 1e6}},
        "gemm_tflops": {"fprop": FLOP_GEMM / statistics.mean(s_[2] for s_ in seg) / 1e9,
                        "dgrad": FLOP_GEMM / statistics.mean(s_[4] for s_ in seg) / 1e9,
                        "wgrad": FLOP_GEMM / statistics.mean(s_[5] for s_ in seg) / 1e9},
        "calls_ms_per_step": calls_ms_per_step,
        "cached_w_step": cached_w,
        "clocks": clocks,
        "e2e": e2e,
        "c1_small_fprop": c1_latency(nv, dev) if args.c1 else None,
        "ffn_step": ffn,
        "mxfp4_step": variants["mxfp4_step"] if variants else None,
        "bf16_step": variants["bf16_step"] if variants else None,
        "wgrad_reduce_scatter": variants["wgrad_reduce_scatter"] if variants else None,
        "fprop_amax_epilogue": variants["fprop_amax_epilogue"] if variants else None,
        "gpu_launches": launches_per_step * args.steps,
        "impl": "ours",
    }
    if args.cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_with_one_core(args)
    return line


# ---------------------------------------------------------------------------------------
# --workload ffn: the one-FFN training step (up-projection, GeLU, down-projection; forward and
# backward: six NVFP4 GEMMs, every quantize, both GeLU kernels) at T=16384, 5120 -> 20480 -> 5120
# ---------------------------------------------------------------------------------------
FFN_T, FFN_D, FFN_F = 16384, 5120, 20480
FFN_FLOP = 6 * 2 * FFN_T * FFN_D * FFN_F


class FFNStep:
    """The one-FFN training step on one rank's batch, its buffers allocated once."""

    def __init__(self, nv, dev):
        import synth
        self.nv = nv
        self.x = synth.activations(FFN_T, FFN_D, seed=0, outlier_frac=0.001).to(dev)
        self.w1 = synth.weights(FFN_F, FFN_D, seed=1).to(dev)
        self.w2 = synth.weights(FFN_D, FFN_F, seed=3).to(dev)
        self.dy = synth.grad_output(FFN_T, FFN_D, seed=4).to(dev)
        self.up = nv.LinearContext(FFN_T, FFN_D, FFN_F, rht_seed=0, device=dev)
        self.down = nv.LinearContext(FFN_T, FFN_F, FFN_D, rht_seed=0, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.h, self.g, self.dg, self.dh = (torch.empty((FFN_T, FFN_F), **bf) for _ in range(4))
        self.y, self.dx = torch.empty((FFN_T, FFN_D), **bf), torch.empty((FFN_T, FFN_D), **bf)
        self.dw1 = torch.empty((FFN_F, FFN_D), dtype=torch.float32, device=dev)
        self.dw2 = torch.empty((FFN_D, FFN_F), dtype=torch.float32, device=dev)

    @staticmethod
    def launches_per_step(fused: bool) -> int:
        # 2 x (W quantize 2 + X/G quantize 2 + fprop 1) + 2 x (dY/dH quantize 2 + dgrad 1 + wgrad 1)
        # + 2 GeLU; the fused variant drops the amax passes of G and dH
        return 2 * 5 + 2 * 4 + 2 - (2 if fused else 0)

    def step(self, seed: int, fused: bool):
        nv = self.nv
        nv.nvfp4_linear_fwd(self.up, self.x, self.w1, self.h)
        if fused:   # the GeLU kernels reduce their output's amax; G's and dH's quantize skip pass 1
            nv.nvfp4_gelu_fwd_amax(self.h, self.g, rht_seed=0, ws=self.down.ws)
            self.down.amax_ready = True
        else:
            nv.nvfp4_gelu_fwd(self.h, self.g)
        nv.nvfp4_linear_fwd(self.down, self.g, self.w2, self.y)
        nv.nvfp4_linear_bwd(self.down, self.dy, 2 * seed, self.dg, self.dw2)
        if fused:
            nv.nvfp4_gelu_bwd_amax(self.h, self.dg, self.dh, rht_seed=0, ws=self.up.ws)
            self.up.amax_ready = True
        else:
            nv.nvfp4_gelu_bwd(self.h, self.dg, self.dh)
        nv.nvfp4_linear_bwd(self.up, self.dh, 2 * seed + 1, self.dx, self.dw1)

    def poll(self, what: str):
        for c in (self.up, self.down):
            if self.nv.nvfp4_poll(c.ws) != 0:
                raise RuntimeError(f"device status {what}")

    def time(self, steps, warmup, fused, flush, dist, dev, clk_gpu=None):
        """ms per step (max over ranks) and the clock summary of the timed region."""
        for i in range(warmup):
            self.step(1000 + i, fused)
        torch.cuda.synchronize()
        self.poll("after warm-up")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with ClockSampler(clk_gpu if clk_gpu is not None else dev.index) as clk:
            if dist:
                dist.barrier()
            torch.cuda.synchronize()
            for k in range(steps):
                flush.fill_(k & 0xFF)                  # evict L2 between steps (outside the events)
                ev[k][0].record()
                self.step(k, fused)
                ev[k][1].record()
            torch.cuda.synchronize()
            if dist:
                dist.barrier()
        self.poll("during timing")
        return reduce_max(sum(a.elapsed_time(b) for a, b in ev), dist, dev) / steps, clk.summary()


def ffn_config(fused: bool) -> dict:
    return {"workload": "one FFN training step: up 5120->20480, GeLU, down 20480->5120, forward and "
                        "backward (6 GEMMs), weights quantized every step"
                        + (", amax of G and dH fused into the GeLU kernels" if fused else ""),
            "tokens": FFN_T, "d": FFN_D, "ffn": FFN_F, "flop_per_step": FFN_FLOP,
            "l2": "256 MiB buffer written between timed steps (outside the events)"}


def ffn_fields(args, world, dev, dist, flush) -> dict:
    """The FFN step, plain and with the GeLU-fused amax, as a nested field of the main line."""
    import nvfp4_bit_quantized_02_b200 as nv
    f = FFNStep(nv, dev)
    out = {}
    for fused in (False, True):
        ms, clocks = f.time(args.steps, args.warmup, fused, flush, dist, dev)
        out["fused_amax" if fused else "plain"] = {
            "value": world * FFN_FLOP / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms,
            "gpu_launches": f.launches_per_step(fused) * args.steps, "clocks": clocks, "config": ffn_config(fused)}
    del f
    torch.cuda.empty_cache()
    return out


def run_ffn(args, rank, world, local_rank):
    import nvfp4_bit_quantized_02_b200 as nv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = torch.distributed if world > 1 else None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    fused = args.ffn_fused_amax
    f = FFNStep(nv, dev)
    ms_per_step, clocks = f.time(args.steps, args.warmup, fused, flush, dist, dev)
    if rank != 0:
        return None
    return {
        "metric": "NVFP4 FFN training step TFLOPS at 16384x5120x20480",
        "value": world * FFN_FLOP / (ms_per_step * 1e-3) / 1e12,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3/16, fp32 scale) operands, fp32 accumulate; GeLU fp32 math, bf16 in/out",
        "data": "synthetic (seeded N(0,1) X with 0.1% x50 outlier channels, N(0,0.02) W1 and W2, N(0,1e-4) dY; bf16)",
        "config": ffn_config(fused),
        "clocks": clocks,
        "e2e": None,
        "gpu_launches": f.launches_per_step(fused) * args.steps,
        "impl": "ours",
    }


def time_calls(calls, steps, warmup, flush):
    """Mean device time of each named call of a step (events between calls on the current stream)
    and of the whole step, over `steps` steps after `warmup`, L2 flushed between steps."""
    for i in range(warmup):
        for _, fn in calls:
            fn(1000 + i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(steps)]
    for k in range(steps):
        flush.fill_(k & 0xFF)
        ev[k][0].record()
        for i, (_, fn) in enumerate(calls):
            fn(k)
            ev[k][i + 1].record()
    torch.cuda.synchronize()
    per = {name: statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps))
           for i, (name, _) in enumerate(calls)}
    return per, statistics.mean(ev[k][0].elapsed_time(ev[k][-1]) for k in range(steps))


def variant_fields(args, dev, flush, x, w, dy) -> dict:
    """The same layer step in the pages' comparison format (MXFP4: three single-pass quantizes, each
    giving both forms from one read, and three kind::mxf4 GEMMs) and on the BF16 path of the high-precision layers (three kind::f16
    GEMMs and the transposes of their K-major operands)."""
    import nvfp4_bit_quantized_02_b200 as nv
    ws = nv.Workspace(dev)
    f = {k: nv.MXTensor.empty(R, K, dev) for k, R, K in (("xr", T_TOK, D_IN), ("xc", D_IN, T_TOK), ("wr", D_OUT, D_IN),
                                                         ("wc", D_IN, D_OUT), ("dyr", T_TOK, D_OUT),
                                                         ("dyc", D_OUT, T_TOK))}
    y = torch.empty((T_TOK, D_OUT), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((T_TOK, D_IN), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((D_OUT, D_IN), dtype=torch.float32, device=dev)
    mq = nv.nvfp4_mx_quantize_dual
    mx_calls = [
        ("quantize X (row, column)", lambda k: mq(x, out_row=f["xr"], out_col=f["xc"], ws=ws)),
        ("quantize W (row, column)", lambda k: mq(w, out_row=f["wr"], out_col=f["wc"], ws=ws)),
        ("fprop", lambda k: nv.nvfp4_mx_gemm(f["xr"], f["wr"], out=y, ws=ws)),
        ("quantize dY (row, column; SR)", lambda k: mq(dy, nv.SR, k, 1, 2, out_row=f["dyr"], out_col=f["dyc"], ws=ws)),
        ("dgrad", lambda k: nv.nvfp4_mx_gemm(f["dyr"], f["wc"], out=dx, ws=ws)),
        ("wgrad", lambda k: nv.nvfp4_mx_gemm(f["dyc"], f["xc"], out=dw, ws=ws)),
    ]
    per, ms = time_calls(mx_calls, args.steps, args.warmup, flush)
    out = {"mxfp4_step": {
        "value": FLOP_STEP / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms, "per_call_ms": per,
        "gemm_tflops": {g: FLOP_GEMM / per[g] / 1e9 for g in ("fprop", "dgrad", "wgrad")},
        "workload": "the same layer with MXFP4 operands (blocks of 32, UE8M0 scales, no tensor scale): X, W and "
                    "dY each quantized in both forms from one read (dY with SR), three kind::mxf4 GEMMs"}}
    del f
    lay = nv.LinearBF16(T_TOK, D_IN, D_OUT, device=dev)
    bf_calls = [("fwd", lambda k: lay.fwd(x, w, y)), ("bwd", lambda k: lay.bwd(x, w, dy, dx, dw))]
    per, ms = time_calls(bf_calls, args.steps, args.warmup, flush)
    if nv.nvfp4_poll(ws) != 0 or nv.nvfp4_poll(lay.ws) != 0:
        raise RuntimeError("device status in the MXFP4 / BF16 steps")
    out["bf16_step"] = {
        "value": FLOP_STEP / (ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": ms, "per_call_ms": per,
        "fprop_tflops": FLOP_GEMM / per["fwd"] / 1e9,
        "workload": "the same layer on the BF16 path: kind::f16 GEMMs with fp32 accumulation; the backward "
                    "includes the bf16 transposes of W, dY and X (K-major operands)"}
    del lay
    torch.cuda.empty_cache()
    out["wgrad_reduce_scatter"] = wgrad_reduce_scatter_fields(args, dev, flush, x, dy, dw)
    out["fprop_amax_epilogue"] = fprop_amax_fields(args, dev, flush, x, w, y)
    return out


def fprop_amax_fields(args, dev, flush, x, w, y) -> dict:
    """The layer's fprop (Y 8192 x 20480 bf16) with Y's amax for the next quantize: the plain GEMM
    followed by the amax pass over Y, against the GEMM whose epilogue produces the same amax words;
    the calls interleaved, each timed with L2 flushed before it."""
    import nvfp4_bit_quantized_02_b200 as nv
    ws, ws_a, ws_b = nv.Workspace(dev), nv.Workspace(dev), nv.Workspace(dev)
    xq = nv.nvfp4_quantize(x, ws=ws)
    wq = nv.nvfp4_quantize(w, block=nv.BLOCK_16x16, ws=ws)
    calls = (("gemm", lambda: nv.nvfp4_gemm(xq, wq, out=y, ws=ws)),
             ("amax pass", lambda: nv.nvfp4_amax(y, True, 0, ws_a)),
             ("gemm with amax epilogue", lambda: nv.nvfp4_gemm_amax(xq, wq, ws_b, rht_seed=0, out=y, ws=ws)))
    for _ in range(args.warmup):
        for _, fn in calls:
            fn()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(args.steps)]
    for k in range(args.steps):
        for i, (_, fn) in enumerate(calls):
            flush.fill_((k + i) & 0xFF)
            ev[k][i][0].record()
            fn()
            ev[k][i][1].record()
    torch.cuda.synchronize()
    if nv.nvfp4_poll(ws) != 0 or not torch.equal(ws_a.amax_words(), ws_b.amax_words()):
        raise RuntimeError("the epilogue amax differs from the amax pass")
    res = {name: statistics.mean(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps))
           for i, (name, _) in enumerate(calls)}
    return {"ms": res, "saved_ms": res["gemm"] + res["amax pass"] - res["gemm with amax epilogue"],
            "workload": "fprop 8192x20480x5120 producing Y's plain and RHT amax: GEMM + amax pass over Y, "
                        "against the GEMM with the amax epilogue (equal words checked)"}


def wgrad_reduce_scatter_fields(args, dev, flush, x, dy, dw) -> dict:
    """The wgrad GEMM (M = 20480, N = 5120, K = 8192 tokens) with its output stored (fp32), added
    into 8 row shards of 2560 rows (the epilogue of the data-parallel reduce-scatter, here into
    local buffers) and added into one fp32 buffer (gradient accumulation); the three calls
    interleaved, each timed alone with L2 flushed before it."""
    import nvfp4_bit_quantized_02_b200 as nv
    ws = nv.Workspace(dev)
    _, xc = nv.nvfp4_quantize_dual(x, mode=nv.RNE, rht_seed=3, ws=ws)
    _, dyc = nv.nvfp4_quantize_dual(dy, mode=nv.SR, rht_seed=3, sr_seed=4, stream_row=1, stream_col=2, ws=ws)
    share = D_OUT // 8
    shards = [dw[o * share:(o + 1) * share] for o in range(8)]
    calls = (("stored", lambda: nv.nvfp4_gemm(dyc, xc, out=dw, ws=ws)),
             ("8 owners", lambda: nv.nvfp4_gemm_reduce_scatter(dyc, xc, shards, share, ws=ws)),
             ("1 owner", lambda: nv.nvfp4_gemm_reduce_scatter(dyc, xc, [dw], D_OUT, ws=ws)))
    for _ in range(args.warmup):
        for _, fn in calls:
            fn()
    # the three interleaved, each with L2 flushed before it, so drifts of clock or power hit all alike
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
          for _ in range(args.steps)]
    for k in range(args.steps):
        for i, (_, fn) in enumerate(calls):
            flush.fill_((k + i) & 0xFF)
            ev[k][i][0].record()
            fn()
            ev[k][i][1].record()
    torch.cuda.synchronize()
    res = {name: statistics.mean(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps))
           for i, (name, _) in enumerate(calls)}
    if nv.nvfp4_poll(ws) != 0:
        raise RuntimeError("device status in the wgrad reduce-scatter timing")
    return {"ms": res, "tflops": {k: FLOP_GEMM / v / 1e9 for k, v in res.items()},
            "workload": "the layer's wgrad GEMM, fp32 output stored, reduce-added into 8 local row shards, and "
                        "reduce-added into one buffer"}


def c1_latency(nv, dev) -> dict:
    """The 256 x 256 x 256 fprop of the small single-GEMM workload, reported as latency: the GEMM
    launch alone and the whole fprop (both quantize calls + GEMM), each as the median of 200
    back-to-back calls from Python (host-bound at this size) and per call of a CUDA graph of 100
    replayed five times (the device latency).  The operands are L2-resident: a latency, not a
    bandwidth figure."""
    import synth
    x = synth.activations(256, 256, seed=0).to(dev)
    w = synth.weights(256, 256, seed=1).to(dev)
    ws = nv.Workspace(dev)
    xq = nv.nvfp4_quantize(x, ws=ws)
    wq = nv.nvfp4_quantize(w, block=nv.BLOCK_16x16, ws=ws)
    y = torch.empty((256, 256), dtype=torch.bfloat16, device=dev)

    def fprop():
        nv.nvfp4_quantize(x, out=xq, ws=ws)
        nv.nvfp4_quantize(w, block=nv.BLOCK_16x16, out=wq, ws=ws)
        nv.nvfp4_gemm(xq, wq, out=y, ws=ws)

    res = {}
    for name, fn in (("gemm_us", lambda: nv.nvfp4_gemm(xq, wq, out=y, ws=ws)), ("fprop_us", fprop)):
        for _ in range(20):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(200):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        res[name] = statistics.median(a.elapsed_time(b) for a, b in ts) * 1e3
        # the same calls captured once into a CUDA graph of 100 and replayed: the device-side
        # latency without the host's per-call work (Python, argument checks, tensor-map encoding)
        try:
            s_cap = torch.cuda.Stream(dev)
            s_cap.wait_stream(torch.cuda.current_stream(dev))
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(s_cap):
                with torch.cuda.graph(graph, stream=s_cap):
                    for _ in range(100):
                        fn()
            torch.cuda.current_stream(dev).wait_stream(s_cap)
            graph.replay()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(5):
                graph.replay()
            b.record()
            torch.cuda.synchronize()
            res[name.replace("_us", "_graph_us")] = a.elapsed_time(b) * 1e3 / 500
            del graph
        except RuntimeError as e:   # a capture the runtime refused: report it, keep the line
            torch.cuda.synchronize()
            res[name.replace("_us", "_graph_us")] = None
            res["graph_error"] = str(e)[:200]
    if nv.nvfp4_poll(ws) != 0:
        raise RuntimeError("device status in the small fprop")
    res["workload"] = "fprop 256x256x256: X N(0,1) 1x16 RNE, W N(0,0.02) 16x16 RNE, bf16 out"
    return res


# ---------------------------------------------------------------------------------------
# the CPU oracle (reference arm and the cpu_baseline field)
# ---------------------------------------------------------------------------------------
def cpu_baseline(args, n_cols: int | None = None, threads: int | None = None):
    """The oracle as it stands on a bounded slice of the same layer: the first T_s tokens and the
    first n_s output features with the full d = 5120 (all six quantized forms, the three GEMMs
    over every output of the slice), on `threads` host threads (all cores by default).  The
    default slice is sized for about 10 s of oracle work."""
    import numpy as np

    import oracle
    import synth

    cores = threads or os.cpu_count() or 1
    T_s = 256
    n_s = n_cols or min(D_OUT, 4096 * max(1, cores // 8))   # about 10 s of oracle work on all cores
    x = synth.bf16_bits(synth.activations(T_TOK, D_IN, seed=0, outlier_frac=0.001)[:T_s])
    w = synth.bf16_bits(synth.weights(D_OUT, D_IN, seed=1)[:n_s])
    dy = synth.bf16_bits(synth.grad_output(T_TOK, D_OUT, seed=2)[:T_s, :n_s])
    t0 = time.perf_counter()
    xq = oracle.quantize(x, nthreads=cores)
    xr = oracle.quantize(x, along=1, rht=True, nthreads=cores)
    wq = oracle.quantize(w, block=oracle.BLOCK_16x16, nthreads=cores)
    wqt = oracle.transpose_2d(wq)
    dq = oracle.quantize(dy, mode=oracle.SR, stream_id=1, nthreads=cores)
    dr = oracle.quantize(dy, along=1, mode=oracle.SR, rht=True, stream_id=2, nthreads=cores)

    def every(a, b):
        ii, jj = np.meshgrid(np.arange(a.R), np.arange(b.R), indexing="ij")
        return oracle.gemm_sampled(a, b, ii.reshape(-1), jj.reshape(-1), nthreads=cores)

    every(xq, wq)
    every(dq, wqt)
    every(dr, xr)
    dt = time.perf_counter() - t0
    flop = 3 * 2 * T_s * D_IN * n_s
    return {"value": flop / dt / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "seconds": dt,
            "sample": f"layer slice T={T_s} tokens x n={n_s} out-features x d={D_IN}: six quantized forms and the "
                      f"fprop/dgrad/wgrad GEMMs (fp64 over dequantized operands) of the slice, {flop / 1e9:.1f} GFLOP"}


def cpu_baseline_with_one_core(args):
    """All host cores (the reported value) and, beside it, one core on a 16x smaller slice (the
    oracle is scalar code: one core is its plain speed)."""
    n_all = min(D_OUT, 4096 * max(1, (os.cpu_count() or 1) // 8))
    allc = cpu_baseline(args, n_cols=n_all)
    one = cpu_baseline(args, n_cols=max(256, n_all // 16), threads=1)
    allc["one_core"] = {k: one[k] for k in ("value", "unit", "cores", "seconds", "sample")}
    return allc


def run_reference(args, rank, world):
    if rank != 0:
        return None
    samples = []
    for _ in range(args.warmup):
        cpu_baseline(args, n_cols=256)
    for _ in range(args.steps):
        samples.append(cpu_baseline(args, n_cols=256))
    value = statistics.mean(s["value"] for s in samples)
    sec = statistics.mean(s["seconds"] for s in samples)
    return {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp64 GEMM over dequantized NVFP4 operands (CPU)", "data": "synthetic",
            "config": linear_config(),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": samples[0]["cores"], "kind": "oracle",
                             "sample": samples[0]["sample"]},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--workload", choices=["linear", "ffn"], default="linear",
                    help="linear: the 8192x5120x20480 layer (the default line); ffn: the one-FFN step")
    ap.add_argument("--no-ffn", dest="ffn", action="store_false",
                    help="linear: skip the nested one-FFN step fields")
    ap.add_argument("--no-c1", dest="c1", action="store_false",
                    help="linear: skip the 256^3 fprop latency field")
    ap.add_argument("--no-variants", dest="variants", action="store_false",
                    help="linear: skip the nested MXFP4 and BF16 step fields")
    ap.add_argument("--ffn-fused-amax", action="store_true",
                    help="ffn: the GeLU kernels that also reduce their output's amax (slower as they stand)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if rank != 0:
        args.cpu_baseline = False
    try:
        line = (run_ffn if args.workload == "ffn" else run_ours)(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
