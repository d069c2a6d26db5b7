#!/usr/bin/env python
"""Throughput of the quantized attention forward on B200.

One step = one pass of the whole hot path over one batch: smoothing + INT8/FP8
quantization of Q, K, V (libsage quantize kernels) and the fused attention
kernel, all through the C ABI (libsage.so).

Default workload: LLM prefill, B1 H32 N8192 d128 bf16, causal, INT8 QK / FP8 PV
(FP32 accumulator).  Inputs (192 MB of bf16 Q, K, V) are larger than the 126 MB
L2, so no flush runs between steps.

Prints ONE JSON line (rank 0).  `value` is whole-job attention TOPS,
4*B*H*N^2*d per step over the step time (the workload's metric, causal runs
included); `value_executed` counts only the (query, key) pairs the mask
leaves visible (causal: N(N+1)/2 pairs per slice), the work the kernel does,
and the roofline fractions use that count.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun each rank runs its own copy of the workload (independent
(b, h) slices, no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import signal
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_attention_sub_b200 import api, inputs, replicas  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense ratio 4.5 / 2.25 PFLOP/s (INT8 dense equals FP8 dense)
# one metric for both arms: 4*B*H*N^2*d over the step time; the fraction of
# the tensor peak is in `roofline`
METRIC = "attention TOPS (4·B·H·N²·d/time) vs N; % of dense FP8/INT8 tensor peak"
FP4_OVER_BF16 = 4.0   # nominal dense ratio 9 / 2.25 PFLOP/s

# DRAM bytes (read + write) of one attention launch at the workload's full
# size, from one ncu capture of the kernel as it stands on a smaller case
# (inputs still above L2), scaled by the token count (attention traffic is
# the codes read once plus the output, linear in N).  null for other sizes.
TRAFFIC_BYTES = {"llm_prefill": 129.9e6, "video_dit": 200.6e6, "nvfp4": 66.8e6}

# per mode: tensor peak ratio to bf16, attention kernel, arithmetic description
MODE_INFO = {
    0: (FP8_OVER_BF16, "attn_i8f8_kernel", "int8 QK / e4m3 PV, fp32 softmax and accumulation"),
    1: (FP8_OVER_BF16, "attn_i8f8_kernel (FP16 accumulator)",
        "int8 QK / e4m3 PV, fp16 PV accumulation per 64 keys, fp32 softmax"),
    2: (FP4_OVER_BF16, "attn_fp4_kernel", "e2m1 QK and PV with ue4m3 block scales, fp32 softmax and accumulation"),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return PEAKS_FALLBACK, "fallback"


def dist_init():
    return replicas.init("nccl")


def barrier(ws):
    replicas.barrier(ws)


def allreduce_max(x, ws):
    return replicas.max_over_ranks(x, ws, "cuda")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.send_signal(signal.SIGTERM)
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_sample(w, max_rows):
    """The CPU oracle as it stands on a bounded sample of the workload: slice
    (b=0, h=0) quantized in full, attention for `max_rows` evenly spaced
    query rows.  Returns (ops of the sampled rows at 4*d per key of the row,
    all N keys, as the metric counts them; seconds; threads; rows)."""
    import oracle as orc
    q, k, v = inputs.generate(inputs.variant(w, B=1, H=1))
    f = lambda t: t.float().reshape(1, w.N, w.d).numpy()
    rows = np.unique(np.linspace(0, w.N - 1, min(max_rows, w.N)).astype(np.int32))
    t0 = time.perf_counter()
    if w.mode == 2:
        qz = orc.quantize_nvfp4(f(q), f(k), f(v), smooth_q=w.smooth_q)
        orc.attention_nvfp4(qz, w.causal, rows=rows)
    else:
        qz = orc.quantize_int8_fp8(f(q), f(k), f(v), smooth_q=w.smooth_q, mode=w.mode)
        orc.attention_int8_fp8(qz, w.causal, rows=rows)
    dt = time.perf_counter() - t0
    ops = float(4.0 * w.d * w.N * len(rows))
    return ops, dt, orc.num_threads(), len(rows)


def run_reference(args, w, ws, rank):
    if rank != 0:
        return
    import oracle as orc
    orc.build()
    rows = 512
    for _ in range(args.warmup):
        oracle_sample(w, rows)
    tot_ops, tot_t, thr, nr = 0.0, 0.0, 1, rows
    for _ in range(args.steps):
        ops, dt, thr, nr = oracle_sample(w, rows)
        tot_ops += ops
        tot_t += dt
    value = tot_ops / tot_t / 1e12
    sample = "slice (b0,h0) of %s quantized in full + attention of %d evenly spaced query rows per step" % (w.name, nr)
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": MODE_INFO[w.mode][2] + " (CPU oracle)", "data": "synthetic",
            "config": config_of(w, args, ws),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, args, ws):
    return {"workload": w.name, "B": w.B * ws, "H": w.H, "N": w.N, "d": w.d, "dtype": w.dtype,
            "causal": w.causal, "mode": ["INT8_FP8", "INT8_FP8_F16ACC", "NVFP4"][w.mode], "smooth_q": w.smooth_q,
            "parallelism": "replicas x%d (independent (b,h) slices per rank)" % ws,
            "l2": "inputs (3 x %.0f MB) larger than the 126 MB L2; no flush" % (
                w.B * w.H * w.N * w.d * 2 / 1e6)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llm_prefill")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--N", type=int, default=0,
                    help="override the workload's sequence length (small cases for profiling; "
                         "the headline runs use the workload's own N)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    w = inputs.WORKLOADS[args.workload] if args.workload in inputs.WORKLOADS else None
    if w is None and args.workload.startswith("sweep_"):
        _, n, d, c = args.workload.split("_")
        w = inputs.sweep(int(n[1:]), int(d[1:]), c == "causal")
    if args.N > 0:
        w = inputs.variant(w, N=args.N)
    ws, rank, local = dist_init() if args.impl == "ours" or int(os.environ.get("WORLD_SIZE", "1")) > 1 else (1, 0, 0)

    if args.impl == "reference":
        run_reference(args, w, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = w.shape()
    dcode = api.DTYPE_CODE[inputs.DTYPES[w.dtype]]
    # each rank draws its own slice batch (seed offset by rank)
    wr = inputs.variant(w, seed=replicas.rank_seed(w.seed, rank))
    q, k, v = [t.to(dev) for t in inputs.generate(wr, device="cuda")]
    out = torch.empty_like(q)
    wsbuf = api.alloc_workspace(B, H, N, d, w.mode, dev)
    nbytes = wsbuf.numel()
    stream = torch.cuda.current_stream()

    def step():
        ev_q.record(stream)
        api.sage_quantize_qkv(q, k, v, dcode, B, H, N, d, w.smooth_q, w.mode, wsbuf, nbytes, stream)
        ev_a.record(stream)
        api.sage_attn_quantized(wsbuf, nbytes, out, dcode, B, H, N, d, w.causal, w.smooth_q, w.mode, stream)
        ev_b.record(stream)

    ev_q, ev_a, ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(args.warmup):
        step()
    api.sage_check(wsbuf, nbytes, stream)

    # timed region: K steps; per-step attention-kernel events on the launch stream
    attn_ms = []
    ev_pairs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        ev_q, ev_a, ev_b = ev_pairs[i]
        step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    api.sage_check(wsbuf, nbytes, stream)
    ms = t_start.elapsed_time(t_stop) / args.steps
    attn_ms = [a_.elapsed_time(b_) for _, a_, b_ in ev_pairs]
    quant_ms = [q_.elapsed_time(a_) for q_, a_, _ in ev_pairs]
    ms = allreduce_max(ms, ws)
    attn_avg = allreduce_max(float(np.mean(attn_ms)), ws)
    quant_avg = allreduce_max(float(np.mean(quant_ms)), ws)

    ops_visible = inputs.executed_ops(w) * ws
    ops_square = inputs.attention_ops(w) * ws
    value = replicas.job_throughput(inputs.attention_ops(w), ms, ws) / 1e12

    # roofline of the dominant kernel (attention), live CUDA-event time
    peaks, peak_src = load_peaks()
    ratio, kname, dtype_desc = MODE_INFO[w.mode]
    peak_fp8 = peaks["bf16_tflops_sustained"] * ratio
    achieved = inputs.executed_ops(w) / (attn_avg * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak_fp8,
                "unit": "TFLOP/s", "frac": achieved / peak_fp8,
                "peak_source": "%s bf16_tflops_sustained x %.0f (nominal dense %s : BF16 ratio)" % (
                    peak_src, ratio, "FP4" if w.mode == 2 else "FP8/INT8"),
                "traffic": TRAFFIC_BYTES.get(w.name) if args.N == 0 else None,
                "traffic_unit": "bytes per launch", "attn_ms": attn_avg}
    # the quantization pass (HBM-bound): 16-bit Q, K, V read once, int8/e4m3
    # codes written, statistics and scales (small) not counted
    Np = (N + 127) // 128 * 128
    # NVFP4: half a byte of code plus 1/16 byte of block scale per element
    q_bytes = 3 * B * H * N * d * 2 + (3 * B * H * Np * d * 9 // 16 if w.mode == 2 else 3 * B * H * Np * d)
    hbm = peaks["hbm_gbs"]
    quant_line = {"bound": "hbm", "kernel": "quant_pass_kernel (stats) + quant_fold_kernel + quant_pass_kernel (codes)", "ms": quant_avg,
                  "algorithmic_bytes": q_bytes, "achieved": q_bytes / (quant_avg * 1e-3) / 1e9,
                  "peak": hbm, "unit": "GB/s", "frac": q_bytes / (quant_avg * 1e-3) / 1e9 / hbm}

    # End to end through the C ABI with host buffers (pinned): every step's
    # host->device copy of Q, K, V and device->host copy of O are inside the
    # timed region.  Steps are pipelined the way a serving loop runs them:
    # step i+1's inputs cross the host link while step i computes and step
    # i-1's output comes back (two device buffer sets; copy-in, compute and
    # copy-out on their own streams, ordered by events).
    hq, hk, hv = [t.cpu().pin_memory() for t in (q, k, v)]
    houts = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dins = [[torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)] for _ in range(2)]
    douts = [torch.empty_like(out) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_c = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        for i in range(nsteps):
            sl = i % 2
            if i >= 2:
                s_in.wait_event(ev_c[i - 2])  # step i-2 has read this slot's inputs
            with torch.cuda.stream(s_in):
                for dst, src in zip(dins[sl], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # this slot's output has been copied out
            api.sage_attn_fwd(dins[sl][0], dins[sl][1], dins[sl][2], douts[sl], B, H, N, d, w.causal, w.mode,
                              dcode, w.smooth_q, wsbuf, nbytes, stream)
            ev_c[i].record(stream)
            s_out.wait_event(ev_c[i])
            with torch.cuda.stream(s_out):
                houts[sl].copy_(douts[sl], non_blocking=True)
            ev_out[i].record(s_out)
        return ev_out[-1]

    e2e_run(2)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(4, min(args.steps, 12))
    e0.record(s_in)
    last = e2e_run(e2e_steps)
    s_out.wait_event(last)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(e0.elapsed_time(e1) / e2e_steps, ws)
    api.sage_check(wsbuf, nbytes, stream)
    in_bytes = 3 * q.numel() * q.element_size()
    out_bytes = out.numel() * out.element_size()

    line = {"metric": METRIC, "value": value,
            "unit": "TOPS", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_desc, "data": "synthetic",
            "config": config_of(w, args, ws),
            "value_executed": ops_visible / (ms * 1e-3) / 1e12,
            "roofline": roofline,
            "quant_roofline": quant_line,
            "e2e": {"value": ops_square / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
                    "pipelined": "step i+1's H2D copy overlaps step i's compute and step i-1's D2H copy"},
            # per step: the stats, fold and codes quantization kernels and the attention kernel
            "gpu_launches": 4 * args.steps,
            "clocks": clk}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle as orc
        orc.build()
        ops, dt, thr, nr = oracle_sample(w, 2048)
        line["cpu_baseline"] = {"value": ops / dt / 1e12, "unit": "TOPS", "cores": thr, "kind": "oracle",
                                "sample": "slice (b0,h0) quantized in full + attention of %d evenly spaced "
                                          "query rows; %.1f s" % (nr, dt)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
