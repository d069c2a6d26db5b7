#!/usr/bin/env python
"""Throughput of the quantized attention forward on B200.

One step = one pass of the whole hot path over one batch: smoothing + INT8/FP8
quantization of Q, K, V (libsage quantize kernels) and the fused attention
kernel, all through the C ABI (libsage.so).

Headline workload: the kernel-speed sweep's target point, B4 H32 N32768 d128
fp16, non-causal, INT8 QK / FP8 PV with the FP32 accumulator (the point the
kernel's roofline aim is quoted on: N >= 16K, d = 128).  Its inputs (3 x 1.07
GB) are far larger than the 126 MB L2, so no flush runs between steps.

Prints ONE JSON line (rank 0).  `value` is whole-job attention TOPS,
4*B*H*N^2*d per step over the step time (the metric as stated, causal runs
included); `value_executed` counts only the (query, key) pairs the mask leaves
visible (causal: N(N+1)/2 per slice), the work the kernel does, and the
roofline fractions use that count.  With one GPU the line also carries:
  per_config   every other point of the sweep (B4 H32, N 1K..32K, d 64/128,
               causal and not) and the llm_prefill, video_dit and nvfp4
               workloads, each timed the same way;
  tensor_peaks the tensor-core rate probe (sage_probe_mma_rate) per
               instruction kind, the denominators of the fractions;
  accuracy     cos / relative L1 / RMSE of the output against fp64 attention
               and max-abs against the CPU oracle, on sampled rows
               (SageAttention2++ summary, App. A.2).

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun each rank runs its own copy of the workload (independent
(b, h) slices, no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import json
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
# nominal dense datasheet rates per GPU (TFLOP/s), context beside the probe
NOMINAL_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0, "int8": 4500.0, "fp4": 9000.0}
METRIC = "attention TOPS (4·B·H·N²·d/time) vs N; % of dense FP8/INT8 tensor peak"
HEADLINE = "sweep_N32768_d128_full"

# DRAM bytes (read + write) of one attention launch of the headline workload:
# one ncu capture of the kernel as it stands on B4 H32 N8192 d128 (inputs
# above L2), scaled by the token count (non-causal attention traffic is the
# codes read once plus the output, linear in N): 403,055,360 B read +
# 232,906,752 B written at N = 8192, times 4.
TRAFFIC_BYTES = {"sweep_N32768_d128_full": 4 * (403055360 + 232906752)}

MODE_NAMES = ["INT8_FP8", "INT8_FP8_F16ACC", "NVFP4"]
MODE_INFO = {
    0: ("attn_i8f8_kernel", "int8 QK / e4m3 PV, fp32 softmax and accumulation"),
    1: ("attn_i8f8_kernel (FP16 accumulator)", "int8 QK / e4m3 PV, fp16 PV accumulation per 64 keys, fp32 softmax"),
    2: ("attn_fp4_kernel", "e2m1 QK and PV with ue4m3 block scales, fp32 softmax and accumulation"),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return PEAKS_FALLBACK, "fallback"


def workload(name):
    if name in inputs.WORKLOADS:
        return inputs.WORKLOADS[name]
    if name.startswith("sweep_"):
        _, n, d, c = name.split("_")
        return inputs.sweep(int(n[1:]), int(d[1:]), c == "causal")
    raise SystemExit("unknown workload %s" % name)


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


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample(w, max_rows, threads=0, keep=None):
    """The CPU oracle as it stands on a bounded sample of the workload: slice
    (b=0, h=0) quantized in full, attention for `max_rows` evenly spaced
    query rows.  Returns (ops of the sampled rows at 4*d per key the row sees
    -- all N keys, or i+1 for row i under a causal mask; seconds; threads;
    rows).  keep: a dict that receives the inputs, rows and oracle output."""
    import oracle as orc
    if threads:
        orc.set_num_threads(threads)
    q, k, v = inputs.generate(inputs.variant(w, B=1, H=1))
    f = lambda t: t.float().reshape(1, w.N, w.d).numpy()
    rows = np.unique(np.linspace(0, w.N - 1, min(max_rows, w.N)).astype(np.int32))
    t0 = time.perf_counter()
    if w.mode == 2:
        qz = orc.quantize_nvfp4(f(q), f(k), f(v), smooth_q=w.smooth_q)
        o = orc.attention_nvfp4(qz, w.causal, rows=rows)
    else:
        qz = orc.quantize_int8_fp8(f(q), f(k), f(v), smooth_q=w.smooth_q, mode=w.mode)
        o = orc.attention_int8_fp8(qz, w.causal, rows=rows)
    dt = time.perf_counter() - t0
    if keep is not None:
        keep.update(q=q, k=k, v=v, rows=rows, out=o)
    keys = (rows.astype(np.float64) + 1.0).sum() if w.causal else float(w.N) * len(rows)
    return float(4.0 * w.d * keys), dt, orc.num_threads(), len(rows)


def gpu_vs_oracle(w, keep, dev):
    """The GPU path (sage_attn_fwd) on the oracle sample's slice: max-abs and
    relative L1 of its output against the oracle's, both in the output dtype."""
    q, k, v = [keep[n].to(dev) for n in ("q", "k", "v")]
    out = api.attn_fwd(q, k, v, causal=w.causal, mode=w.mode, smooth_q=w.smooth_q)
    torch.cuda.synchronize()
    got = out.float().cpu().reshape(w.N, w.d).numpy()[keep["rows"]].astype(np.float64)
    ref = torch.from_numpy(keep["out"][0]).to(inputs.DTYPES[w.dtype]).double().numpy()
    diff = np.abs(got - ref)
    return {"max_abs": float(diff.max()), "rel_l1": float(diff.sum() / np.abs(ref).sum()),
            "sample": "slice (b0,h0) of the CPU sample, %d rows" % len(keep["rows"])}


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
    sample = ("slice (b0,h0) of %s quantized in full + attention of %d evenly spaced query rows per step "
              "(ops counted over the keys each row sees)" % (w.name, nr))
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": MODE_INFO[w.mode][1] + " (CPU oracle)", "data": "synthetic",
            "config": config_of(w, ws),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w, ws, q_blocks=False):
    return {"workload": w.name, "B": w.B * ws, "H": w.H, "N": w.N, "d": w.d, "dtype": w.dtype,
            "causal": w.causal, "mode": MODE_NAMES[w.mode], "smooth_q": w.smooth_q, "q_blocks": q_blocks,
            "parallelism": "replicas x%d (independent (b,h) slices per rank)" % ws,
            "l2": "inputs (3 x %.0f MB) larger than the 126 MB L2; no flush" % (
                w.B * w.H * w.N * w.d * 2 / 1e6)}


# --------------------------------------------------------------------------
# Tensor-core rate probe
# --------------------------------------------------------------------------
PROBE_KINDS = {"int8": api.PROBE_I8, "fp8_f32acc": api.PROBE_F8_F32ACC, "fp8_f16acc": api.PROBE_F8_F16ACC,
               "bf16": api.PROBE_BF16, "fp4": api.PROBE_FP4}


def probe_peaks(dev, sm_count):
    """TFLOP/s of back-to-back tcgen05.mma per kind, one CTA per SM: `burst`
    = one ~20 ms launch after a warm-up launch (the rate a kernel timed alone
    sees), `sustained` = back-to-back launches for ~1.5 s (under the power
    cap).  Each figure is the CUDA-event time of its launches."""
    wsb = api.alloc_workspace(1, 1, 128, 64, 0, dev)
    stream = torch.cuda.current_stream()
    out = {}
    for name, kind in PROBE_KINDS.items():
        ops1 = api.sage_probe_mma_rate(kind, sm_count, 256, wsb, wsb.numel(), stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        api.sage_probe_mma_rate(kind, sm_count, 256, wsb, wsb.numel(), stream)
        e1.record(stream)
        torch.cuda.synchronize()
        t_small = e0.elapsed_time(e1) * 1e-3
        # size one launch at ~20 ms from the small one's rate
        iters = int(min(1 << 20, max(256, 256 * 0.02 / max(t_small, 1e-6))))
        time.sleep(0.2)
        e0.record(stream)
        ops = api.sage_probe_mma_rate(kind, sm_count, iters, wsb, wsb.numel(), stream)
        e1.record(stream)
        torch.cuda.synchronize()
        burst = ops / (e0.elapsed_time(e1) * 1e-3) / 1e12
        n_launch = 75
        e0.record(stream)
        for _ in range(n_launch):
            api.sage_probe_mma_rate(kind, sm_count, iters, wsb, wsb.numel(), stream)
        e1.record(stream)
        torch.cuda.synchronize()
        sustained = n_launch * ops / (e0.elapsed_time(e1) * 1e-3) / 1e12
        out[name] = {"burst": burst, "sustained": sustained, "unit": "TFLOP/s",
                     "launch": "%d CTAs x %d x 4 MMAs M128 N256" % (sm_count, iters)}
        del ops1
    api.sage_check(wsb, wsb.numel(), stream)
    out["fp8_f16acc_over_f32acc"] = out["fp8_f16acc"]["burst"] / out["fp8_f32acc"]["burst"]
    return out


def mode_peak(mode, probe, which="burst"):
    """Tensor peak of one attention step's mix: half the operations are the
    QK^T product, half the PV product, so the peak is the harmonic mean of
    the two instruction rates (INT8 and FP8 with the mode's accumulator), or
    the FP4 rate."""
    if mode == 2:
        return probe["fp4"][which]
    pv = probe["fp8_f16acc" if mode == 1 else "fp8_f32acc"][which]
    return 2.0 / (1.0 / probe["int8"][which] + 1.0 / pv)


# --------------------------------------------------------------------------
# Device timing of one workload
# --------------------------------------------------------------------------
def time_workload(w, dev, steps, warmup, seed_rank=0, clocks=None, ws=1, q_blocks=False):
    """Quantize + attention steps on device-resident inputs; CUDA events on
    the launch stream around each kernel group.  Returns the timings and the
    tensors (for the accuracy and e2e legs).  q_blocks: Q smoothed per
    128-row block (the sage_*_blocksmooth calls)."""
    B, H, N, d = w.shape()
    dcode = api.DTYPE_CODE[inputs.DTYPES[w.dtype]]
    wr = inputs.variant(w, seed=replicas.rank_seed(w.seed, seed_rank))
    q, k, v = [t.to(dev) for t in inputs.generate(wr, device="cuda")]
    out = torch.empty_like(q)
    wsbuf = (api.alloc_workspace_blocksmooth if q_blocks else api.alloc_workspace)(B, H, N, d, w.mode, dev)
    nbytes = wsbuf.numel()
    stream = torch.cuda.current_stream()

    def step(ev):
        ev[0].record(stream)
        if q_blocks:
            api.sage_quantize_qkv_blocksmooth(q, k, v, dcode, B, H, N, d, w.mode, wsbuf, nbytes, stream)
        else:
            api.sage_quantize_qkv(q, k, v, dcode, B, H, N, d, w.smooth_q, w.mode, wsbuf, nbytes, stream)
        ev[1].record(stream)
        if q_blocks:
            api.sage_attn_quantized_blocksmooth(wsbuf, nbytes, out, dcode, B, H, N, d, w.causal, w.mode, stream)
        else:
            api.sage_attn_quantized(wsbuf, nbytes, out, dcode, B, H, N, d, w.causal, w.smooth_q, w.mode, stream)
        ev[2].record(stream)

    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    for i in range(warmup):
        step(evs[i % steps])
    api.sage_check(wsbuf, nbytes, stream)
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    replicas.barrier(ws)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(steps):
        step(evs[i])
    t_stop.record(stream)
    torch.cuda.synchronize()
    replicas.barrier(ws)
    clk = clocks.stop() if clocks is not None else None
    api.sage_check(wsbuf, nbytes, stream)
    ms = t_start.elapsed_time(t_stop) / steps
    attn_ms = float(np.mean([a.elapsed_time(b) for _, a, b in evs]))
    quant_ms = float(np.mean([s.elapsed_time(a) for s, a, _ in evs]))
    return dict(ms=ms, attn_ms=attn_ms, quant_ms=quant_ms, clocks=clk, q=q, k=k, v=v, out=out, ws=wsbuf,
                dcode=dcode)


def quant_bytes(w):
    """Algorithmic bytes of the quantization pass: 16-bit Q, K, V read once,
    the codes written once (INT8/e4m3: 1 byte; NVFP4: half a byte plus 1/16
    byte of block scale); statistics and per-granule scales not counted."""
    B, H, N, d = w.shape()
    Np = (N + 127) // 128 * 128
    return 3 * B * H * N * d * 2 + (3 * B * H * Np * d * 9 // 16 if w.mode == 2 else 3 * B * H * Np * d)


def summarize(w, t, probe, hbm):
    """Figures of one timed workload (single rank)."""
    ex = inputs.executed_ops(w)
    attn_tops = ex / (t["attn_ms"] * 1e-3) / 1e12
    qb = quant_bytes(w)
    s = {"workload": w.name, "mode": MODE_NAMES[w.mode], "causal": w.causal,
         "ms_per_step": t["ms"], "value": inputs.attention_ops(w) / (t["ms"] * 1e-3) / 1e12,
         "value_executed": ex / (t["ms"] * 1e-3) / 1e12,
         "attn_ms": t["attn_ms"], "attn_tops_executed": attn_tops,
         "quant_ms": t["quant_ms"], "quant_gbs": qb / (t["quant_ms"] * 1e-3) / 1e9,
         "quant_frac_hbm": qb / (t["quant_ms"] * 1e-3) / 1e9 / hbm}
    if probe is not None:
        s["attn_frac_of_probe_burst"] = attn_tops / mode_peak(w.mode, probe)
    return s


def accuracy_metrics(o_test, o_ref) -> dict:
    """Cosine similarity, relative L1 and RMSE of O' against O (the metrics of
    the SageAttention2++ summary, App. A.2)."""
    a = np.asarray(o_test, np.float64).ravel()
    b = np.asarray(o_ref, np.float64).ravel()
    return {"cos": float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b))),
            "rel_l1": float(np.abs(a - b).sum() / np.abs(b).sum()),
            "rmse": float(np.sqrt(np.mean((a - b) ** 2)))}


def accuracy_leg(w, t, rows_n=48):
    """cos / rel-L1 / RMSE of the GPU output against softmax(Q K^T / sqrt(d)) V
    of the unquantized inputs, computed in float64 (torch, on the device), on
    `rows_n` evenly spaced query rows of slice (b0, h0)."""
    B, H, N, d = w.shape()
    sl = lambda x: x.reshape(B * H, N, d)[0].double()
    q, k, v = sl(t["q"]), sl(t["k"]), sl(t["v"])
    rows = torch.from_numpy(np.unique(np.linspace(0, N - 1, rows_n).astype(np.int64))).to(q.device)
    s = (q[rows] @ k.T) / np.sqrt(d)
    if w.causal:
        s = s.masked_fill(torch.arange(N, device=q.device)[None, :] > rows[:, None], float("-inf"))
    ref = torch.softmax(s, dim=1) @ v
    got = t["out"].reshape(B * H, N, d)[0, rows].double()
    return {"vs_fp64": accuracy_metrics(got.cpu().numpy(), ref.cpu().numpy()),
            "sample": "slice (b0,h0), %d evenly spaced query rows" % len(rows)}


def e2e_leg(w, t, dev, steps, ws, q_blocks=False):
    """End to end through the C ABI with host buffers (pinned): every step's
    host->device copy of Q, K, V and device->host copy of O are inside the
    timed region.  Steps are pipelined the way a serving loop runs them:
    step i+1's inputs cross the host link while step i computes and step
    i-1's output comes back (two device buffer sets; copy-in, compute and
    copy-out on their own streams, ordered by events)."""
    B, H, N, d = w.shape()
    q, k, v, out, wsbuf = t["q"], t["k"], t["v"], t["out"], t["ws"]
    nbytes = wsbuf.numel()
    stream = torch.cuda.current_stream()
    hq, hk, hv = [x.cpu().pin_memory() for x in (q, k, v)]
    houts = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dins = [[q, k, v], [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]]
    douts = [out, torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def run(nsteps):
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
            if q_blocks:
                api.sage_attn_fwd_blocksmooth(dins[sl][0], dins[sl][1], dins[sl][2], douts[sl], B, H, N, d,
                                              w.causal, w.mode, t["dcode"], wsbuf, nbytes, stream)
            else:
                api.sage_attn_fwd(dins[sl][0], dins[sl][1], dins[sl][2], douts[sl], B, H, N, d, w.causal, w.mode,
                                  t["dcode"], w.smooth_q, wsbuf, nbytes, stream)
            ev_c[i].record(stream)
            s_out.wait_event(ev_c[i])
            with torch.cuda.stream(s_out):
                houts[sl].copy_(douts[sl], non_blocking=True)
            ev_out[i].record(s_out)
        return ev_out[-1]

    run(2)
    torch.cuda.synchronize()
    replicas.barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    last = run(steps)
    s_out.wait_event(last)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks(e0.elapsed_time(e1) / steps, ws, "cuda")
    api.sage_check(wsbuf, nbytes, stream)
    in_bytes = 3 * q.numel() * q.element_size()
    out_bytes = out.numel() * out.element_size()
    return {"value": inputs.attention_ops(w) * ws / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
            "pipelined": "step i+1's H2D copy overlaps step i's compute and step i-1's D2H copy"}


def fused_leg(w, dev, steps, warmup):
    """The whole step through sage_attn_fwd_fused (Q quantized inside the
    attention kernel) against the same step through sage_attn_fwd, CUDA
    events on the launch stream; device-resident inputs."""
    B, H, N, d = w.shape()
    dcode = api.DTYPE_CODE[inputs.DTYPES[w.dtype]]
    q, k, v = [t.to(dev) for t in inputs.generate(w, device="cuda")]
    out = torch.empty_like(q)
    wsbuf = api.alloc_workspace(B, H, N, d, w.mode, dev)
    stream = torch.cuda.current_stream()
    fns = (("unfused", api.sage_attn_fwd), ("fused", api.sage_attn_fwd_fused))
    for _, fn in fns:
        for _ in range(warmup):
            fn(q, k, v, out, B, H, N, d, w.causal, w.mode, dcode, w.smooth_q, wsbuf, wsbuf.numel(), stream)
    # the two calls alternate (three rounds, median of each), so that clock
    # drift under the power cap falls on both alike
    times = {name: [] for name, _ in fns}
    for _ in range(3):
        for name, fn in fns:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn(q, k, v, out, B, H, N, d, w.causal, w.mode, dcode, w.smooth_q, wsbuf, wsbuf.numel(), stream)
            e1.record(stream)
            torch.cuda.synchronize()
            times[name].append(e0.elapsed_time(e1) / steps)
    api.sage_check(wsbuf, wsbuf.numel(), stream)
    res = {name + "_ms": float(np.median(t)) for name, t in times.items()}
    res["rounds"] = "3 alternating rounds of %d steps each, medians" % steps
    res["value_fused"] = inputs.attention_ops(w) / (res["fused_ms"] * 1e-3) / 1e12
    return res


def visible_pairs(Nq, Nk, causal):
    """(query, key) pairs a slice computes: all Nq * Nk, or under the causal
    mask aligned to the last key (query row i sees keys j <= i + Nk - Nq)
    sum over i of min(Nk, i + Nk - Nq + 1)."""
    if not causal:
        return Nq * Nk
    koff = Nk - Nq
    # rows with i + koff + 1 < Nk see i + koff + 1 keys; the rest see Nk
    full_from = max(0, Nk - koff - 1)
    n_part = min(Nq, full_from)
    part = n_part * (koff + 1) + n_part * (n_part - 1) // 2
    return part + (Nq - n_part) * Nk


GQA_CASES = (
    # (name, base workload for the value law, B, Hq, Hkv, Nq, Nk, causal)
    ("llm_prefill_gqa4", "llm_prefill", 1, 32, 8, 8192, 8192, True),
    ("chunked_prefill_gqa4", "llm_prefill", 1, 32, 8, 2048, 32768, True),
)


def gqa_leg(dev, steps, warmup, probe):
    """Grouped key/value heads and separate lengths (sage_*_gqa): quantization
    and attention timed apart with CUDA events on the launch stream, inputs
    drawn from the workload's value law (Q with Hq heads and Nq rows, K and V
    with Hkv heads and Nk rows).  Operations count the visible pairs."""
    res = {}
    for name, base, B, Hq, Hkv, Nq, Nk, causal in GQA_CASES:
        w0 = workload(base)
        q = inputs.generate(inputs.variant(w0, B=B, H=Hq, N=Nq), device="cuda")[0].to(dev)
        _, k, v = inputs.generate(inputs.variant(w0, B=B, H=Hkv, N=Nk, seed=w0.seed + 1), device="cuda")
        k, v = k.to(dev), v.to(dev)
        d = q.shape[-1]
        dcode = api.DTYPE_CODE[q.dtype]
        out = torch.empty_like(q)
        wsbuf = api.alloc_workspace_gqa(B, Hq, Hkv, Nq, Nk, d, w0.mode, dev)
        stream = torch.cuda.current_stream()
        fq = lambda: api.sage_quantize_qkv_gqa(q, k, v, dcode, B, Hq, Hkv, Nq, Nk, d, False, w0.mode, wsbuf,
                                               wsbuf.numel(), stream)
        fa = lambda: api.sage_attn_quantized_gqa(wsbuf, wsbuf.numel(), out, dcode, B, Hq, Hkv, Nq, Nk, d, causal,
                                                 False, w0.mode, stream)
        for _ in range(warmup):
            fq()
            fa()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e in evs:
            e[0].record(stream)
            fq()
            e[1].record(stream)
            fa()
            e[2].record(stream)
        torch.cuda.synchronize()
        api.sage_check(wsbuf, wsbuf.numel(), stream)
        quant_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in evs]))
        attn_ms = float(np.mean([b.elapsed_time(c) for _, b, c in evs]))
        ops = 4.0 * B * Hq * visible_pairs(Nq, Nk, causal) * d
        r = {"B": B, "Hq": Hq, "Hkv": Hkv, "Nq": Nq, "Nk": Nk, "d": d, "dtype": w0.dtype, "causal": causal,
             "mode": MODE_NAMES[w0.mode], "quant_ms": quant_ms, "attn_ms": attn_ms,
             "attn_tops_executed": ops / (attn_ms * 1e-3) / 1e12,
             "step_tops_executed": ops / ((quant_ms + attn_ms) * 1e-3) / 1e12}
        if probe is not None:
            r["attn_frac_of_probe_burst"] = r["attn_tops_executed"] / mode_peak(w0.mode, probe, "burst")
        res[name] = r
        del q, k, v, out, wsbuf
        torch.cuda.empty_cache()
    return res


def q_blocks_leg(w, dev, steps, warmup):
    """Q smoothed per slice (sage_quantize_qkv + sage_attn_quantized with
    smooth_q) against Q smoothed per 128-row block (the sage_*_blocksmooth
    calls) on the same inputs: quantization and attention timed apart, CUDA
    events on the launch stream, the two paths alternating (three rounds,
    medians).  The per-block quantization adds the block means and one bias
    row per block: Npad^2 * d / 128 fp32 multiply-adds per slice."""
    w = inputs.variant(w, smooth_q=True)
    B, H, N, d = w.shape()
    dcode = api.DTYPE_CODE[inputs.DTYPES[w.dtype]]
    q, k, v = [t.to(dev) for t in inputs.generate(w, device="cuda")]
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    ws_s = api.alloc_workspace(B, H, N, d, w.mode, dev)
    ws_b = api.alloc_workspace_blocksmooth(B, H, N, d, w.mode, dev)
    paths = {
        "per_slice": (lambda: api.sage_quantize_qkv(q, k, v, dcode, B, H, N, d, True, w.mode, ws_s, ws_s.numel(),
                                                    stream),
                      lambda: api.sage_attn_quantized(ws_s, ws_s.numel(), out, dcode, B, H, N, d, w.causal, True,
                                                      w.mode, stream)),
        "per_block": (lambda: api.sage_quantize_qkv_blocksmooth(q, k, v, dcode, B, H, N, d, w.mode, ws_b,
                                                                ws_b.numel(), stream),
                      lambda: api.sage_attn_quantized_blocksmooth(ws_b, ws_b.numel(), out, dcode, B, H, N, d,
                                                                  w.causal, w.mode, stream)),
    }
    for fq, fa in paths.values():
        for _ in range(warmup):
            fq()
            fa()
    times = {name: ([], []) for name in paths}
    for _ in range(3):
        for name, (fq, fa) in paths.items():
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
            for e in evs:
                e[0].record(stream)
                fq()
                e[1].record(stream)
                fa()
                e[2].record(stream)
            torch.cuda.synchronize()
            times[name][0].append(float(np.mean([a.elapsed_time(b) for a, b, _ in evs])))
            times[name][1].append(float(np.mean([b.elapsed_time(c) for _, b, c in evs])))
    api.sage_check(ws_s, ws_s.numel(), stream)
    api.sage_check(ws_b, ws_b.numel(), stream)
    res = {}
    for name, (tq, ta) in times.items():
        res[name + "_quant_ms"] = float(np.median(tq))
        res[name + "_attn_ms"] = float(np.median(ta))
    Np = (N + 127) // 128 * 128
    fma = B * H * (Np // 128) * Np * d
    extra = res["per_block_quant_ms"] - res["per_slice_quant_ms"]
    res["bias_fma_per_step"] = fma
    res["bias_fma_rate_lower_bound_tfma_s"] = fma / (extra * 1e-3) / 1e12 if extra > 0 else None
    res["value_per_block"] = inputs.attention_ops(w) / ((res["per_block_quant_ms"] + res["per_block_attn_ms"]) *
                                                        1e-3) / 1e12
    res["rounds"] = "3 alternating rounds of %d steps each, medians; the rate bound charges the whole extra " \
                    "quantization time to the bias rows" % steps
    return res


def per_config_leg(dev, steps, probe, hbm, skip):
    names = ["sweep_N%d_d%d_%s" % (n, d, c) for d in (128, 64) for c in ("full", "causal")
             for n in (1024, 2048, 4096, 8192, 16384, 32768)]
    names += ["llm_prefill", "video_dit", "nvfp4"]
    res = {}
    for name in names:
        if name == skip:
            continue
        w = workload(name)
        t = time_workload(w, dev, steps, 3)
        res[name] = summarize(w, t, probe, hbm)
        del t
        torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the per-config sweep, the tensor-core probe and the accuracy leg")
    ap.add_argument("--q-blocks", action="store_true",
                    help="smooth Q per 128-row block (sage_*_blocksmooth calls; implies smooth_q)")
    ap.add_argument("--N", type=int, default=0,
                    help="override the workload's sequence length (small cases for profiling; "
                         "the headline runs use the workload's own N)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    w = workload(args.workload)
    if args.N > 0:
        w = inputs.variant(w, N=args.N)
    if args.q_blocks:
        w = inputs.variant(w, smooth_q=True)
    ws, rank, local = replicas.init("nccl") if args.impl == "ours" or int(
        os.environ.get("WORLD_SIZE", "1")) > 1 else (1, 0, 0)

    if args.impl == "reference":
        run_reference(args, w, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    extras = ws == 1 and not args.no_extras and not args.q_blocks

    # every rank probes its own GPU (no collective), so the roofline fraction
    # has the same denominator at every N
    probe = probe_peaks(dev, sm_count) if not args.no_extras else None

    clocks = ClockSampler(local)
    t = time_workload(w, dev, args.steps, args.warmup, seed_rank=rank, clocks=clocks, ws=ws, q_blocks=args.q_blocks)
    ms = replicas.max_over_ranks(t["ms"], ws, "cuda")
    attn_avg = replicas.max_over_ranks(t["attn_ms"], ws, "cuda")
    quant_avg = replicas.max_over_ranks(t["quant_ms"], ws, "cuda")
    value = replicas.job_throughput(inputs.attention_ops(w), ms, ws) / 1e12

    # roofline of the dominant kernel (attention), live CUDA-event time
    kname, dtype_desc = MODE_INFO[w.mode]
    achieved = inputs.executed_ops(w) / (attn_avg * 1e-3) / 1e12
    nominal = NOMINAL_TFLOPS["fp4" if w.mode == 2 else "fp8"]
    if probe is not None:
        peak = mode_peak(w.mode, probe, "burst")
        peak_source = ("tensor-core probe (sage_probe_mma_rate), burst: harmonic mean of the INT8 and FP8 "
                       "(accumulator of the mode) rates, half the operations each" if w.mode != 2 else
                       "tensor-core probe (sage_probe_mma_rate), burst: block-scaled FP4 rate")
    else:
        peak = peaks["bf16_tflops"] * (4.0 if w.mode == 2 else 2.0)
        peak_source = "%s bf16_tflops (burst) x nominal dense %s:BF16 ratio" % (peak_src, "FP4" if w.mode == 2
                                                                              else "FP8")
    traffic = TRAFFIC_BYTES.get(w.name) if args.N == 0 else None
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": peak_source,
                "frac_of_nominal": achieved / nominal,
                "nominal": "%.0f TFLOP/s dense datasheet" % nominal,
                "traffic": traffic, "traffic_unit": "bytes per launch", "attn_ms": attn_avg,
                "algorithmic_ops_per_launch": inputs.executed_ops(w)}
    qb = quant_bytes(w)
    qkern = "quant_pass_kernel (stats) + quant_fold_kernel + quant_pass_kernel (codes)"
    if args.q_blocks:
        qkern += " + quant_fold_qblock_kernel + qblock_bias_kernel (bias rows not counted in the bytes)"
    quant_line = {"bound": "hbm", "kernel": qkern,
                  "ms": quant_avg, "algorithmic_bytes": qb, "achieved": qb / (quant_avg * 1e-3) / 1e9,
                  "peak": hbm, "unit": "GB/s", "frac": qb / (quant_avg * 1e-3) / 1e9 / hbm,
                  "peak_source": "%s hbm_gbs" % peak_src}

    acc = accuracy_leg(w, t) if rank == 0 and extras else None
    # up to 20 pipelined steps: the first copy-in and the last compute and
    # copy-out are not overlapped, a fixed cost that more steps amortize
    e2e = e2e_leg(w, t, dev, max(4, min(args.steps, 20)), ws, q_blocks=args.q_blocks)
    clk = t["clocks"]
    del t
    torch.cuda.empty_cache()

    per_config = per_config_leg(dev, min(args.steps, 10), probe, hbm, w.name) if extras else None
    fused = None
    if extras and w.mode != 2:
        fused = {w.name: fused_leg(w, dev, min(args.steps, 10), 3)}
        torch.cuda.empty_cache()
        fused["llm_prefill"] = fused_leg(workload("llm_prefill"), dev, 10, 3)
        torch.cuda.empty_cache()
    gqa = gqa_leg(dev, 10, 3, probe) if extras else None
    q_blocks = None
    if extras and w.mode != 2:
        q_blocks = {}
        for name in ("video_dit", "llm_prefill"):
            q_blocks[name] = q_blocks_leg(workload(name), dev, 10, 3)
            torch.cuda.empty_cache()

    line = {"metric": METRIC, "value": value,
            "unit": "TOPS", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_desc, "data": "synthetic",
            "config": config_of(w, ws, args.q_blocks),
            "value_executed": inputs.executed_ops(w) * ws / (ms * 1e-3) / 1e12,
            "roofline": roofline,
            "quant_roofline": quant_line,
            "e2e": e2e,
            # per step: the stats, fold and codes quantization kernels and the attention kernel
            # (Q smoothed per block: also the block-mean fold and the bias rows)
            "gpu_launches": (6 if args.q_blocks else 4) * args.steps,
            "clocks": clk}
    if probe is not None:
        line["tensor_peaks"] = probe
    if acc is not None:
        line["accuracy"] = acc
    if per_config is not None:
        line["per_config"] = per_config
    if fused is not None:
        # Q quantized inside the attention kernel (sage_attn_fwd_fused), whole step
        line["fused_q"] = fused
    if q_blocks is not None:
        # Q smoothed per slice vs per 128-row block (sage_*_blocksmooth)
        line["q_blocks"] = q_blocks
    if gqa is not None:
        # grouped key/value heads and separate query / key lengths (sage_*_gqa)
        line["gqa"] = gqa
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle as orc
        orc.build()
        keep = {}
        ops, dt, thr, nr = oracle_sample(w, 2048, keep=keep)
        if "accuracy" in line:
            line["accuracy"]["vs_oracle"] = gpu_vs_oracle(w, keep, dev)
        cpu = {"value": ops / dt / 1e12, "unit": "TOPS", "cores": thr, "kind": "oracle",
               "sample": "slice (b0,h0) quantized in full + attention of %d evenly spaced query rows; %.1f s "
                         "(ops counted over the keys each row sees)" % (nr, dt)}
        if extras:
            single = {}
            for name, rows_n in (("unit", 128), ("llm_prefill", 64)):
                o1, d1, _, n1 = oracle_sample(workload(name), rows_n, threads=1)
                single[name] = {"value": o1 / d1 / 1e12, "unit": "TOPS", "seconds": d1, "rows": n1}
            orc.set_num_threads(thr)
            cpu["single_thread"] = single
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
