"""Seeded synthetic inputs shaped like the workloads the SageAttention pages name.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle may consume its
tensors.  Values are drawn in float32 and cast to the workload dtype; the cast
tensors are what every side sees.

Workloads (the pages evaluate language, image and video models, SageAttention2
abstract and SageAttention2++ summary Sec. 4.1 / App. A.2; their datasets and
weights are not used -- these shapes and value laws stand in for them):

  unit        B1 H2  N128   d64  fp16  non-causal  Q,V ~ N(0,1), K ~ N(0,1) + b_c, b_c ~ N(0,2^2)
  llm_prefill B1 H32 N8192  d128 bf16  causal      as unit with b_c ~ N(0,3^2); one K channel in
                                                   a hundred (rounded, >= 1) per head scaled x10
  video_dit   B1 H12 N32760 d128 fp16  non-causal  Q,K,V ~ N(0,1); per-channel bias N(0,2^2) on Q and K
  sweep       B4 H32 N in 1K..32K, d in {64,128}, fp16, K bias N(0,2^2)
  nvfp4       B1 H16 N16384 d128 bf16  non-causal  Q,K,V Student-t with 3 degrees of freedom
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

MODE_INT8_FP8, MODE_INT8_FP8_F16ACC, MODE_NVFP4 = 0, 1, 2
DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str
    causal: bool
    mode: int
    smooth_q: bool
    law: str            # "k_bias", "k_bias_outlier", "qk_bias", "student_t3"
    bias_std: float = 2.0
    seed: int = 1000

    def shape(self):
        return (self.B, self.H, self.N, self.d)


WORKLOADS = {
    "unit": Workload("unit", 1, 2, 128, 64, "fp16", False, MODE_INT8_FP8, False, "k_bias", 2.0, 1001),
    "llm_prefill": Workload("llm_prefill", 1, 32, 8192, 128, "bf16", True, MODE_INT8_FP8, False,
                            "k_bias_outlier", 3.0, 1002),
    "video_dit": Workload("video_dit", 1, 12, 32760, 128, "fp16", False, MODE_INT8_FP8_F16ACC, True,
                          "qk_bias", 2.0, 1003),
    "nvfp4": Workload("nvfp4", 1, 16, 16384, 128, "bf16", False, MODE_NVFP4, False, "student_t3",
                      0.0, 1005),
}


def sweep(N: int, d: int, causal: bool) -> Workload:
    """One point of the kernel-speed sweep (B4 H32 fp16, K bias N(0,2^2))."""
    return Workload("sweep_N%d_d%d_%s" % (N, d, "causal" if causal else "full"), 4, 32, N, d, "fp16",
                    causal, MODE_INT8_FP8, False, "k_bias", 2.0, 1004 + 7919 * N + 31 * d + int(causal))


def variant(w: Workload, **kw) -> Workload:
    """The same value law with other sizes or flags (used for small parity cases)."""
    return replace(w, **kw)


def generate(w: Workload, device: str = "cpu"):
    """Return (q, k, v) of shape [B, H, N, d] in the workload dtype on `device`.

    Draws happen on `device` with a generator seeded by the workload seed, so
    the CPU and CUDA streams differ; each is reproducible on its own."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    B, H, N, d = w.shape()
    f32 = dict(dtype=torch.float32, device=device, generator=g)

    def randn(*s):
        return torch.randn(*s, **f32)

    if w.law == "student_t3":
        def t3(*s):
            z = randn(*s)
            chi2 = randn(3, *s).pow_(2).sum(0)
            return z / torch.sqrt(chi2 / 3.0)
        q, k, v = t3(B, H, N, d), t3(B, H, N, d), t3(B, H, N, d)
    else:
        q, k, v = randn(B, H, N, d), randn(B, H, N, d), randn(B, H, N, d)
        k += w.bias_std * randn(B, H, 1, d)
        if w.law == "qk_bias":
            q += w.bias_std * randn(B, H, 1, d)
        if w.law == "k_bias_outlier":
            n_out = max(1, int(round(0.01 * d)))
            for h in range(H):
                ch = torch.randperm(d, generator=g, device=device)[:n_out]
                k[:, h, :, ch] *= 10.0
    dt = DTYPES[w.dtype]
    return q.to(dt), k.to(dt), v.to(dt)


def attention_ops(w: Workload) -> float:
    """Operation count 4*B*H*N^2*d of the attention (two matmuls, 2 ops per MAC)."""
    return 4.0 * w.B * w.H * w.N * w.N * w.d


def executed_ops(w: Workload) -> float:
    """Operations over the (query, key) pairs the mask leaves visible: all
    N^2 pairs, or N(N+1)/2 under a causal mask."""
    if not w.causal:
        return attention_ops(w)
    return 4.0 * w.B * w.H * (w.N * (w.N + 1) / 2.0) * w.d
