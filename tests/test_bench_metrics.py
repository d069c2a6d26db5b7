"""The bench line's arithmetic (CPU): algorithmic operation counts and
quantization bytes against brute-force counts over small shapes."""
import importlib.util
import os

import numpy as np
import pytest

from quantized_attention_sub_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("N,d,causal", [(1, 64, False), (1, 64, True), (7, 128, True), (130, 64, False),
                                         (257, 128, True)])
def test_operation_counts_match_visible_pairs(N, d, causal):
    """4*d operations per visible (query, key) pair (two matmuls, 2 ops per
    multiply-add): all N^2 pairs, or the pairs j <= i under a causal mask."""
    w = inputs.variant(inputs.WORKLOADS["unit"], B=2, H=3, N=N, d=d, causal=causal)
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    visible = int(np.count_nonzero(j <= i)) if causal else N * N
    assert inputs.attention_ops(w) == 4.0 * 2 * 3 * N * N * d
    assert inputs.executed_ops(w) == 4.0 * 2 * 3 * visible * d


@pytest.mark.parametrize("N,d,mode", [(1, 64, 0), (300, 128, 0), (300, 128, 1), (128, 128, 2), (1000, 64, 2)])
def test_quantization_bytes(N, d, mode):
    """Q, K and V read once at 2 bytes per element; codes written once for the
    padded tokens: 1 byte (INT8 / e4m3) or, in NVFP4, half a byte plus one
    1-byte block scale per 16 elements."""
    b = _bench()
    w = inputs.variant(inputs.WORKLOADS["unit"], B=1, H=2, N=N, d=d, mode=mode)
    Np = -(-N // 128) * 128
    reads = 3 * 2 * N * d * 2
    codes = 3 * 2 * Np * d * (0.5 + 1.0 / 16) if mode == 2 else 3 * 2 * Np * d
    assert b.quant_bytes(w) == reads + codes


@pytest.mark.parametrize("Nq,Nk,causal", [(1, 1, True), (5, 5, True), (3, 10, True), (7, 130, True), (128, 128, False),
                                           (2048, 4096, True), (10, 3, False)])
def test_visible_pairs_match_brute_force(Nq, Nk, causal):
    """Pairs the grouped-head leg counts: query row i sees keys j <= i + Nk - Nq
    under the causal mask (aligned to the last key), every key otherwise."""
    b = _bench()
    i, j = np.meshgrid(np.arange(Nq), np.arange(Nk), indexing="ij")
    brute = int(np.count_nonzero(j <= i + (Nk - Nq))) if causal else Nq * Nk
    assert b.visible_pairs(Nq, Nk, causal) == brute
