"""Pins of the oracle's per-block Q smoothing (CPU): Q smoothed per block of
128 query rows, each block's bias row added to its rows' logits.  Checked
against closed forms, the per-slice path it reduces to, fp64 identities and
fp64 attention."""
import numpy as np
import pytest

import oracle as orc


def _fp64_attention(q, k, v, causal):
    BH, N, d = q.shape
    s = np.einsum("bid,bjd->bij", q.astype(np.float64), k.astype(np.float64)) / np.sqrt(d)
    if causal:
        s = np.where(np.arange(N)[None, None, :] > np.arange(N)[None, :, None], -np.inf, s)
    p = np.exp(s - s.max(-1, keepdims=True))
    return np.einsum("bij,bjd->bid", p / p.sum(-1, keepdims=True), v.astype(np.float64))


def _qkv(N, d, seed, block_offsets=True, BH=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((BH, N, d)).astype(np.float32)
    if block_offsets:
        # a different per-channel offset in every 128-row block
        for b in range(0, N, 128):
            q[:, b:b + 128] += (4.0 * rng.standard_normal((BH, 1, d))).astype(np.float32)
    k = (rng.standard_normal((BH, N, d)) + 2.0 * rng.standard_normal((BH, 1, d))).astype(np.float32)
    v = rng.standard_normal((BH, N, d)).astype(np.float32)
    return q, k, v


def test_block_mean_closed_form():
    """Block b = offset_b + (+x, -x) pairs inside each 64-row chunk: every
    chunk sum is the offset times the rows, exactly, so the block mean is the
    offset."""
    d, N = 16, 300
    offs = np.array([0.5, -2.25, 3.0], np.float32)  # blocks 0-127, 128-255, 256-299
    q = np.zeros((1, N, d), np.float32)
    for b, o in enumerate(offs):
        r0, r1 = 128 * b, min(N, 128 * (b + 1))
        q[0, r0:r1] = o
        for t in range(r0, r1 - 1, 2):
            q[0, t] += 0.125
            q[0, t + 1] -= 0.125
    k = np.ones((1, N, d), np.float32)
    qz = orc.quantize_int8_fp8_blocksmooth(q, k, k, orc.MODE_INT8_FP8)
    # the last block has 44 rows: 22 (+,-) pairs
    assert np.array_equal(qz["q_mean"][0], np.repeat(offs[:, None], d, 1))


def test_reduces_to_per_slice_smoothing():
    """When every block's mean equals the slice's (each block carries the same
    exactly representable offset and its zero-sum noise), the block path
    gives the per-slice path's codes, scales and bias, bit for bit, and the
    same attention output."""
    d, N = 64, 384
    rng = np.random.default_rng(3)
    base = rng.integers(-8, 8, (2, 1, d)).astype(np.float32) * 0.25
    half = (rng.integers(1, 16, (2, N // 2, d)).astype(np.float32) * 0.0625)
    noise = np.empty((2, N, d), np.float32)
    noise[:, 0::2] = half
    noise[:, 1::2] = -half
    q = base + noise
    k = rng.standard_normal((2, N, d)).astype(np.float32)
    v = rng.standard_normal((2, N, d)).astype(np.float32)
    g = orc.quantize_int8_fp8(q, k, v, smooth_q=True, mode=orc.MODE_INT8_FP8)
    b = orc.quantize_int8_fp8_blocksmooth(q, k, v, orc.MODE_INT8_FP8)
    assert np.array_equal(g["q_mean"], b["q_mean"][:, 0]) and np.array_equal(g["q_mean"], b["q_mean"][:, 2])
    for name in ("q_codes", "q_scale", "k_codes", "k_scale", "vt_codes", "v_scale"):
        assert np.array_equal(g[name], b[name]), name
    for blk in range(N // 128):
        assert np.array_equal(g["q_bias"], b["q_bias"][:, blk])
    og = orc.attention_int8_fp8(g, True)
    ob = orc.attention_int8_fp8_blocksmooth(b, True)
    assert np.array_equal(og, ob)


def test_bias_identity_fp64():
    """q_i . k~_j = (q_i - mean_b) . k~_j + bias_b[j] for every row i of block
    b: the stored mean is the block's fp64 mean within fp32 rounding and the
    bias is mean_b . k~ within the fp32 chain's error."""
    q, k, v = _qkv(300, 64, 11)
    qz = orc.quantize_int8_fp8_blocksmooth(q, k, v, orc.MODE_INT8_FP8)
    kt = k.astype(np.float64) - qz["k_mean"][:, None, :].astype(np.float64)
    for b in range(3):
        r0, r1 = 128 * b, min(300, 128 * (b + 1))
        m64 = q[:, r0:r1].astype(np.float64).mean(1)
        assert np.allclose(qz["q_mean"][:, b], m64, rtol=1e-5, atol=1e-5)
        ref = np.einsum("bc,bjc->bj", qz["q_mean"][:, b].astype(np.float64), kt)
        got = qz["q_bias"][:, b, :300].astype(np.float64)
        assert np.allclose(got, ref, rtol=1e-5, atol=1e-4 * np.abs(ref).max())
        assert not qz["q_bias"][:, b, 300:].any()


@pytest.mark.parametrize("causal", [False, True])
def test_block_smoothing_close_to_fp64_and_better_than_per_slice(causal):
    """On Q whose 128-row blocks carry different offsets, block smoothing stays
    within cos 0.999 of fp64 attention and has a smaller relative-L1 error
    than per-slice smoothing (the offsets then stay in Q's INT8 range)."""
    q, k, v = _qkv(384, 128, 21)
    ref = _fp64_attention(q, k, v, causal)
    ob = orc.attention_int8_fp8_blocksmooth(orc.quantize_int8_fp8_blocksmooth(q, k, v, orc.MODE_INT8_FP8), causal)
    og = orc.attention_int8_fp8(orc.quantize_int8_fp8(q, k, v, smooth_q=True, mode=orc.MODE_INT8_FP8), causal)
    cos = (ob.astype(np.float64) * ref).sum() / np.linalg.norm(ob) / np.linalg.norm(ref)
    assert cos >= 0.999
    err_b = np.abs(ob - ref).sum() / np.abs(ref).sum()
    err_g = np.abs(og - ref).sum() / np.abs(ref).sum()
    assert err_b < err_g, (err_b, err_g)


def test_rows_of_one_block_use_that_blocks_bias():
    """Rows of block 1 computed alone equal those rows of the full output; a
    row computed with block 0's bias row instead differs."""
    q, k, v = _qkv(300, 64, 5)
    qz = orc.quantize_int8_fp8_blocksmooth(q, k, v, orc.MODE_INT8_FP8)
    full = orc.attention_int8_fp8_blocksmooth(qz, False)
    rows = np.array([128, 200, 255], np.int32)
    part = orc.attention_int8_fp8_blocksmooth(qz, False, rows=rows)
    assert np.array_equal(part, full[:, rows])
    wrong = orc.attention_int8_fp8(dict(qz, q_bias=np.ascontiguousarray(qz["q_bias"][:, 0])), False, rows=rows)
    assert not np.allclose(wrong, part, atol=1e-3)
