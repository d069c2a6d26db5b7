"""Pins for the CPU oracle: each check ties it to something other than itself
(the pages' printed numbers, closed forms, library routines, brute force,
invariants of the mathematics).  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc
from quantized_attention_sub_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Small-float encoders.
# --------------------------------------------------------------------------
def e4m3_values_brute():
    """Every finite e4m3fn magnitude from the bit layout: 1 sign, 4 exponent
    (bias 7), 3 mantissa bits; exponent 0 is subnormal; S.1111.111 is NaN."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    return vals


def test_e4m3_table_matches_bit_layout_and_roundtrips():
    vals = e4m3_values_brute()
    assert len(vals) == 127 and vals[-1] == 448.0 and vals[1] == 2.0 ** -9
    for code, v in enumerate(vals):
        assert orc.e4m3_decode(code) == v
        assert orc.e4m3_encode(v) == code
        assert orc.e4m3_encode(-v) == (0x80 | code)
        assert orc.e4m3_decode(0x80 | code) == -v
    assert math.isnan(orc.e4m3_decode(0x7F))


def test_e4m3_midpoints_go_to_even_code_and_saturate():
    vals = e4m3_values_brute()
    for c in range(126):
        mid = 0.5 * (vals[c] + vals[c + 1])
        even = c if c % 2 == 0 else c + 1
        assert orc.e4m3_encode(mid) == even, (c, mid)
        assert orc.e4m3_encode(np.nextafter(mid, 0)) == c
        assert orc.e4m3_encode(np.nextafter(mid, 1e9)) == c + 1
    for big in (448.0, 449.0, 464.0, 465.0, 1e6, float("inf")):
        assert orc.e4m3_encode(big) == 126
        assert orc.e4m3_encode(-big) == 0x80 | 126


def test_e4m3_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.1, 1, 30, 150)])
    x = x.clamp(-464, 464).to(torch.float32)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([orc.e4m3_encode(float(v)) for v in x.numpy()])
    # torch keeps the sign of zero results; so does the oracle (0x80).
    assert np.array_equal(mine, ref)


def test_e4m3_matches_linear_scan():
    vals = np.array(e4m3_values_brute())
    rng = np.random.default_rng(3)
    for a in np.abs(rng.standard_normal(3000)) * rng.choice([1e-3, 1, 100], 3000):
        d = np.abs(vals - a)
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert orc.e4m3_encode(float(a)) == code


def test_e2m1_and_ue4m3():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c, v in enumerate(mags):
        assert orc.e2m1_decode(c) == v and orc.e2m1_encode(v) == c
        if v:
            assert orc.e2m1_encode(-v) == 8 | c and orc.e2m1_decode(8 | c) == -v
    # midpoints: 0.25->0, 0.75->1(code 2, even), 1.25->1(code 2), 1.75->2(code 4),
    # 2.5->2(code 4), 3.5->4(code 6), 5->4(code 6)
    for mid, code in [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6)]:
        assert orc.e2m1_encode(mid) == code, mid
    assert orc.e2m1_encode(100.0) == 7
    vals = e4m3_values_brute()
    for c, v in enumerate(vals):
        assert orc.ue4m3_encode(v) == c
    assert orc.ue4m3_encode(-1.0) == 0 and orc.ue4m3_encode(1e9) == 126


def test_f16_round_matches_numpy():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(5000) * s for s in (1e-6, 1e-3, 1, 300, 3e4)])
    # exact ties between neighbouring halves
    h = np.arange(1, 2000, dtype=np.float16).astype(np.float64)
    ties = (h[:-1] + h[1:]) / 2
    for v in np.concatenate([x, ties, -ties]):
        if abs(v) >= 65520.0:
            continue
        assert orc.f16_round(v) == float(np.float16(v)), v
    assert orc.f16_round(65504.0) == 65504.0
    assert math.isinf(orc.f16_round(65520.0)) and orc.f16_round(65519.0) == 65504.0


# --------------------------------------------------------------------------
# Smoothing statistics and the INT8 quantizer.
# --------------------------------------------------------------------------
def test_channel_mean_closed_form():
    N, d = 300, 8
    t = np.arange(N, dtype=np.float32)[:, None]
    c = np.arange(d, dtype=np.float32)[None, :]
    x = (t + 4 * c)[None]                 # sums are small integers: exact in fp32
    m = orc.channel_mean(x)
    assert np.array_equal(m[0], ((N - 1) / 2 + 4 * np.arange(d)).astype(np.float32))
    const = np.full((2, 777, 4), 0.375, np.float32)
    assert np.all(orc.channel_mean(const) == 0.375)


def test_channel_mean_close_to_fp64():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((3, 1000, 16)) * 3 + 7).astype(np.float32)
    m = orc.channel_mean(x)
    ref = x.astype(np.float64).mean(axis=1)
    assert np.max(np.abs(m - ref)) < 1e-5 * 10


def test_int8_quantizer_closed_forms():
    G, d = 32, 4
    x = np.zeros((1, 64, d), np.float32)
    x[0, 3, 1] = -2.0                    # granule 0 absmax 2 -> scale 2/127, this code -127
    x[0, 5, 2] = 1.0 * 2.0 / 127 * 2.5   # exactly 2.5 steps -> rint even -> 2
    x[0, 6, 2] = 2.0 / 127 * 3.5         # 3.5 steps -> 4
    codes, scale = orc.quant_int8(x, None, G)
    assert codes.shape == (1, 128, d) and scale.shape == (1, 4)
    assert scale[0, 0] == np.float32(2.0) / np.float32(127.0)
    assert codes[0, 3, 1] == -127
    inv = np.float32(127.0) / np.float32(2.0)
    assert codes[0, 5, 2] == int(np.rint(np.float32(x[0, 5, 2]) * inv))
    assert codes[0, 6, 2] == int(np.rint(np.float32(x[0, 6, 2]) * inv))
    assert np.all(scale[0, 1:] == 0) and np.all(codes[0, 32:] == 0)   # zero + pad granules


def test_int8_quantizer_error_bound_and_padding():
    rng = np.random.default_rng(9)
    N, d = 200, 64
    x = rng.standard_normal((2, N, d)).astype(np.float32) * 3
    mean = orc.channel_mean(x)
    codes, scale = orc.quant_int8(x, mean, 64)
    xs = x - mean[:, None, :]
    deq = codes[:, :N].astype(np.float64) * np.repeat(scale, 64, axis=1)[:, :N, None]
    step = np.repeat(scale, 64, axis=1)[:, :N, None]
    assert np.all(np.abs(deq - xs) <= step * (0.5 + 1e-5))
    assert np.all(codes[:, N:] == 0) and np.abs(codes).max() == 127
    # per granule, the largest |x~| maps to +-127
    for bh in range(2):
        for g in range(4):
            blk = codes[bh, g * 64:min((g + 1) * 64, N)]
            assert np.abs(blk).max() == 127


def test_v_fp8_quantizer():
    rng = np.random.default_rng(13)
    N, d = 150, 16
    v = rng.standard_normal((1, N, d)).astype(np.float32)
    v[0, :, 3] = 0.0                        # constant-zero channel
    amax = orc.channel_absmax(v)
    assert np.array_equal(amax[0], np.abs(v[0]).max(axis=0))
    for Vr in (448.0, 4.5):
        vt, sv = orc.quant_v_fp8(v, amax, Vr)
        assert vt.shape == (1, d, 256) and np.all(vt[:, :, N:] == 0)
        assert sv[0, 3] == 0 and np.all(vt[0, 3] == 0)
        dec = orc.e4m3_decode_array(vt[0, :, :N]).T            # [N, d]
        assert np.max(np.abs(dec)) == Vr if Vr == 448.0 else np.max(np.abs(dec)) <= 4.5
        # e4m3 round-to-nearest: half an ulp is 2^-4 relative for normals and
        # 2^-10 absolute (in code units) in the subnormal range
        err = np.abs(dec * sv[0] - v[0])
        bound = 2.0 ** -4 * np.abs(v[0]) + 2.0 ** -10 * sv[0] + 1e-7
        assert np.all(err <= bound)


def test_q_bias_restores_logits():
    """Smoothing Q: q.k~ == q~.k~ + bias exactly in real arithmetic."""
    rng = np.random.default_rng(21)
    q = (rng.standard_normal((1, 96, 32)) + 2).astype(np.float32)
    k = (rng.standard_normal((1, 96, 32)) - 1).astype(np.float32)
    mk, mq = orc.channel_mean(k), orc.channel_mean(q)
    bias = orc.q_bias(k, mk, mq)
    kt = k.astype(np.float64) - mk[:, None]
    qt = q.astype(np.float64) - mq[:, None]
    lhs = q[0].astype(np.float64) @ kt[0].T
    rhs = qt[0] @ kt[0].T + bias[0, :96][None, :]
    assert np.max(np.abs(lhs - rhs)) < 1e-4
    assert np.all(bias[0, 96:] == 0)


def test_smoothing_leaves_softmax_unchanged_fp64():
    """K smoothing adds a per-row constant q_i . mean_k to every logit."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 70, 16))
    k = rng.standard_normal((2, 70, 16)) + rng.standard_normal((2, 1, 16)) * 4
    v = rng.standard_normal((2, 70, 16))
    mk = orc.channel_mean(k.astype(np.float32)).astype(np.float64)
    for causal in (False, True):
        a = orc.attention_fp64(q, k, v, causal)
        b = orc.attention_fp64(q, k - mk[:, None, :], v, causal)
        assert np.max(np.abs(a - b)) < 1e-12


def test_qk_s32_equals_int64_matmul():
    rng = np.random.default_rng(2)
    a = rng.integers(-127, 128, (40, 128), dtype=np.int64)
    b = rng.integers(-127, 128, (50, 128), dtype=np.int64)
    a[0] = 127
    b[0] = 127
    b[1] = -127
    s = orc.qk_s32(a.astype(np.int8), b.astype(np.int8))
    assert np.array_equal(s.astype(np.int64), a @ b.T)
    assert s[0, 0] == 128 * 127 * 127 and s[0, 1] == -128 * 127 * 127


# --------------------------------------------------------------------------
# The tiled quantized attention.
# --------------------------------------------------------------------------
def _small(N, d=64, H=2, dtype="fp16", seed=1001, law="k_bias", causal=False, smooth_q=False):
    w = inputs.variant(inputs.WORKLOADS["unit"], N=N, d=d, H=H, dtype=dtype, seed=seed, law=law,
                       causal=causal, smooth_q=smooth_q)
    q, k, v = inputs.generate(w)
    f = lambda t: t.float().reshape(-1, N, d).numpy()
    return w, f(q), f(k), f(v)


@pytest.mark.parametrize("mode", [orc.MODE_INT8_FP8, orc.MODE_INT8_FP8_F16ACC])
@pytest.mark.parametrize("causal", [False, True])
def test_quantized_attention_close_to_fp64(mode, causal):
    """Oracle accuracy check: cos >= 0.999 against unquantized fp64 attention."""
    w, q, k, v = _small(128)
    qz = orc.quantize_int8_fp8(q, k, v, smooth_q=False, mode=mode)
    o = orc.attention_int8_fp8(qz, causal)
    ref = orc.attention_fp64(q, k, v, causal)
    acc = orc.accuracy(o, ref)
    assert acc["cos"] >= 0.999, acc
    assert acc["rel_l1"] < 0.05, acc


@pytest.mark.parametrize("mode", [orc.MODE_INT8_FP8, orc.MODE_INT8_FP8_F16ACC])
def test_multi_tile_ragged_close_to_fp64(mode):
    w, q, k, v = _small(333, d=128, law="qk_bias", smooth_q=True)
    for smooth_q in (False, True):
        qz = orc.quantize_int8_fp8(q, k, v, smooth_q=smooth_q, mode=mode)
        for causal in (False, True):
            o = orc.attention_int8_fp8(qz, causal)
            acc = orc.accuracy(o, orc.attention_fp64(q, k, v, causal))
            assert acc["cos"] >= 0.999, (smooth_q, causal, acc)


def test_f16acc_same_accuracy_as_fp32acc():
    """SageAttention2++ keeps SageAttention2's attention accuracy (summary Sec. 1, 4)."""
    w, q, k, v = _small(512, d=128)
    ref = orc.attention_fp64(q, k, v, False)
    a32 = orc.accuracy(orc.attention_int8_fp8(orc.quantize_int8_fp8(q, k, v, False, 0), False), ref)
    a16 = orc.accuracy(orc.attention_int8_fp8(orc.quantize_int8_fp8(q, k, v, False, 1), False), ref)
    assert abs(a16["cos"] - a32["cos"]) < 5e-4
    assert a16["rel_l1"] < 1.5 * a32["rel_l1"] + 1e-3


def test_dropping_the_rescale_is_caught():
    """The online softmax over several tiles against a single global-max
    softmax of the same codes (rows whose max sits in the first tile), and
    the quantized attention against fp64 on random data, where the running
    max grows across tiles.  tests/test_oracle_plants.py plants a dropped
    rescale and a wrong K-scale granule in a copy of the oracle and checks
    that this test rejects both."""
    w, q, k, v = _small(1024, d=64)
    ref = orc.attention_fp64(q, k, v, False)
    qz = orc.quantize_int8_fp8(q, k, v, False, 0)
    good = orc.accuracy(orc.attention_int8_fp8(qz, False), ref)
    assert good["cos"] >= 0.999
    # re-evaluate with all logits of tiles after the first shifted so that the
    # first tile holds the row max: then alpha == 1 on every later tile and the
    # oracle must agree with a single global-max softmax of the same codes.
    N = 256
    w2, q2, k2, v2 = _small(N, d=64, seed=77)
    k2[:, 0, :] = q2[:, :, :].mean(axis=1) * 0 + 3.0 * np.sign(q2.sum(axis=1))  # key 0 aligns with most rows
    qz2 = orc.quantize_int8_fp8(q2, k2, v2, False, 0)
    o2 = orc.attention_int8_fp8(qz2, False)
    s = np.stack([orc.qk_s32(qz2["q_codes"][b, :N], qz2["k_codes"][b, :N]) for b in range(2)])
    sq = np.repeat(qz2["q_scale"], 32, axis=1)[:, :N]
    sk = np.repeat(qz2["k_scale"], 64, axis=1)[:, :N]
    t = s.astype(np.float64) * sq[:, :, None] * sk[:, None, :] / math.sqrt(64) * math.log2(math.e)
    first_tile_max = t[:, :, :128].max(axis=2) >= t.max(axis=2)
    rows = np.flatnonzero(first_tile_max.all(axis=0))
    assert len(rows) > 10
    p = np.exp2(t - t.max(axis=2, keepdims=True))
    ptil = np.vectorize(lambda x: orc.e4m3_decode(orc.e4m3_encode(x)))(np.float32(p * 448.0))
    vdq = np.stack([orc.e4m3_decode_array(qz2["vt_codes"][b, :, :N]).T for b in range(2)])
    o_plain = (ptil @ vdq) * qz2["v_scale"][:, None, :] / (448.0 * p.sum(axis=2, keepdims=True))
    # fp64 logits and exponentials here against the oracle's fp32 steps: the
    # row sums differ in the last bits and a P~ code may flip where p*448 sits
    # that close to a rounding midpoint; a dropped rescale, or a wrong scale
    # granule, gives errors of the size of O itself
    err = np.abs(o2[:, rows] - o_plain[:, rows])
    assert np.max(err) < 5e-3 and np.mean(err) < 3e-4


# The oracle's exp2 is the library exp2 rounded to fp32; single-key and
# equal-logit rows reproduce V up to the rounding of the logits and of l.
EXP2_RTOL = 1e-5


def test_exp2_is_correctly_rounded_powers_of_two():
    """orc_exp2 agrees with 2^x rounded once to fp32 (half an ulp) over the
    range the softmax uses; exact at integers; 2^-inf = +0; monotonic."""
    xs = np.concatenate([np.linspace(-126, 9, 200001), np.arange(-126, 10, dtype=np.float64)]).astype(np.float32)
    got = np.array([orc.exp2(float(x)) for x in xs], np.float64)
    ref = np.exp2(xs.astype(np.float64))
    assert np.max(np.abs(got / ref - 1)) <= 2.0 ** -24
    assert all(orc.exp2(float(i)) == 2.0 ** i for i in range(-126, 10))
    assert orc.exp2(float("-inf")) == 0.0
    g = np.array([orc.exp2(float(x)) for x in np.linspace(-20, 9, 100001, dtype=np.float32)])
    assert np.all(np.diff(g) >= 0)


def test_single_key_returns_dequantized_v():
    for mode in (0, 1):
        w, q, k, v = _small(1, d=64)
        qz = orc.quantize_int8_fp8(q, k, v, False, mode)
        o = orc.attention_int8_fp8(qz, False)
        vdq = orc.e4m3_decode_array(qz["vt_codes"][:, :, 0]) * qz["v_scale"]
        assert np.allclose(o[:, 0], vdq, rtol=EXP2_RTOL, atol=0)


def test_zero_q_gives_mean_of_dequantized_v():
    w, q, k, v = _small(300, d=64)
    q[:] = 0
    qz = orc.quantize_int8_fp8(q, k, v, False, 0)
    o = orc.attention_int8_fp8(qz, False)
    vdq = np.stack([orc.e4m3_decode_array(qz["vt_codes"][b, :, :300]).T for b in range(2)])
    mean = (vdq * qz["v_scale"][:, None, :]).mean(axis=1)
    assert np.allclose(o, mean[:, None, :], rtol=EXP2_RTOL, atol=1e-6)
    # causal: row 0 sees only key 0
    oc = orc.attention_int8_fp8(qz, True)
    assert np.allclose(oc[:, 0], vdq[:, 0] * qz["v_scale"], rtol=EXP2_RTOL, atol=0)
    assert np.allclose(oc[:, 9], (vdq[:, :10] * qz["v_scale"][:, None, :]).mean(axis=1), rtol=EXP2_RTOL,
                       atol=1e-6)


def test_pages_fp16_range_pairs():
    g = json.load(open(os.path.join(GOLDEN, "sa2pp_fp16_range.json")))
    assert (orc.PR_F16ACC, orc.VR_F16ACC) == (g["sec_3_1_chosen"]["Pr"], g["sec_3_1_chosen"]["Vr"])
    fmax = g["fp16_max_finite"]
    assert orc.f16_round(fmax) == fmax and math.isinf(orc.f16_round(fmax + 16))
    assert 32 * g["sec_3_1_example"]["p_max"] * g["sec_3_1_example"]["v_max"] <= fmax
    assert 32 * g["sec_3_2"]["mma_results_accumulated_in_fp16"] * 224 * 4.5 <= fmax
    # both constants are exact e4m3 values, so P~ = 1 and |v^| = Vr are representable
    assert orc.e4m3_decode(orc.e4m3_encode(224.0)) == 224.0
    assert orc.e4m3_decode(orc.e4m3_encode(4.5)) == 4.5


def test_f16acc_worst_case_stays_finite_and_wider_range_overflows():
    """All P~ = Pr and all |v^| = Vr in a 64-key chunk: 64*224*4.5 = 64512 is
    finite in FP16; with Vr = 9 the same chunk overflows, which the emulated
    FP16 accumulator must show."""
    N, d = 128, 16
    q = np.zeros((1, N, d), np.float32)
    k = np.random.default_rng(0).standard_normal((1, N, d)).astype(np.float32)
    v = np.full((1, N, d), 2.0, np.float32)
    qz = orc.quantize_int8_fp8(q, k, v, False, orc.MODE_INT8_FP8_F16ACC)
    assert np.all(orc.e4m3_decode_array(qz["vt_codes"][:, :, :N]) == 4.5)
    o = orc.attention_int8_fp8(qz, False)
    assert np.all(np.isfinite(o)) and np.allclose(o, 2.0, rtol=EXP2_RTOL)
    vt9, sv9 = orc.quant_v_fp8(v, orc.channel_absmax(v), 9.0)
    qz9 = dict(qz, vt_codes=vt9, v_scale=sv9)
    o9 = orc.attention_int8_fp8(qz9, False)
    assert np.all(np.isinf(o9))


# --------------------------------------------------------------------------
# NVFP4 mode.
# --------------------------------------------------------------------------
def test_nvfp4_quantizer_block_properties():
    rng = np.random.default_rng(4)
    N, d = 100, 32
    x = rng.standard_t(3, (2, N, d)).astype(np.float32)
    qz = orc.quantize_nvfp4(x, x, x, smooth_q=False)
    codes, bs, gs = qz["q_codes"], qz["q_bscale"], qz["q_gscale"]
    assert np.allclose(gs, np.abs(x).reshape(2, -1).max(axis=1) / 2688.0, rtol=1e-7)
    deq = np.vectorize(orc.e2m1_decode)(codes[:, :N]) * np.repeat(
        np.vectorize(lambda c: orc.e4m3_decode(c))(bs[:, :N]), 16, axis=2) * gs[:, None, None]
    # every block's largest element lands on +-6 (or the ue4m3 rounding moves it to 4..6)
    mag = np.abs(np.vectorize(orc.e2m1_decode)(codes[:, :N])).reshape(2, N, d // 16, 16).max(axis=3)
    assert np.all((mag >= 4) | (bs[:, :N] == 0))
    err = np.abs(deq - x)
    blk_amax = np.abs(x).reshape(2, N, d // 16, 16).max(axis=3, keepdims=True)
    assert np.all(err.reshape(2, N, d // 16, 16) <= blk_amax * 0.26 + 1e-6)
    assert np.all(codes[:, N:] == 0)


def test_nvfp4_attention_single_key_and_accuracy():
    w, q, k, v = _small(1, d=64, law="student_t3")
    qz = orc.quantize_nvfp4(q, k, v, False)
    o = orc.attention_nvfp4(qz, False)
    vdq = np.vectorize(orc.e2m1_decode)(qz["vt_codes"][:, :, 0]) * np.vectorize(orc.e4m3_decode)(
        qz["vt_bscale"][:, :, 0]) * qz["v_gscale"][:, None]
    assert np.allclose(o[:, 0], vdq, rtol=1e-6, atol=0)
    # FP4 keeps about 2 significant bits, so near-uniform attention over random
    # V carries ~10-20% relative error; the bound only catches gross mistakes.
    w, q, k, v = _small(256, d=128, law="student_t3")
    o = orc.attention_nvfp4(orc.quantize_nvfp4(q, k, v, False), False)
    acc = orc.accuracy(o, orc.attention_fp64(q, k, v, False))
    assert acc["cos"] > 0.95, acc


def test_nvfp4_zero_q_gives_mean_of_dequantized_v():
    """Q = 0: every p is 1, each P~ block is exactly 6 * 448 * (1/2688) = 1,
    so O is the plain mean of the dequantized V (also across several tiles)."""
    w, q, k, v = _small(300, d=64, law="student_t3")
    q[:] = 0
    qz = orc.quantize_nvfp4(q, k, v, False)
    o = orc.attention_nvfp4(qz, False)
    dec = np.vectorize(orc.e2m1_decode)(qz["vt_codes"][:, :, :300]) * np.repeat(
        np.vectorize(orc.e4m3_decode)(qz["vt_bscale"]), 16, axis=2)[:, :, :300]
    mean = dec.mean(axis=2) * qz["v_gscale"][:, None]
    assert np.allclose(o, mean[:, None, :], rtol=1e-5, atol=1e-7)
