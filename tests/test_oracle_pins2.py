"""More pins for the CPU oracle, each built so that a plausible mistake fails:
the FP16-accumulator chunk rounding (SageAttention2++ summary, Sec. 3.2:
two consecutive MMA results summed in FP16 before the FP32 buffer) on a
constructed 64-key chunk whose three groupings round differently, and the
NVFP4 P~ block quantization (SageAttention3 abstract: microscaled FP4) on
non-uniform p, against a numpy restatement from the e2m1 / ue4m3 value
tables.  tests/test_oracle_plants.py plants mistakes in copies of the oracle
and checks that these pins catch them.  CPU only."""
import math

import numpy as np

import oracle as orc
from quantized_attention_sub_b200 import inputs


# --------------------------------------------------------------------------
# FP16 accumulator: the grouping of a 64-key chunk.
# --------------------------------------------------------------------------
def e4m3_table():
    """Finite non-negative e4m3fn values from the bit layout (bias 7, 3 mantissa bits)."""
    out = []
    for e in range(16):
        for m in range(8):
            if not (e == 15 and m == 7):
                out.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


# Per channel: first 32 keys 4.5 except key 0 = x; key 32 = y; keys 33..63 = 0.
# With Q = 0 every p is 1 and P~ = e4m3(224) = 224, so the chunk's two halves
# sum to s0 = 224 (31 * 4.5 + x) and s1 = 224 y exactly.
CHUNK_CASES = [(2.0 ** -9, 0.25), (2.0 ** -9, 0.03515625), (2.0 ** -8, 1.25), (2.0 ** -8, 2.25)]


def f16acc_chunk_case():
    N, d = 64, 16
    q = np.zeros((1, N, d), np.float32)
    k = np.random.default_rng(3).standard_normal((1, N, d)).astype(np.float32)
    v = np.zeros((1, N, d), np.float32)
    for c in range(d):
        x, y = CHUNK_CASES[c % len(CHUNK_CASES)]
        v[0, :32, c] = 4.5
        v[0, 0, c] = x
        v[0, 32, c] = y
    return q, k, v


def f16acc_chunk_expected():
    """The delayed-FP32 result by hand: h = f16(f16(s0) + s1), O = h / (Pr * l)
    with l = 64 keys of p = 1 and scale_v = 4.5 / Vr = 1."""
    out = []
    for c in range(16):
        x, y = CHUNK_CASES[c % len(CHUNK_CASES)]
        s0, s1 = 224.0 * (31 * 4.5 + x), 224.0 * y
        h = np.float16(np.float64(np.float16(s0)) + s1)
        out.append(np.float32(np.float32(h) / np.float32(224.0 * 64)))
    return np.array(out, np.float32)


def check_f16acc_chunk():
    q, k, v = f16acc_chunk_case()
    qz = orc.quantize_int8_fp8(q, k, v, smooth_q=False, mode=orc.MODE_INT8_FP8_F16ACC)
    o = orc.attention_int8_fp8(qz, False)
    return bool(np.array_equal(o[0, 0], f16acc_chunk_expected())), o[0, 0]


def test_f16acc_chunk_groupings_differ_and_oracle_takes_the_delayed_one():
    # the case separates the readings: two roundings, one rounding, 32-key flushes
    for x, y in CHUNK_CASES:
        s0, s1 = 224.0 * (31 * 4.5 + x), 224.0 * y
        two = float(np.float16(float(np.float16(s0)) + s1))
        one = float(np.float16(s0 + s1))
        flushed = float(np.float32(np.float16(s0)) + np.float32(np.float16(s1)))
        assert len({two, one, flushed, s0 + s1}) == 4, (x, y)
    # the inputs quantize to exactly the constructed codes
    q, k, v = f16acc_chunk_case()
    qz = orc.quantize_int8_fp8(q, k, v, smooth_q=False, mode=orc.MODE_INT8_FP8_F16ACC)
    assert np.all(qz["q_codes"] == 0) and np.all(qz["v_scale"] == 1.0)
    assert np.array_equal(orc.e4m3_decode_array(qz["vt_codes"][0, :, :64]).T, v[0].astype(np.float64))
    ok, got = check_f16acc_chunk()
    assert ok, (got, f16acc_chunk_expected())
    # first channel: s0 + s1 = 31304.4375; the chunk rounds f16(s0) = 31248,
    # then 31248 + 56 = 31304 is a tie between 31296 and 31312 -> even 31296
    assert got[0] == np.float32(31296.0 / 14336.0)


# --------------------------------------------------------------------------
# NVFP4: the block quantizer and the P~ blocks of the attention.
# --------------------------------------------------------------------------
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def nearest_even(tab, a):
    """Index of the nearest table entry by a linear scan; ties to the even
    index; saturating at the last entry."""
    if not a > 0:
        return 0
    if a >= tab[-1]:
        return len(tab) - 1
    dist = np.abs(tab - a)
    best = np.flatnonzero(dist == dist.min())
    return int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])


def np_nvfp4_block(x, g):
    """The NVFP4 block reading restated with numpy float32 steps: scale code
    bs = ue4m3(max|x| / (6 g)); each value times r = fl32(1 / fl32(g * dec(bs)))
    rounded to the nearest e2m1 value (ties to even, saturating)."""
    x = np.asarray(x, np.float32)
    e4 = e4m3_table()
    a = np.float32(np.max(np.abs(x)))
    bs = nearest_even(e4, float(np.float32(a / np.float32(np.float32(6.0) * np.float32(g))))) if g > 0 else 0
    sd = np.float32(e4[bs])
    if sd == 0:
        return bs, np.zeros(16, np.uint8)
    r = np.float32(np.float32(1.0) / np.float32(np.float32(g) * sd))
    codes = []
    for xv in x:
        y = np.float32(xv * r)
        c = nearest_even(E2M1, abs(float(y)))
        codes.append(c | (8 if np.signbit(y) else 0))
    return bs, np.array(codes, np.uint8)


def check_nvfp4_blocks():
    """Random heavy-tailed blocks, ramps and softmax-like p blocks (g = 1/2688)."""
    rng = np.random.default_rng(12)
    blocks = [rng.standard_t(3, 16) for _ in range(150)]
    blocks += [np.linspace(0.0, 1.0, 16), 2.0 ** -np.arange(16), np.exp2(-0.37 * np.arange(16)),
               np.exp2(-rng.uniform(0, 12, 16)), np.exp2(-rng.uniform(0, 3, 16))]
    gs = [1.0 / 2688.0] * len(blocks)
    blocks += [rng.standard_normal(16) * 3 for _ in range(50)]
    gs += list(rng.uniform(1e-4, 1e-2, 50))
    for x, g in zip(blocks, gs):
        x = np.asarray(x, np.float32)
        bs, codes = orc.nvfp4_block(x, g)
        bs2, codes2 = np_nvfp4_block(x, g)
        if bs != bs2 or not np.array_equal(codes, codes2):
            return False
    return True


def test_nvfp4_block_quantizer_matches_table_restatement():
    assert check_nvfp4_blocks()
    # a softmax-like block: p = 1 (the row max) maps to e2m1 6 at scale 448
    bs, codes = orc.nvfp4_block(np.exp2(-0.37 * np.arange(16)), 1.0 / 2688.0)
    assert bs == 126 and codes[0] == 7
    assert len(set(codes.tolist())) > 4          # non-uniform codes within the block


def nvfp4_row_restated(qz, i, N):
    """One query row of a one-tile NVFP4 problem restated from the codes:
    exact dot products, t = ((x (g_q g_k)) + 0) log2(e)/sqrt(d) in fp32,
    p = exp2(t - max t), P~ blocks of 16 consecutive keys, O = sum P~ V / l."""
    d = qz["q_codes"].shape[2]
    e4 = e4m3_table()
    dec = lambda c: np.where(np.asarray(c) & 8, -1.0, 1.0) * E2M1[np.asarray(c) & 7]
    qd = dec(qz["q_codes"][0, i]) * np.repeat(e4[qz["q_bscale"][0, i]], 16)
    kd = dec(qz["k_codes"][0, :N]) * np.repeat(e4[qz["k_bscale"][0, :N]], 16, axis=1)
    x = (kd @ qd).astype(np.float32)
    gqk = np.float32(qz["q_gscale"][0] * qz["k_gscale"][0])
    c = np.float32(1.4426950408889634 / math.sqrt(d))
    t = (x * gqk) * c
    p = np.exp2((t - t.max()).astype(np.float64)).astype(np.float32)
    l = np.float32(0)
    for pv in p:
        l = np.float32(l + pv)
    gp = np.float32(1.0) / np.float32(6.0 * 448.0)
    pdq = np.zeros(N)
    for b in range(0, N, 16):
        bs, codes = np_nvfp4_block(p[b:b + 16], gp)
        pdq[b:b + 16] = dec(codes) * e4[bs]
    vd = dec(qz["vt_codes"][0, :, :N]) * np.repeat(e4[qz["vt_bscale"][0]], 16, axis=1)[:, :N]
    acc = (vd @ pdq).astype(np.float32)
    return acc * np.float32(gp * qz["v_gscale"][0]) / l


def check_nvfp4_attention_blocks():
    N, d = 128, 64
    w = inputs.variant(inputs.WORKLOADS["unit"], N=N, d=d, H=1, law="student_t3", seed=4242)
    q, k, v = [t.float().reshape(1, N, d).numpy() for t in inputs.generate(w)]
    q *= 3.0                                   # sharper rows: p spreads over many codes
    qz = orc.quantize_nvfp4(q, k, v, smooth_q=False)
    rows = [0, 5, 63, 100, 127]
    o = orc.attention_nvfp4(qz, False, rows=np.array(rows))
    for r, i in enumerate(rows):
        ref = nvfp4_row_restated(qz, i, N)
        if not np.allclose(o[0, r], ref, rtol=2e-6, atol=1e-7):
            return False
    return True


def test_nvfp4_attention_p_blocks_match_restatement():
    assert check_nvfp4_attention_blocks()
