"""Pins for the oracle's grouped key/value heads and separate query and key
lengths (query head hq reads key/value head hq / G; a causal row i sees keys
j <= i + Nk - Nq): reduces exactly to the per-head oracle when G = 1 and
Nq = Nk, equals the per-head oracle on key/value heads repeated G times, and
matches fp64 attention under the same mask.  CPU only."""
import numpy as np
import pytest

import oracle as orc


def _data(B, Hq, Hkv, Nq, Nk, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, Nq, d)).astype(np.float32)
    k = (rng.standard_normal((B, Hkv, Nk, d)) + 2.0 * rng.standard_normal((B, Hkv, 1, d))).astype(np.float32)
    v = rng.standard_normal((B, Hkv, Nk, d)).astype(np.float32)
    return q, k, v


def check_gqa_equals_repeated_heads(smooth_q=True, causal=True):
    B, Hq, Hkv, Nq, Nk, d = 2, 6, 2, 200, 200, 64
    q, k, v = _data(B, Hq, Hkv, Nq, Nk, d, 11)
    G = Hq // Hkv
    qz = orc.quantize_int8_fp8_gqa(q, k, v, smooth_q, 0)
    o_gqa = orc.attention_int8_fp8_gqa(qz, causal)
    kx, vx = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    f = lambda t: t.reshape(B * Hq, Nq, d)
    qz_mha = orc.quantize_int8_fp8(f(q), f(kx), f(vx), smooth_q, 0)
    o_mha = orc.attention_int8_fp8(qz_mha, causal)
    return bool(np.array_equal(o_gqa, o_mha))


@pytest.mark.parametrize("smooth_q,causal", [(False, False), (True, True), (True, False)])
def test_gqa_equals_per_head_oracle_on_repeated_kv(smooth_q, causal):
    assert check_gqa_equals_repeated_heads(smooth_q, causal)


def test_one_group_same_length_is_the_per_head_oracle():
    B, H, N, d = 1, 3, 300, 128
    q, k, v = _data(B, H, H, N, N, d, 12)
    for mode in (0, 1):
        qz = orc.quantize_int8_fp8_gqa(q, k, v, True, mode)
        f = lambda t: t.reshape(B * H, N, d)
        qz2 = orc.quantize_int8_fp8(f(q), f(k), f(v), True, mode)
        for causal in (False, True):
            assert np.array_equal(orc.attention_int8_fp8_gqa(qz, causal), orc.attention_int8_fp8(qz2, causal))


def check_cross_length_causal(Nq=100, Nk=333):
    B, Hq, Hkv, d = 1, 4, 1, 64
    q, k, v = _data(B, Hq, Hkv, Nq, Nk, d, 13)
    qz = orc.quantize_int8_fp8_gqa(q, k, v, False, 0)
    o = orc.attention_int8_fp8_gqa(qz, True)
    ref = orc.attention_fp64(q.reshape(Hq, Nq, d), np.repeat(k, Hq, axis=1).reshape(Hq, Nk, d),
                             np.repeat(v, Hq, axis=1).reshape(Hq, Nk, d), True)
    ok = orc.accuracy(o, ref)["cos"] >= 0.999
    # the last query row sees every key: the same as without the mask
    full = orc.attention_int8_fp8_gqa(qz, False, rows=np.array([Nq - 1]))
    ok = ok and np.array_equal(o[:, Nq - 1], full[:, 0])
    # row 0 sees keys 0 .. Nk - Nq
    part = orc.attention_int8_fp8_gqa(qz, False, rows=np.array([0]))
    ok = ok and not np.array_equal(o[:, 0], part[:, 0])
    return bool(ok)


def test_cross_length_causal_is_bottom_right():
    assert check_cross_length_causal()


def test_cross_length_noncausal_close_to_fp64():
    B, Hq, Hkv, Nq, Nk, d = 1, 2, 2, 77, 500, 128
    q, k, v = _data(B, Hq, Hkv, Nq, Nk, d, 14)
    for mode in (0, 1):
        qz = orc.quantize_int8_fp8_gqa(q, k, v, True, mode)
        o = orc.attention_int8_fp8_gqa(qz, False)
        ref = orc.attention_fp64(q.reshape(2, Nq, d), k.reshape(2, Nk, d), v.reshape(2, Nk, d), False)
        assert orc.accuracy(o, ref)["cos"] >= 0.999
