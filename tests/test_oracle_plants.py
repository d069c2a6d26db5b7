"""Planted mistakes: each test compiles a copy of the CPU oracle with one
plausible error edited into its source (a dropped term, a wrong sign or
index, another rounding grouping, a wrong block) and checks that one of the
oracle's pins fails on it.  The oracle itself is never modified; the copies
live in a temporary folder.  CPU only."""
import numpy as np
import pytest

import oracle as orc
import test_oracle as t1
import test_oracle_gqa as t3
import test_oracle_pins2 as t2

PLANTS = {
    # FP16 accumulator: one rounding of the whole 64-key sum (no delayed buffer)
    "f16_single_rounding": [("          double h = orc_f16_round(s0);\n          if (chunk == 64) h = orc_f16_round(h + s1);",
                             "          double h = orc_f16_round(s0 + s1);")],
    # FP16 accumulator: each 32-key MMA result flushed to fp32 on its own
    "f16_flush_every_32": [("          double h = orc_f16_round(s0);\n          if (chunk == 64) h = orc_f16_round(h + s1);",
                            "          a = a + (float)orc_f16_round(s0);\n          double h = orc_f16_round(s1);")],
    # NVFP4 block scale against the wrong e2m1 range (4 instead of 6)
    "fp4_scale_range": [("bs = orc_ue4m3_encode((double)(a / (6.0f * g)));",
                         "bs = orc_ue4m3_encode((double)(a / (4.0f * g)));")],
    # NVFP4 P~: the block of keys quantized into the wrong block's slot
    "fp4_p_block_index": [("pbs[b] = (uint8_t)fp4_block(pvals + b * 16, 1, gp, pcodes + b * 16);",
                           "pbs[b] = (uint8_t)fp4_block(pvals + (7 - b) * 16, 1, gp, pcodes + b * 16);")],
    # NVFP4 P~: one block scale applied to every block
    "fp4_p_block_scale": [("sum += orc_e2m1_decode(pcodes[j]) * orc_ue4m3_decode(pbs[b]) * vj;",
                           "sum += orc_e2m1_decode(pcodes[j]) * orc_ue4m3_decode(pbs[0]) * vj;")],
    # online softmax: the accumulator never rescaled (alpha dropped)
    "no_rescale": [("        acc[c] = alpha * acc[c] + (float)sum;\n      } else {",
                    "        acc[c] = acc[c] + (float)sum;\n      } else {")],
    # K scale of the wrong granule (32-key instead of 64-key index)
    "k_granule_index": [("float deq = (float)s * (sq * sk[j / 64]);", "float deq = (float)s * (sq * sk[j / 32]);")],
    # Q-smoothing bias subtracted instead of added
    "bias_sign": [("      if (bias) deq = deq + bias[j];\n      const float t = deq * c_log2;\n      tvals[j - j0] = t;\n"
                   "      if (t > mt) mt = t;\n    }\n    const float m_new = m > mt ? m : mt;\n    const float alpha = "
                   "orc_exp2(m - m_new);   /* first tile",
                   "      if (bias) deq = deq - bias[j];\n      const float t = deq * c_log2;\n      tvals[j - j0] = t;\n"
                   "      if (t > mt) mt = t;\n    }\n    const float m_new = m > mt ? m : mt;\n    const float alpha = "
                   "orc_exp2(m - m_new);   /* first tile")],
    # grouped heads: query head read against the wrong key/value head
    "gqa_head_map": [("const int bkv = (bh / Hq) * Hkv + (bh % Hq) / G;",
                      "const int bkv = (bh / Hq) * Hkv + (bh % Hq) % Hkv;")],
    # separate lengths: causal mask aligned at the top left instead of the bottom right
    "cross_causal_offset": [("const int BH = B * Hq, G = Hq / Hkv, koff = Nk - Nq;",
                             "const int BH = B * Hq, G = Hq / Hkv, koff = 0;")],
    # P~ quantized without its range factor Pr
    "p_without_range": [("pcode[j] = (j0 + j <= jmax) ? orc_e4m3_encode((double)(p * Pr)) : -1;",
                         "pcode[j] = (j0 + j <= jmax) ? orc_e4m3_encode((double)p) : -1;")],
}


def _fails(check):
    """True if `check` (a pin: returns False or raises AssertionError on a
    mismatch) rejects the oracle in use."""
    try:
        return check() is False
    except AssertionError:
        return True


CATCHERS = {
    "f16_single_rounding": lambda: t2.check_f16acc_chunk()[0],
    "f16_flush_every_32": lambda: t2.check_f16acc_chunk()[0],
    "fp4_scale_range": t2.check_nvfp4_blocks,
    "fp4_p_block_index": t2.check_nvfp4_attention_blocks,
    "fp4_p_block_scale": t2.check_nvfp4_attention_blocks,
    "no_rescale": t1.test_dropping_the_rescale_is_caught,
    "k_granule_index": t1.test_dropping_the_rescale_is_caught,
    "bias_sign": lambda: t1.test_multi_tile_ragged_close_to_fp64(orc.MODE_INT8_FP8),
    "gqa_head_map": t3.check_gqa_equals_repeated_heads,
    "cross_causal_offset": t3.check_cross_length_causal,
    "p_without_range": lambda: t1.test_quantized_attention_close_to_fp64(orc.MODE_INT8_FP8, False),
}


def test_pins_accept_the_oracle_as_it_stands():
    for name, check in CATCHERS.items():
        assert not _fails(check), name


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_planted_mistake_is_caught(name):
    path = orc.build_variant(PLANTS[name])
    with orc.using(path):
        assert _fails(CATCHERS[name]), name
