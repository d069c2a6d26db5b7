"""The (Pr, Vr) x FP16 chunk-depth accuracy sweep on the CPU oracle
(SageAttention2++ summary: Sec. 3.1 narrows the P~ and V ranges so that an
FP16 accumulator cannot overflow and picks Pr = 224, Vr = 4.5 among the
qualifying pairs; Sec. 3.2 sums two MMA results in FP16; App. A.2 measures
attention accuracy by cosine similarity, relative L1 and RMSE).  A pair
qualifies at chunk depth D when D * Pr * Vr <= 65504 (all D products at
their maxima stay finite in FP16).  Accuracy is measured against fp64
softmax attention of the same dequantized logits with the unquantized V, so
it isolates what the P~ / V quantization and the accumulator contribute.
Also the host-side checks of sage_attn_fwd_ranges.  CPU only."""
import ctypes
import math

import numpy as np
import pytest

import oracle as orc
from quantized_attention_sub_b200 import api, inputs

PR = (56.0, 112.0, 224.0, 448.0)
VR = (1.125, 2.25, 4.5, 9.0, 18.0)


def feasible(depth, Pr, Vr):
    return depth * Pr * Vr <= 65504.0


def pv_reference(qz, v):
    """fp64 softmax over the exact dequantized logits the method forms, times
    the unquantized V."""
    BH, Np, d = qz["q_codes"].shape
    N = qz["N"]
    out = []
    for b in range(BH):
        s = orc.qk_s32(qz["q_codes"][b, :N], qz["k_codes"][b, :N]).astype(np.float64)
        t = s * np.repeat(qz["q_scale"][b], 32)[:N, None] * np.repeat(qz["k_scale"][b], 64)[None, :N]
        if qz["q_bias"] is not None:
            t = t + qz["q_bias"][b, :N][None, :]
        t = t / math.sqrt(d)
        p = np.exp(t - t.max(axis=1, keepdims=True))
        out.append((p / p.sum(axis=1, keepdims=True)) @ v[b].astype(np.float64))
    return np.stack(out)


def sweep(law, N=256, H=2):
    w = inputs.variant(inputs.WORKLOADS["video_dit"], H=H, N=N, law=law, seed=2505)
    q, k, v = [t.float().reshape(H, N, w.d).numpy() for t in inputs.generate(w)]
    ref = pv_reference(orc.quantize_int8_fp8(q, k, v, True, 0), v)
    table = {("fp32acc", 448.0, 448.0): orc.accuracy(orc.attention_int8_fp8(
        orc.quantize_int8_fp8(q, k, v, True, 0), False), ref)}
    for depth in (64, 32):
        for Pr in PR:
            for Vr in VR:
                if not feasible(depth, Pr, Vr):
                    continue
                o = orc.attention_int8_fp8(orc.quantize_int8_fp8(q, k, v, True, 1, Vr=Vr), False, Pr=Pr,
                                           chunk=depth)
                assert np.all(np.isfinite(o)), (depth, Pr, Vr)
                table[(depth, Pr, Vr)] = orc.accuracy(o, ref)
    return table


@pytest.mark.parametrize("law", ["qk_bias", "student_t3"])
def test_range_sweep(law):
    t = sweep(law)
    for key, a in sorted(t.items(), key=lambda kv: str(kv[0])):
        print("sweep", law, key, "cos %.7f rel_l1 %.6f rmse %.3e" % (a["cos"], a["rel_l1"], a["rmse"]))
    best = min(a["rel_l1"] for k, a in t.items() if k[0] == 64)
    pages = t[(64, 224.0, 4.5)]
    # the pages' pair is as good as the best qualifying pair at its depth
    assert pages["rel_l1"] <= 1.01 * best and pages["cos"] > 0.999
    # the FP16 accumulator costs little against the FP32 one ("same accuracy")
    assert pages["rel_l1"] <= 1.1 * t[("fp32acc", 448.0, 448.0)]["rel_l1"]
    # delayed buffering (two MMA results per FP16 partial) against one
    assert abs(t[(64, 224.0, 4.5)]["rel_l1"] - t[(32, 224.0, 4.5)]["rel_l1"]) <= 0.01 * best


def test_narrow_v_range_costs_accuracy_on_heavy_tails():
    """With a heavy-tailed V a small Vr pushes many V codes into the e4m3
    subnormal range."""
    t = sweep("student_t3")
    assert t[(64, 224.0, 1.125)]["rel_l1"] > 1.01 * t[(64, 224.0, 4.5)]["rel_l1"]


@pytest.fixture(scope="module")
def lib():
    from quantized_attention_sub_b200 import build
    build.build()
    return api.lib()


@pytest.mark.parametrize("mode,Pr,Vr,status", [
    (1, 224.0, 9.0, api.SAGE_ERR_INVALID_ARG),      # 64 * 224 * 9 > 65504
    (1, 448.0, 4.5, api.SAGE_ERR_INVALID_ARG),
    (0, 0.0, 4.5, api.SAGE_ERR_INVALID_ARG),
    (0, 448.0, 500.0, api.SAGE_ERR_INVALID_ARG),
    (2, 224.0, 4.5, api.SAGE_ERR_UNSUPPORTED),
])
def test_ranges_rejected_on_host(lib, mode, Pr, Vr, status):
    vp = ctypes.c_void_p
    ws = api.sage_workspace_size(1, 2, 128, 128, mode)
    st = lib.sage_attn_fwd_ranges(vp(4096), vp(4096), vp(4096), vp(4096), 1, 2, 128, 128, 0, mode, 0, 0, Pr, Vr,
                                  vp(4096), ws, vp(0))
    assert st == status
