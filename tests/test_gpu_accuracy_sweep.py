"""sage_attn_fwd_ranges on the GPU for qualifying (Pr, Vr) pairs of the
FP16-accumulator mode (SageAttention2++ summary, Sec. 3.1), against the CPU
oracle with the same pair: parity within the usual bounds, and the accuracy
figures against fp64 attention (App. A.2) reproduced."""
import numpy as np
import pytest
import torch

import oracle as orc
from parity_check import compare_out
from quantized_attention_sub_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_sub_b200 import build
    build.build()
    api.lib()


@pytest.mark.parametrize("mode,Pr,Vr", [(1, 224.0, 4.5), (1, 112.0, 9.0), (1, 448.0, 2.25), (1, 56.0, 18.0),
                                        (1, 224.0, 1.125), (0, 448.0, 448.0), (0, 224.0, 4.5)])
def test_ranges_match_oracle(mode, Pr, Vr):
    N, H, d = 700, 2, 128
    w = inputs.variant(inputs.WORKLOADS["video_dit"], H=H, N=N, seed=2506)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(1, H, N, d, mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd_ranges(q, k, v, out, 1, H, N, d, False, mode, 0, True, Pr, Vr, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    f = lambda t: t.float().cpu().reshape(H, N, d).numpy()
    qz = orc.quantize_int8_fp8(f(q), f(k), f(v), True, mode, Vr=Vr)
    ref32, flip = orc.attention_int8_fp8(qz, False, Pr=Pr, with_flip=True)
    got = f(out)
    compare_out(got, ref32, flip, "fp16", (mode, Pr, Vr))
    ref64 = orc.attention_fp64(f(q), f(k), f(v), False)
    a_gpu, a_orc = orc.accuracy(got, ref64), orc.accuracy(ref32, ref64)
    print("ranges", mode, Pr, Vr, "gpu", a_gpu, "oracle", a_orc)
    assert abs(a_gpu["rel_l1"] - a_orc["rel_l1"]) <= 2e-4 and abs(a_gpu["cos"] - a_orc["cos"]) <= 1e-5
