"""sage_attn_fwd_fused (Q quantized inside the attention kernel) against
sage_attn_fwd: the same codes feed the same attention, so the outputs must
be bit-identical, and the workspace's K/V codes, scales, means and bias must
equal the oracle's."""
import numpy as np
import pytest
import torch

import oracle as orc
from quantized_attention_sub_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_sub_b200 import build
    build.build()
    api.lib()


CASES = [
    # (B, H, N, d, dtype, law, causal, smooth_q, mode)
    (1, 2, 128, 64, "fp16", "k_bias", False, False, 0),
    (1, 2, 1, 128, "bf16", "k_bias", False, False, 0),
    (1, 3, 333, 128, "fp16", "qk_bias", True, True, 0),
    (2, 2, 1000, 64, "bf16", "qk_bias", False, True, 0),
    (1, 4, 700, 128, "fp16", "qk_bias", False, True, 1),
    (1, 2, 257, 64, "bf16", "k_bias_outlier", True, False, 1),
    (1, 32, 8192, 128, "bf16", "k_bias_outlier", True, False, 0),
    (4, 8, 4096, 128, "fp16", "k_bias", False, False, 0),
]


@pytest.mark.parametrize("B,H,N,d,dtype,law,causal,smooth_q,mode", CASES)
def test_fused_equals_unfused(B, H, N, d, dtype, law, causal, smooth_q, mode):
    w = inputs.variant(inputs.WORKLOADS["unit"], B=B, H=H, N=N, d=d, dtype=dtype, law=law, causal=causal,
                       smooth_q=smooth_q, mode=mode, seed=6100 + N + d)
    q, k, v = [t.cuda() for t in inputs.generate(w, device="cuda")]
    dt = api.DTYPE_CODE[q.dtype]
    ws1 = api.alloc_workspace(B, H, N, d, mode)
    ws2 = api.alloc_workspace(B, H, N, d, mode)
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, o1, B, H, N, d, causal, mode, dt, smooth_q, ws1, ws1.numel())
    api.sage_attn_fwd_fused(q, k, v, o2, B, H, N, d, causal, mode, dt, smooth_q, ws2, ws2.numel())
    api.sage_check(ws2, ws2.numel())
    api.sage_check(ws1, ws1.numel())
    assert torch.equal(o1, o2)
    g1, g2 = api.ws_views(ws1, B, H, N, d, mode), api.ws_views(ws2, B, H, N, d, mode)
    names = ["k_codes", "vt_codes", "k_scale", "v_scale", "k_mean"] + (["q_mean", "q_bias"] if smooth_q else [])
    for n in names:
        assert torch.equal(g1[n].view(torch.uint8), g2[n].view(torch.uint8)), n


def test_fused_rejects_nvfp4():
    q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    ws = api.alloc_workspace(1, 1, 128, 128, api.MODE_NVFP4)
    with pytest.raises(api.SageError) as e:
        api.sage_attn_fwd_fused(q, q, q, torch.empty_like(q), 1, 1, 128, 128, False, api.MODE_NVFP4, 1, False, ws,
                                ws.numel())
    assert e.value.status == api.SAGE_ERR_UNSUPPORTED
