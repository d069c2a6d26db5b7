"""Grouped key/value heads and separate query / key lengths through the C ABI
(sage_*_gqa) against the CPU oracle: quantization bit-exact, the output
within the parity bounds, and the per-head calls reproduced exactly when
Hq == Hkv and Nq == Nk."""
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


def _inputs(B, Hq, Hkv, Nq, Nk, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Nq, d, generator=g) + 1.5 * torch.randn(B, Hq, 1, d, generator=g)
    k = torch.randn(B, Hkv, Nk, d, generator=g) + 2.0 * torch.randn(B, Hkv, 1, d, generator=g)
    v = torch.randn(B, Hkv, Nk, d, generator=g)
    dt = inputs.DTYPES[dtype]
    return [t.to(dt).cuda() for t in (q, k, v)]


CASES = [
    # (B, Hq, Hkv, Nq, Nk, d, dtype, causal, smooth_q, mode)
    (2, 8, 2, 500, 500, 128, "bf16", True, True, 0),
    (1, 4, 1, 200, 1000, 64, "fp16", True, False, 1),
    (1, 6, 3, 129, 333, 128, "fp16", False, True, 0),
    (1, 8, 2, 1, 2000, 128, "bf16", True, True, 0),
    (2, 4, 4, 300, 700, 128, "fp16", True, True, 1),
    (1, 2, 1, 1000, 257, 64, "bf16", False, False, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dtype,causal,smooth_q,mode", CASES)
def test_gqa_matches_oracle(B, Hq, Hkv, Nq, Nk, d, dtype, causal, smooth_q, mode):
    q, k, v = _inputs(B, Hq, Hkv, Nq, Nk, d, dtype, 9000 + Nq + Nk + Hq)
    ws = api.alloc_workspace_gqa(B, Hq, Hkv, Nq, Nk, d, mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd_gqa(q, k, v, out, B, Hq, Hkv, Nq, Nk, d, causal, mode, api.DTYPE_CODE[q.dtype], smooth_q, ws,
                          ws.numel())
    api.sage_check(ws, ws.numel())
    f = lambda t: t.float().cpu().numpy()
    oz = orc.quantize_int8_fp8_gqa(f(q), f(k), f(v), smooth_q, mode)
    g = {n: t.cpu().numpy() for n, t in api.ws_views_gqa(ws, B, Hq, Hkv, Nq, Nk, d, mode).items()}
    for name in ("q_codes", "k_codes", "vt_codes"):
        assert np.array_equal(g[name].view(np.uint8), oz[name].view(np.uint8)), name
    for name in ("q_scale", "k_scale", "v_scale", "k_mean"):
        assert np.array_equal(g[name].view(np.uint32), oz[name].view(np.uint32)), name
    if smooth_q:
        assert np.array_equal(g["q_mean"].view(np.uint32), oz["q_mean"].view(np.uint32)), "q_mean"
        assert np.array_equal(g["q_bias"].view(np.uint32), oz["q_bias"].view(np.uint32)), "q_bias"
    ref32, flip = orc.attention_int8_fp8_gqa(oz, causal, with_flip=True)
    got = out.float().cpu().reshape(B * Hq, Nq, d).numpy()
    compare_out(got, ref32, flip, dtype, (B, Hq, Hkv, Nq, Nk, d, causal, mode))


def test_gqa_calls_equal_per_head_calls_for_equal_shapes():
    B, H, N, d = 1, 3, 600, 128
    q, k, v = _inputs(B, H, H, N, N, d, "fp16", 9100)
    for mode in (0, 1, 2):
        for causal in (False, True):
            ws1 = api.alloc_workspace(B, H, N, d, mode)
            ws2 = api.alloc_workspace_gqa(B, H, H, N, N, d, mode)
            assert ws1.numel() == ws2.numel()
            o1, o2 = torch.empty_like(q), torch.empty_like(q)
            api.sage_attn_fwd(q, k, v, o1, B, H, N, d, causal, mode, 0, True, ws1, ws1.numel())
            api.sage_attn_fwd_gqa(q, k, v, o2, B, H, H, N, N, d, causal, mode, 0, True, ws2, ws2.numel())
            api.sage_check(ws2, ws2.numel())
            assert torch.equal(o1, o2), (mode, causal)
