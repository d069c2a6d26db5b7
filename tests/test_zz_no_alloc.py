"""sage_quantize_qkv_static, the quantization entry point for callers that
cannot allocate device memory (graph captures that must not grow the pool,
plugins whose host owns all allocations, real-time loops).  Its statistics
scratch is a fixed device array inside the library; this checks, through the
C ABI, that two calls in a row give exactly what the regular entry point
(workspace scratch) gives, and that oversized problems are refused.

Kept in its own file so pytest collects it last."""
import numpy as np
import pytest
import torch

from quantized_attention_sub_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_sub_b200 import build
    build.build()
    api.lib()


def _regular(q, k, v, w, mode):
    B, H, N, d = w.shape()
    ws = api.alloc_workspace(B, H, N, d, mode)
    api.sage_quantize_qkv(q, k, v, api.DTYPE_CODE[q.dtype], B, H, N, d, w.smooth_q, mode, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    return {n: t.clone() for n, t in api.ws_views(ws, B, H, N, d, mode).items()}


def _static(q, k, v, w, mode, out):
    B, H, N, d = w.shape()
    L = api.sage_workspace_layout(B, H, N, d, mode)
    api.sage_quantize_qkv_static(q, k, v, api.DTYPE_CODE[q.dtype], B, H, N, d, w.smooth_q, mode, out, L.scratch)
    api.sage_check(out, L.scratch)
    return {n: t.clone() for n, t in api.ws_views(out, B, H, N, d, mode).items()}


def _same(a, b, smooth_q):
    if "q_sf_atoms" in a:   # NVFP4: packed codes, scale atoms, global scales
        names = ["q_codes", "k_codes", "vt_codes", "q_sf_atoms", "k_sf_atoms", "v_sf_atoms", "global_scale", "k_mean"]
    else:
        names = ["q_codes", "k_codes", "vt_codes", "q_scale", "k_scale", "v_scale", "k_mean"]
    if smooth_q:
        names += ["q_mean", "q_bias"]
    for n in names:
        assert torch.equal(a[n].reshape(-1).view(torch.uint8), b[n].reshape(-1).view(torch.uint8)), n


def test_static_scratch_matches_regular_entry_point_twice():
    # two different problems back to back: the second call must not depend on
    # what the first one left in the shared array
    cases = [
        (inputs.variant(inputs.WORKLOADS["video_dit"], H=3, N=4000), 1),
        (inputs.variant(inputs.WORKLOADS["llm_prefill"], H=4, N=2500), 0),
    ]
    for w, mode in cases:
        q, k, v = [t.cuda() for t in inputs.generate(w)]
        B, H, N, d = w.shape()
        out = api.alloc_workspace(B, H, N, d, mode)
        ref = _regular(q, k, v, w, mode)
        got = _static(q, k, v, w, mode, out)
        _same(got, ref, w.smooth_q)
    # and the first problem again after the second
    w, mode = cases[0]
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H, N, d = w.shape()
    _same(_static(q, k, v, w, mode, api.alloc_workspace(B, H, N, d, mode)), _regular(q, k, v, w, mode), w.smooth_q)


def test_static_scratch_refuses_oversized_problem():
    # 3*BH*(Npad/64)*d + BH*d floats must stay within 4 Mi
    B, H, N, d = 1, 32, 32768, 128
    L = api.sage_workspace_layout(B, H, N, d, 0)
    q = torch.empty(16, dtype=torch.float16, device="cuda")
    out = api.alloc_workspace(1, 1, 128, 64, 0)
    with pytest.raises(api.SageError) as e:
        api.sage_quantize_qkv_static(q, q, q, 0, B, H, N, d, False, 0, out, L.scratch)
    assert e.value.status == api.SAGE_ERR_UNSUPPORTED
    assert "static scratch" in str(e.value)


def test_static_scratch_nvfp4_matches_regular_entry_point():
    """The NVFP4 layout (seven partial planes, no V multipliers) through the
    static array, twice in a row, bit for bit against the regular entry point."""
    w = inputs.variant(inputs.WORKLOADS["nvfp4"], H=3, N=1500, smooth_q=True)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H, N, d = w.shape()
    ref = _regular(q, k, v, w, api.MODE_NVFP4)
    for _ in range(2):
        out = api.alloc_workspace(B, H, N, d, api.MODE_NVFP4)
        _same(_static(q, k, v, w, api.MODE_NVFP4, out), ref, w.smooth_q)


def test_static_scratch_refuses_oversized_nvfp4_problem():
    # 7*BH*(Npad/64)*d floats must stay within 4 Mi: B1 H32 N16384 d128 needs 7.3 Mi
    B, H, N, d = 1, 32, 16384, 128
    L = api.sage_workspace_layout(B, H, N, d, api.MODE_NVFP4)
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    out = api.alloc_workspace(1, 1, 128, 64, 0)
    with pytest.raises(api.SageError) as e:
        api.sage_quantize_qkv_static(q, q, q, 1, B, H, N, d, False, api.MODE_NVFP4, out, L.scratch)
    assert e.value.status == api.SAGE_ERR_UNSUPPORTED


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_attention_runs_on_the_static_output(mode):
    """A caller that sized its buffer as documented (sage_ws_layout.scratch
    bytes, no statistics scratch) runs sage_attn_quantized on it and gets the
    output of the regular path bit for bit."""
    base = inputs.WORKLOADS["nvfp4" if mode == 2 else ("video_dit" if mode == 1 else "llm_prefill")]
    w = inputs.variant(base, H=2, N=700, causal=mode == 0)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H, N, d = w.shape()
    dt = api.DTYPE_CODE[q.dtype]
    L = api.sage_workspace_layout(B, H, N, d, mode)
    out_q = api.alloc_workspace(B, H, N, d, mode)[:L.scratch]
    api.sage_quantize_qkv_static(q, k, v, dt, B, H, N, d, w.smooth_q, mode, out_q, L.scratch)
    o_static = torch.empty_like(q)
    api.sage_attn_quantized(out_q, L.scratch, o_static, dt, B, H, N, d, w.causal, w.smooth_q, mode)
    api.sage_check(out_q, L.scratch)
    ws = api.alloc_workspace(B, H, N, d, mode)
    o_reg = api.attn_fwd(q, k, v, causal=w.causal, mode=mode, smooth_q=w.smooth_q, ws=ws)
    api.sage_check(ws, ws.numel())
    assert torch.equal(o_static, o_reg)
