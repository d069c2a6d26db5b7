"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Codes, scales and INT32 QK^T tiles must be bit-exact; the
output within max-abs 2e-3 and relative-L1 5e-4 of the oracle's, with the two
derived exemptions of parity_check.compare_out (counted and printed)."""
import numpy as np
import pytest
import torch

import oracle as orc
from parity_check import compare_out, to_dtype_np
from quantized_attention_sub_b200 import api, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_attention_sub_b200 import build
    build.build()
    api.lib()


def run_quant(w, mode, smooth_q, device_inputs=None):
    q, k, v = device_inputs if device_inputs is not None else [t.cuda() for t in inputs.generate(w)]
    B, H, N, d = w.shape()
    ws = api.alloc_workspace(B, H, N, d, mode)
    api.sage_quantize_qkv(q, k, v, api.DTYPE_CODE[q.dtype], B, H, N, d, smooth_q, mode, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    return (q, k, v), ws, {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, mode).items()}


def oracle_quant(qkv, mode, smooth_q):
    B, H, N, d = qkv[0].shape
    f = lambda t: t.float().cpu().reshape(B * H, N, d).numpy()
    return orc.quantize_int8_fp8(f(qkv[0]), f(qkv[1]), f(qkv[2]), smooth_q=smooth_q, mode=mode)


def assert_quant_bitexact(g, o, smooth_q):
    for name in ("q_codes", "k_codes", "vt_codes"):
        assert np.array_equal(g[name].view(np.uint8), o[name].view(np.uint8)), name
    for name in ("q_scale", "k_scale", "v_scale", "k_mean"):
        assert np.array_equal(g[name].view(np.uint32), o[name].view(np.uint32)), name
    if smooth_q:
        assert np.array_equal(g["q_mean"].view(np.uint32), o["q_mean"].view(np.uint32))
        assert np.array_equal(g["q_bias"].view(np.uint32), o["q_bias"].view(np.uint32))


SMALL = [
    # (N, d, dtype, law, smooth_q, mode)
    (128, 64, "fp16", "k_bias", False, 0),
    (1, 64, "fp16", "k_bias", False, 0),
    (31, 128, "bf16", "k_bias_outlier", False, 0),
    (129, 128, "fp16", "qk_bias", True, 0),
    (333, 64, "bf16", "qk_bias", True, 1),
    (1000, 128, "bf16", "k_bias_outlier", False, 0),
    (700, 128, "fp16", "qk_bias", True, 1),
]


def small_workload(N, d, dtype, law, smooth_q, mode, H=2, causal=False):
    return inputs.variant(inputs.WORKLOADS["unit"], N=N, d=d, H=H, dtype=dtype, law=law, smooth_q=smooth_q,
                          mode=mode, causal=causal, seed=5000 + N + d)


@pytest.mark.parametrize("N,d,dtype,law,smooth_q,mode", SMALL)
def test_quantize_bitexact(N, d, dtype, law, smooth_q, mode):
    w = small_workload(N, d, dtype, law, smooth_q, mode)
    qkv, ws, g = run_quant(w, mode, smooth_q)
    assert_quant_bitexact(g, oracle_quant(qkv, mode, smooth_q), smooth_q)


@pytest.mark.parametrize("H,N,d,smooth_q", [(40, 2048, 128, False), (80, 2048, 64, True)])
def test_quantize_many_slices_bitexact(H, N, d, smooth_q):
    """Many slices (40 and 80, more than the persistent passes' CTAs can
    take in one round of chunks): every code, scale, mean and bias equals
    the oracle's."""
    w = small_workload(N, d, "fp16", "qk_bias" if smooth_q else "k_bias", smooth_q, 0, H=H)
    qkv, ws, g = run_quant(w, 0, smooth_q)
    assert_quant_bitexact(g, oracle_quant(qkv, 0, smooth_q), smooth_q)


def test_quantize_edge_values():
    """Zero channels, constant tokens, a zero granule, huge and tiny values."""
    w = small_workload(200, 64, "fp16", "k_bias", True, 0)
    q, k, v = [t.clone() for t in inputs.generate(w)]
    v[:, :, :, 5] = 0          # zero V channel -> scale 0, codes 0
    k[:, :, 64:128, :] = 3.0   # constant K granule -> after smoothing mostly nonzero
    q[:, 1, 32:64, :] = 0      # zero Q granule when not smoothed
    v[:, 0, 7, 9] = 60000.0    # big value: other codes of channel 9 go subnormal
    for smooth_q in (False, True):
        qkv, ws, g = run_quant(w, 0, smooth_q, [t.cuda() for t in (q, k, v)])
        o = oracle_quant(qkv, 0, smooth_q)
        assert_quant_bitexact(g, o, smooth_q)
    assert np.all(g["vt_codes"][:, 5] == 0) and np.all(g["v_scale"][:, 5] == 0)


@pytest.mark.parametrize("N,d", [(128, 64), (333, 128), (1000, 64)])
def test_qk_s32_tiles_bitexact(N, d):
    w = small_workload(N, d, "fp16", "k_bias", False, 0)
    qkv, ws, g = run_quant(w, 0, False)
    B, H = 1, 2
    T = (N + 127) // 128
    out = torch.empty(128, 128, dtype=torch.int32, device="cuda")
    for bh in range(B * H):
        for qt, kt in {(0, 0), (T - 1, 0), (0, T - 1), (T - 1, T - 1), (T // 2, (T + 1) // 3)}:
            api.sage_debug_qk_s32(ws, ws.numel(), B, H, N, d, bh, qt, kt, out)
            api.sage_check(ws, ws.numel())
            ref = orc.qk_s32(g["q_codes"][bh, qt * 128:(qt + 1) * 128], g["k_codes"][bh, kt * 128:(kt + 1) * 128])
            assert np.array_equal(out.cpu().numpy(), ref), (bh, qt, kt)


@pytest.mark.parametrize("N,d", [(32768, 128), (8192, 64)])
def test_qk_s32_tiles_bitexact_long(N, d):
    """One slice at the sweep's token counts (the headline N = 32768, d = 128):
    INT32 S tiles across the whole key range -- first, last, diagonal and
    off-diagonal -- equal the oracle's integer products."""
    w = inputs.variant(inputs.sweep(N, d, False), B=1, H=1)
    qkv, ws, g = run_quant(w, 0, False)
    T = N // 128
    out = torch.empty(128, 128, dtype=torch.int32, device="cuda")
    for qt, kt in [(0, 0), (T - 1, T - 1), (0, T - 1), (T - 1, 0), (T // 2, T // 3), (T // 3, 2 * T // 3)]:
        api.sage_debug_qk_s32(ws, ws.numel(), 1, 1, N, d, 0, qt, kt, out)
        api.sage_check(ws, ws.numel())
        ref = orc.qk_s32(g["q_codes"][0, qt * 128:(qt + 1) * 128], g["k_codes"][0, kt * 128:(kt + 1) * 128])
        assert np.array_equal(out.cpu().numpy(), ref), (qt, kt)


ATTN_SMALL = [
    # (N, d, dtype, law, smooth_q, causal, mode)
    (128, 64, "fp16", "k_bias", False, False, 0),
    (1, 128, "bf16", "k_bias", False, False, 0),
    (33, 64, "fp16", "k_bias", False, True, 0),
    (129, 128, "bf16", "k_bias_outlier", False, True, 0),
    (333, 128, "fp16", "qk_bias", True, False, 0),
    (640, 64, "bf16", "qk_bias", True, True, 0),
    (1000, 128, "bf16", "k_bias_outlier", False, True, 0),
    (1000, 128, "fp16", "k_bias", False, False, 0),
    # FP16 PV accumulator (SageAttention2++)
    (1, 128, "fp16", "qk_bias", True, False, 1),
    (128, 64, "fp16", "k_bias", False, False, 1),
    (200, 128, "fp16", "qk_bias", True, True, 1),
    (700, 128, "fp16", "qk_bias", True, False, 1),
    (1000, 64, "bf16", "k_bias_outlier", False, True, 1),
]


@pytest.mark.parametrize("N,d,dtype,law,smooth_q,causal,mode", ATTN_SMALL)
def test_attention_matches_oracle(N, d, dtype, law, smooth_q, causal, mode):
    w = small_workload(N, d, dtype, law, smooth_q, mode, causal=causal)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H = 1, 2
    ws = api.alloc_workspace(B, H, N, d, mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, causal, mode, api.DTYPE_CODE[q.dtype], smooth_q, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    oz = oracle_quant((q, k, v), mode, smooth_q)
    ref32, flip = orc.attention_int8_fp8(oz, causal, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()
    compare_out(got, ref32, flip, dtype, (N, d, dtype, causal, mode))


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("case", ["zero_k_granules", "zero_q_granule"])
def test_attention_zero_scale_granules_with_masks(mode, case):
    """Degenerate scales under causal and ragged masks.  zero_k_granules: K is
    the same vector for every token, so the smoothed K and every K scale are
    0 and every logit is 0 (each row averages the V of the keys it sees).
    zero_q_granule: Q rows 32..63 are 0 (no Q smoothing), so that granule's
    scale is 0.  Masked keys must stay out in both."""
    N, d = 300, 128
    w = small_workload(N, d, "fp16", "k_bias", False, mode, causal=True)
    q, k, v = [t.clone() for t in inputs.generate(w)]
    if case == "zero_k_granules":
        k[:] = k[:, :, :1, :]
    else:
        q[:, :, 32:64, :] = 0
    q, k, v = [t.cuda() for t in (q, k, v)]
    B, H = 1, 2
    ws = api.alloc_workspace(B, H, N, d, mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, True, mode, 0, False, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    oz = oracle_quant((q, k, v), mode, False)
    if case == "zero_k_granules":
        assert not np.any(oz["k_scale"])
    ref32, flip = orc.attention_int8_fp8(oz, True, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()
    compare_out(got, ref32, flip, "fp16", (case, mode))


def test_full_size_llm_prefill_sampled_rows():
    """The B1 H32 N8192 d128 bf16 causal workload at full size, in the launch
    configuration the bench times: quantization bit-exact everywhere, the
    output on 24 sampled rows per head (first, last, tile edges, random)."""
    w = inputs.WORKLOADS["llm_prefill"]
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(B, H, N, d, 0)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, True, 0, 1, False, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, 0).items()}
    oz = oracle_quant((q, k, v), 0, False)
    assert_quant_bitexact(g, oz, False)
    rng = np.random.default_rng(8192)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, N - 129, N - 128, N - 1],
                                     rng.integers(0, N, 15)])).astype(np.int32)
    ref32, flip = orc.attention_int8_fp8(oz, True, rows=rows, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()[:, rows]
    compare_out(got, ref32, flip, "bf16", "llm_prefill")


def test_full_size_video_dit_sampled_rows():
    """B1 H12 N32760 d128 fp16, non-causal, FP16 PV accumulator, Q smoothing:
    quantization bit-exact everywhere, the output on sampled rows per head."""
    w = inputs.WORKLOADS["video_dit"]
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(B, H, N, d, w.mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, False, w.mode, 0, True, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, w.mode).items()}
    oz = oracle_quant((q, k, v), w.mode, True)
    assert_quant_bitexact(g, oz, True)
    rng = np.random.default_rng(32760)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 121, N - 120, N - 1], rng.integers(0, N, 10)])).astype(np.int32)
    ref32, flip = orc.attention_int8_fp8(oz, False, rows=rows, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()[:, rows]
    compare_out(got, ref32, flip, "fp16", "video_dit")


def test_max_size_sampled_slices():
    """The largest problem the C ABI accepts in element count: B1 H16383
    N1024 d128, B*H*Npad*d = 2^31 - 2^17 (the limit is < 2^31), 16383
    slices in the attention grid.  Inputs drawn on the GPU (12.9 GB), the
    whole problem quantized and attended; three slices spread over the index
    range are checked: codes and scales bit-exact, the output on sampled
    rows within the parity bounds (so no index past 2^31 bytes wraps)."""
    w = inputs.variant(inputs.sweep(1024, 128, False), B=1, H=16383)
    B, H, N, d = w.shape()
    assert B * H * N * d < (1 << 31) <= B * (H + 1) * N * d  # one more slice is refused
    q, k, v = inputs.generate(w, device="cuda")
    ws = api.alloc_workspace(B, H, N, d, 0)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, False, 0, 0, False, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    views = api.ws_views(ws, B, H, N, d, 0)
    rows = np.array([0, 1, 127, 128, 511, 512, 1022, 1023], np.int32)
    for bh in (0, H // 2, H - 1):
        sl = lambda t: t[:, bh:bh + 1].contiguous()
        oz = oracle_quant((sl(q), sl(k), sl(v)), 0, False)
        g = {n: views[n][bh:bh + 1].cpu().numpy() for n in ("q_codes", "k_codes", "vt_codes", "q_scale", "k_scale",
                                                              "v_scale", "k_mean")}
        assert_quant_bitexact(g, oz, False)
        ref32, flip = orc.attention_int8_fp8(oz, False, rows=rows, with_flip=True)
        got = out[0, bh].float().cpu().numpy()[rows][None]
        compare_out(got, ref32, flip, "fp16", "max size, slice %d" % bh)
    del q, k, v, ws, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("N,d,causal", [(8192, 128, False), (2048, 64, True), (8192, 64, True), (16384, 64, True),
                                         (4096, 128, True), (16384, 128, True), (1024, 64, False)])
def test_sweep_points_sampled_rows(N, d, causal):
    """Points of the kernel-speed sweep (B4 H32 fp16, K bias N(0, 2^2)):
    quantization bit-exact everywhere, the output on sampled rows of every
    head (tile edges, the last row, random rows).  The causal points cover
    the causal CTA orders: longest-first across all 128 slices (N 2048), in
    two groups of 64 slices (N 8192), and per slice (N 16384)."""
    w = inputs.sweep(N, d, causal)
    B, H = w.B, w.H
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(B, H, N, d, 0)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, causal, 0, 0, False, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, 0).items()}
    oz = oracle_quant((q, k, v), 0, False)
    assert_quant_bitexact(g, oz, False)
    rng = np.random.default_rng(N + d)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.integers(0, N, 4)])).astype(np.int32)
    ref32, flip = orc.attention_int8_fp8(oz, causal, rows=rows, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()[:, rows]
    compare_out(got, ref32, flip, "fp16", w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_target_point_n32k_d128_sampled(causal):
    """The sweep's target point B4 H32 N32768 d128 fp16 (the point the kernel's
    50 %-of-peak aim is quoted on), in the launch configuration the bench
    times: codes and scales bit-exact on four of the 128 slices, the output on
    sampled rows of those slices."""
    w = inputs.sweep(32768, 128, causal)
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w, device="cuda")]
    ws = api.alloc_workspace(B, H, N, d, 0)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, causal, 0, 0, False, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    slices = np.array([0, 45, 90, 127])
    views = api.ws_views(ws, B, H, N, d, 0)
    g = {n: views[n][slices].cpu().numpy() for n in ("q_codes", "k_codes", "vt_codes", "q_scale", "k_scale",
                                                       "v_scale", "k_mean")}
    f = lambda t: t.reshape(B * H, N, d)[slices].float().cpu().numpy()
    oz = orc.quantize_int8_fp8(f(q), f(k), f(v), smooth_q=False, mode=0)
    assert_quant_bitexact(g, oz, False)
    rng = np.random.default_rng(32768 + int(causal))
    rows = np.unique(np.concatenate([[0, 127, 128, N - 129, N - 1], rng.integers(0, N, 7)])).astype(np.int32)
    ref32, flip = orc.attention_int8_fp8(oz, causal, rows=rows, with_flip=True)
    got = out.reshape(B * H, N, d)[slices][:, rows].float().cpu().numpy()
    compare_out(got, ref32, flip, "fp16", w.name)


def test_repeated_calls_identical_and_no_error():
    w = small_workload(1000, 128, "bf16", "k_bias", False, 0, causal=True)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(1, 2, 1000, 128, 0)
    outs = []
    for _ in range(3):
        out = torch.empty_like(q)
        api.sage_attn_fwd(q, k, v, out, 1, 2, 1000, 128, True, 0, 1, False, ws, ws.numel())
        outs.append(out)
    api.sage_check(ws, ws.numel())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = api.alloc_workspace(1, 2, 128, 64, 0)
    api.sage_debug_timeout_probe(ws, ws.numel())
    with pytest.raises(api.SageError) as e:
        api.sage_check(ws, ws.numel())
    assert e.value.status == api.SAGE_ERR_TIMEOUT
    # the context still runs work and the word was cleared
    api.sage_check(ws, ws.numel())
    w = small_workload(128, 64, "fp16", "k_bias", False, 0)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    out = api.attn_fwd(q, k, v, ws=ws)
    api.sage_check(ws, ws.numel())
    assert torch.isfinite(out.float()).all()
