"""Q smoothed per 128-row block through the C ABI (sage_*_blocksmooth) against
the CPU oracle: codes, scales, block means and bias rows bit-exact, the
output within the parity bounds, and the one-call forward equal to the
quantize + attention pair."""
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


def _inputs(B, H, N, d, dtype, seed, block_std=3.0):
    """Q with a different per-channel offset in every 128-row block (the case
    per-block smoothing is for), K with a per-channel bias, V standard normal."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g)
    nb = (N + 127) // 128
    off = block_std * torch.randn(B, H, nb, d, generator=g)
    q += off.repeat_interleave(128, dim=2)[:, :, :N]
    k = torch.randn(B, H, N, d, generator=g) + 2.0 * torch.randn(B, H, 1, d, generator=g)
    v = torch.randn(B, H, N, d, generator=g)
    dt = inputs.DTYPES[dtype]
    return [t.to(dt).cuda() for t in (q, k, v)]


def _np(t):
    return t.float().cpu().reshape(-1, t.shape[-2], t.shape[-1]).numpy()


def _assert_quant_bitexact(g, oz):
    for name in ("q_codes", "k_codes", "vt_codes"):
        assert np.array_equal(g[name].view(np.uint8), oz[name].view(np.uint8)), name
    for name in ("q_scale", "k_scale", "v_scale", "k_mean", "q_mean", "q_bias"):
        assert np.array_equal(g[name].view(np.uint32), oz[name].view(np.uint32)), name


CASES = [
    # (B, H, N, d, dtype, causal, mode)
    (1, 2, 300, 128, "fp16", False, 0),
    (2, 2, 1000, 64, "bf16", True, 1),
    (1, 3, 129, 128, "bf16", True, 0),
    (1, 1, 1, 64, "fp16", False, 0),
    (1, 2, 64, 128, "fp16", True, 1),
    (1, 1, 8300, 128, "bf16", False, 0),   # 65 blocks: a second group of 64 holding one block
    (1, 2, 8192 + 65, 64, "fp16", True, 1),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,mode", CASES)
def test_blocksmooth_matches_oracle(B, H, N, d, dtype, causal, mode):
    q, k, v = _inputs(B, H, N, d, dtype, 9300 + N + d + H)
    ws = api.alloc_workspace_blocksmooth(B, H, N, d, mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd_blocksmooth(q, k, v, out, B, H, N, d, causal, mode, api.DTYPE_CODE[q.dtype], ws, ws.numel())
    api.sage_check(ws, ws.numel())
    oz = orc.quantize_int8_fp8_blocksmooth(_np(q), _np(k), _np(v), mode)
    g = {n: t.cpu().numpy() for n, t in api.ws_views_blocksmooth(ws, B, H, N, d, mode).items()}
    _assert_quant_bitexact(g, oz)
    if N <= 1024:
        rows = None
    else:
        rng = np.random.default_rng(N)
        rows = np.unique(np.concatenate([[0, 127, 128, 8191 if N > 8191 else 1, N - 65, N - 64, N - 1],
                                         rng.integers(0, N, 12)])).astype(np.int32)
    ref32, flip = orc.attention_int8_fp8_blocksmooth(oz, causal, rows=rows, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()
    if rows is not None:
        got = got[:, rows]
    compare_out(got, ref32, flip, dtype, (B, H, N, d, causal, mode))


def test_fwd_equals_quantize_then_attention():
    B, H, N, d = 1, 2, 700, 128
    q, k, v = _inputs(B, H, N, d, "fp16", 9400)
    for mode in (0, 1):
        for causal in (False, True):
            ws1 = api.alloc_workspace_blocksmooth(B, H, N, d, mode)
            ws2 = api.alloc_workspace_blocksmooth(B, H, N, d, mode)
            o1, o2 = torch.empty_like(q), torch.empty_like(q)
            api.sage_attn_fwd_blocksmooth(q, k, v, o1, B, H, N, d, causal, mode, 0, ws1, ws1.numel())
            api.sage_quantize_qkv_blocksmooth(q, k, v, 0, B, H, N, d, mode, ws2, ws2.numel())
            api.sage_attn_quantized_blocksmooth(ws2, ws2.numel(), o2, 0, B, H, N, d, causal, mode)
            api.sage_check(ws2, ws2.numel())
            assert torch.equal(o1, o2), (mode, causal)


def test_blocksmooth_beats_per_slice_on_drifting_q():
    """Where Q's offset changes from block to block, per-block smoothing is
    closer to fp64 attention than per-slice smoothing, on the GPU as in the
    oracle (B1 H4 N2048 d128 fp16, block offsets N(0, 4^2))."""
    B, H, N, d = 1, 4, 2048, 128
    q, k, v = _inputs(B, H, N, d, "fp16", 9500, block_std=4.0)
    ob, og = torch.empty_like(q), torch.empty_like(q)
    wb = api.alloc_workspace_blocksmooth(B, H, N, d, 0)
    wg = api.alloc_workspace(B, H, N, d, 0)
    api.sage_attn_fwd_blocksmooth(q, k, v, ob, B, H, N, d, False, 0, 0, wb, wb.numel())
    api.sage_attn_fwd(q, k, v, og, B, H, N, d, False, 0, 0, True, wg, wg.numel())
    api.sage_check(wb, wb.numel())
    ref = orc.attention_fp64(_np(q), _np(k), _np(v), False)
    eb = np.abs(_np(ob) - ref).sum() / np.abs(ref).sum()
    eg = np.abs(_np(og) - ref).sum() / np.abs(ref).sum()
    assert eb < eg, (eb, eg)


def test_full_size_video_dit_blocksmooth_sampled():
    """The video_dit shape (B1 H12 N32760 d128 fp16, FP16 PV accumulator) with
    per-block Q smoothing: K and V codes and scales bit-exact everywhere; Q's
    block means, codes, scales and bias rows bit-exact on sampled blocks (the
    oracle's per-block steps on those blocks' rows); the output on rows of
    those blocks."""
    w = inputs.WORKLOADS["video_dit"]
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace_blocksmooth(B, H, N, d, w.mode)
    out = torch.empty_like(q)
    api.sage_attn_fwd_blocksmooth(q, k, v, out, B, H, N, d, False, w.mode, 0, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views_blocksmooth(ws, B, H, N, d, w.mode).items()}
    qn, kn, vn = _np(q), _np(k), _np(v)
    # every block's bias row in the oracle takes minutes at this size: K and V
    # come from the oracle whole, the Q side of the sampled blocks from the
    # oracle's per-block steps (block mean, granule codes, bias row)
    nb = (N + 127) // 128
    blocks = np.array([0, 1, 128, nb - 2, nb - 1])
    oz = orc.quantize_int8_fp8(qn, kn, vn, smooth_q=False, mode=w.mode)
    for name in ("k_codes", "vt_codes"):
        assert np.array_equal(g[name].view(np.uint8), oz[name].view(np.uint8)), name
    for name in ("k_scale", "v_scale", "k_mean"):
        assert np.array_equal(g[name].view(np.uint32), oz[name].view(np.uint32)), name
    qc, sq = np.zeros_like(oz["q_codes"]), np.zeros_like(oz["q_scale"])
    for b in blocks:
        r0, r1 = 128 * b, min(N, 128 * b + 128)
        mb = orc.channel_mean(np.ascontiguousarray(qn[:, r0:r1]))
        assert np.array_equal(g["q_mean"][:, b].view(np.uint32), mb.view(np.uint32)), b
        cb, sb = orc.quant_int8(np.ascontiguousarray(qn[:, r0:r1]), mb, orc.Q_GRANULE)
        qc[:, r0:r0 + 128], sq[:, r0 // 32:r0 // 32 + 4] = cb, sb
        assert np.array_equal(g["q_codes"][:, r0:r0 + 128], cb), b
        assert np.array_equal(g["q_scale"][:, r0 // 32:r0 // 32 + 4].view(np.uint32), sb.view(np.uint32)), b
        bias = orc.q_bias(kn, oz["k_mean"], mb)
        assert np.array_equal(g["q_bias"][:, b].view(np.uint32), bias.view(np.uint32)), b
        # rows of block b read only block b's Q codes and scales
        view = dict(oz, q_codes=qc, q_scale=sq, q_bias=bias)
        rows = np.array(sorted({r0, (r0 + r1) // 2, r1 - 1}), np.int32)
        ref32, flip = orc.attention_int8_fp8(view, False, rows=rows, with_flip=True)
        got = out.float().cpu().reshape(B * H, N, d).numpy()[:, rows]
        compare_out(got, ref32, flip, "fp16", ("video_dit_blocksmooth", int(b)))


def test_sweep_point_blocksmooth_sampled():
    """The shape `bench.py --q-blocks` times (B4 H32 N8192 d128 fp16, FP32
    accumulator, non-causal): on three of the 128 slices, K and V codes and
    scales bit-exact; on sampled blocks of those slices the block means, Q
    codes, scales and bias rows bit-exact (the oracle's per-block steps), and
    the output on rows of those blocks."""
    w = inputs.variant(inputs.sweep(8192, 128, False), smooth_q=True)
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w, device="cuda")]
    ws = api.alloc_workspace_blocksmooth(B, H, N, d, 0)
    out = torch.empty_like(q)
    api.sage_attn_fwd_blocksmooth(q, k, v, out, B, H, N, d, False, 0, 0, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    slices = np.array([0, 77, 127])
    views = api.ws_views_blocksmooth(ws, B, H, N, d, 0)
    g = {n: views[n][slices].cpu().numpy() for n in views}
    f = lambda t: t.reshape(B * H, N, d)[slices].float().cpu().numpy()
    qn, kn, vn = f(q), f(k), f(v)
    oz = orc.quantize_int8_fp8(qn, kn, vn, smooth_q=False, mode=0)
    for name in ("k_codes", "vt_codes"):
        assert np.array_equal(g[name].view(np.uint8), oz[name].view(np.uint8)), name
    for name in ("k_scale", "v_scale", "k_mean"):
        assert np.array_equal(g[name].view(np.uint32), oz[name].view(np.uint32)), name
    got_all = out.reshape(B * H, N, d)[slices].float().cpu().numpy()
    qc, sq = np.zeros_like(oz["q_codes"]), np.zeros_like(oz["q_scale"])
    for b in (0, 1, 31, 63):
        r0 = 128 * b
        mb = orc.channel_mean(np.ascontiguousarray(qn[:, r0:r0 + 128]))
        assert np.array_equal(g["q_mean"][:, b].view(np.uint32), mb.view(np.uint32)), b
        cb, sb = orc.quant_int8(np.ascontiguousarray(qn[:, r0:r0 + 128]), mb, orc.Q_GRANULE)
        qc[:, r0:r0 + 128], sq[:, r0 // 32:r0 // 32 + 4] = cb, sb
        assert np.array_equal(g["q_codes"][:, r0:r0 + 128], cb), b
        assert np.array_equal(g["q_scale"][:, r0 // 32:r0 // 32 + 4].view(np.uint32), sb.view(np.uint32)), b
        bias = orc.q_bias(kn, oz["k_mean"], mb)
        assert np.array_equal(g["q_bias"][:, b].view(np.uint32), bias.view(np.uint32)), b
        # rows of block b read only block b's Q codes and scales
        view = dict(oz, q_codes=qc, q_scale=sq, q_bias=bias)
        rows = np.array([r0, r0 + 63, r0 + 127], np.int32)
        ref32, flip = orc.attention_int8_fp8(view, False, rows=rows, with_flip=True)
        compare_out(got_all[:, rows], ref32, flip, "fp16", ("sweep_N8192_blocksmooth", b))
