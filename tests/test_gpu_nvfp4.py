"""GPU parity of the NVFP4 mode (SageAttention3 abstract: microscaling FP4):
the CUDA quantizers through the C ABI against the CPU oracle, bit for bit on
codes, block scales, global scales, means and bias."""
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


def unpack_nibbles(b):
    """[..., n] bytes -> [..., 2n] e2m1 codes, low nibble first."""
    b = np.asarray(b, np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def atoms_to_rows(atoms):
    """Q/K scale atoms [BH, Npad/128, d/64, 512] -> [BH, Npad, d/16]."""
    BH, T, KA, _ = atoms.shape
    m = np.arange(128)
    out = np.empty((BH, T * 128, KA * 4), np.uint8)
    for ka in range(KA):
        for kb in range(4):
            out[:, :, ka * 4 + kb] = atoms[:, :, ka, 16 * (m % 32) + 4 * (m // 32) + kb].reshape(BH, T * 128)
    return out


def atoms_to_vt(atoms, d):
    """V^T scale atoms [BH, Npad/128, 2, 512] -> [BH, d, Npad/16]; also the
    unused rows (channels d..127), which must be 0."""
    BH, T, _, _ = atoms.shape
    c = np.arange(128)
    full = np.empty((BH, 128, T * 8), np.uint8)
    for t in range(T):
        for ka in range(2):
            for kb in range(4):
                full[:, :, t * 8 + ka * 4 + kb] = atoms[:, t, ka, 16 * (c % 32) + 4 * (c // 32) + kb]
    return full[:, :d], full[:, d:]


def run_quant_fp4(q, k, v, smooth_q):
    B, H, N, d = q.shape
    ws = api.alloc_workspace(B, H, N, d, api.MODE_NVFP4)
    api.sage_quantize_qkv(q, k, v, api.DTYPE_CODE[q.dtype], B, H, N, d, smooth_q, api.MODE_NVFP4, ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, api.MODE_NVFP4).items()}
    return ws, g


def oracle_fp4(q, k, v, smooth_q):
    B, H, N, d = q.shape
    f = lambda t: t.float().cpu().reshape(B * H, N, d).numpy()
    return orc.quantize_nvfp4(f(q), f(k), f(v), smooth_q)


def assert_fp4_bitexact(g, o, d, smooth_q):
    assert np.array_equal(unpack_nibbles(g["q_codes"]), o["q_codes"]), "q_codes"
    assert np.array_equal(unpack_nibbles(g["k_codes"]), o["k_codes"]), "k_codes"
    assert np.array_equal(unpack_nibbles(g["vt_codes"]), o["vt_codes"]), "vt_codes"
    assert np.array_equal(atoms_to_rows(g["q_sf_atoms"]), o["q_bscale"]), "q block scales"
    assert np.array_equal(atoms_to_rows(g["k_sf_atoms"]), o["k_bscale"]), "k block scales"
    vbs, vpad = atoms_to_vt(g["v_sf_atoms"], d)
    assert np.array_equal(vbs, o["vt_bscale"]), "v block scales"
    assert not vpad.any(), "unused V scale rows must be 0"
    gs = g["global_scale"]
    for col, name in ((0, "q_gscale"), (1, "k_gscale"), (2, "v_gscale")):
        assert np.array_equal(gs[:, col].view(np.uint32), o[name].view(np.uint32)), name
    assert np.array_equal(g["k_mean"].view(np.uint32), o["k_mean"].view(np.uint32)), "k_mean"
    if smooth_q:
        assert np.array_equal(g["q_mean"].view(np.uint32), o["q_mean"].view(np.uint32)), "q_mean"
        assert np.array_equal(g["q_bias"].view(np.uint32), o["q_bias"].view(np.uint32)), "q_bias"


FP4_QUANT = [
    # (N, d, dtype, law, smooth_q)
    (128, 128, "bf16", "student_t3", False),
    (1, 64, "fp16", "student_t3", False),
    (77, 128, "fp16", "qk_bias", True),
    (200, 64, "bf16", "k_bias_outlier", True),
    (1000, 128, "bf16", "student_t3", False),
]


@pytest.mark.parametrize("N,d,dtype,law,smooth_q", FP4_QUANT)
def test_nvfp4_quantize_bitexact(N, d, dtype, law, smooth_q):
    w = inputs.variant(inputs.WORKLOADS["unit"], N=N, d=d, H=2, dtype=dtype, law=law, smooth_q=smooth_q,
                       mode=api.MODE_NVFP4, seed=7000 + N + d)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    _, g = run_quant_fp4(q, k, v, smooth_q)
    assert_fp4_bitexact(g, oracle_fp4(q, k, v, smooth_q), d, smooth_q)


def test_nvfp4_quantize_many_slices_bitexact():
    """B1 H40 N2048 d128 with Q smoothing: codes, block scales, global
    scales, means and bias of many slices equal the oracle's."""
    w = inputs.variant(inputs.WORKLOADS["unit"], N=2048, d=128, H=40, dtype="bf16", law="student_t3",
                       smooth_q=True, mode=api.MODE_NVFP4, seed=7400)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    _, g = run_quant_fp4(q, k, v, True)
    assert_fp4_bitexact(g, oracle_fp4(q, k, v, True), 128, True)


def test_nvfp4_quantize_edge_values():
    """A zero V channel, an all-zero Q slice (global scale 0), a constant K
    block, a value far above the rest (subnormal block scales elsewhere)."""
    w = inputs.variant(inputs.WORKLOADS["unit"], N=150, d=64, H=2, dtype="fp16", law="student_t3",
                       mode=api.MODE_NVFP4, seed=7777)
    q, k, v = [t.clone() for t in inputs.generate(w)]
    v[:, :, :, 3] = 0
    q[:, 1] = 0
    k[:, 0, 16:32, :] = 2.5
    v[:, 0, 5, 7] = 3000.0
    q, k, v = [t.cuda() for t in (q, k, v)]
    for smooth_q in (False, True):
        _, g = run_quant_fp4(q, k, v, smooth_q)
        assert_fp4_bitexact(g, oracle_fp4(q, k, v, smooth_q), 64, smooth_q)
    assert g["global_scale"][1, 0] == 0 and not unpack_nibbles(g["q_codes"][1]).any()


def dequant_rows(codes, bscale):
    """e2m1 codes [.., n] and ue4m3 scales [.., n/16] -> values (float64)."""
    e2m1 = np.array([orc.e2m1_decode(c) for c in range(16)])
    ue4m3 = np.array([orc.e4m3_decode(c & 0x7F) for c in range(256)])
    return e2m1[codes] * np.repeat(ue4m3[bscale], 16, axis=-1)


@pytest.mark.parametrize("N,law", [(256, "student_t3"), (300, "qk_bias")])
def test_nvfp4_s_tile_tensor_core(N, law):
    """One block-scaled S tile through tcgen05.cp + kind::mxf4nvf4 equals the
    exact sum of products of the dequantized codes (FP32 accumulation)."""
    w = inputs.variant(inputs.WORKLOADS["unit"], N=N, d=128, H=2, dtype="bf16", law=law, smooth_q=False,
                       mode=api.MODE_NVFP4, seed=7100 + N)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H, d = 1, 2, 128
    ws, g = run_quant_fp4(q, k, v, False)
    qd = dequant_rows(unpack_nibbles(g["q_codes"]), atoms_to_rows(g["q_sf_atoms"]))
    kd = dequant_rows(unpack_nibbles(g["k_codes"]), atoms_to_rows(g["k_sf_atoms"]))
    T = (N + 127) // 128
    out = torch.empty(128, 128, dtype=torch.float32, device="cuda")
    for bh in range(B * H):
        for qt, kt in {(0, 0), (T - 1, 0), (0, T - 1), (T - 1, T - 1)}:
            api.sage_debug_fp4_s(ws, ws.numel(), B, H, N, d, bh, qt, kt, out)
            api.sage_check(ws, ws.numel())
            ref = qd[bh, qt * 128:(qt + 1) * 128] @ kd[bh, kt * 128:(kt + 1) * 128].T
            got = out.cpu().numpy().astype(np.float64)
            scale = np.abs(ref).max() + 1e-30
            assert np.abs(got - ref).max() <= 1e-5 * scale, (bh, qt, kt, np.abs(got - ref).max(), scale)


ATTN_FP4 = [
    # (N, dtype, law, smooth_q, causal)
    (128, "bf16", "student_t3", False, False),
    (1, "bf16", "student_t3", False, False),
    (33, "fp16", "k_bias", False, True),
    (256, "bf16", "student_t3", False, False),
    (300, "fp16", "qk_bias", True, True),
    (1000, "bf16", "student_t3", False, True),
    (640, "fp16", "k_bias_outlier", True, False),
]


@pytest.mark.parametrize("N,dtype,law,smooth_q,causal", ATTN_FP4)
def test_nvfp4_attention_matches_oracle(N, dtype, law, smooth_q, causal):
    """The fused kind::mxf4nvf4 attention against the oracle's NVFP4
    attention on the same (bit-identical) codes and scales, output rounded to
    the dtype, with the INT8/FP8 modes' bounds."""
    w = inputs.variant(inputs.WORKLOADS["unit"], N=N, d=128, H=2, dtype=dtype, law=law, smooth_q=smooth_q,
                       mode=api.MODE_NVFP4, causal=causal, seed=7300 + N)
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    B, H, d = 1, 2, 128
    ws = api.alloc_workspace(B, H, N, d, api.MODE_NVFP4)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, causal, api.MODE_NVFP4, api.DTYPE_CODE[q.dtype], smooth_q, ws,
                      ws.numel())
    api.sage_check(ws, ws.numel())
    ref32, flip = orc.attention_nvfp4(oracle_fp4(q, k, v, smooth_q), causal, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()
    compare_out(got, ref32, flip, dtype, (N, dtype, law, smooth_q, causal))


def test_nvfp4_attention_rejects_d64():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    ws = api.alloc_workspace(1, 1, 128, 64, api.MODE_NVFP4)
    with pytest.raises(api.SageError) as e:
        api.sage_attn_fwd(q, q, q, torch.empty_like(q), 1, 1, 128, 64, False, api.MODE_NVFP4, 1, False, ws,
                          ws.numel())
    assert e.value.status == api.SAGE_ERR_UNSUPPORTED


def test_full_size_nvfp4_sampled_rows():
    """The B1 H16 N16384 d128 bf16 NVFP4 workload at full size, in the launch
    configuration the bench times: quantization bit-exact everywhere, the
    output on sampled rows per head (first, tile edges, last, random)."""
    w = inputs.WORKLOADS["nvfp4"]
    B, H, N, d = w.shape()
    q, k, v = [t.cuda() for t in inputs.generate(w)]
    ws = api.alloc_workspace(B, H, N, d, api.MODE_NVFP4)
    out = torch.empty_like(q)
    api.sage_attn_fwd(q, k, v, out, B, H, N, d, w.causal, api.MODE_NVFP4, api.DTYPE_CODE[q.dtype], w.smooth_q,
                      ws, ws.numel())
    api.sage_check(ws, ws.numel())
    g = {n: t.cpu().numpy() for n, t in api.ws_views(ws, B, H, N, d, api.MODE_NVFP4).items()}
    oz = oracle_fp4(q, k, v, w.smooth_q)
    assert_fp4_bitexact(g, oz, d, w.smooth_q)
    rng = np.random.default_rng(16384)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 129, N - 1], rng.integers(0, N, 11)])).astype(np.int32)
    ref32, flip = orc.attention_nvfp4(oz, w.causal, rows=rows, with_flip=True)
    got = out.float().cpu().reshape(B * H, N, d).numpy()[:, rows]
    compare_out(got, ref32, flip, w.dtype, "nvfp4 full size")
