"""The C-ABI library loads and exports every symbol include/sage.h declares;
host-side argument checks and the workspace layout (no GPU needed)."""
import ctypes
import os
import re

import pytest

from quantized_attention_sub_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sage.h")).read()
    return sorted(set(re.findall(r"SAGE_API\s+[\w\s\*]+?\b(sage_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from quantized_attention_sub_b200 import build
    build.build()
    return api.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(api.EXPORTED) <= set(names)


def test_workspace_layout_is_aligned_and_disjoint(lib):
    for (B, H, N, d, mode) in [(1, 2, 128, 64, 0), (1, 32, 8192, 128, 0), (1, 12, 32760, 128, 1), (4, 3, 1, 64, 0),
                               (1, 16, 16384, 128, 2)]:
        L = api.sage_workspace_layout(B, H, N, d, mode)
        offs = [getattr(L, f) for f, _ in api.WsLayout._fields_ if f != "total"]
        assert all(o % 1024 == 0 for o in offs)
        assert L.total >= max(offs) and api.sage_workspace_size(B, H, N, d, mode) == L.total
        Np = (N + 127) // 128 * 128
        if mode != 2:
            assert L.k_codes - L.q_codes >= B * H * Np * d
            assert L.vt_codes - L.k_codes >= B * H * Np * d


@pytest.mark.parametrize("args,status", [
    ((1, 1, 128, 96, 0), api.SAGE_ERR_UNSUPPORTED),
    ((0, 1, 128, 64, 0), api.SAGE_ERR_INVALID_ARG),
    ((1, 1, 0, 64, 0), api.SAGE_ERR_INVALID_ARG),
    ((1, 1, 128, 64, 7), api.SAGE_ERR_INVALID_ARG),
    ((64, 64, 1 << 20, 128, 0), api.SAGE_ERR_UNSUPPORTED),
])
def test_bad_shapes_rejected_on_host(lib, args, status):
    out = api.WsLayout()
    assert lib.sage_workspace_layout(*args, ctypes.byref(out)) == status
    assert api.sage_workspace_size(*args) == 0
    assert len(lib.sage_last_error()) > 0


def test_bad_pointers_rejected_before_any_launch(lib):
    vp = ctypes.c_void_p
    ws_bytes = api.sage_workspace_size(1, 2, 128, 64, 0)
    # null inputs
    st = lib.sage_quantize_qkv(vp(0), vp(0), vp(0), 0, 1, 2, 128, 64, 0, 0, vp(1024), ws_bytes, vp(0))
    assert st == api.SAGE_ERR_INVALID_ARG
    # misaligned workspace
    st = lib.sage_quantize_qkv(vp(4096), vp(4096), vp(4096), 0, 1, 2, 128, 64, 0, 0, vp(1040), ws_bytes, vp(0))
    assert st == api.SAGE_ERR_INVALID_ARG
    # workspace too small
    st = lib.sage_quantize_qkv(vp(4096), vp(4096), vp(4096), 0, 1, 2, 128, 64, 0, 0, vp(4096), 16, vp(0))
    assert st == api.SAGE_ERR_INVALID_ARG
    # bad dtype
    st = lib.sage_attn_quantized(vp(4096), ws_bytes, vp(4096), 5, 1, 2, 128, 64, 0, 0, 0, vp(0))
    assert st == api.SAGE_ERR_INVALID_ARG
    # debug tile out of range
    st = lib.sage_debug_qk_s32(vp(4096), ws_bytes, 1, 2, 128, 64, 0, 1, 0, vp(4096), vp(0))
    assert st == api.SAGE_ERR_INVALID_ARG


@pytest.mark.parametrize("args,status", [
    ((1, 6, 4, 128, 128, 64, 0), api.SAGE_ERR_INVALID_ARG),      # Hq not a multiple of Hkv
    ((1, 8, 2, 128, 128, 128, 2), api.SAGE_ERR_UNSUPPORTED),     # NVFP4 with grouped heads
    ((1, 8, 0, 128, 128, 64, 0), api.SAGE_ERR_INVALID_ARG),
    ((1, 8, 2, 128, 0, 64, 0), api.SAGE_ERR_INVALID_ARG),
])
def test_gqa_shapes_rejected_on_host(lib, args, status):
    out = api.WsLayout()
    assert lib.sage_workspace_layout_gqa(*args, ctypes.byref(out)) == status


def test_gqa_layout_reduces_to_per_head_layout(lib):
    for (B, H, N, d, mode) in [(1, 4, 1000, 128, 0), (2, 3, 257, 64, 1), (1, 2, 512, 128, 2)]:
        a, b = api.sage_workspace_layout(B, H, N, d, mode), api.sage_workspace_layout_gqa(B, H, H, N, N, d, mode)
        assert all(getattr(a, f) == getattr(b, f) for f, _ in api.WsLayout._fields_)
    L = api.sage_workspace_layout_gqa(2, 8, 2, 100, 3000, 128, 0)
    assert L.k_codes - L.q_codes >= 2 * 8 * 128 * 128 and L.vt_codes - L.k_codes >= 2 * 2 * 3072 * 128


def test_gqa_causal_needs_nq_le_nk(lib):
    vp = ctypes.c_void_p
    ws = api.sage_workspace_layout_gqa(1, 4, 2, 300, 200, 64, 0).total
    st = lib.sage_attn_fwd_gqa(vp(4096), vp(4096), vp(4096), vp(4096), 1, 4, 2, 300, 200, 64, 1, 0, 0, 0, vp(4096), ws,
                               vp(0))
    assert st == api.SAGE_ERR_UNSUPPORTED


def test_blocksmooth_layout_holds_a_row_per_block(lib):
    """The per-block Q smoothing layout is the per-head one with q_mean and
    q_bias grown to one row per 128-row block; the NVFP4 mode is refused."""
    for (B, H, N, d, mode) in [(1, 2, 300, 128, 0), (2, 3, 8300, 64, 1), (1, 1, 1, 64, 0)]:
        a, b = api.sage_workspace_layout(B, H, N, d, mode), api.sage_workspace_layout_blocksmooth(B, H, N, d, mode)
        Np = (N + 127) // 128 * 128
        nb = Np // 128
        for f in ("q_codes", "k_codes", "vt_codes", "q_scale", "k_scale", "v_scale", "k_mean", "q_mean"):
            assert getattr(a, f) == getattr(b, f), f
        assert b.q_bias - b.q_mean >= B * H * nb * d * 4
        assert b.scratch - b.q_bias >= B * H * nb * Np * 4
        offs = [getattr(b, f) for f, _ in api.WsLayout._fields_ if f != "total"]
        assert all(o % 1024 == 0 for o in offs) and b.total > b.scratch
    out = api.WsLayout()
    assert lib.sage_workspace_layout_blocksmooth(1, 2, 300, 128, 2, ctypes.byref(out)) == api.SAGE_ERR_UNSUPPORTED
    vp = ctypes.c_void_p
    st = lib.sage_attn_fwd_blocksmooth(vp(4096), vp(4096), vp(4096), vp(4096), 1, 2, 300, 128, 0, 2, 0, vp(4096),
                                       1 << 30, vp(0))
    assert st == api.SAGE_ERR_UNSUPPORTED


def test_blocksmooth_bias_view_follows_the_key_tile_major_layout(lib):
    """The workspace stores block b's bias at key j at element
    ((bh * nkt + j // 128) * nblk + b) * 128 + j % 128; the binding's q_bias
    view reads it back as [bh, b, j]."""
    import torch
    B, H, N, d, mode = 1, 2, 300, 64, 0
    L = api.sage_workspace_layout_blocksmooth(B, H, N, d, mode)
    ws = torch.zeros(L.total, dtype=torch.uint8)
    BH, Np = B * H, (N + 127) // 128 * 128
    nb = Np // 128
    flat = ws[L.q_bias:L.q_bias + BH * nb * Np * 4].view(torch.float32)
    for bh in range(BH):
        for b in range(nb):
            for j in range(Np):
                flat[((bh * nb + j // 128) * nb + b) * 128 + j % 128] = bh * 1e6 + b * 1e4 + j
    v = api.ws_views_blocksmooth(ws, B, H, N, d, mode)["q_bias"]
    want = (torch.arange(BH)[:, None, None] * 1e6 + torch.arange(nb)[None, :, None] * 1e4
            + torch.arange(Np)[None, None, :]).float()
    assert torch.equal(v, want)
