"""Thin Python binding of libsage.so (include/sage.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
passes torch tensors' device pointers and the current CUDA stream through
ctypes.  There is no fallback: if the library is missing, or a call returns a
non-OK status, a RuntimeError is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsage.so")

SAGE_OK, SAGE_ERR_INVALID_ARG, SAGE_ERR_UNSUPPORTED, SAGE_ERR_CUDA, SAGE_ERR_TIMEOUT = range(5)
MODE_INT8_FP8, MODE_INT8_FP8_F16ACC, MODE_NVFP4 = 0, 1, 2
DTYPE_CODE = {torch.float16: 0, torch.bfloat16: 1}

EXPORTED = ("sage_workspace_layout", "sage_workspace_size", "sage_quantize_qkv", "sage_quantize_qkv_static",
            "sage_attn_quantized",
            "sage_attn_fwd", "sage_attn_fwd_fused", "sage_attn_fwd_ranges", "sage_workspace_layout_gqa", "sage_quantize_qkv_gqa",
            "sage_attn_quantized_gqa", "sage_attn_fwd_gqa", "sage_workspace_layout_blocksmooth",
            "sage_quantize_qkv_blocksmooth", "sage_attn_quantized_blocksmooth", "sage_attn_fwd_blocksmooth",
            "sage_debug_qk_s32", "sage_debug_fp4_s", "sage_debug_timeout_probe", "sage_probe_mma_rate",
            "sage_check", "sage_last_error")
PROBE_I8, PROBE_F8_F32ACC, PROBE_F8_F16ACC, PROBE_BF16, PROBE_FP4 = range(5)


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("q_codes", "k_codes", "vt_codes", "q_scale", "k_scale", "v_scale",
                                               "k_mean", "q_mean", "q_bias", "global_scale", "error", "scratch",
                                               "total")]


class SageError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("sage status %d: %s" % (status, message))
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsage.so (built in-tree by quantized_attention_sub_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libsage.so is not built (run __graft_entry__.build() or "
                               "python -m quantized_attention_sub_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        i, sz, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        L.sage_workspace_layout.argtypes = [i, i, i, i, i, ctypes.POINTER(WsLayout)]
        L.sage_workspace_layout.restype = i
        L.sage_workspace_size.argtypes = [i, i, i, i, i]
        L.sage_workspace_size.restype = sz
        L.sage_quantize_qkv.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_quantize_qkv.restype = i
        L.sage_quantize_qkv_static.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_quantize_qkv_static.restype = i
        L.sage_attn_quantized.argtypes = [vp, sz, vp, i, i, i, i, i, i, i, i, vp]
        L.sage_attn_quantized.restype = i
        L.sage_attn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_attn_fwd.restype = i
        L.sage_attn_fwd_fused.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_attn_fwd_fused.restype = i
        f = ctypes.c_float
        L.sage_attn_fwd_ranges.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, f, vp, sz, vp]
        L.sage_attn_fwd_ranges.restype = i
        L.sage_workspace_layout_gqa.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(WsLayout)]
        L.sage_workspace_layout_gqa.restype = i
        L.sage_quantize_qkv_gqa.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_quantize_qkv_gqa.restype = i
        L.sage_attn_quantized_gqa.argtypes = [vp, sz, vp, i, i, i, i, i, i, i, i, i, i, vp]
        L.sage_attn_quantized_gqa.restype = i
        L.sage_attn_fwd_gqa.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_attn_fwd_gqa.restype = i
        L.sage_workspace_layout_blocksmooth.argtypes = [i, i, i, i, i, ctypes.POINTER(WsLayout)]
        L.sage_workspace_layout_blocksmooth.restype = i
        L.sage_quantize_qkv_blocksmooth.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]
        L.sage_quantize_qkv_blocksmooth.restype = i
        L.sage_attn_quantized_blocksmooth.argtypes = [vp, sz, vp, i, i, i, i, i, i, i, vp]
        L.sage_attn_quantized_blocksmooth.restype = i
        L.sage_attn_fwd_blocksmooth.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        L.sage_attn_fwd_blocksmooth.restype = i
        L.sage_debug_qk_s32.argtypes = [vp, sz, i, i, i, i, i, i, i, vp, vp]
        L.sage_debug_qk_s32.restype = i
        L.sage_debug_fp4_s.argtypes = [vp, sz, i, i, i, i, i, i, i, vp, vp]
        L.sage_debug_fp4_s.restype = i
        L.sage_debug_timeout_probe.argtypes = [vp, sz, vp]
        L.sage_debug_timeout_probe.restype = i
        L.sage_probe_mma_rate.argtypes = [i, i, i, vp, sz, ctypes.POINTER(ctypes.c_double), vp]
        L.sage_probe_mma_rate.restype = i
        L.sage_check.argtypes = [vp, sz, vp]
        L.sage_check.restype = i
        L.sage_last_error.argtypes = []
        L.sage_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _raise(st):
    if st != SAGE_OK:
        raise SageError(st, lib().sage_last_error().decode())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


# ------------------------------------------------------------------ C names
def sage_workspace_layout(B, H, N, d, mode) -> WsLayout:
    out = WsLayout()
    _raise(lib().sage_workspace_layout(B, H, N, d, mode, ctypes.byref(out)))
    return out


def sage_workspace_size(B, H, N, d, mode) -> int:
    return lib().sage_workspace_size(B, H, N, d, mode)


def sage_quantize_qkv(q, k, v, dtype, B, H, N, d, smooth_q, mode, ws, ws_bytes, stream=None):
    _raise(lib().sage_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, N, d, int(smooth_q), mode, _ptr(ws),
                                   ws_bytes, _stream(stream)))


def sage_quantize_qkv_static(q, k, v, dtype, B, H, N, d, smooth_q, mode, out, out_bytes, stream=None):
    """No-allocation quantization (see include/sage.h): `out` receives the
    quantized region of the workspace layout; the statistics scratch lives in
    a fixed 16 MiB device array inside the library."""
    _raise(lib().sage_quantize_qkv_static(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, N, d, int(smooth_q), mode,
                                          _ptr(out), out_bytes, _stream(stream)))


def sage_attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, smooth_q, mode, stream=None):
    _raise(lib().sage_attn_quantized(_ptr(ws), ws_bytes, _ptr(out), dtype, B, H, N, d, int(causal), int(smooth_q),
                                     mode, _stream(stream)))


def sage_attn_fwd(q, k, v, out, B, H, N, d, causal, mode, dtype, smooth_q, ws, ws_bytes, stream=None):
    _raise(lib().sage_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, int(causal), mode, dtype,
                               int(smooth_q), _ptr(ws), ws_bytes, _stream(stream)))


def sage_attn_fwd_fused(q, k, v, out, B, H, N, d, causal, mode, dtype, smooth_q, ws, ws_bytes, stream=None):
    _raise(lib().sage_attn_fwd_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, int(causal), mode, dtype,
                                     int(smooth_q), _ptr(ws), ws_bytes, _stream(stream)))


def sage_attn_fwd_ranges(q, k, v, out, B, H, N, d, causal, mode, dtype, smooth_q, Pr, Vr, ws, ws_bytes,
                         stream=None):
    _raise(lib().sage_attn_fwd_ranges(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, int(causal), mode, dtype,
                                      int(smooth_q), float(Pr), float(Vr), _ptr(ws), ws_bytes, _stream(stream)))


def sage_workspace_layout_gqa(B, Hq, Hkv, Nq, Nk, d, mode) -> WsLayout:
    out = WsLayout()
    _raise(lib().sage_workspace_layout_gqa(B, Hq, Hkv, Nq, Nk, d, mode, ctypes.byref(out)))
    return out


def sage_quantize_qkv_gqa(q, k, v, dtype, B, Hq, Hkv, Nq, Nk, d, smooth_q, mode, ws, ws_bytes, stream=None):
    _raise(lib().sage_quantize_qkv_gqa(_ptr(q), _ptr(k), _ptr(v), dtype, B, Hq, Hkv, Nq, Nk, d, int(smooth_q), mode,
                                       _ptr(ws), ws_bytes, _stream(stream)))


def sage_attn_quantized_gqa(ws, ws_bytes, out, dtype, B, Hq, Hkv, Nq, Nk, d, causal, smooth_q, mode, stream=None):
    _raise(lib().sage_attn_quantized_gqa(_ptr(ws), ws_bytes, _ptr(out), dtype, B, Hq, Hkv, Nq, Nk, d, int(causal),
                                         int(smooth_q), mode, _stream(stream)))


def sage_attn_fwd_gqa(q, k, v, out, B, Hq, Hkv, Nq, Nk, d, causal, mode, dtype, smooth_q, ws, ws_bytes, stream=None):
    _raise(lib().sage_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, Nq, Nk, d, int(causal), mode,
                                   dtype, int(smooth_q), _ptr(ws), ws_bytes, _stream(stream)))


def alloc_workspace_gqa(B, Hq, Hkv, Nq, Nk, d, mode, device="cuda") -> torch.Tensor:
    """Device workspace for the grouped-head / separate-length calls (1024-byte aligned)."""
    n = sage_workspace_layout_gqa(B, Hq, Hkv, Nq, Nk, d, mode).total
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + n]


def ws_views_gqa(ws: torch.Tensor, B, Hq, Hkv, Nq, Nk, d, mode) -> dict:
    """Typed views of the quantized buffers of a grouped-head workspace (INT8/FP8)."""
    L = sage_workspace_layout_gqa(B, Hq, Hkv, Nq, Nk, d, mode)
    BHq, BHk = B * Hq, B * Hkv
    Npq, Npk = (Nq + 127) // 128 * 128, (Nk + 127) // 128 * 128

    def view(off, nbytes, dtype, shape):
        return ws[off:off + nbytes].view(dtype).view(*shape)

    return dict(
        q_codes=view(L.q_codes, BHq * Npq * d, torch.int8, (BHq, Npq, d)),
        k_codes=view(L.k_codes, BHk * Npk * d, torch.int8, (BHk, Npk, d)),
        vt_codes=view(L.vt_codes, BHk * d * Npk, torch.uint8, (BHk, d, Npk)),
        q_scale=view(L.q_scale, BHq * (Npq // 32) * 4, torch.float32, (BHq, Npq // 32)),
        k_scale=view(L.k_scale, BHk * (Npk // 64) * 4, torch.float32, (BHk, Npk // 64)),
        v_scale=view(L.v_scale, BHk * d * 4, torch.float32, (BHk, d)),
        k_mean=view(L.k_mean, BHk * d * 4, torch.float32, (BHk, d)),
        q_mean=view(L.q_mean, BHq * d * 4, torch.float32, (BHq, d)),
        q_bias=view(L.q_bias, BHq * Npk * 4, torch.float32, (BHq, Npk)),
    )


def sage_workspace_layout_blocksmooth(B, H, N, d, mode) -> WsLayout:
    out = WsLayout()
    _raise(lib().sage_workspace_layout_blocksmooth(B, H, N, d, mode, ctypes.byref(out)))
    return out


def sage_quantize_qkv_blocksmooth(q, k, v, dtype, B, H, N, d, mode, ws, ws_bytes, stream=None):
    _raise(lib().sage_quantize_qkv_blocksmooth(_ptr(q), _ptr(k), _ptr(v), dtype, B, H, N, d, mode, _ptr(ws), ws_bytes,
                                               _stream(stream)))


def sage_attn_quantized_blocksmooth(ws, ws_bytes, out, dtype, B, H, N, d, causal, mode, stream=None):
    _raise(lib().sage_attn_quantized_blocksmooth(_ptr(ws), ws_bytes, _ptr(out), dtype, B, H, N, d, int(causal), mode,
                                                 _stream(stream)))


def sage_attn_fwd_blocksmooth(q, k, v, out, B, H, N, d, causal, mode, dtype, ws, ws_bytes, stream=None):
    _raise(lib().sage_attn_fwd_blocksmooth(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, int(causal), mode, dtype,
                                           _ptr(ws), ws_bytes, _stream(stream)))


def alloc_workspace_blocksmooth(B, H, N, d, mode, device="cuda") -> torch.Tensor:
    """Device workspace for the per-block Q smoothing calls (1024-byte aligned)."""
    n = sage_workspace_layout_blocksmooth(B, H, N, d, mode).total
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + n]


def ws_views_blocksmooth(ws: torch.Tensor, B, H, N, d, mode) -> dict:
    """Typed views of a per-block Q smoothing workspace: the per-head buffers
    with q_mean [BH, Npad/128, d], and q_bias as [BH, Npad/128 blocks, Npad]
    (a copy: the workspace stores the rows key-tile-major, [BH][key tile]
    [block][128])."""
    L = sage_workspace_layout_blocksmooth(B, H, N, d, mode)
    BH, Np = B * H, (N + 127) // 128 * 128
    nb = Np // 128

    def view(off, nbytes, dtype, shape):
        return ws[off:off + nbytes].view(dtype).view(*shape)

    return dict(
        q_codes=view(L.q_codes, BH * Np * d, torch.int8, (BH, Np, d)),
        k_codes=view(L.k_codes, BH * Np * d, torch.int8, (BH, Np, d)),
        vt_codes=view(L.vt_codes, BH * d * Np, torch.uint8, (BH, d, Np)),
        q_scale=view(L.q_scale, BH * (Np // 32) * 4, torch.float32, (BH, Np // 32)),
        k_scale=view(L.k_scale, BH * (Np // 64) * 4, torch.float32, (BH, Np // 64)),
        v_scale=view(L.v_scale, BH * d * 4, torch.float32, (BH, d)),
        k_mean=view(L.k_mean, BH * d * 4, torch.float32, (BH, d)),
        q_mean=view(L.q_mean, BH * nb * d * 4, torch.float32, (BH, nb, d)),
        q_bias=view(L.q_bias, BH * nb * Np * 4, torch.float32, (BH, nb, nb, 128)).permute(0, 2, 1, 3)
        .reshape(BH, nb, Np),
    )


def sage_debug_qk_s32(ws, ws_bytes, B, H, N, d, bh, q_tile, k_tile, out, stream=None):
    _raise(lib().sage_debug_qk_s32(_ptr(ws), ws_bytes, B, H, N, d, bh, q_tile, k_tile, _ptr(out), _stream(stream)))


def sage_debug_fp4_s(ws, ws_bytes, B, H, N, d, bh, q_tile, k_tile, out, stream=None):
    _raise(lib().sage_debug_fp4_s(_ptr(ws), ws_bytes, B, H, N, d, bh, q_tile, k_tile, _ptr(out), _stream(stream)))


def sage_debug_timeout_probe(ws, ws_bytes, stream=None):
    _raise(lib().sage_debug_timeout_probe(_ptr(ws), ws_bytes, _stream(stream)))


def sage_probe_mma_rate(kind, ctas, iters, ws, ws_bytes, stream=None) -> float:
    """Launch the tensor-core rate probe; returns the operation count of the
    launch (the caller times it with events on the same stream)."""
    ops = ctypes.c_double(0.0)
    _raise(lib().sage_probe_mma_rate(kind, ctas, iters, _ptr(ws), ws_bytes, ctypes.byref(ops), _stream(stream)))
    return ops.value


def sage_check(ws, ws_bytes, stream=None):
    _raise(lib().sage_check(_ptr(ws), ws_bytes, _stream(stream)))


# ------------------------------------------------------------------ torch helpers
def alloc_workspace(B, H, N, d, mode, device="cuda") -> torch.Tensor:
    """A device byte tensor big enough for the problem (torch's allocator
    returns blocks aligned to at least 512 bytes; the library needs 1024, so
    one extra KiB is taken and the view is offset)."""
    n = sage_workspace_size(B, H, N, d, mode)
    if n == 0:
        _raise(lib().sage_workspace_layout(B, H, N, d, mode, ctypes.byref(WsLayout())))
    raw = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-raw.data_ptr()) % 1024
    return raw[off:off + n]


def ws_views(ws: torch.Tensor, B, H, N, d, mode) -> dict:
    """Typed views of the quantized buffers inside a workspace.  NVFP4: packed
    codes as bytes and the block scales as raw 512-byte atoms (the layout the
    tensor cores read; include/sage.h gives the indexing)."""
    L = sage_workspace_layout(B, H, N, d, mode)
    BH, Np = B * H, (N + 127) // 128 * 128

    def view(off, nbytes, dtype, shape):
        return ws[off:off + nbytes].view(dtype).view(*shape)

    if mode == MODE_NVFP4:
        return dict(
            q_codes=view(L.q_codes, BH * Np * d // 2, torch.uint8, (BH, Np, d // 2)),
            k_codes=view(L.k_codes, BH * Np * d // 2, torch.uint8, (BH, Np, d // 2)),
            vt_codes=view(L.vt_codes, BH * d * Np // 2, torch.uint8, (BH, d, Np // 2)),
            q_sf_atoms=view(L.q_scale, BH * Np * d // 16, torch.uint8, (BH, Np // 128, d // 64, 512)),
            k_sf_atoms=view(L.k_scale, BH * Np * d // 16, torch.uint8, (BH, Np // 128, d // 64, 512)),
            v_sf_atoms=view(L.v_scale, BH * Np * 8, torch.uint8, (BH, Np // 128, 2, 512)),
            global_scale=view(L.global_scale, BH * 16, torch.float32, (BH, 4)),
            k_mean=view(L.k_mean, BH * d * 4, torch.float32, (BH, d)),
            q_mean=view(L.q_mean, BH * d * 4, torch.float32, (BH, d)),
            q_bias=view(L.q_bias, BH * Np * 4, torch.float32, (BH, Np)),
        )
    return dict(
        q_codes=view(L.q_codes, BH * Np * d, torch.int8, (BH, Np, d)),
        k_codes=view(L.k_codes, BH * Np * d, torch.int8, (BH, Np, d)),
        vt_codes=view(L.vt_codes, BH * d * Np, torch.uint8, (BH, d, Np)),
        q_scale=view(L.q_scale, BH * (Np // 32) * 4, torch.float32, (BH, Np // 32)),
        k_scale=view(L.k_scale, BH * (Np // 64) * 4, torch.float32, (BH, Np // 64)),
        v_scale=view(L.v_scale, BH * d * 4, torch.float32, (BH, d)),
        k_mean=view(L.k_mean, BH * d * 4, torch.float32, (BH, d)),
        q_mean=view(L.q_mean, BH * d * 4, torch.float32, (BH, d)),
        q_bias=view(L.q_bias, BH * Np * 4, torch.float32, (BH, Np)),
    )


def attn_fwd(q, k, v, causal=False, mode=MODE_INT8_FP8, smooth_q=False, out=None, ws=None, stream=None):
    """Quantized attention of [B,H,N,d] fp16/bf16 CUDA tensors (one library call)."""
    B, H, N, d = q.shape
    for t in (q, k, v):
        if not (t.is_cuda and t.is_contiguous() and t.shape == q.shape and t.dtype == q.dtype):
            raise ValueError("q, k, v must be contiguous CUDA tensors of one shape and dtype")
    if q.dtype not in DTYPE_CODE:
        raise ValueError("dtype must be float16 or bfloat16")
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = alloc_workspace(B, H, N, d, mode, q.device)
    sage_attn_fwd(q, k, v, out, B, H, N, d, causal, mode, DTYPE_CODE[q.dtype], smooth_q, ws, ws.numel(), stream)
    return out
