"""CPU oracle for the SageAttention-family quantized attention forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA product path (``quantized_attention_sub_b200``) neither
imports it nor shares code with it.

The arithmetic lives in ``sage_oracle.c`` (plain scalar C, one function per step
of the method, each citing the passage it follows).  This module marshals numpy
arrays to it and adds the two pieces that are plain definitions rather than
emulations: the fp64 unquantized attention and the three accuracy metrics the
SageAttention2++ summary (App. A.2) uses to compare O' with O.

Every function takes and returns numpy arrays; inputs are the float32 values of
the fp16/bf16 tensors both sides consume.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "libsage_oracle.so")

# Quantization constants (SageAttention2++ summary, Sec. 3.1): Pr = 224 and
# Vr = 4.5 in the FP16-accumulator mode; the full e4m3 range 448 otherwise
# (the pages do not name a range for the FP32-accumulator mode).
E4M3_MAX = 448.0
PR_F16ACC, VR_F16ACC = 224.0, 4.5
PR_FP32ACC, VR_FP32ACC = 448.0, 448.0
Q_GRANULE, K_GRANULE, TILE = 32, 64, 128

MODE_INT8_FP8, MODE_INT8_FP8_F16ACC, MODE_NVFP4 = 0, 1, 2

_lib = None


def _compile(src: str, out: str) -> None:
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile sage_oracle.c into libsage_oracle.so (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        _compile(_SRC, _LIB)
    return _LIB


def build_variant(edits) -> str:
    """Compile a copy of sage_oracle.c with textual edits [(old, new), ...]
    applied (each `old` must occur exactly once) into a temporary library and
    return its path.  Used by the tests that plant a mistake in the oracle and
    check that a pin catches it; the product never calls it."""
    src = open(_SRC).read()
    for old, new in edits:
        n = src.count(old)
        if n != 1:
            raise ValueError("edit target found %d times: %r" % (n, old[:60]))
        src = src.replace(old, new)
    d = tempfile.mkdtemp(prefix="orc_variant_")
    path = os.path.join(d, "sage_oracle_variant.c")
    with open(path, "w") as f:
        f.write(src)
    out = os.path.join(d, "libsage_oracle_variant.so")
    _compile(path, out)
    return out


@contextlib.contextmanager
def using(path: str):
    """Run the wrappers of this module against another build of the oracle
    (a variant from build_variant) inside the `with` block."""
    global _lib
    saved = lib()
    _lib = _declare(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_int]
    L.orc_e4m3_encode.restype = ctypes.c_int
    L.orc_e4m3_encode.argtypes = [ctypes.c_double]
    L.orc_ue4m3_encode.restype = ctypes.c_int
    L.orc_ue4m3_encode.argtypes = [ctypes.c_double]
    L.orc_ue4m3_decode.restype = ctypes.c_double
    L.orc_ue4m3_decode.argtypes = [ctypes.c_int]
    L.orc_e2m1_encode.restype = ctypes.c_int
    L.orc_e2m1_encode.argtypes = [ctypes.c_double]
    L.orc_e2m1_decode.restype = ctypes.c_double
    L.orc_e2m1_decode.argtypes = [ctypes.c_int]
    L.orc_f16_round.restype = ctypes.c_double
    L.orc_f16_round.argtypes = [ctypes.c_double]
    L.orc_num_threads.restype = ctypes.c_int
    L.orc_exp2.restype = ctypes.c_float
    L.orc_exp2.argtypes = [ctypes.c_float]
    L.orc_nvfp4_block.restype = ctypes.c_int
    L.orc_nvfp4_block.argtypes = [ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p]
    return L


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def npad(N: int) -> int:
    return ((N + TILE - 1) // TILE) * TILE


# --------------------------------------------------------------------------
# Scalar encoders (exposed for the pins).
# --------------------------------------------------------------------------
def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(float(x))


def e4m3_decode(c: int) -> float:
    return lib().orc_e4m3_decode(int(c))


def ue4m3_encode(x: float) -> int:
    return lib().orc_ue4m3_encode(float(x))


def e2m1_encode(x: float) -> int:
    return lib().orc_e2m1_encode(float(x))


def e2m1_decode(c: int) -> float:
    return lib().orc_e2m1_decode(int(c))


def f16_round(x: float) -> float:
    return lib().orc_f16_round(float(x))


def exp2(d: float) -> float:
    """The softmax's exp2: the library exp2 in double, rounded to fp32."""
    return lib().orc_exp2(float(d))


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    tab = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return tab[np.asarray(codes, dtype=np.uint8)]


# --------------------------------------------------------------------------
# Quantization steps.
# --------------------------------------------------------------------------
def channel_mean(x: np.ndarray) -> np.ndarray:
    """x: [BH, N, d] float32 -> per-channel mean over tokens [BH, d] (fixed fp32 order)."""
    x = _f32(x)
    BH, N, d = x.shape
    out = np.empty((BH, d), np.float32)
    lib().orc_channel_mean(_p(x), BH, N, d, _p(out))
    return out


def channel_absmax(x: np.ndarray) -> np.ndarray:
    x = _f32(x)
    BH, N, d = x.shape
    out = np.empty((BH, d), np.float32)
    lib().orc_channel_absmax(_p(x), BH, N, d, _p(out))
    return out


def quant_int8(x: np.ndarray, mean: np.ndarray | None, G: int):
    """Smooth (if mean is given) and quantize to INT8 per G-token granule.
    Returns (codes [BH,Npad,d] int8, scale [BH,Npad/G] float32)."""
    x = _f32(x)
    BH, N, d = x.shape
    Np = npad(N)
    codes = np.empty((BH, Np, d), np.int8)
    scale = np.empty((BH, Np // G), np.float32)
    m = _f32(mean) if mean is not None else None
    lib().orc_quant_int8(_p(x), _p(m), BH, N, Np, d, G, _p(codes), _p(scale))
    return codes, scale


def q_bias(k: np.ndarray, mean_k: np.ndarray, mean_q: np.ndarray) -> np.ndarray:
    k = _f32(k)
    BH, N, d = k.shape
    Np = npad(N)
    out = np.empty((BH, Np), np.float32)
    lib().orc_q_bias(_p(k), _p(_f32(mean_k)), _p(_f32(mean_q)), BH, N, Np, d, _p(out))
    return out


def quant_v_fp8(v: np.ndarray, amax: np.ndarray, Vr: float):
    """Returns (vt codes [BH,d,Npad] uint8 e4m3, scale_v [BH,d] float32)."""
    v = _f32(v)
    BH, N, d = v.shape
    Np = npad(N)
    vt = np.empty((BH, d, Np), np.uint8)
    sv = np.empty((BH, d), np.float32)
    lib().orc_quant_v_fp8(_p(v), _p(_f32(amax)), BH, N, Np, d, ctypes.c_float(Vr), _p(vt), _p(sv))
    return vt, sv


def qk_s32(qc: np.ndarray, kc: np.ndarray) -> np.ndarray:
    """Exact int32 Q^ K^T of two code blocks [nq,d] x [nk,d]."""
    qc = np.ascontiguousarray(qc, np.int8)
    kc = np.ascontiguousarray(kc, np.int8)
    out = np.empty((qc.shape[0], kc.shape[0]), np.int32)
    lib().orc_qk_s32(_p(qc), _p(kc), qc.shape[0], kc.shape[0], qc.shape[1], _p(out))
    return out


def quantize_int8_fp8(q, k, v, smooth_q: bool, mode: int, Vr: float | None = None) -> dict:
    """The whole preprocessing of the INT8/FP8 modes for [BH, N, d] inputs:
    K smoothing, optional Q smoothing with its bias, INT8 Q/K, FP8 V (range
    Vr: the mode's default unless given)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    if Vr is None:
        Vr = VR_F16ACC if mode == MODE_INT8_FP8_F16ACC else VR_FP32ACC
    mean_k = channel_mean(k)
    mean_q = channel_mean(q) if smooth_q else None
    amax_v = channel_absmax(v)
    qc, sq = quant_int8(q, mean_q, Q_GRANULE)
    kc, sk = quant_int8(k, mean_k, K_GRANULE)
    bias = q_bias(k, mean_k, mean_q) if smooth_q else None
    vt, sv = quant_v_fp8(v, amax_v, Vr)
    return dict(q_codes=qc, q_scale=sq, k_codes=kc, k_scale=sk, vt_codes=vt, v_scale=sv,
                k_mean=mean_k, q_mean=mean_q, q_bias=bias, v_absmax=amax_v,
                N=q.shape[1], d=q.shape[2], mode=mode)


def attention_int8_fp8(qz: dict, causal: bool, rows=None, with_flip: bool = False, Pr: float | None = None,
                       chunk: int = 64):
    """Tiled online-softmax attention on quantized inputs.  rows: None (all)
    or an int array of query rows (same rows for every slice).
    Returns float32 [BH, nrows, d] before the cast to the output dtype; with
    `with_flip`, also the per-element change one P~ code moved to a
    neighbouring code would cause (a sensitivity figure for comparisons).
    Pr: the P~ range (the mode's default unless given); chunk: keys per FP16
    partial in the FP16-accumulator mode (64, or 32 without delayed
    buffering)."""
    qc, kc, vt = qz["q_codes"], qz["k_codes"], qz["vt_codes"]
    BH, Np, d = qc.shape
    N = qz["N"]
    mode = qz["mode"]
    if Pr is None:
        Pr = PR_F16ACC if mode == MODE_INT8_FP8_F16ACC else PR_FP32ACC
    if rows is None:
        r = None
        nrows = N
    else:
        r = np.ascontiguousarray(rows, np.int32)
        nrows = len(r)
    out = np.empty((BH, nrows, d), np.float32)
    flip = np.empty((BH, nrows, d), np.float32) if with_flip else None
    bias = qz["q_bias"]
    lib().orc_attn_int8_fp8(_p(qc), _p(qz["q_scale"]), _p(kc), _p(qz["k_scale"]), _p(vt),
                            _p(qz["v_scale"]), _p(bias), BH, N, Np, d, int(causal), int(mode), int(chunk),
                            ctypes.c_float(Pr), _p(r), nrows, _p(out), _p(flip))
    return (out, flip) if with_flip else out


Q_BLOCK = 128  # query rows per smoothing block (the attention's query tile)


def quantize_int8_fp8_blocksmooth(q, k, v, mode: int, Vr: float | None = None) -> dict:
    """Preprocessing with Q smoothed per block of 128 query rows instead of
    per slice (the pages say only that Q is smoothed, SageAttention2
    abstract): block b's mean is the channel mean of its valid rows (the
    per-slice mean's fixed order applied to the block), its rows are
    quantized in their 32-row granules after subtracting that mean, and its
    bias row is the per-slice bias formula with that mean, over every key.
    K, V and their statistics as in quantize_int8_fp8.  Returns the same
    dict with q_mean [BH, nblk, d] and q_bias [BH, nblk, Npad]."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, d = q.shape
    Np = npad(N)
    nblk = Np // Q_BLOCK
    if Vr is None:
        Vr = VR_F16ACC if mode == MODE_INT8_FP8_F16ACC else VR_FP32ACC
    mean_k = channel_mean(k)
    amax_v = channel_absmax(v)
    kc, sk = quant_int8(k, mean_k, K_GRANULE)
    vt, sv = quant_v_fp8(v, amax_v, Vr)
    qc = np.zeros((BH, Np, d), np.int8)
    sq = np.zeros((BH, Np // Q_GRANULE), np.float32)
    mean_q = np.empty((BH, nblk, d), np.float32)
    bias = np.empty((BH, nblk, Np), np.float32)
    for b in range(nblk):
        r0, r1 = b * Q_BLOCK, min(N, (b + 1) * Q_BLOCK)
        xb = np.ascontiguousarray(q[:, r0:r1])
        mb = channel_mean(xb)
        cb, sb = quant_int8(xb, mb, Q_GRANULE)
        qc[:, r0:r0 + Q_BLOCK] = cb
        sq[:, r0 // Q_GRANULE:(r0 + Q_BLOCK) // Q_GRANULE] = sb
        mean_q[:, b] = mb
        bias[:, b] = q_bias(k, mean_k, mb)
    return dict(q_codes=qc, q_scale=sq, k_codes=kc, k_scale=sk, vt_codes=vt, v_scale=sv,
                k_mean=mean_k, q_mean=mean_q, q_bias=bias, v_absmax=amax_v,
                N=N, d=d, mode=mode)


def attention_int8_fp8_blocksmooth(qz: dict, causal: bool, rows=None, with_flip: bool = False):
    """attention_int8_fp8 on quantize_int8_fp8_blocksmooth's output: each
    query row takes the bias row of its 128-row block.  Runs the per-slice
    attention once per block on that block's rows with that block's bias."""
    N, d = qz["N"], qz["d"]
    BH = qz["q_codes"].shape[0]
    all_rows = np.arange(N, dtype=np.int32) if rows is None else np.asarray(rows, np.int32)
    out = np.empty((BH, len(all_rows), d), np.float32)
    flip = np.empty((BH, len(all_rows), d), np.float32) if with_flip else None
    blocks = all_rows // Q_BLOCK
    for b in np.unique(blocks):
        sel = np.nonzero(blocks == b)[0]
        view = dict(qz, q_bias=np.ascontiguousarray(qz["q_bias"][:, b]))
        res = attention_int8_fp8(view, causal, rows=all_rows[sel], with_flip=with_flip)
        if with_flip:
            out[:, sel], flip[:, sel] = res
        else:
            out[:, sel] = res
    return (out, flip) if with_flip else out


def quantize_int8_fp8_gqa(q, k, v, smooth_q: bool, mode: int, Vr: float | None = None) -> dict:
    """Preprocessing with grouped key/value heads and separate lengths: q
    [B, Hq, Nq, d], k and v [B, Hkv, Nk, d].  Each tensor is smoothed and
    quantized per its own heads and tokens as in quantize_int8_fp8; the
    Q-smoothing bias of query head hq is mean_q(hq) . k~ over the keys of its
    key/value head hq / G, G = Hq / Hkv."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nk, _ = k.shape
    G = Hq // Hkv
    if Vr is None:
        Vr = VR_F16ACC if mode == MODE_INT8_FP8_F16ACC else VR_FP32ACC
    qf, kf, vf = q.reshape(B * Hq, Nq, d), k.reshape(B * Hkv, Nk, d), v.reshape(B * Hkv, Nk, d)
    mean_k = channel_mean(kf)
    mean_q = channel_mean(qf) if smooth_q else None
    qc, sq = quant_int8(qf, mean_q, Q_GRANULE)
    kc, sk = quant_int8(kf, mean_k, K_GRANULE)
    vt, sv = quant_v_fp8(vf, channel_absmax(vf), Vr)
    bias = None
    if smooth_q:
        # each query head against its key/value head's keys
        kx = np.repeat(kf.reshape(B, Hkv, Nk, d), G, axis=1).reshape(B * Hq, Nk, d)
        mkx = np.repeat(mean_k.reshape(B, Hkv, d), G, axis=1).reshape(B * Hq, d)
        bias = q_bias(kx, mkx, mean_q)
    return dict(q_codes=qc, q_scale=sq, k_codes=kc, k_scale=sk, vt_codes=vt, v_scale=sv, k_mean=mean_k,
                q_mean=mean_q, q_bias=bias, B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, mode=mode)


def attention_int8_fp8_gqa(qz: dict, causal: bool, rows=None, with_flip: bool = False, Pr: float | None = None,
                           chunk: int = 64):
    """Attention on quantize_int8_fp8_gqa's output: query head hq reads
    key/value head hq / G; causal rows see keys j <= i + (Nk - Nq).
    Returns float32 [B*Hq, nrows, d] (and the P~ sensitivity with with_flip)."""
    B, Hq, Hkv, Nq, Nk, d = qz["B"], qz["Hq"], qz["Hkv"], qz["Nq"], qz["Nk"], qz["d"]
    mode = qz["mode"]
    if Pr is None:
        Pr = PR_F16ACC if mode == MODE_INT8_FP8_F16ACC else PR_FP32ACC
    if rows is None:
        r, nrows = None, Nq
    else:
        r = np.ascontiguousarray(rows, np.int32)
        nrows = len(r)
    out = np.empty((B * Hq, nrows, d), np.float32)
    flip = np.empty((B * Hq, nrows, d), np.float32) if with_flip else None
    lib().orc_attn_int8_fp8_gqa(_p(qz["q_codes"]), _p(qz["q_scale"]), _p(qz["k_codes"]), _p(qz["k_scale"]),
                                _p(qz["vt_codes"]), _p(qz["v_scale"]), _p(qz["q_bias"]), B, Hq, Hkv, Nq, Nk,
                                npad(Nq), npad(Nk), d, int(causal), int(mode), int(chunk), ctypes.c_float(Pr),
                                _p(r), nrows, _p(out), _p(flip))
    return (out, flip) if with_flip else out


# --------------------------------------------------------------------------
# NVFP4 mode.
# --------------------------------------------------------------------------
def quantize_nvfp4(q, k, v, smooth_q: bool) -> dict:
    """NVFP4 preprocessing: K smoothed (and Q if smooth_q), blocks of 16 along
    d for Q/K and along tokens for V^T; ue4m3 block scales; fp32 global scale
    per slice.  Codes are returned unpacked (one e2m1 code per byte)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    BH, N, d = q.shape
    Np = npad(N)
    mean_k = channel_mean(k)
    mean_q = channel_mean(q) if smooth_q else None
    out = {}
    for name, x, mean in (("q", q, mean_q), ("k", k, mean_k)):
        codes = np.empty((BH, Np, d), np.uint8)
        bs = np.empty((BH, Np, d // 16), np.uint8)
        gs = np.empty((BH,), np.float32)
        lib().orc_quant_nvfp4_rows(_p(x), _p(_f32(mean) if mean is not None else None), BH, N, Np,
                                   d, _p(codes), _p(bs), _p(gs))
        out[name + "_codes"], out[name + "_bscale"], out[name + "_gscale"] = codes, bs, gs
    vc = np.empty((BH, d, Np), np.uint8)
    vbs = np.empty((BH, d, Np // 16), np.uint8)
    vg = np.empty((BH,), np.float32)
    lib().orc_quant_nvfp4_vt(_p(v), BH, N, Np, d, _p(vc), _p(vbs), _p(vg))
    out.update(vt_codes=vc, vt_bscale=vbs, v_gscale=vg, k_mean=mean_k, q_mean=mean_q,
               q_bias=q_bias(k, mean_k, mean_q) if smooth_q else None, N=N, d=d,
               mode=MODE_NVFP4)
    return out


def attention_nvfp4(qz: dict, causal: bool, rows=None, with_flip: bool = False):
    """NVFP4 attention (see attention_int8_fp8 for rows and with_flip)."""
    BH, Np, d = qz["q_codes"].shape
    N = qz["N"]
    if rows is None:
        r, nrows = None, N
    else:
        r = np.ascontiguousarray(rows, np.int32)
        nrows = len(r)
    out = np.empty((BH, nrows, d), np.float32)
    flip = np.empty((BH, nrows, d), np.float32) if with_flip else None
    lib().orc_attn_nvfp4(_p(qz["q_codes"]), _p(qz["q_bscale"]), _p(qz["q_gscale"]),
                         _p(qz["k_codes"]), _p(qz["k_bscale"]), _p(qz["k_gscale"]),
                         _p(qz["vt_codes"]), _p(qz["vt_bscale"]), _p(qz["v_gscale"]),
                         _p(qz["q_bias"]), BH, N, Np, d, int(causal), _p(r), nrows, _p(out), _p(flip))
    return (out, flip) if with_flip else out


def nvfp4_block(x, g: float):
    """The NVFP4 block quantizer on 16 values with global scale g: returns
    (ue4m3 scale code, 16 e2m1 codes)."""
    x = _f32(np.asarray(x).reshape(16))
    codes = np.empty(16, np.uint8)
    bs = lib().orc_nvfp4_block(_p(x), ctypes.c_float(g), _p(codes))
    return bs, codes


# --------------------------------------------------------------------------
# Plain definitions: unquantized attention and the accuracy metrics.
# --------------------------------------------------------------------------
def attention_fp64(q, k, v, causal: bool, rows=None) -> np.ndarray:
    """softmax(Q K^T / sqrt(d)) V in float64.  q [BH, Nq, d], k and v
    [BH, Nk, d] (Nq may differ from Nk; a causal row i sees keys
    j <= i + Nk - Nq)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    BH, Nq, d = q.shape
    Nk = k.shape[1]
    idx = np.arange(Nq) if rows is None else np.asarray(rows)
    out = np.empty((BH, len(idx), d), np.float64)
    for bh in range(BH):
        s = q[bh, idx] @ k[bh].T / np.sqrt(d)
        if causal:
            s = np.where(np.arange(Nk)[None, :] <= idx[:, None] + (Nk - Nq), s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[bh] = (p / p.sum(axis=1, keepdims=True)) @ v[bh]
    return out


def accuracy(o_test, o_ref) -> dict:
    """Cosine similarity, relative L1 and RMSE of O' against O (SageAttention2++
    summary, App. A.2)."""
    a = np.asarray(o_test, np.float64).ravel()
    b = np.asarray(o_ref, np.float64).ravel()
    cos = float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))
    rel_l1 = float(np.abs(a - b).sum() / np.abs(b).sum())
    rmse = float(np.sqrt(np.mean((a - b) ** 2)))
    return dict(cos=cos, rel_l1=rel_l1, rmse=rmse)
