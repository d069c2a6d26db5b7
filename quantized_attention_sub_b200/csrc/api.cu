// api.cu -- the C ABI of libsage.so (declared in include/sage.h): argument
// checks, workspace layout, tensor-map encoding and kernel launches.
#include <stdio.h>
#include <string.h>

#include <string>

#include "../../include/sage.h"
#include "sage_internal.h"

namespace {

thread_local std::string g_last_error;

sage_status set_err(sage_status st, const char* fmt, const char* detail = "") {
  char buf[512];
  snprintf(buf, sizeof(buf), fmt, detail);
  g_last_error = buf;
  return st;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kAlign = 1024;

sage_status check_shape(int B, int H, int N, int d, int mode) {
  if (B < 1 || H < 1 || N < 1) return set_err(SAGE_ERR_INVALID_ARG, "B, H and N must be >= 1%s");
  if (d != 64 && d != 128) return set_err(SAGE_ERR_UNSUPPORTED, "head dimension must be 64 or 128%s");
  if (mode != SAGE_MODE_INT8_FP8 && mode != SAGE_MODE_INT8_FP8_F16ACC && mode != SAGE_MODE_NVFP4)
    return set_err(SAGE_ERR_INVALID_ARG, "unknown mode%s");
  const long long npad = ((long long)N + 127) / 128 * 128;
  if ((long long)B * H * npad * d >= (1LL << 31) || (long long)B * H > 65535)
    return set_err(SAGE_ERR_UNSUPPORTED, "problem too large (B*H*Npad*d must be < 2^31, B*H <= 65535)%s");
  return SAGE_OK;
}

// Grouped key/value heads (Hq query heads per batch, Hkv key/value heads,
// Hq % Hkv == 0) and separate query / key lengths.  INT8/FP8 modes only
// unless the shapes coincide (then the per-head checks and layout apply).
sage_status check_shape_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mode) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1)
    return set_err(SAGE_ERR_INVALID_ARG, "B, Hq, Hkv, Nq and Nk must be >= 1%s");
  if (Hq % Hkv) return set_err(SAGE_ERR_INVALID_ARG, "Hq must be a multiple of Hkv%s");
  sage_status st = check_shape(B, Hq, Nq, d, mode);
  if (st != SAGE_OK) return st;
  if ((st = check_shape(B, Hkv, Nk, d, mode)) != SAGE_OK) return st;
  if (mode == SAGE_MODE_NVFP4 && (Hq != Hkv || Nq != Nk))
    return set_err(SAGE_ERR_UNSUPPORTED, "the NVFP4 mode needs Hq == Hkv and Nq == Nk%s");
  const long long npk = ((long long)Nk + 127) / 128 * 128;
  if ((long long)B * Hq * npk >= (1LL << 31))
    return set_err(SAGE_ERR_UNSUPPORTED, "problem too large (B*Hq*Npad_k must be < 2^31)%s");
  return SAGE_OK;
}

// q_blocks: Q smoothed per 128-row block (per-head shapes): q_mean and q_bias
// hold one row per block instead of one per slice.
sage_ws_layout layout_of_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mode, bool q_blocks = false);

sage_ws_layout layout_of(int B, int H, int N, int d, int mode, bool q_blocks = false) {
  return layout_of_gqa(B, H, H, N, N, d, mode, q_blocks);
}

sage_ws_layout layout_of_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mode, bool q_blocks) {
  sage_ws_layout L;
  memset(&L, 0, sizeof(L));
  const bool split = Hq != Hkv || Nq != Nk;
  const size_t BH = (size_t)B * Hq, Np = ((size_t)Nq + 127) / 128 * 128;
  const size_t BHk = (size_t)B * Hkv, Npk = ((size_t)Nk + 127) / 128 * 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.error = take(sizeof(int));
  if (mode == SAGE_MODE_NVFP4) {
    L.q_codes = take(BH * Np * d / 2);
    L.k_codes = take(BH * Np * d / 2);
    L.vt_codes = take(BH * d * Np / 2);
    L.q_scale = take(BH * Np * d / 16);
    L.k_scale = take(BH * Np * d / 16);
    L.v_scale = take(BH * Np * 8);  // two 128-channel scale atoms per 128 tokens
    L.global_scale = take(BH * 4 * sizeof(float));
  } else {
    L.q_codes = take(BH * Np * d);
    L.k_codes = take(BHk * Npk * d);
    L.vt_codes = take(BHk * d * Npk);
    L.q_scale = take(BH * (Np / 32) * sizeof(float));
    L.k_scale = take(BHk * (Npk / 64) * sizeof(float));
    L.v_scale = take(BHk * d * sizeof(float));
    L.global_scale = take(0);
  }
  L.k_mean = take(BHk * d * sizeof(float));
  const size_t qrows = q_blocks ? Np / 128 : 1;  // mean and bias rows per slice
  L.q_mean = take(BH * qrows * d * sizeof(float));
  L.q_bias = take(BH * qrows * Npk * sizeof(float));
  // statistics partials and V multipliers of the quantize pass
  L.scratch = take((split ? sage::quant_scratch_floats_split((int)BH, (int)Np, (int)BHk, (int)Npk, d)
                          : sage::quant_scratch_floats((int)BH, (int)Np, d, mode)) *
                   sizeof(float));
  L.total = off;
  return L;
}

sage::WsPtrs resolve(void* ws, const sage_ws_layout& L) {
  char* b = (char*)ws;
  sage::WsPtrs w;
  w.q_codes = (int8_t*)(b + L.q_codes);
  w.k_codes = (int8_t*)(b + L.k_codes);
  w.vt_codes = (uint8_t*)(b + L.vt_codes);
  w.q_scale = (float*)(b + L.q_scale);
  w.k_scale = (float*)(b + L.k_scale);
  w.v_scale = (float*)(b + L.v_scale);
  w.k_mean = (float*)(b + L.k_mean);
  w.q_mean = (float*)(b + L.q_mean);
  w.q_bias = (float*)(b + L.q_bias);
  w.global_scale = (float*)(b + L.global_scale);
  w.error = (int*)(b + L.error);
  w.scratch = (float*)(b + L.scratch);
  return w;
}

// `need`: bytes the call touches -- L.total for the quantization pass (it
// writes the statistics scratch), L.scratch for the calls that only read the
// quantized region below it (attention, the debug tiles).
sage_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return set_err(SAGE_ERR_INVALID_ARG, "workspace pointer is null%s");
  if (((uintptr_t)ws) % kAlign) return set_err(SAGE_ERR_INVALID_ARG, "workspace must be 1024-byte aligned%s");
  if (ws_bytes < need) return set_err(SAGE_ERR_INVALID_ARG, "workspace too small%s");
  return SAGE_OK;
}

sage_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SAGE_OK;
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
  g_last_error = buf;
  return SAGE_ERR_CUDA;
}

}  // namespace

namespace sage {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  // initialized once, thread-safely (C++11 static initialization)
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return (EncodeTiledFn)p;
    return nullptr;
  }();
  return fn;
}

bool make_tmap_u8_3d(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                     uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0, dim0 * dim1};  // bytes, dims 1 and 2
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMapSwizzle sw = box0 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8_nd(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                     const uint32_t* box, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 2 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sage

extern "C" {

const char* sage_last_error(void) { return g_last_error.c_str(); }

sage_status sage_workspace_layout(int B, int H, int N, int d, int mode, sage_ws_layout* out) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "layout pointer is null%s");
  *out = layout_of(B, H, N, d, mode);
  return SAGE_OK;
}

size_t sage_workspace_size(int B, int H, int N, int d, int mode) {
  if (check_shape(B, H, N, d, mode) != SAGE_OK) return 0;
  return layout_of(B, H, N, d, mode).total;
}

// Default quantization ranges of a mode (SageAttention2++ summary, Sec. 3.1:
// Pr = 224 and Vr = 4.5 with the FP16 accumulator; the full e4m3 range 448
// with the FP32 one).
static float default_vr(int mode) { return mode == SAGE_MODE_INT8_FP8_F16ACC ? 4.5f : 448.0f; }
static float default_pr(int mode) { return mode == SAGE_MODE_INT8_FP8_F16ACC ? 224.0f : 448.0f; }

static sage_status quantize(const void* q, const void* k, const void* v, int dtype, int B, int H, int N, int d,
                            int smooth_q, int mode, float Vr, void* ws, size_t ws_bytes, sage_stream_t stream,
                            bool q_blocks = false);
static sage_status attn_quantized(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int H, int N, int d,
                                  int causal, int smooth_q, int mode, float Pr, sage_stream_t stream,
                                  bool after_quantize, bool q_blocks = false);

sage_status sage_quantize_qkv(const void* q, const void* k, const void* v, int dtype, int B, int H, int N, int d,
                              int smooth_q, int mode, void* ws, size_t ws_bytes, sage_stream_t stream) {
  return quantize(q, k, v, dtype, B, H, N, d, smooth_q, mode, default_vr(mode), ws, ws_bytes, stream);
}

static sage_status quantize(const void* q, const void* k, const void* v, int dtype, int B, int H, int N, int d,
                            int smooth_q, int mode, float Vr, void* ws, size_t ws_bytes, sage_stream_t stream,
                            bool q_blocks) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (!q || !k || !v) return set_err(SAGE_ERR_INVALID_ARG, "null input pointer%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  if ((((uintptr_t)q) | ((uintptr_t)k) | ((uintptr_t)v)) % 16)
    return set_err(SAGE_ERR_INVALID_ARG, "inputs must be 16-byte aligned%s");
  const sage_ws_layout L = layout_of(B, H, N, d, mode, q_blocks);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SAGE_OK) return st;
  sage::Problem pb{B * H, N, (N + 127) / 128 * 128, d, dtype, smooth_q ? 1 : 0, mode, 0};
  pb.q_blocks = q_blocks ? 1 : 0;
  if ((st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_quant_int8_fp8(q, k, v, pb, Vr, resolve(ws, L), (cudaStream_t)stream),
                     "quantize launch");
}

sage_status sage_quantize_qkv_static(const void* q, const void* k, const void* v, int dtype, int B, int H, int N,
                                     int d, int smooth_q, int mode, void* out, size_t out_bytes,
                                     sage_stream_t stream) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (!q || !k || !v) return set_err(SAGE_ERR_INVALID_ARG, "null input pointer%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  if ((((uintptr_t)q) | ((uintptr_t)k) | ((uintptr_t)v)) % 16)
    return set_err(SAGE_ERR_INVALID_ARG, "inputs must be 16-byte aligned%s");
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "output buffer pointer is null%s");
  if (((uintptr_t)out) % kAlign) return set_err(SAGE_ERR_INVALID_ARG, "output buffer must be 1024-byte aligned%s");
  const sage_ws_layout L = layout_of(B, H, N, d, mode);
  if (out_bytes < L.scratch)
    return set_err(SAGE_ERR_INVALID_ARG, "output buffer smaller than the layout's quantized region (layout.scratch)%s");
  const size_t Np = ((size_t)N + 127) / 128 * 128, BH = (size_t)B * H;
  const size_t need = sage::quant_scratch_floats((int)BH, (int)Np, d, mode);
  if (need > sage::static_scratch_floats()) {
    char buf[200];
    snprintf(buf, sizeof(buf), "problem needs %zu floats of static scratch; the maximum is %zu (16 MiB)", need,
             sage::static_scratch_floats());
    g_last_error = buf;
    return SAGE_ERR_UNSUPPORTED;
  }
  sage::Problem pb{B * H, N, (int)Np, d, dtype, smooth_q ? 1 : 0, mode, 0};
  const float Vr = default_vr(mode);
  if ((st = cuda_status(cudaMemsetAsync((char*)out + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_quant_static(q, k, v, pb, Vr, resolve(out, L), (cudaStream_t)stream),
                     "static quantize launch");
}

// The attention launch behind sage_attn_quantized and sage_attn_fwd.  After
// sage_quantize_qkv on the same stream (sage_attn_fwd) the workspace error
// word is already clear; called on its own it clears it first.
static sage_status attn_quantized(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int H, int N, int d,
                                  int causal, int smooth_q, int mode, float Pr, sage_stream_t stream,
                                  bool after_quantize, bool q_blocks) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "null output pointer%s");
  if (((uintptr_t)out) % 16) return set_err(SAGE_ERR_INVALID_ARG, "output must be 16-byte aligned%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  if (mode == SAGE_MODE_NVFP4 && d != 128)
    return set_err(SAGE_ERR_UNSUPPORTED, "the NVFP4 attention kernel needs d = 128%s");
  const sage_ws_layout L = layout_of(B, H, N, d, mode, q_blocks);
  if ((st = check_ws(ws, ws_bytes, L.scratch)) != SAGE_OK) return st;
  sage::Problem pb{B * H, N, (N + 127) / 128 * 128, d, dtype, smooth_q ? 1 : 0, mode, causal ? 1 : 0};
  pb.q_blocks = q_blocks ? 1 : 0;
  if (!after_quantize &&
      (st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  if (mode == SAGE_MODE_NVFP4)
    return cuda_status(
        sage::launch_attn_fp4(resolve(const_cast<void*>(ws), L), out, pb, (cudaStream_t)stream),
        "attention launch");
  return cuda_status(
      sage::launch_attn_i8f8(resolve(const_cast<void*>(ws), L), out, pb, Pr, (cudaStream_t)stream),
      "attention launch");
}

sage_status sage_attn_quantized(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int H, int N, int d,
                                int causal, int smooth_q, int mode, sage_stream_t stream) {
  return attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, smooth_q, mode, default_pr(mode), stream,
                        false);
}

sage_status sage_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                          int causal, int mode, int dtype, int smooth_q, void* ws, size_t ws_bytes,
                          sage_stream_t stream) {
  sage_status st = sage_quantize_qkv(q, k, v, dtype, B, H, N, d, smooth_q, mode, ws, ws_bytes, stream);
  if (st != SAGE_OK) return st;
  return attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, smooth_q, mode, default_pr(mode), stream,
                        true);
}

sage_status sage_attn_fwd_ranges(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                                 int causal, int mode, int dtype, int smooth_q, float Pr, float Vr, void* ws,
                                 size_t ws_bytes, sage_stream_t stream) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (mode == SAGE_MODE_NVFP4)
    return set_err(SAGE_ERR_UNSUPPORTED, "the NVFP4 mode has no P~ / V ranges (its block scales are fixed)%s");
  if (!(Pr > 0.0f && Pr <= 448.0f) || !(Vr > 0.0f && Vr <= 448.0f))
    return set_err(SAGE_ERR_INVALID_ARG, "Pr and Vr must lie in (0, 448], the finite e4m3 range%s");
  // the worst 64-key FP16 partial (all P~ = Pr, all |v^| = Vr) must stay finite
  if (mode == SAGE_MODE_INT8_FP8_F16ACC && 64.0 * (double)Pr * (double)Vr > 65504.0)
    return set_err(SAGE_ERR_INVALID_ARG, "64 * Pr * Vr exceeds 65504: the FP16 partial could overflow%s");
  st = quantize(q, k, v, dtype, B, H, N, d, smooth_q, mode, Vr, ws, ws_bytes, stream);
  if (st != SAGE_OK) return st;
  return attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, smooth_q, mode, Pr, stream, true);
}

sage_status sage_attn_fwd_fused(const void* q, const void* k, const void* v, void* out, int B, int H, int N, int d,
                                int causal, int mode, int dtype, int smooth_q, void* ws, size_t ws_bytes,
                                sage_stream_t stream) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (mode == SAGE_MODE_NVFP4)
    return set_err(SAGE_ERR_UNSUPPORTED, "the fused forward covers the INT8/FP8 modes%s");
  if (!q || !k || !v || !out) return set_err(SAGE_ERR_INVALID_ARG, "null input or output pointer%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  if ((((uintptr_t)q) | ((uintptr_t)k) | ((uintptr_t)v) | ((uintptr_t)out)) % 16)
    return set_err(SAGE_ERR_INVALID_ARG, "inputs and output must be 16-byte aligned%s");
  const sage_ws_layout L = layout_of(B, H, N, d, mode);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SAGE_OK) return st;
  sage::Problem pb{B * H, N, (N + 127) / 128 * 128, d, dtype, smooth_q ? 1 : 0, mode, causal ? 1 : 0};
  if ((st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  const sage::WsPtrs w = resolve(ws, L);
  if ((st = cuda_status(sage::launch_quant_split(q, k, v, pb, default_vr(mode), w, (cudaStream_t)stream, true),
                        "quantize launch")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_attn_i8f8_fused_q(w, q, out, pb, default_pr(mode), (cudaStream_t)stream),
                     "attention launch");
}

sage_status sage_workspace_layout_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int mode, sage_ws_layout* out) {
  sage_status st = check_shape_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if (st != SAGE_OK) return st;
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "layout pointer is null%s");
  *out = layout_of_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  return SAGE_OK;
}

static sage::Problem problem_gqa(int B, int Hq, int Hkv, int Nq, int Nk, int d, int dtype, int smooth_q, int mode,
                                 int causal) {
  sage::Problem pb{B * Hq, Nq, (Nq + 127) / 128 * 128, d, dtype, smooth_q ? 1 : 0, mode, causal ? 1 : 0};
  pb.Hq = Hq;
  pb.G = Hq / Hkv;
  pb.Nk = Nk;
  pb.Npad_k = (Nk + 127) / 128 * 128;
  return pb;
}

sage_status sage_quantize_qkv_gqa(const void* q, const void* k, const void* v, int dtype, int B, int Hq, int Hkv,
                                  int Nq, int Nk, int d, int smooth_q, int mode, void* ws, size_t ws_bytes,
                                  sage_stream_t stream) {
  sage_status st = check_shape_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if (st != SAGE_OK) return st;
  if (Hq == Hkv && Nq == Nk) return sage_quantize_qkv(q, k, v, dtype, B, Hq, Nq, d, smooth_q, mode, ws, ws_bytes, stream);
  if (!q || !k || !v) return set_err(SAGE_ERR_INVALID_ARG, "null input pointer%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  if ((((uintptr_t)q) | ((uintptr_t)k) | ((uintptr_t)v)) % 16)
    return set_err(SAGE_ERR_INVALID_ARG, "inputs must be 16-byte aligned%s");
  const sage_ws_layout L = layout_of_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if ((st = check_ws(ws, ws_bytes, L.total)) != SAGE_OK) return st;
  const sage::Problem pb = problem_gqa(B, Hq, Hkv, Nq, Nk, d, dtype, smooth_q, mode, 0);
  if ((st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_quant_split(q, k, v, pb, default_vr(mode), resolve(ws, L), (cudaStream_t)stream),
                     "quantize launch");
}

static sage_status attn_quantized_gqa(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int Hq, int Hkv,
                                      int Nq, int Nk, int d, int causal, int smooth_q, int mode,
                                      sage_stream_t stream, bool after_quantize) {
  sage_status st = check_shape_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if (st != SAGE_OK) return st;
  if (Hq == Hkv && Nq == Nk)
    return attn_quantized(ws, ws_bytes, out, dtype, B, Hq, Nq, d, causal, smooth_q, mode, default_pr(mode), stream,
                          after_quantize);
  if (causal && Nq > Nk)
    return set_err(SAGE_ERR_UNSUPPORTED, "a causal mask with Nq > Nk leaves query rows without keys%s");
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "null output pointer%s");
  if (((uintptr_t)out) % 16) return set_err(SAGE_ERR_INVALID_ARG, "output must be 16-byte aligned%s");
  if (dtype != SAGE_F16 && dtype != SAGE_BF16) return set_err(SAGE_ERR_INVALID_ARG, "dtype must be 0 (f16) or 1 (bf16)%s");
  const sage_ws_layout L = layout_of_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if ((st = check_ws(ws, ws_bytes, L.scratch)) != SAGE_OK) return st;
  const sage::Problem pb = problem_gqa(B, Hq, Hkv, Nq, Nk, d, dtype, smooth_q, mode, causal);
  if (!after_quantize &&
      (st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_attn_i8f8(resolve(const_cast<void*>(ws), L), out, pb, default_pr(mode),
                                            (cudaStream_t)stream),
                     "attention launch");
}

sage_status sage_attn_quantized_gqa(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int Hq, int Hkv,
                                    int Nq, int Nk, int d, int causal, int smooth_q, int mode, sage_stream_t stream) {
  return attn_quantized_gqa(ws, ws_bytes, out, dtype, B, Hq, Hkv, Nq, Nk, d, causal, smooth_q, mode, stream, false);
}

sage_status sage_attn_fwd_gqa(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv, int Nq,
                              int Nk, int d, int causal, int mode, int dtype, int smooth_q, void* ws, size_t ws_bytes,
                              sage_stream_t stream) {
  sage_status st = check_shape_gqa(B, Hq, Hkv, Nq, Nk, d, mode);
  if (st != SAGE_OK) return st;
  if (causal && Nq > Nk)
    return set_err(SAGE_ERR_UNSUPPORTED, "a causal mask with Nq > Nk leaves query rows without keys%s");
  st = sage_quantize_qkv_gqa(q, k, v, dtype, B, Hq, Hkv, Nq, Nk, d, smooth_q, mode, ws, ws_bytes, stream);
  if (st != SAGE_OK) return st;
  return attn_quantized_gqa(ws, ws_bytes, out, dtype, B, Hq, Hkv, Nq, Nk, d, causal, smooth_q, mode, stream, true);
}

// Q smoothed per 128-row block: the per-head entry points with smooth_q set
// and one Q mean and one bias row per block.
static sage_status check_blocksmooth(int B, int H, int N, int d, int mode) {
  sage_status st = check_shape(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (mode == SAGE_MODE_NVFP4)
    return set_err(SAGE_ERR_UNSUPPORTED, "per-block Q smoothing covers the INT8/FP8 modes%s");
  return SAGE_OK;
}

sage_status sage_workspace_layout_blocksmooth(int B, int H, int N, int d, int mode, sage_ws_layout* out) {
  sage_status st = check_blocksmooth(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  if (!out) return set_err(SAGE_ERR_INVALID_ARG, "layout pointer is null%s");
  *out = layout_of(B, H, N, d, mode, true);
  return SAGE_OK;
}

sage_status sage_quantize_qkv_blocksmooth(const void* q, const void* k, const void* v, int dtype, int B, int H, int N,
                                          int d, int mode, void* ws, size_t ws_bytes, sage_stream_t stream) {
  sage_status st = check_blocksmooth(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  return quantize(q, k, v, dtype, B, H, N, d, 1, mode, default_vr(mode), ws, ws_bytes, stream, true);
}

sage_status sage_attn_quantized_blocksmooth(const void* ws, size_t ws_bytes, void* out, int dtype, int B, int H, int N,
                                            int d, int causal, int mode, sage_stream_t stream) {
  sage_status st = check_blocksmooth(B, H, N, d, mode);
  if (st != SAGE_OK) return st;
  return attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, 1, mode, default_pr(mode), stream, false, true);
}

sage_status sage_attn_fwd_blocksmooth(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                                      int d, int causal, int mode, int dtype, void* ws, size_t ws_bytes,
                                      sage_stream_t stream) {
  sage_status st = sage_quantize_qkv_blocksmooth(q, k, v, dtype, B, H, N, d, mode, ws, ws_bytes, stream);
  if (st != SAGE_OK) return st;
  return attn_quantized(ws, ws_bytes, out, dtype, B, H, N, d, causal, 1, mode, default_pr(mode), stream, true, true);
}

sage_status sage_debug_qk_s32(const void* ws, size_t ws_bytes, int B, int H, int N, int d, int bh, int q_tile,
                              int k_tile, int32_t* out, sage_stream_t stream) {
  sage_status st = check_shape(B, H, N, d, SAGE_MODE_INT8_FP8);
  if (st != SAGE_OK) return st;
  const int ntiles = (N + 127) / 128;
  if (!out || bh < 0 || bh >= B * H || q_tile < 0 || q_tile >= ntiles || k_tile < 0 || k_tile >= ntiles)
    return set_err(SAGE_ERR_INVALID_ARG, "debug tile out of range%s");
  const sage_ws_layout L = layout_of(B, H, N, d, SAGE_MODE_INT8_FP8);
  if ((st = check_ws(ws, ws_bytes, L.scratch)) != SAGE_OK) return st;
  sage::Problem pb{B * H, N, ntiles * 128, d, 0, 0, 0, 0};
  if ((st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_debug_qk(resolve(const_cast<void*>(ws), L), pb, bh, q_tile, k_tile, out,
                                           (cudaStream_t)stream),
                     "debug launch");
}

sage_status sage_debug_fp4_s(const void* ws, size_t ws_bytes, int B, int H, int N, int d, int bh, int q_tile,
                             int k_tile, float* out, sage_stream_t stream) {
  sage_status st = check_shape(B, H, N, d, SAGE_MODE_NVFP4);
  if (st != SAGE_OK) return st;
  if (d != 128) return set_err(SAGE_ERR_UNSUPPORTED, "the NVFP4 tensor-core path needs d = 128%s");
  const int ntiles = (N + 127) / 128;
  if (!out || bh < 0 || bh >= B * H || q_tile < 0 || q_tile >= ntiles || k_tile < 0 || k_tile >= ntiles)
    return set_err(SAGE_ERR_INVALID_ARG, "debug tile out of range%s");
  const sage_ws_layout L = layout_of(B, H, N, d, SAGE_MODE_NVFP4);
  if ((st = check_ws(ws, ws_bytes, L.scratch)) != SAGE_OK) return st;
  sage::Problem pb{B * H, N, ntiles * 128, d, 0, 0, SAGE_MODE_NVFP4, 0};
  if ((st = cuda_status(cudaMemsetAsync((char*)ws + L.error, 0, sizeof(int), (cudaStream_t)stream), "clear")) != SAGE_OK)
    return st;
  return cuda_status(sage::launch_debug_fp4_s(resolve(const_cast<void*>(ws), L), pb, bh, q_tile, k_tile, out,
                                              (cudaStream_t)stream),
                     "debug launch");
}

sage_status sage_debug_timeout_probe(void* ws, size_t ws_bytes, sage_stream_t stream) {
  if (!ws || ws_bytes < sizeof(int) || ((uintptr_t)ws) % kAlign)
    return set_err(SAGE_ERR_INVALID_ARG, "workspace pointer is null or misaligned%s");
  sage_ws_layout L;
  memset(&L, 0, sizeof(L));  // only the error word (offset 0) is used
  sage_status st = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int), (cudaStream_t)stream), "clear");
  if (st != SAGE_OK) return st;
  return cuda_status(sage::launch_timeout_probe(resolve(ws, L), (cudaStream_t)stream), "probe launch");
}

sage_status sage_probe_mma_rate(int kind, int ctas, int iters, void* ws, size_t ws_bytes, double* ops,
                               sage_stream_t stream) {
  if (!ws || ws_bytes < sizeof(int) || ((uintptr_t)ws) % kAlign)
    return set_err(SAGE_ERR_INVALID_ARG, "workspace pointer is null or misaligned%s");
  if (kind < SAGE_PROBE_I8 || kind > SAGE_PROBE_FP4) return set_err(SAGE_ERR_INVALID_ARG, "unknown probe kind%s");
  if (ctas < 1 || ctas > 65535 || iters < 1 || iters > (1 << 20))
    return set_err(SAGE_ERR_INVALID_ARG, "ctas must be in [1, 65535] and iters in [1, 2^20]%s");
  if (ops) *ops = sage::mma_rate_ops(kind, ctas, iters);
  sage_status st = cuda_status(cudaMemsetAsync(ws, 0, sizeof(int), (cudaStream_t)stream), "clear");
  if (st != SAGE_OK) return st;
  return cuda_status(sage::launch_mma_rate(kind, ctas, iters, (int*)ws, (cudaStream_t)stream), "probe launch");
}

sage_status sage_check(void* ws, size_t ws_bytes, sage_stream_t stream) {
  if (!ws || ws_bytes < sizeof(int)) return set_err(SAGE_ERR_INVALID_ARG, "workspace pointer is null%s");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "stream synchronize");
  int word = 0;
  // the error word sits at offset 0 of every layout
  e = cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e, "error word read");
  if (word != 0) {
    const int zero = 0;
    cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice);
    char buf[64];
    snprintf(buf, sizeof(buf), "device wait timed out (site 0x%x)", word);
    g_last_error = buf;
    return SAGE_ERR_TIMEOUT;
  }
  return SAGE_OK;
}

}  // extern "C"
