// sage_internal.h -- declarations shared by the library's translation units
// (launchers and the resolved workspace pointers).  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sage {

// Device pointers into one workspace, resolved from sage_ws_layout.
struct WsPtrs {
  int8_t* q_codes;
  int8_t* k_codes;
  uint8_t* vt_codes;
  float* q_scale;
  float* k_scale;
  float* v_scale;
  float* k_mean;
  float* q_mean;
  float* q_bias;
  float* global_scale;
  int* error;
  float* scratch;  // statistics partials, then the per-channel V multipliers
};

// BH = B * Hq query slices of N query rows (padded to Npad); with grouped
// key/value heads (G = Hq / Hkv > 1) and / or a key length Nk != N the last
// fields describe the keys; 0 there means "the same as the queries".
struct Problem {
  int BH, N, Npad, d, dtype, smooth_q, mode, causal;
  int Hq = 0, G = 1, Nk = 0, Npad_k = 0;
  // Q smoothed per 128-row block (per-head shapes, INT8/FP8 modes): q_mean
  // [BH][Npad/128][d] and q_bias [BH][Npad/128][Npad], one row per block
  int q_blocks = 0;
  int nk() const { return Nk ? Nk : N; }
  int npk() const { return Npad_k ? Npad_k : Npad; }
  int bh_kv() const { return BH / G; }
  int hq() const { return Hq ? Hq : 1; }
};

// Causal attention grids run (G, query blocks, B*H/G): the CTAs of G slices
// launch longest-first together, then the next G.  G is the largest divisor
// of B*H whose K and V codes (slice_bytes each) fit in `budget` bytes of L2,
// at least 1.
inline int causal_slice_group(int BH, double slice_bytes, double budget) {
  int g = 1;
  for (int c = 1; c <= BH; ++c)
    if (BH % c == 0 && c * slice_bytes <= budget) g = c;
  return g;
}

// Launch `kern` on `s`; with `pdl` it may start while the previous kernel on
// the stream is still running (programmatic stream serialization): the kernel
// must call grid_dep_wait before it reads what that kernel wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                                 Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Floats of scratch the quantization pass needs.  INT8/FP8 modes: statistics
// partials [3][BH][Npad/64][d] (K sums, Q sums, |V| maxima) and V multipliers
// [BH][d].  NVFP4: partials [7][BH][Npad/64][d] (the same three planes, then
// K maxima, K minima, Q maxima, Q minima of the raw values).
size_t quant_scratch_floats(int BH, int Npad, int d, int mode);

// The same with grouped key/value heads or separate query and key lengths
// (INT8/FP8 modes): separate passes over Q and over K/V.
size_t quant_scratch_floats_split(int BHq, int Npq, int BHkv, int Npk, int d);
// skip_q_codes: Q statistics only (the fused forward quantizes Q in the
// attention kernel); with equal shapes the per-head layout's scratch serves.
cudaError_t launch_quant_split(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                               const WsPtrs& w, cudaStream_t s, bool skip_q_codes = false);

// Smoothing statistics + INT8 Q/K + FP8 V (+ bias), enqueued on `s`.
cudaError_t launch_quant_int8_fp8(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                                  const WsPtrs& w, cudaStream_t s);

// The same quantization pass with its statistics scratch in a file-scope
// device array (quant_static.cu) instead of w.scratch, which is ignored.
cudaError_t launch_quant_static(const void* q, const void* k, const void* v, const Problem& pb, float Vr, WsPtrs w,
                                cudaStream_t s);
size_t static_scratch_floats();

// Fused attention (FP32 or FP16 PV accumulator).  Launched normally: a
// programmatic launch behind the codes pass measured slower on video_dit.
cudaError_t launch_attn_i8f8(const WsPtrs& w, void* out, const Problem& pb, float Pr, cudaStream_t s);
// The same with Q quantized inside the attention kernel from the caller's
// 16-bit Q ([BH, N, d]); the workspace holds K/V codes, scales, means, bias.
cudaError_t launch_attn_i8f8_fused_q(const WsPtrs& w, const void* q_raw, void* out, const Problem& pb, float Pr,
                                     cudaStream_t s);

// Fused NVFP4 attention (kind::mxf4nvf4 for S and P~V, FP32 accumulator); d = 128.
cudaError_t launch_attn_fp4(const WsPtrs& w, void* out, const Problem& pb, cudaStream_t s);

// INT32 S tile through the tensor-core path.
cudaError_t launch_debug_qk(const WsPtrs& w, const Problem& pb, int bh, int q_tile, int k_tile, int32_t* out,
                            cudaStream_t s);

// One NVFP4 S tile (raw block-scaled dot products, FP32) through the
// kind::mxf4nvf4 tensor-core path; d = 128.
cudaError_t launch_debug_fp4_s(const WsPtrs& w, const Problem& pb, int bh, int q_tile, int k_tile, float* out,
                               cudaStream_t s);

// Tensor-core rate probe (probe.cu): `ctas` CTAs each issue `iters` x 4
// back-to-back M=128 N=256 MMAs of one kind on shared-memory operands.
enum { kProbeI8 = 0, kProbeF8F32 = 1, kProbeF8F16 = 2, kProbeBF16 = 3, kProbeFP4 = 4 };
cudaError_t launch_mma_rate(int kind, int ctas, int iters, int* err, cudaStream_t s);
double mma_rate_ops(int kind, int ctas, int iters);  // 2*M*N*K per instruction, summed

// A kernel whose only wait can never complete: exercises the bounded-wait path.
cudaError_t launch_timeout_probe(const WsPtrs& w, cudaStream_t s);

// Tensor maps (cuTensorMapEncodeTiled through the runtime's driver entry point).
// A 3-D uint8 tensor [dim2][dim1][dim0] with a box of box0 x box1 x 1 and
// the swizzle that matches a row of box0 bytes (64 or 128).
bool make_tmap_u8_3d(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                     uint32_t box0, uint32_t box1);
// A uint8 tensor of `rank` (2..5) dimensions, dims[0] innermost and
// contiguous, strides[i] = bytes between consecutive indices of dimension
// i + 1 (any order: a map may walk rows out of their memory order), a box of
// box[0..rank) elements; swizzle_bytes 128, 64 or 0.
bool make_tmap_u8_nd(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
                     const uint32_t* box, int swizzle_bytes);

}  // namespace sage
