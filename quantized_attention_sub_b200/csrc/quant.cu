// quant.cu -- smoothing and quantization kernels of the INT8/FP8 modes
// (SageAttention2 abstract: smooth, INT-quantize Q/K, FP8-quantize V;
// SageAttention2++ summary Sec. 2.1: per-block Q/K scales, per-channel V
// scales; Sec. 3.1: the narrowed V range Vr).
//
// All arithmetic that decides a code is IEEE fp32 with explicit _rn
// intrinsics (no contraction), in the order below, so the codes and scales
// are bit-reproducible:
//   mean_c   = (sum over 64-token chunks, in order, of the sequential fp32
//               sum of the chunk) / N
//   x~       = x - mean_c                       (Q only when smooth_q)
//   granule  : a = max |x~| over its valid tokens (Q 32 tokens, K 64)
//              scale = a / 127, inv = 127 / a, code = rint_even(x~ * inv)
//              (a == 0: scale 0, codes 0)
//   bias_n   = fma chain over c of mean_q[c] * k~[n,c]  (smooth_q)
//   V        : scale_c = a_c / Vr, code = e4m3_rn_satfinite(v * (Vr / a_c))
//
// Pass 1 (stats_partials) reads K, V (and Q) once per 64-token chunk and
// writes per-chunk partial sums / maxima; pass 2 (stats_finalize) folds them
// per channel; pass 3 (quant_rows / quant_v) reads the inputs again and
// writes codes.  The three passes are HBM-bound.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

template <typename T>
SAGE_DEV float to_f(T x);
template <>
SAGE_DEV float to_f<__half>(__half x) { return __half2float(x); }
template <>
SAGE_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Four consecutive 16-bit values -> float4.
template <typename T>
SAGE_DEV void load4(const T* p, float* f) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  const T* h = reinterpret_cast<const T*>(&u);
  f[0] = to_f(h[0]);
  f[1] = to_f(h[1]);
  f[2] = to_f(h[2]);
  f[3] = to_f(h[3]);
}

// ---------------------------------------------------------------- pass 1
// grid (Npad/64, BH), block D threads; thread c owns channel c of one chunk.
template <typename T, int D>
__global__ void __launch_bounds__(D) stats_partials_kernel(const T* __restrict__ k, const T* __restrict__ q,
                                                           const T* __restrict__ v, int N, int nchunks,
                                                           float* __restrict__ part) {
  const int chunk = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const int t0 = chunk * 64;
  const int t1 = min(t0 + 64, N);
  const size_t base = (size_t)bh * N * D + c;
  float sk = 0.f, sq = 0.f, av = 0.f;
  for (int t = t0; t < t1; ++t) {
    const size_t o = base + (size_t)t * D;
    sk = __fadd_rn(sk, to_f(k[o]));
    if (q) sq = __fadd_rn(sq, to_f(q[o]));
    av = fmaxf(av, fabsf(to_f(v[o])));
  }
  // part layout: [3][BH][nchunks][D] = sums of K, sums of Q, maxima of |V|
  const size_t plane = (size_t)gridDim.y * nchunks * D;
  const size_t o = ((size_t)bh * nchunks + chunk) * D + c;
  part[o] = sk;
  part[plane + o] = sq;
  part[2 * plane + o] = av;
}

// ---------------------------------------------------------------- pass 2
// grid BH, block D: channel means in chunk order, V absmax, V scale/multiplier.
template <int D>
__global__ void __launch_bounds__(D) stats_finalize_kernel(const float* __restrict__ part, int N, int nchunks,
                                                           int with_q, float Vr, float* __restrict__ k_mean,
                                                           float* __restrict__ q_mean, float* __restrict__ v_scale,
                                                           float* __restrict__ v_mul) {
  const int bh = blockIdx.x, c = threadIdx.x;
  const int nvalid = (N + 63) / 64;
  const size_t plane = (size_t)gridDim.x * nchunks * D;
  float tk = 0.f, tq = 0.f, a = 0.f;
  for (int g = 0; g < nvalid; ++g) {
    const size_t o = ((size_t)bh * nchunks + g) * D + c;
    tk = __fadd_rn(tk, part[o]);
    if (with_q) tq = __fadd_rn(tq, part[plane + o]);
    a = fmaxf(a, part[2 * plane + o]);
  }
  k_mean[bh * D + c] = __fdiv_rn(tk, (float)N);
  if (with_q) q_mean[bh * D + c] = __fdiv_rn(tq, (float)N);
  v_scale[bh * D + c] = a > 0.f ? __fdiv_rn(a, Vr) : 0.f;
  v_mul[bh * D + c] = a > 0.f ? __fdiv_rn(Vr, a) : 0.f;
}

// ---------------------------------------------------------------- pass 3a
// INT8 quantization of 64 tokens of Q or K: grid (Npad/64, BH), 256 threads.
// G = granule (32 for Q, 64 for K).  mean may be null (no smoothing).  When
// bias_mq is set (K with smooth_q), also writes bias[n] for the 64 tokens.
template <typename T, int D, int G>
__global__ void __launch_bounds__(256) quant_rows_int8_kernel(const T* __restrict__ x, const float* __restrict__ mean,
                                                              int N, int Npad, int8_t* __restrict__ codes,
                                                              float* __restrict__ scale,
                                                              const float* __restrict__ bias_mq,
                                                              float* __restrict__ bias) {
  constexpr int kRows = 64, kVec = D / 4, kNG = kRows / G;
  __shared__ float xs[kRows][D + 1];
  __shared__ float wmax[8][kNG];
  __shared__ float ginv[kNG];
  __shared__ float smq[D];
  const int blk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int t0 = blk * kRows;

  float amax0 = 0.f, amax1 = 0.f;  // the block's one or two granules
  for (int e = tid; e < kRows * kVec; e += 256) {
    const int r = e / kVec, c = (e % kVec) * 4;
    const int t = t0 + r;
    float f[4] = {0.f, 0.f, 0.f, 0.f};
    if (t < N) {
      load4(x + ((size_t)bh * N + t) * D + c, f);
      if (mean) {
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __fsub_rn(f[i], mean[bh * D + c + i]);
      }
    }
    const float fa = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
    if (kNG == 1 || r < G) amax0 = fmaxf(amax0, fa);
    else amax1 = fmaxf(amax1, fa);
#pragma unroll
    for (int i = 0; i < 4; ++i) xs[r][c + i] = f[i];
  }
  if (bias_mq && tid < D) smq[tid] = bias_mq[bh * D + tid];
#pragma unroll
  for (int g = 0; g < kNG; ++g) {
    float a = g == 0 ? amax0 : amax1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) wmax[tid >> 5][g] = a;
  }
  __syncthreads();
  if (tid < kNG) {
    float a = 0.f;
    for (int w = 0; w < 8; ++w) a = fmaxf(a, wmax[w][tid]);
    const int gi = (t0 / G) + tid;
    scale[(size_t)bh * (Npad / G) + gi] = a > 0.f ? __fdiv_rn(a, 127.0f) : 0.f;
    ginv[tid] = a > 0.f ? __fdiv_rn(127.0f, a) : 0.f;
  }
  __syncthreads();
  // codes: each thread writes 4 consecutive codes per step
  for (int e = tid; e < kRows * kVec; e += 256) {
    const int r = e / kVec, c = (e % kVec) * 4;
    const float inv = ginv[r / G];
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int qv = __float2int_rn(__fmul_rn(xs[r][c + i], inv));
      qv = max(-127, min(127, qv));
      packed |= ((uint32_t)(qv & 0xFF)) << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(codes + ((size_t)bh * Npad + t0 + r) * D + c) = packed;
  }
  if (bias_mq && tid < kRows) {
    const int t = t0 + tid;
    float acc = 0.f;
    if (t < N)
      for (int c = 0; c < D; ++c) acc = __fmaf_rn(smq[c], xs[tid][c], acc);
    bias[(size_t)bh * Npad + t] = acc;
  }
}

// ---------------------------------------------------------------- pass 3b
// FP8 quantization of V, 128 tokens per block, written transposed:
// grid (Npad/128, BH), 256 threads.
template <typename T, int D>
__global__ void __launch_bounds__(256) quant_v_fp8_kernel(const T* __restrict__ v, const float* __restrict__ v_mul,
                                                          int N, int Npad, uint8_t* __restrict__ vt) {
  constexpr int kTok = 128, kVec = D / 4;
  __shared__ __align__(16) uint8_t tile[D][kTok + 16];
  __shared__ float mul[D];
  const int blk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int t0 = blk * kTok;
  if (tid < D) mul[tid] = v_mul[bh * D + tid];
  __syncthreads();
  for (int e = tid; e < kTok * kVec; e += 256) {
    const int r = e / kVec, c = (e % kVec) * 4;
    const int t = t0 + r;
    uint8_t cd[4] = {0, 0, 0, 0};
    if (t < N) {
      float f[4];
      load4(v + ((size_t)bh * N + t) * D + c, f);
      const uint16_t a = e4m3x2(__fmul_rn(f[0], mul[c]), __fmul_rn(f[1], mul[c + 1]));
      const uint16_t b = e4m3x2(__fmul_rn(f[2], mul[c + 2]), __fmul_rn(f[3], mul[c + 3]));
      cd[0] = (uint8_t)(a & 0xFF);
      cd[1] = (uint8_t)(a >> 8);
      cd[2] = (uint8_t)(b & 0xFF);
      cd[3] = (uint8_t)(b >> 8);
      // a zero multiplier (all-zero channel) gives code 0 as the oracle's rule
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (mul[c + i] == 0.f) cd[i] = 0;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) tile[c + i][r] = cd[i];
  }
  __syncthreads();
  for (int e = tid; e < D * (kTok / 16); e += 256) {
    const int c = e / (kTok / 16), s = e % (kTok / 16);
    const uint4 val = *reinterpret_cast<const uint4*>(&tile[c][s * 16]);
    *reinterpret_cast<uint4*>(vt + ((size_t)bh * D + c) * Npad + t0 + s * 16) = val;
  }
}

template <typename T, int D>
static cudaError_t quant_all(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                             const WsPtrs& w, cudaStream_t s) {
  const T* qp = (const T*)q;
  const T* kp = (const T*)k;
  const T* vp = (const T*)v;
  const int nchunks = pb.Npad / 64;
  float* part = w.scratch;
  float* v_mul = w.scratch + (size_t)3 * pb.BH * nchunks * D;
  stats_partials_kernel<T, D><<<dim3(nchunks, pb.BH), D, 0, s>>>(kp, pb.smooth_q ? qp : nullptr, vp, pb.N,
                                                                   nchunks, part);
  stats_finalize_kernel<D><<<pb.BH, D, 0, s>>>(part, pb.N, nchunks, pb.smooth_q, Vr, w.k_mean, w.q_mean,
                                               w.v_scale, v_mul);
  quant_rows_int8_kernel<T, D, 32><<<dim3(nchunks, pb.BH), 256, 0, s>>>(
      qp, pb.smooth_q ? w.q_mean : nullptr, pb.N, pb.Npad, w.q_codes, w.q_scale, nullptr, nullptr);
  quant_rows_int8_kernel<T, D, 64><<<dim3(nchunks, pb.BH), 256, 0, s>>>(
      kp, w.k_mean, pb.N, pb.Npad, w.k_codes, w.k_scale, pb.smooth_q ? w.q_mean : nullptr, w.q_bias);
  quant_v_fp8_kernel<T, D><<<dim3(pb.Npad / 128, pb.BH), 256, 0, s>>>(vp, v_mul, pb.N, pb.Npad, w.vt_codes);
  return cudaGetLastError();
}

cudaError_t launch_quant_int8_fp8(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                                  const WsPtrs& w, cudaStream_t s) {
  if (pb.dtype == 0) {
    return pb.d == 128 ? quant_all<__half, 128>(q, k, v, pb, Vr, w, s) : quant_all<__half, 64>(q, k, v, pb, Vr, w, s);
  }
  return pb.d == 128 ? quant_all<__nv_bfloat16, 128>(q, k, v, pb, Vr, w, s)
                     : quant_all<__nv_bfloat16, 64>(q, k, v, pb, Vr, w, s);
}

}  // namespace sage
