// quant.cu -- smoothing and quantization of the INT8/FP8 modes
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
// Three kernels on the stream, none of which waits on another CTA:
//   stats : per 64-token chunk of each (b, h) slice, the sequential sums of K
//           (and Q) per channel and the maxima of |V| per channel;
//   fold  : per slice and tensor, the sequential sum (maximum) over the
//           chunk partials in chunk order -> means, V scales and multipliers;
//   codes : per 64-token chunk, K/Q codes and scales, the bias, V codes.
// The stats and codes kernels are persistent: one loader warp streams each
// CTA's chunks with TMA into a double buffer while eight compute warps work
// on the other half.
//
// The K and Q granule maxima come from exact packed 16-bit max / min per
// channel: RN(x - mean) is monotone in x, so the largest |x~| of a channel is
// the larger of |RN(max - mean)| and |RN(min - mean)|.  Codes use packed fp32
// adds (each lane rounds like the scalar operation) and take the rounded
// integer from the low mantissa bits of y + 1.5 * 2^23.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

namespace {

constexpr int kComputeWarps = 8;
constexpr int kCompute = 32 * kComputeWarps;  // threads of the compute warps
constexpr int kThreadsQ = kCompute + 32;      // + one loader warp
constexpr int kTok = 64;        // tokens per work item (one K granule, two Q granules)
constexpr int kBoxBytes = 128;  // TMA box row: 64 16-bit channels, SWIZZLE_128B
constexpr int kBarCompute = 1;  // named barrier of the compute warps

// error code of a CTA whose own tile loads did not land in time
constexpr int kErrTileWait = 0x202;

template <typename T>
SAGE_DEV float to_f(T x);
template <>
SAGE_DEV float to_f<__half>(__half x) { return __half2float(x); }
template <>
SAGE_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Two 16-bit values packed in a word -> floats (low half first).
template <typename T>
SAGE_DEV void unpack2(uint32_t u, float& lo, float& hi) {
  T h[2];
  *reinterpret_cast<uint32_t*>(h) = u;
  lo = to_f(h[0]);
  hi = to_f(h[1]);
}

struct QuantArgs {
  int8_t* q_codes;
  int8_t* k_codes;
  uint8_t* vt_codes;
  float* q_scale;
  float* k_scale;
  float* v_scale;
  float* k_mean;
  float* q_mean;
  float* q_bias;
  float* part;   // [3 or 7][BH][Npad/64][d] per-chunk partials (see quant_scratch_floats)
  float* v_mul;  // [BH][d] (INT8/FP8 modes)
  float* gscale; // [BH][4] NVFP4 global scales (Q, K, V, 0)
  int* err;
  int BH, N, Npad, smooth_q, n_items;
  float Vr;
  // tensors this pass handles: kRolesQ, kRolesKV or both (the per-head
  // problem: Q, K and V share heads and tokens).  With grouped key/value heads
  // the K/V pass writes the Q-smoothing bias of the G query heads of each
  // key/value slice, reading their means from q_mean_g.
  int roles, G;
  const float* q_mean_g;
  // Q smoothed per 128-row block: the codes pass reads block blk / 2's mean
  // from q_mean [BH][Npad/128][d] and writes no bias (qblock_bias_kernel does)
  int q_blocks;
};
constexpr int kRolesQ = 1, kRolesKV = 2;

// Shared-memory image of one 64-token tile of a [.., D] 16-bit tensor as TMA
// writes it with SWIZZLE_128B: D/64 boxes of 64 rows x 128 bytes, the 16-byte
// chunk c of row r stored at chunk c ^ (r & 7).  Byte offset of byte `b` of row `r`:
SAGE_DEV uint32_t swz(int r, int b) {
  return (uint32_t)((b >> 7) * (kTok * kBoxBytes) + r * kBoxBytes + ((((b >> 4) & 7) ^ (r & 7)) << 4) + (b & 15));
}

// Packed max / min of two 16-bit values (exact comparisons) and the
// identities of those reductions.
template <typename T>
struct P16;
template <>
struct P16<__nv_bfloat16> {
  static constexpr uint32_t kNegInf = 0xFF80FF80u, kPosInf = 0x7F807F80u;
  static SAGE_DEV uint32_t max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  static SAGE_DEV uint32_t min(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
};
template <>
struct P16<__half> {
  static constexpr uint32_t kNegInf = 0xFC00FC00u, kPosInf = 0x7C007C00u;
  static SAGE_DEV uint32_t max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
  static SAGE_DEV uint32_t min(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
  }
};

// Low bytes of four floats -> one word (byte i from z[i]).
SAGE_DEV uint32_t low_bytes4(float z0, float z1, float z2, float z3) {
  const uint32_t lo = __byte_perm(__float_as_uint(z0), __float_as_uint(z1), 0x0040);
  const uint32_t hi = __byte_perm(__float_as_uint(z2), __float_as_uint(z3), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// 1.5 * 2^23: for |y| < 2^22, y + kRound rounds y to an integer (ties to
// even) and leaves it, in two's complement, in the low mantissa bits.
constexpr float kRound = 12582912.0f;

// Offsets, within one tile, of the 4-byte column `word` in rows r0 + k,
// k = 0..7 (r0 a multiple of 8); row r0 + 8 j + k is at o[k] + 1024 j.
SAGE_DEV void col_offsets(int word, int r0, uint32_t (&o)[8]) {
  const int b = 4 * word;
  const uint32_t base = (uint32_t)((b >> 7) * (kTok * kBoxBytes) + r0 * kBoxBytes + (b & 15));
  const uint32_t c = (uint32_t)((b >> 4) & 7);
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] = base + k * kBoxBytes + ((c ^ k) << 4);
}

// Shared-memory loads at 32-bit shared addresses (tile bytes land through
// the async proxy; these follow the mbarrier waits that publish them).
template <typename U>
SAGE_DEV U lds(uint32_t addr);
template <>
SAGE_DEV uint32_t lds<uint32_t>(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
template <>
SAGE_DEV float lds<float>(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
template <>
SAGE_DEV uint4 lds<uint4>(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Calls f(r) for the rows r < rows of a tile, in order; FULL: rows == kTok.
template <bool FULL, typename F>
SAGE_DEV void each_row(int rows, F&& f) {
#pragma unroll
  for (int r = 0; r < kTok; ++r)
    if (FULL || r < rows) f(r);
}

template <int D>
struct QLayout {
  static constexpr int W = D / 2;              // 32-bit words per token row
  static constexpr int kTile = kTok * D * 2;   // bytes of one tensor tile
  static constexpr int kItem = 3 * kTile;      // K, Q, V
  static constexpr int kTiles = 2 * kItem;     // double buffer
  static constexpr int kSlot = 3 * D * 4;      // k_mean, q_mean, v_mul of one buffer
  static constexpr int kBytes = kTiles + 2 * kSlot;
};

enum Pass { kStatsPass = 0, kCodesPass = 1 };

// One streaming pass over the 64-token chunks of all slices (chunk i of the
// list is slice i / (Npad/64), block i % (Npad/64)); CTA c takes chunks
// c, c + grid, ...  PASS selects the per-chunk work.
template <typename T, int D, int PASS, bool FP4>
__global__ void __launch_bounds__(kThreadsQ, 2) quant_pass_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                 const __grid_constant__ CUtensorMap tm_k,
                                                                 const __grid_constant__ CUtensorMap tm_v,
                                                                 const QuantArgs a) {
  using L = QLayout<D>;
  using P = P16<T>;
  constexpr int W = L::W;
  extern __shared__ __align__(1024) uint8_t qsm[];
  __shared__ __align__(8) uint64_t full[2], empty[2];
  __shared__ int4 info[2];  // (item, bh, blk, -) per buffer; item -1: end
  __shared__ int abort_s;
  __shared__ uint2 mm[2][kCompute];  // K, Q: (max, min) pairs per (row group, word)
  __shared__ float red[kComputeWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = a.Npad / kTok;
  const int nchunks = a.Npad / 64;
  const size_t plane = (size_t)a.BH * nchunks * D;
  // 1024-byte aligned start of the tiles (SWIZZLE_128B boxes)
  uint8_t* const sm = qsm + ((1024u - (smem_u32(qsm) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(sm);

  if (tid == 0) {
    abort_s = 0;
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&empty[0], kComputeWarps);
    mbar_init(&empty[1], kComputeWarps);
    fence_mbar_init();
  }
  __syncthreads();
  // the codes pass may start while the fold kernel runs (programmatic
  // launch): nothing it wrote is read before this point
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------- loader
    if (lane != 0) return;
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    const bool do_q = (a.roles & kRolesQ) != 0, do_kv = (a.roles & kRolesKV) != 0;
    const bool need_q = do_q && (PASS == kCodesPass || a.smooth_q || FP4);
    for (int it = 0;; ++it) {
      const int b = it & 1;
      // the codes pass walks the items backwards: the slices the statistics
      // pass read last are the likeliest to be still in L2
      const int idx = blockIdx.x + it * gridDim.x;
      const int item = PASS == kCodesPass ? a.n_items - 1 - idx : idx;
      if (it >= 2 && !mbar_wait(&empty[b], ((it >> 1) - 1) & 1, &abort_s)) {
        atomicCAS(a.err, 0, kErrTileWait);
        abort_s = 1;
        return;
      }
      if (idx >= a.n_items) {
        info[b] = make_int4(-1, 0, 0, 0);
        mbar_arrive(&full[b]);
        return;
      }
      const int bh = item / nb, blk = item % nb;
      info[b] = make_int4(item, bh, blk, 0);
      uint32_t bytes = (uint32_t)L::kTile * ((need_q ? 1 : 0) + (do_kv ? 2 : 0));
      if (PASS == kCodesPass)
        bytes += FP4 ? (uint32_t)(D * 4) * (a.smooth_q ? 2 : 1) + 16u
                     : (uint32_t)(D * 4) * ((do_kv ? 2 : 0) + (do_q && a.smooth_q ? 1 : 0));
      mbar_arrive_expect_tx(&full[b], bytes);
      uint8_t* dst = sm + b * L::kItem;
#pragma unroll
      for (int x = 0; x < D / 64; ++x) {
        const int off = x * kTok * kBoxBytes;
        if (do_kv) tma_load_3d(dst + off, &tm_k, &full[b], x * kBoxBytes, blk * kTok, bh);
        if (need_q) tma_load_3d(dst + L::kTile + off, &tm_q, &full[b], x * kBoxBytes, blk * kTok, bh);
        if (do_kv) tma_load_3d(dst + 2 * L::kTile + off, &tm_v, &full[b], x * kBoxBytes, blk * kTok, bh);
      }
      if (PASS == kCodesPass) {
        // the slice's means and V multipliers (written by the fold kernel)
        float* sl = reinterpret_cast<float*>(sm + L::kTiles) + b * (3 * D);
        if (do_kv || FP4) bulk_load(sl, a.k_mean + (size_t)bh * D, D * 4, &full[b]);
        if (a.smooth_q && (do_q || FP4)) {
          const size_t mrow = a.q_blocks ? (size_t)bh * (a.Npad / 128) + (blk >> 1) : (size_t)bh;
          bulk_load(sl + D, a.q_mean + mrow * D, D * 4, &full[b]);
        }
        if (FP4)
          bulk_load(sl + 2 * D, a.gscale + (size_t)bh * 4, 16, &full[b]);
        else if (do_kv)
          bulk_load(sl + 2 * D, a.v_mul + (size_t)bh * D, D * 4, &full[b]);
      }
    }
  }

  // --------------------------------------------------------------- compute
  for (int it = 0;; ++it) {
    const int b = it & 1;
    const bool landed = mbar_wait(&full[b], (it >> 1) & 1, &abort_s);
    if (!named_bar_and(kBarCompute, kCompute, landed)) {
      if (tid == 0) {
        atomicCAS(a.err, 0, kErrTileWait);
        abort_s = 1;
      }
      return;
    }
    const int4 inf = info[b];
    if (inf.x < 0) return;
    const int bh = inf.y, blk = inf.z;
    const int t0 = blk * kTok;
    const int rows = min(kTok, a.N - t0);  // valid tokens (may be <= 0 in the padding)
    const uint32_t tk = b * L::kItem, tq = tk + L::kTile, tv = tk + 2 * L::kTile;

    if (PASS == kStatsPass && FP4) {
      // Thread u < W: word u of the K rows: two sequential sums in token order
      // and the raw maxima and minima; W <= u < 2W: the same for Q (the sums
      // only with smooth_q); 2W <= u < 3W: |V| maxima of word u - 2W.
      const int role = tid / W, word = tid % W;
      if (role < 3) {
        uint32_t o[8];
        col_offsets(word, 0, o);
        const size_t cell = ((size_t)bh * nchunks + blk) * D + 2 * word;
        const uint32_t src = role == 0 ? tk : role == 1 ? tq : tv;
        const bool want_sum = role == 0 || (role == 1 && a.smooth_q);
        uint32_t mx = P::kNegInf, mn = P::kPosInf;
        uint64_t sum = f2pack(0.f, 0.f);
        auto f = [&](int r) {
          const uint32_t u = lds<uint32_t>(sb + src + o[r & 7] + 1024 * (r >> 3));
          mx = P::max(mx, u);
          mn = P::min(mn, u);
          if (want_sum) {
            float lo, hi;
            unpack2<T>(u, lo, hi);
            sum = add2(sum, f2pack(lo, hi));
          }
        };
        if (rows == kTok)
          each_row<true>(rows, f);
        else
          each_row<false>(rows, f);
        float x0 = 0.f, x1 = 0.f, n0 = 0.f, n1 = 0.f;
        if (rows > 0) {
          unpack2<T>(mx, x0, x1);
          unpack2<T>(mn, n0, n1);
        }
        if (role == 2) {
          *reinterpret_cast<float2*>(a.part + 2 * plane + cell) =
              make_float2(fmaxf(fabsf(x0), fabsf(n0)), fmaxf(fabsf(x1), fabsf(n1)));
        } else {
          if (want_sum) {
            float s0, s1;
            f2unpack(sum, s0, s1);
            *reinterpret_cast<float2*>(a.part + role * plane + cell) = make_float2(s0, s1);
          }
          *reinterpret_cast<float2*>(a.part + (3 + 2 * role) * plane + cell) = make_float2(x0, x1);
          *reinterpret_cast<float2*>(a.part + (4 + 2 * role) * plane + cell) = make_float2(n0, n1);
        }
      }
    } else if (PASS == kStatsPass) {
      // Thread u < W: word u of the K rows, two sequential sums in token
      // order; W <= u < 2W: the same for Q (smooth_q); 2W <= u < 3W: |V|
      // maxima of word u - 2W (exact max / min of the raw values).
      const int role = tid / W, word = tid % W;
      const bool mine = role == 1 ? (a.roles & kRolesQ) && a.smooth_q : (a.roles & kRolesKV) != 0;
      if (role < 3 && mine) {
        uint32_t o[8];
        col_offsets(word, 0, o);
        float* p = a.part + role * plane + ((size_t)bh * nchunks + blk) * D + 2 * word;
        if (role == 2) {
          uint32_t mx = P::kNegInf, mn = P::kPosInf;
          auto f = [&](int r) {
            const uint32_t u = lds<uint32_t>(sb + tv + o[r & 7] + 1024 * (r >> 3));
            mx = P::max(mx, u);
            mn = P::min(mn, u);
          };
          if (rows == kTok)
            each_row<true>(rows, f);
          else
            each_row<false>(rows, f);
          float a0 = 0.f, a1 = 0.f;
          if (rows > 0) {
            float x0, x1, n0, n1;
            unpack2<T>(mx, x0, x1);
            unpack2<T>(mn, n0, n1);
            a0 = fmaxf(fabsf(x0), fabsf(n0));
            a1 = fmaxf(fabsf(x1), fabsf(n1));
          }
          *reinterpret_cast<float2*>(p) = make_float2(a0, a1);
        } else {
          const uint32_t src = role == 0 ? tk : tq;
          uint64_t sum = f2pack(0.f, 0.f);
          auto f = [&](int r) {
            float lo, hi;
            unpack2<T>(lds<uint32_t>(sb + src + o[r & 7] + 1024 * (r >> 3)), lo, hi);
            sum = add2(sum, f2pack(lo, hi));
          };
          if (rows == kTok)
            each_row<true>(rows, f);
          else
            each_row<false>(rows, f);
          float s0, s1;
          f2unpack(sum, s0, s1);
          *reinterpret_cast<float2*>(p) = make_float2(s0, s1);
        }
      }
    } else if (FP4) {
      // NVFP4 codes: Q and K rows in blocks of 16 channels, V^T in blocks of
      // 16 tokens per channel; per block a = max |x|, bs = ue4m3(a / (6 g)),
      // r = 1 / (g * dec(bs)), code = e2m1(x * r), all IEEE fp32 steps.
      const uint32_t kmean = sb + L::kTiles + 4 * (b * (3 * D));
      const uint32_t qmean = kmean + 4 * D;
      const uint32_t gsa = kmean + 8 * D;  // g_q, g_k, g_v, 0
      const int tiles_per_slice = a.Npad / 128;
      {
        constexpr int CB = D / 16;
        constexpr int RPT = kTok * CB / kCompute;  // rows per thread: 2 (d=128) or 1 (d=64)
        const int cb = (tid & 3) + (CB == 8 ? 4 * ((tid >> 3) & 1) : 0);
        const int rbase = (CB == 8 ? 2 * (tid >> 4) : 2 * (tid >> 3)) + ((tid >> 2) & 1);
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const bool isk = which == 0;
          const bool sub = isk || a.smooth_q;
          const uint32_t src = isk ? tk : tq;
          const uint32_t mean = isk ? kmean : qmean;
          const float g = lds<float>(gsa + (isk ? 4 : 0));
          const float six_g = __fmul_rn(6.0f, g);
          uint64_t negm[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            negm[j] = sub ? f2pack(-lds<float>(mean + 4 * (16 * cb + 2 * j)), -lds<float>(mean + 4 * (16 * cb + 2 * j + 1)))
                          : f2pack(0.f, 0.f);
          uint8_t* codes = reinterpret_cast<uint8_t*>(isk ? a.k_codes : a.q_codes);
          uint8_t* sf = reinterpret_cast<uint8_t*>(isk ? a.k_scale : a.q_scale);
#pragma unroll
          for (int k = 0; k < RPT; ++k) {
            const int row = rbase + 32 * k;
            const uint4 h0 = lds<uint4>(sb + src + swz(row, 32 * cb));
            const uint4 h1 = lds<uint4>(sb + src + swz(row, 32 * cb + 16));
            const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            float x[16];
            float am = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float lo, hi;
              unpack2<T>(hw[j], lo, hi);
              if (sub) f2unpack(add2(f2pack(lo, hi), negm[j]), lo, hi);
              x[2 * j] = lo;
              x[2 * j + 1] = hi;
              am = fmaxf(am, fmaxf(fabsf(lo), fabsf(hi)));
            }
            uint32_t bs = 0;
            float r = 0.f;
            if (g > 0.f) {
              bs = e4m3x2(__fdiv_rn(am, six_g), 0.f) & 0xFFu;
              const float sd = e4m3_to_f32(bs);
              if (sd > 0.f) r = __fdiv_rn(1.0f, __fmul_rn(g, sd));
            }
            uint2 cw = make_uint2(0u, 0u);
            if (r > 0.f && row < rows) {
#pragma unroll
              for (int j = 0; j < 16; ++j) x[j] = __fmul_rn(x[j], r);
              cw.x = e2m1x8(x);
              cw.y = e2m1x8(x + 8);
            }
            if (row >= rows) bs = 0;
            const int t = t0 + row;
            *reinterpret_cast<uint2*>(codes + ((size_t)bh * a.Npad + t) * (D / 2) + 8 * cb) = cw;
            const int m = t % 128;
            sf[(((size_t)bh * tiles_per_slice + t / 128) * (D / 64) + cb / 4) * 512 + 16 * (m % 32) + 4 * (m / 32) +
               (cb % 4)] = (uint8_t)bs;
          }
        }
      }
      if (a.smooth_q && tid < kTok) {
        // Q-smoothing bias of token t0 + tid, as in the INT8/FP8 modes
        const int row = tid;
        float acc = 0.f;
        if (row < rows) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 8) {
            const uint4 v4 = lds<uint4>(sb + tk + swz(row, 2 * c0));
            const uint32_t uu[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float lo, hi;
              unpack2<T>(uu[j], lo, hi);
              const int c = c0 + 2 * j;
              acc = __fmaf_rn(lds<float>(qmean + 4 * c), __fsub_rn(lo, lds<float>(kmean + 4 * c)), acc);
              acc = __fmaf_rn(lds<float>(qmean + 4 * c + 4), __fsub_rn(hi, lds<float>(kmean + 4 * c + 4)), acc);
            }
          }
        }
        a.q_bias[(size_t)bh * a.Npad + t0 + row] = acc;
      }
      if (tid < 4 * W) {
        // V^T: thread = word (channels 2w, 2w+1) x one block of 16 tokens;
        // tokens past N read as 0 (TMA fill), like the zero padding they stand for
        const int word = tid % W, vb = tid / W;
        uint32_t ov[8];
        col_offsets(word, 16 * vb, ov);
        const float g = lds<float>(gsa + 8);
        const float six_g = __fmul_rn(6.0f, g);
        float v0[16], v1[16];
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          unpack2<T>(lds<uint32_t>(sb + tv + ov[r & 7] + 1024 * (r >> 3)), v0[r], v1[r]);
          a0 = fmaxf(a0, fabsf(v0[r]));
          a1 = fmaxf(a1, fabsf(v1[r]));
        }
        uint8_t* sfv = reinterpret_cast<uint8_t*>(a.v_scale);
        const int tt = t0 / 128, ka = (t0 % 128) / 64;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          float* vv = ch == 0 ? v0 : v1;
          const float am = ch == 0 ? a0 : a1;
          const int c = 2 * word + ch;
          uint32_t bs = 0;
          float r = 0.f;
          if (g > 0.f) {
            bs = e4m3x2(__fdiv_rn(am, six_g), 0.f) & 0xFFu;
            const float sd = e4m3_to_f32(bs);
            if (sd > 0.f) r = __fdiv_rn(1.0f, __fmul_rn(g, sd));
          }
          uint2 cw = make_uint2(0u, 0u);
          if (r > 0.f) {
#pragma unroll
            for (int j = 0; j < 16; ++j) vv[j] = __fmul_rn(vv[j], r);
            cw.x = e2m1x8(vv);
            cw.y = e2m1x8(vv + 8);
          }
          *reinterpret_cast<uint2*>(a.vt_codes + ((size_t)bh * D + c) * (a.Npad / 2) + (t0 + 16 * vb) / 2) = cw;
          sfv[(((size_t)bh * tiles_per_slice + tt) * 2 + ka) * 512 + 16 * (c % 32) + 4 * (c / 32) + vb] = (uint8_t)bs;
        }
      }
    } else {
        // shared addresses of this buffer's k_mean, q_mean, v_mul
        const uint32_t kmean = sb + L::kTiles + 4 * (b * (3 * D));
        const uint32_t qmean = kmean + 4 * D;
        const uint32_t vmul = kmean + 8 * D;
        constexpr int RG = kCompute / W;  // row groups: 4 (d=128) or 8 (d=64)
        constexpr int RPG = kTok / RG;    // rows per group: 16 or 8
        const int cw = tid % W, r0 = (tid / W) * RPG;  // this thread's column word and first row
        uint32_t o[8];
        col_offsets(cw, r0, o);
        const bool do_q = (a.roles & kRolesQ) != 0, do_kv = (a.roles & kRolesKV) != 0;
        // A: per (row group, word) max and min of the raw K and Q values
        {
          uint32_t kx = P::kNegInf, kn = P::kPosInf, qx = P::kNegInf, qn = P::kPosInf;
#pragma unroll
          for (int r = 0; r < RPG; ++r) {
            if (rows == kTok || r0 + r < rows) {
              const uint32_t off = o[r & 7] + 1024 * (r >> 3);
              if (do_kv) {
                const uint32_t uk = lds<uint32_t>(sb + tk + off);
                kx = P::max(kx, uk);
                kn = P::min(kn, uk);
              }
              if (do_q) {
                const uint32_t uq = lds<uint32_t>(sb + tq + off);
                qx = P::max(qx, uq);
                qn = P::min(qn, uq);
              }
            }
          }
          mm[0][tid] = make_uint2(kx, kn);
          mm[1][tid] = make_uint2(qx, qn);
        }
        named_bar_sync(kBarCompute, kCompute);
        // B: granule maxima of |x~|.  RN(x - mean) is monotone in x, so the
        // largest |x~| of a channel is at its largest or smallest raw value.
        if (tid < 3 * W) {
          const bool isk = tid < W;
          const int g = isk ? 0 : (tid - W) / W, word = tid % W;
          const int rg0 = isk ? 0 : g * (RG / 2), nrg = isk ? RG : RG / 2;
          uint32_t x = P::kNegInf, n = P::kPosInf;
          for (int i = 0; i < nrg; ++i) {
            const uint2 e = mm[isk ? 0 : 1][(rg0 + i) * W + word];
            x = P::max(x, e.x);
            n = P::min(n, e.y);
          }
          float am = 0.f;
          if ((isk ? do_kv : do_q) && (isk ? rows : rows - 32 * g) > 0) {
            float x0, x1, n0, n1;
            unpack2<T>(x, x0, x1);
            unpack2<T>(n, n0, n1);
            if (isk || a.smooth_q) {
              const uint32_t mean = isk ? kmean : qmean;
              const float m0 = lds<float>(mean + 8 * word), m1 = lds<float>(mean + 8 * word + 4);
              x0 = __fsub_rn(x0, m0);
              n0 = __fsub_rn(n0, m0);
              x1 = __fsub_rn(x1, m1);
              n1 = __fsub_rn(n1, m1);
            }
            am = fmaxf(fmaxf(fabsf(x0), fabsf(n0)), fmaxf(fabsf(x1), fabsf(n1)));
          }
#pragma unroll
          for (int s = 16; s > 0; s >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, s));
          if (lane == 0) red[warp] = am;
        }
        named_bar_sync(kBarCompute, kCompute);
        // C: scales, then codes.  K granule: warps [0, W/32); Q granule g:
        // warps [W/32 (1 + g), W/32 (2 + g)).
        constexpr int WPG = W / 32;
        float mk = 0.f, mq0 = 0.f, mq1 = 0.f;
#pragma unroll
        for (int i = 0; i < WPG; ++i) {
          mk = fmaxf(mk, red[i]);
          mq0 = fmaxf(mq0, red[WPG + i]);
          mq1 = fmaxf(mq1, red[2 * WPG + i]);
        }
        if (tid == 0 && do_kv) a.k_scale[(size_t)bh * (a.Npad / 64) + t0 / 64] = mk > 0.f ? __fdiv_rn(mk, 127.0f) : 0.f;
        if ((tid == 1 || tid == 2) && do_q) {
          const float m = tid == 1 ? mq0 : mq1;
          a.q_scale[(size_t)bh * (a.Npad / 32) + t0 / 32 + (tid - 1)] = m > 0.f ? __fdiv_rn(m, 127.0f) : 0.f;
        }
        const float ik = mk > 0.f ? __fdiv_rn(127.0f, mk) : 0.f;
        const float iq0 = mq0 > 0.f ? __fdiv_rn(127.0f, mq0) : 0.f;
        const float iq1 = mq1 > 0.f ? __fdiv_rn(127.0f, mq1) : 0.f;
        {
          // thread: 16-channel block cb of two adjacent rows' worth of lanes;
          // each group of 8 lanes reads 8 distinct 16-byte bank groups
          constexpr int CB = D / 16;
          constexpr int RPT = kTok * CB / kCompute;  // rows per thread: 2 (d=128) or 1 (d=64)
          const int cb = (tid & 3) + (CB == 8 ? 4 * ((tid >> 3) & 1) : 0);
          const int rbase = (CB == 8 ? 2 * (tid >> 4) : 2 * (tid >> 3)) + ((tid >> 2) & 1);
          const uint64_t rnd = f2pack(kRound, kRound);
#pragma unroll 1
          for (int which = 0; which < 2; ++which) {
            const bool isk = which == 0;
            if (!(isk ? do_kv : do_q)) continue;
            const bool sub = isk || a.smooth_q;
            const uint32_t src = isk ? tk : tq;
            const uint32_t mean = isk ? kmean : qmean;
            uint64_t negm[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              negm[j] = sub ? f2pack(-lds<float>(mean + 4 * (16 * cb + 2 * j)), -lds<float>(mean + 4 * (16 * cb + 2 * j + 1)))
                            : f2pack(0.f, 0.f);
            int8_t* dstc = isk ? a.k_codes : a.q_codes;
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
              const int row = rbase + 32 * k;
              const float inv = isk ? ik : (row < 32 ? iq0 : iq1);
              const uint4 h0 = lds<uint4>(sb + src + swz(row, 32 * cb));
              const uint4 h1 = lds<uint4>(sb + src + swz(row, 32 * cb + 16));
              const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
              float z[16];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float lo, hi;
                unpack2<T>(hw[j], lo, hi);
                if (sub) f2unpack(add2(f2pack(lo, hi), negm[j]), lo, hi);
                // scalar __fmul_rn: never merged into an fma with the add that
                // follows, which would round x~ * inv and the integer rounding
                // in one step (the packed multiply gets contracted)
                lo = __fmul_rn(lo, inv);
                hi = __fmul_rn(hi, inv);
                f2unpack(add2(f2pack(lo, hi), rnd), z[2 * j], z[2 * j + 1]);
              }
              uint4 ov;
              ov.x = low_bytes4(z[0], z[1], z[2], z[3]);
              ov.y = low_bytes4(z[4], z[5], z[6], z[7]);
              ov.z = low_bytes4(z[8], z[9], z[10], z[11]);
              ov.w = low_bytes4(z[12], z[13], z[14], z[15]);
              if (row >= rows) ov = make_uint4(0u, 0u, 0u, 0u);
              *reinterpret_cast<uint4*>(dstc + ((size_t)bh * a.Npad + t0 + row) * D + 16 * cb) = ov;
            }
          }
        }
        const bool pass_bias = a.smooth_q && !a.q_blocks && do_kv && tid < kTok;
        if (pass_bias && do_q) {
          // Q-smoothing bias of token t0 + tid: fma chain over channels of
          // mean_q[c] * k~[c] in channel order (k~ recomputed from the tile)
          const int row = tid;
          float acc = 0.f;
          if (row < rows) {
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 8) {
              const uint4 v4 = lds<uint4>(sb + tk + swz(row, 2 * c0));
              const uint32_t uu[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                float lo, hi;
                unpack2<T>(uu[j], lo, hi);
                const int c = c0 + 2 * j;
                acc = __fmaf_rn(lds<float>(qmean + 4 * c), __fsub_rn(lo, lds<float>(kmean + 4 * c)), acc);
                acc = __fmaf_rn(lds<float>(qmean + 4 * c + 4), __fsub_rn(hi, lds<float>(kmean + 4 * c + 4)), acc);
              }
            }
          }
          a.q_bias[(size_t)bh * a.Npad + t0 + row] = acc;
        } else if (pass_bias) {
          // K/V pass with its own query heads: the bias of each of the G query
          // heads of this key/value slice (query slice bh * G + g), the same
          // chain with that head's mean read from global memory
          const int row = tid;
#pragma unroll 1
          for (int g = 0; g < a.G; ++g) {
            const float* mq = a.q_mean_g + ((size_t)bh * a.G + g) * D;
            float acc = 0.f;
            if (row < rows) {
#pragma unroll 1
              for (int c0 = 0; c0 < D; c0 += 8) {
                const uint4 v4 = lds<uint4>(sb + tk + swz(row, 2 * c0));
                const uint32_t uu[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  float lo, hi;
                  unpack2<T>(uu[j], lo, hi);
                  const int c = c0 + 2 * j;
                  acc = __fmaf_rn(__ldg(mq + c), __fsub_rn(lo, lds<float>(kmean + 4 * c)), acc);
                  acc = __fmaf_rn(__ldg(mq + c + 1), __fsub_rn(hi, lds<float>(kmean + 4 * c + 4)), acc);
                }
              }
            }
            a.q_bias[((size_t)bh * a.G + g) * a.Npad + t0 + row] = acc;
          }
        }
        if (do_kv) {
          // V: thread = word cw (channels 2cw, 2cw+1) x rows r0 .. r0+RPG-1;
          // e4m3 codes of v * (Vr / absmax_c), written transposed [c][t]
          const float mul0 = lds<float>(vmul + 8 * cw), mul1 = lds<float>(vmul + 8 * cw + 4);
          const uint64_t mul2v = f2pack(mul0, mul1);
          uint32_t c0w[RPG / 4], c1w[RPG / 4];
#pragma unroll
          for (int r = 0; r < RPG; r += 4) {
            float f0[4], f1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float lo, hi;
              unpack2<T>(lds<uint32_t>(sb + tv + o[(r + i) & 7] + 1024 * ((r + i) >> 3)), lo, hi);
              f2unpack(mul2(f2pack(lo, hi), mul2v), f0[i], f1[i]);
            }
            uint32_t w0 = __byte_perm(e4m3x2(f0[0], f0[1]), e4m3x2(f0[2], f0[3]), 0x5410);
            uint32_t w1 = __byte_perm(e4m3x2(f1[0], f1[1]), e4m3x2(f1[2], f1[3]), 0x5410);
            if (rows < kTok) {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (r0 + r + i >= rows) {
                  w0 &= ~(0xFFu << (8 * i));
                  w1 &= ~(0xFFu << (8 * i));
                }
            }
            // a zero multiplier (all-zero channel) gives code 0, never -0
            c0w[r / 4] = mul0 == 0.f ? 0u : w0;
            c1w[r / 4] = mul1 == 0.f ? 0u : w1;
          }
          uint8_t* d0 = a.vt_codes + ((size_t)bh * D + 2 * cw) * a.Npad + t0 + r0;
          uint8_t* d1 = d0 + a.Npad;
          if constexpr (RPG == 16) {
            *reinterpret_cast<uint4*>(d0) = make_uint4(c0w[0], c0w[1], c0w[2], c0w[3]);
            *reinterpret_cast<uint4*>(d1) = make_uint4(c1w[0], c1w[1], c1w[2], c1w[3]);
          } else {
            *reinterpret_cast<uint2*>(d0) = make_uint2(c0w[0], c0w[1]);
            *reinterpret_cast<uint2*>(d1) = make_uint2(c1w[0], c1w[1]);
          }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);  // this warp is done with buffer b
  }
}

// Folding the chunk partials of one slice: thread c runs channel c's chain
// over the valid chunks in chunk order.  The partials stream through shared
// memory in 16 KB pieces (bulk copies into a double buffer), so every step of
// a chain reads shared memory.  Pieces are numbered across calls: piece k
// uses buffer k & 1 with barrier parity (k >> 1) & 1.
template <int D>
struct Folder {
  static constexpr int kRows = 4096 / D;  // chunks per 16 KB piece
  float (*piece)[kRows * D];
  uint64_t* bar;
  int* abort;
  int k = 0;
  enum Op { kSum, kMax, kMin };

  SAGE_DEV void issue(const float* src, int nvalid, int p) {
    const int rows = min(kRows, nvalid - p * kRows);
    const uint32_t bytes = (uint32_t)rows * D * 4;
    const int kb = (k + p) & 1;
    mbar_arrive_expect_tx(&bar[kb], bytes);
    bulk_load(piece[kb], src + (size_t)p * kRows * D, bytes, &bar[kb]);
  }
  // Returns false (every thread) if a piece did not land in time.
  SAGE_DEV bool run(const float* src, int nvalid, Op op, float& acc) {
    const int c = threadIdx.x;
    const int npieces = (nvalid + kRows - 1) / kRows;
    acc = op == kSum ? 0.f : op == kMax ? -INFINITY : INFINITY;
    if (c == 0) {
      issue(src, nvalid, 0);
      if (npieces > 1) issue(src, nvalid, 1);
    }
    for (int p = 0; p < npieces; ++p) {
      const int kk = k + p;
      if (!__syncthreads_and(mbar_wait(&bar[kk & 1], (kk >> 1) & 1, abort))) return false;
      const int rows = min(kRows, nvalid - p * kRows);
      const float* pc = piece[kk & 1];
      if (op == kSum) {
        for (int g = 0; g < rows; ++g) acc = __fadd_rn(acc, pc[g * D + c]);
      } else if (op == kMax) {
        for (int g = 0; g < rows; ++g) acc = fmaxf(acc, pc[g * D + c]);
      } else {
        for (int g = 0; g < rows; ++g) acc = fminf(acc, pc[g * D + c]);
      }
      __syncthreads();  // buffer kk & 1 is free
      if (c == 0 && p + 2 < npieces) issue(src, nvalid, p + 2);
    }
    k += npieces;
    return true;
  }
};

// INT8/FP8 modes.  Per slice and tensor (blockIdx.y: 0 K sums, 1 |V| maxima,
// 2 Q sums): means, V scales and multipliers.
template <int D>
__global__ void __launch_bounds__(D) quant_fold_kernel(const QuantArgs a) {
  __shared__ __align__(16) float piece[2][Folder<D>::kRows * D];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_s;
  const int bh = blockIdx.x, c = threadIdx.x;
  // part plane: K sums, V maxima, Q sums (a Q-only pass folds Q sums alone)
  const int which = a.roles == kRolesQ ? 1 : blockIdx.y == 0 ? 0 : blockIdx.y == 1 ? 2 : 1;
  const int nchunks = a.Npad / 64;
  const int nvalid = (a.N + 63) / 64;
  if (c == 0) {
    abort_s = 0;
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // launched while the statistics pass may still run: wait for its partials
  grid_dep_wait();
  grid_dep_launch();
  Folder<D> f{piece, bar, &abort_s};
  const float* src = a.part + ((size_t)which * a.BH + bh) * nchunks * D;
  float acc;
  if (!f.run(src, nvalid, which == 2 ? Folder<D>::kMax : Folder<D>::kSum, acc)) {
    if (c == 0) atomicCAS(a.err, 0, kErrTileWait);
    return;
  }
  if (which == 0) {
    a.k_mean[bh * D + c] = __fdiv_rn(acc, (float)a.N);
  } else if (which == 1) {
    a.q_mean[bh * D + c] = __fdiv_rn(acc, (float)a.N);
  } else {
    a.v_scale[bh * D + c] = acc > 0.f ? __fdiv_rn(acc, a.Vr) : 0.f;
    a.v_mul[bh * D + c] = acc > 0.f ? __fdiv_rn(a.Vr, acc) : 0.f;
  }
}

// Q smoothed per 128-row block: block b = blockIdx.x of slice bh =
// blockIdx.y, thread c = channel.  Its mean is the per-slice mean's chain
// applied to the block's valid rows: the sum of the Q-sum partials of its
// chunks 2b and 2b + 1 (the second only if it holds valid rows), in order,
// from 0, divided by the number of valid rows.
template <int D>
__global__ void __launch_bounds__(D) quant_fold_qblock_kernel(const QuantArgs a) {
  const int b = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const int nchunks = a.Npad / 64, nblk = a.Npad / 128;
  // launched while the fold kernel may still run: the statistics pass it
  // waited for wrote the partials
  grid_dep_wait();
  grid_dep_launch();
  // plane 1 of the partials: Q sums [BH][Npad/64][D]
  const float* p = a.part + ((size_t)a.BH * nchunks + (size_t)bh * nchunks + 2 * b) * D + c;
  const int r0 = 128 * b, rows = min(128, a.N - r0);
  float acc = __fadd_rn(0.f, p[0]);
  if (r0 + 64 < a.N) acc = __fadd_rn(acc, p[D]);
  a.q_mean[((size_t)bh * nblk + b) * D + c] = __fdiv_rn(acc, (float)rows);
}

// Per-block Q-smoothing bias: bias row b of slice bh at key j (stored at
// q_bias[bh][j / 128][b][j % 128], key-tile-major) = the fma chain over channels
// c, in order and from 0, of mean_b[c] * RN(k[j][c] - k_mean[c]) -- the
// per-slice bias with block b's mean -- for keys j < N, and 0 for the
// padding.  A CTA computes 64 blocks x 128 keys of one slice (grid: key
// tiles, block groups, slices) from shared-memory fp32 copies of k~ for its
// keys and of the blocks' means, each row padded by 4 floats so that the
// 16-byte loads of 8 consecutive lanes fall in distinct bank groups.  Warp w
// owns blocks 8w .. 8w+7 of the group, lane l the keys l + 32 q, q < 4.
constexpr int kBiasKeys = 128, kBiasBlocks = 64, kBiasThreads = 256;

template <int D>
constexpr size_t bias_smem_bytes() {
  return (size_t)(kBiasKeys + kBiasBlocks) * (D + 4) * sizeof(float);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBiasThreads, 2) qblock_bias_kernel(const T* __restrict__ k, const QuantArgs a) {
  constexpr int RS = D + 4;  // floats per shared row
  extern __shared__ __align__(16) float bsm[];
  float* const kt = bsm;                     // [kBiasKeys][RS]
  float* const mb = bsm + kBiasKeys * RS;    // [kBiasBlocks][RS]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = blockIdx.x * kBiasKeys, b0 = blockIdx.y * kBiasBlocks, bh = blockIdx.z;
  const int nblk = a.Npad / 128;
  // the K means and block means come from the kernels before this one
  grid_dep_wait();
  grid_dep_launch();
  {
    // k~ of the CTA's keys and the group's block means (0 past the last
    // block).  Every global load is issued before the first is used: each
    // thread holds KIT 16-byte pieces of K (8 channels, always channels c0 ..
    // c0 + 7) and MIT float4 of the means.
    constexpr int PPR = D / 8, QPR = D / 4;
    constexpr int KIT = kBiasKeys * PPR / kBiasThreads, MIT = kBiasBlocks * QPR / kBiasThreads;
    static_assert(kBiasThreads % PPR == 0 && kBiasThreads % QPR == 0, "fixed column per thread");
    const int c0 = 8 * (tid % PPR), r0 = tid / PPR;
    const float* km = a.k_mean + (size_t)bh * D + c0;
    const float4 km0 = __ldg(reinterpret_cast<const float4*>(km)), km1 = __ldg(reinterpret_cast<const float4*>(km + 4));
    uint4 kraw[KIT];
#pragma unroll
    for (int it = 0; it < KIT; ++it) {
      const int j = j0 + r0 + it * (kBiasThreads / PPR);
      kraw[it] = j < a.N ? __ldg(reinterpret_cast<const uint4*>(k + ((size_t)bh * a.N + j) * D + c0))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
    const int mc0 = 4 * (tid % QPR), mr0 = tid / QPR;
    float4 mraw[MIT];
#pragma unroll
    for (int it = 0; it < MIT; ++it) {
      const int b = b0 + mr0 + it * (kBiasThreads / QPR);
      mraw[it] = b < nblk ? __ldg(reinterpret_cast<const float4*>(a.q_mean + ((size_t)bh * nblk + b) * D + mc0))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float kmv[8] = {km0.x, km0.y, km0.z, km0.w, km1.x, km1.y, km1.z, km1.w};
#pragma unroll
    for (int it = 0; it < KIT; ++it) {
      const int r = r0 + it * (kBiasThreads / PPR);
      float x[8];
      const uint32_t w4[4] = {kraw[it].x, kraw[it].y, kraw[it].z, kraw[it].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) unpack2<T>(w4[e], x[2 * e], x[2 * e + 1]);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = j0 + r < a.N ? __fsub_rn(x[e], kmv[e]) : 0.f;
      *reinterpret_cast<float4*>(kt + r * RS + c0) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(kt + r * RS + c0 + 4) = make_float4(x[4], x[5], x[6], x[7]);
    }
#pragma unroll
    for (int it = 0; it < MIT; ++it)
      *reinterpret_cast<float4*>(mb + (mr0 + it * (kBiasThreads / QPR)) * RS + mc0) = mraw[it];
  }
  __syncthreads();
  const int bw = b0 + 8 * warp;  // this warp's first block
  if (bw >= nblk) return;
  float acc[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[m][q] = 0.f;
#pragma unroll 2
  for (int c0 = 0; c0 < D; c0 += 4) {
    float4 kv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) kv[q] = *reinterpret_cast<const float4*>(kt + (lane + 32 * q) * RS + c0);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const float4 mv = *reinterpret_cast<const float4*>(mb + (8 * warp + m) * RS + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float t = acc[m][q];
        t = __fmaf_rn(mv.x, kv[q].x, t);
        t = __fmaf_rn(mv.y, kv[q].y, t);
        t = __fmaf_rn(mv.z, kv[q].z, t);
        t = __fmaf_rn(mv.w, kv[q].w, t);
        acc[m][q] = t;
      }
    }
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    if (bw + m >= nblk) break;
    // key-tile-major: [BH][key tile][block][128 keys]
    float* o = a.q_bias + (((size_t)bh * nblk + blockIdx.x) * nblk + bw + m) * kBiasKeys + lane;
#pragma unroll
    for (int q = 0; q < 4; ++q) o[32 * q] = j0 + lane + 32 * q < a.N ? acc[m][q] : 0.f;
  }
}

// NVFP4.  Per slice and tensor (blockIdx.y: 0 K, 1 V, 2 Q): the means (K;
// Q with smooth_q) and the global scale g = A / (6 * 448), A = the slice's
// max |x~| over valid tokens.  RN(x - mean) is monotone in x, so per channel
// that maximum is the larger of |RN(max - mean)| and |RN(min - mean)|.
template <int D>
__global__ void __launch_bounds__(D) quant_fold_fp4_kernel(const QuantArgs a) {
  __shared__ __align__(16) float piece[2][Folder<D>::kRows * D];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_s;
  __shared__ float red[D / 32];
  const int bh = blockIdx.x, c = threadIdx.x, y = blockIdx.y;
  const int nchunks = a.Npad / 64;
  const int nvalid = (a.N + 63) / 64;
  const size_t plane = (size_t)a.BH * nchunks * D;
  if (c == 0) {
    abort_s = 0;
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // launched while the statistics pass may still run: wait for its partials
  grid_dep_wait();
  grid_dep_launch();
  Folder<D> f{piece, bar, &abort_s};
  auto src = [&](int pl) { return a.part + pl * plane + (size_t)bh * nchunks * D; };
  bool ok = true;
  float am = 0.f;
  if (y == 1) {
    ok = f.run(src(2), nvalid, Folder<D>::kMax, am);
  } else {
    const int role = y == 0 ? 0 : 1;  // 0 K, 1 Q
    const bool has_mean = role == 0 || a.smooth_q;
    float mu = 0.f, mx, mn;
    if (has_mean) {
      float s;
      ok = f.run(src(role), nvalid, Folder<D>::kSum, s);
      mu = __fdiv_rn(s, (float)a.N);
      if (ok) (role == 0 ? a.k_mean : a.q_mean)[bh * D + c] = mu;
    }
    ok = ok && f.run(src(3 + 2 * role), nvalid, Folder<D>::kMax, mx);
    ok = ok && f.run(src(4 + 2 * role), nvalid, Folder<D>::kMin, mn);
    if (ok) {
      if (has_mean) {
        mx = __fsub_rn(mx, mu);
        mn = __fsub_rn(mn, mu);
      }
      am = fmaxf(fabsf(mx), fabsf(mn));
    }
  }
  if (!ok) {
    if (c == 0) atomicCAS(a.err, 0, kErrTileWait);
    return;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((c & 31) == 0) red[c >> 5] = am;
  __syncthreads();
  if (c == 0) {
    float A = 0.f;
    for (int i = 0; i < D / 32; ++i) A = fmaxf(A, red[i]);
    a.gscale[bh * 4 + (y == 0 ? 1 : y == 1 ? 2 : 0)] = __fdiv_rn(A, 2688.0f);
    if (y == 0) a.gscale[bh * 4 + 3] = 0.f;
  }
}

// Per-device launch facts: SM count and resident CTAs per SM.
struct LaunchFacts {
  int sms = 0, per_sm = 0;
};

template <typename T, int D, int PASS, bool FP4>
cudaError_t launch_facts(size_t smem, LaunchFacts* out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static LaunchFacts facts[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (facts[dev].sms == 0) {
    e = cudaFuncSetAttribute(quant_pass_kernel<T, D, PASS, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchFacts f;
    e = cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&f.per_sm, quant_pass_kernel<T, D, PASS, FP4>, kThreadsQ, smem);
    if (e != cudaSuccess) return e;
    if (f.per_sm < 1) return cudaErrorInvalidConfiguration;
    facts[dev] = f;
  }
  *out = facts[dev];
  return cudaSuccess;
}

template <typename T, int D, bool FP4>
cudaError_t quant_run(const void* q, const void* k, const void* v, const Problem& pb, float Vr, const WsPtrs& w,
                      cudaStream_t s) {
  QuantArgs a;
  a.q_codes = w.q_codes;
  a.k_codes = w.k_codes;
  a.vt_codes = w.vt_codes;
  a.q_scale = w.q_scale;
  a.k_scale = w.k_scale;
  a.v_scale = w.v_scale;
  a.k_mean = w.k_mean;
  a.q_mean = w.q_mean;
  a.q_bias = w.q_bias;
  a.part = w.scratch;
  a.v_mul = w.scratch + (size_t)3 * pb.BH * (pb.Npad / 64) * D;
  a.gscale = w.global_scale;
  a.err = w.error;
  a.BH = pb.BH;
  a.N = pb.N;
  a.Npad = pb.Npad;
  a.smooth_q = pb.smooth_q;
  a.Vr = Vr;
  a.n_items = pb.BH * (pb.Npad / kTok);
  a.roles = kRolesQ | kRolesKV;
  a.G = 1;
  a.q_mean_g = w.q_mean;
  a.q_blocks = pb.q_blocks;

  // 16-bit [BH][N][D] inputs seen as bytes: rows of 2D bytes, boxes of
  // 128 bytes x 64 tokens (rows past N read as zero)
  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = (uint64_t)D * 2;
  if (!make_tmap_u8_3d(&tq, q, row_bytes, pb.N, pb.BH, kBoxBytes, kTok) ||
      !make_tmap_u8_3d(&tk, k, row_bytes, pb.N, pb.BH, kBoxBytes, kTok) ||
      !make_tmap_u8_3d(&tv, v, row_bytes, pb.N, pb.BH, kBoxBytes, kTok))
    return cudaErrorInvalidValue;

  const size_t smem = QLayout<D>::kBytes + 1024;  // + alignment slack
  LaunchFacts f0, f1;
  cudaError_t e = launch_facts<T, D, kStatsPass, FP4>(smem, &f0);
  if (e != cudaSuccess) return e;
  e = launch_facts<T, D, kCodesPass, FP4>(smem, &f1);
  if (e != cudaSuccess) return e;
  const int g0 = (int)fmin((double)a.n_items, (double)f0.sms * f0.per_sm);
  const int g1 = (int)fmin((double)a.n_items, (double)f1.sms * f1.per_sm);
  if (FP4 && D == 64) {
    // rows 64..127 of the V^T scale atoms are never written: keep them 0
    e = cudaMemsetAsync(w.v_scale, 0, (size_t)pb.BH * pb.Npad * 8, s);
    if (e != cudaSuccess) return e;
  }
  // The statistics pass follows whatever the caller enqueued and launches
  // normally; the fold and the codes pass follow this library's own kernels
  // and launch programmatically (each waits for its predecessor's results).
  quant_pass_kernel<T, D, kStatsPass, FP4><<<g0, kThreadsQ, smem, s>>>(tq, tk, tv, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (FP4)
    e = launch_kernel(quant_fold_fp4_kernel<D>, dim3(pb.BH, 3), dim3(D), 0, s, true, a);
  else
    e = launch_kernel(quant_fold_kernel<D>, dim3(pb.BH, pb.smooth_q && !pb.q_blocks ? 3 : 2), dim3(D), 0, s, true, a);
  if (e != cudaSuccess) return e;
  const int nblk = pb.Npad / 128;
  if (!FP4 && pb.q_blocks) {
    // Q means per 128-row block (the fold above did K and V only)
    e = launch_kernel(quant_fold_qblock_kernel<D>, dim3(nblk, pb.BH), dim3(D), 0, s, true, a);
    if (e != cudaSuccess) return e;
  }
  e = launch_kernel(quant_pass_kernel<T, D, kCodesPass, FP4>, dim3(g1), dim3(kThreadsQ), smem, s, true, tq, tk, tv,
                    a);
  if (e != cudaSuccess || FP4 || !pb.q_blocks) return e;
  // the bias rows of the blocks (after the codes pass, which rereads the
  // inputs the statistics pass left in L2)
  const size_t bsmem = bias_smem_bytes<D>();
  e = cudaFuncSetAttribute(qblock_bias_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsmem);
  if (e != cudaSuccess) return e;
  return launch_kernel(qblock_bias_kernel<T, D>, dim3(pb.Npad / kBiasKeys, (nblk + kBiasBlocks - 1) / kBiasBlocks, pb.BH),
                       dim3(kBiasThreads), bsmem, s, true, static_cast<const T*>(k), a);
}

// Grouped key/value heads and / or separate query and key lengths (INT8/FP8
// modes): the same kernels in two passes, one over Q's slices and tokens and
// one over K/V's.  Order: Q statistics and fold (Q smoothing only), K/V
// statistics and fold, K/V codes (with the bias of every query head of each
// key/value slice, which needs the Q means), Q codes.  Every launch after the
// first is programmatic and waits for its predecessor, so each sees all
// earlier results.
// skip_q_codes: leave Q's codes and scales to the attention kernel, which
// quantizes each Q tile itself (the fused forward); only Q's statistics run.
// With equal shapes the two passes share the per-head layout's three
// partial planes (K sums 0, Q sums 1, V maxima 2).
template <typename T, int D>
cudaError_t quant_run_split(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                            const WsPtrs& w, cudaStream_t s, bool skip_q_codes) {
  const int BHq = pb.BH, BHkv = pb.bh_kv(), Npq = pb.Npad, Npk = pb.npk();
  const size_t plane_q = (size_t)BHq * (Npq / 64) * D, plane_kv = (size_t)BHkv * (Npk / 64) * D;
  const bool shared_planes = BHq == BHkv && Npq == Npk;
  QuantArgs a;
  a.q_codes = w.q_codes;
  a.k_codes = w.k_codes;
  a.vt_codes = w.vt_codes;
  a.q_scale = w.q_scale;
  a.k_scale = w.k_scale;
  a.v_scale = w.v_scale;
  a.k_mean = w.k_mean;
  a.q_mean = w.q_mean;
  a.q_bias = w.q_bias;
  a.gscale = w.global_scale;
  a.err = w.error;
  a.smooth_q = pb.smooth_q;
  a.Vr = Vr;
  a.G = pb.G;
  a.q_mean_g = w.q_mean;
  a.q_blocks = 0;
  QuantArgs aq = a, akv = a;
  aq.roles = kRolesQ;
  aq.BH = BHq;
  aq.N = pb.N;
  aq.Npad = Npq;
  aq.n_items = BHq * (Npq / kTok);
  aq.part = w.scratch;  // Q sums in plane 1 of two
  aq.v_mul = nullptr;
  akv.roles = kRolesKV;
  akv.BH = BHkv;
  akv.N = pb.nk();
  akv.Npad = Npk;
  akv.n_items = BHkv * (Npk / kTok);
  akv.part = shared_planes ? w.scratch : w.scratch + 2 * plane_q;  // K sums plane 0, V maxima plane 2
  akv.v_mul = akv.part + 3 * plane_kv;

  CUtensorMap tq, tk, tv;
  const uint64_t row_bytes = (uint64_t)D * 2;
  if (!make_tmap_u8_3d(&tq, q, row_bytes, pb.N, BHq, kBoxBytes, kTok) ||
      !make_tmap_u8_3d(&tk, k, row_bytes, pb.nk(), BHkv, kBoxBytes, kTok) ||
      !make_tmap_u8_3d(&tv, v, row_bytes, pb.nk(), BHkv, kBoxBytes, kTok))
    return cudaErrorInvalidValue;
  const size_t smem = QLayout<D>::kBytes + 1024;
  LaunchFacts f0, f1;
  cudaError_t e = launch_facts<T, D, kStatsPass, false>(smem, &f0);
  if (e != cudaSuccess) return e;
  e = launch_facts<T, D, kCodesPass, false>(smem, &f1);
  if (e != cudaSuccess) return e;
  auto grid = [](const QuantArgs& x, const LaunchFacts& f) {
    return dim3((unsigned)fmin((double)x.n_items, (double)f.sms * f.per_sm));
  };
  bool pdl = false;  // the first launch follows the caller's work normally
  if (pb.smooth_q) {
    e = launch_kernel(quant_pass_kernel<T, D, kStatsPass, false>, grid(aq, f0), dim3(kThreadsQ), smem, s, pdl, tq,
                      tq, tq, aq);
    if (e != cudaSuccess) return e;
    e = launch_kernel(quant_fold_kernel<D>, dim3(BHq, 1), dim3(D), 0, s, true, aq);
    if (e != cudaSuccess) return e;
    pdl = true;
  }
  e = launch_kernel(quant_pass_kernel<T, D, kStatsPass, false>, grid(akv, f0), dim3(kThreadsQ), smem, s, pdl, tk, tk,
                    tv, akv);
  if (e != cudaSuccess) return e;
  e = launch_kernel(quant_fold_kernel<D>, dim3(BHkv, 2), dim3(D), 0, s, true, akv);
  if (e != cudaSuccess) return e;
  e = launch_kernel(quant_pass_kernel<T, D, kCodesPass, false>, grid(akv, f1), dim3(kThreadsQ), smem, s, true, tk, tk,
                    tv, akv);
  if (e != cudaSuccess || skip_q_codes) return e;
  return launch_kernel(quant_pass_kernel<T, D, kCodesPass, false>, grid(aq, f1), dim3(kThreadsQ), smem, s, true, tq,
                       tq, tq, aq);
}

}  // namespace

// Scratch floats of the two-pass quantization with grouped key/value heads or
// separate lengths: Q partials (two planes), K/V partials (three planes), V
// multipliers.
size_t quant_scratch_floats_split(int BHq, int Npq, int BHkv, int Npk, int d) {
  return (size_t)2 * BHq * (Npq / 64) * d + (size_t)3 * BHkv * (Npk / 64) * d + (size_t)BHkv * d;
}

cudaError_t launch_quant_split(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                               const WsPtrs& w, cudaStream_t s, bool skip_q_codes) {
  if (pb.dtype == 0)
    return pb.d == 128 ? quant_run_split<__half, 128>(q, k, v, pb, Vr, w, s, skip_q_codes)
                       : quant_run_split<__half, 64>(q, k, v, pb, Vr, w, s, skip_q_codes);
  return pb.d == 128 ? quant_run_split<__nv_bfloat16, 128>(q, k, v, pb, Vr, w, s, skip_q_codes)
                     : quant_run_split<__nv_bfloat16, 64>(q, k, v, pb, Vr, w, s, skip_q_codes);
}

// Scratch floats the quantization pass needs (chunk partials, V multipliers).
size_t quant_scratch_floats(int BH, int Npad, int d, int mode) {
  if (mode == 2) return (size_t)7 * BH * (Npad / 64) * d;
  return (size_t)3 * BH * (Npad / 64) * d + (size_t)BH * d;
}

cudaError_t launch_quant_int8_fp8(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                                  const WsPtrs& w, cudaStream_t s) {
  if (pb.mode == 2) {
    if (pb.dtype == 0)
      return pb.d == 128 ? quant_run<__half, 128, true>(q, k, v, pb, Vr, w, s)
                         : quant_run<__half, 64, true>(q, k, v, pb, Vr, w, s);
    return pb.d == 128 ? quant_run<__nv_bfloat16, 128, true>(q, k, v, pb, Vr, w, s)
                       : quant_run<__nv_bfloat16, 64, true>(q, k, v, pb, Vr, w, s);
  }
  if (pb.dtype == 0)
    return pb.d == 128 ? quant_run<__half, 128, false>(q, k, v, pb, Vr, w, s)
                       : quant_run<__half, 64, false>(q, k, v, pb, Vr, w, s);
  return pb.d == 128 ? quant_run<__nv_bfloat16, 128, false>(q, k, v, pb, Vr, w, s)
                     : quant_run<__nv_bfloat16, 64, false>(q, k, v, pb, Vr, w, s);
}

}  // namespace sage
