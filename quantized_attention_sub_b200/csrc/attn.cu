// attn.cu -- fused quantized attention forward for sm_100a, INT8 QK^T and FP8
// P~V with an FP32 accumulator (SageAttention2 abstract; SageAttention2++
// summary Sec. 2, 2.1: FlashAttention-based, per-block Q/K scales, per-channel
// V scale, rescale at the end), and the same kernel with the FP16 P~V
// accumulator of SageAttention2++ Sec. 3 (F16ACC: one query tile per CTA,
// 320 threads, the 64-key f16 chunk partials folded into the fp32 row).
//
// One CTA owns two 128-query tiles of one (b, h) slice and walks the key
// tiles of 128 in order (causal: the longest query blocks launch first, see
// the grid mapping in the kernel).  Warp roles (576 threads, 18 warps):
//   warps 0-15  softmax: warps 8q..8q+7 handle query tile q; warp w reads the
//               16 TMEM lanes 32 (w%4) + 16 ((w/4)%2) .. +15 with the .16x64b
//               shape, so the two threads of a row (lanes t and t^2) sit in one
//               warp, one per 64-key half (one 64-key scale granule each).
//   warp 16     TMA producer (Q tiles once, then a 3-stage ring of K and V^T
//               tiles); owns the TMEM allocation
//   warp 17     MMA issuer (one thread): S_q = Q_q K^T with tcgen05 kind::i8
//               into TMEM, O_q += P~_q V with kind::f8f6f4 into TMEM
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 after it.
// The K tile rows and the V^T tile rows (channels) arrive in shared memory in
// pair order -- row 2i + e holds key (channel) 64e + i (d/2 e + i) -- through
// the tensor maps' strides, so that in TMEM column 2i + e of S and O belongs
// to half e: a .16x64b load hands each thread of a row one contiguous half of
// the keys and of the output channels.
// Per key tile j the two threads of row i (one per key half):
//   load their 64 S values from TMEM and free the buffer,
//   take the half's logit max and the row max with one shuffle,
//   m_new = max(m, row max), alpha = exp2(m - m_new),
//   p' = 2^d with d = t - m_new + log2(Pr), P~ = e4m3(p'),
//   wait for the previous P~V, multiply their half of the O row by alpha
//   (skipped when alpha == 1 on the whole warp), write their 64 P~ bytes into
//   the 128B-swizzled K-major shared tile the MMA reads, l_h = alpha l_h + sum p'.
// At the end l = l_0 + l_1 and O = acc * scale_v / l is cast and stored (the
// quotient through one reciprocal of l per row and an FMA correction).
// exp2 runs on the special-function unit (ex2.approx; in the FP16 mode a
// quarter on a polynomial, ex2_poly2); the logit is formed as
// fma(x, (sq sk) log2(e)/sqrt(d), ...) and Pr enters the exponent, so a P~ code
// may differ from the CPU reference's e4m3(p * Pr) in rare cases and the
// output is compared within a tolerance.
// Every wait is bounded (sage_ptx.cuh); a timeout records an error code in
// the workspace, makes the other roles stop, and the CTA frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "sage_internal.h"
#include "sage_ptx.cuh"
#include "sage_softmax.cuh"

namespace sage {

using namespace sm;

namespace {

constexpr int kStages = 3;
// Query tiles per CTA: two with the FP32 accumulator (TMEM S_0, S_1, O_0, O_1),
// one with the FP16 accumulator (TMEM S, O, H_0, H_1).
template <bool F16ACC>
struct Roles {
  static constexpr int kNQ = F16ACC ? 1 : 2;
  static constexpr int kSoftmaxWarps = 8 * kNQ;  // 8 warps x 16 rows x 2 halves per query tile
  static constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
};
constexpr uint32_t kTmemCols = 512;

// RING: the softmax warps' bias buffers (kernels with a bias) are present.
template <int D, int NQ, bool RING>
struct Smem {
  static constexpr int kQ = 128 * D;  // one Q tile (int8)
  static constexpr int kK = 128 * D;  // one K tile (int8), rows in pair order
  static constexpr int kV = D * 128;  // one V^T tile (e4m3), rows in pair order
  static constexpr int kP = 128 * 128;
  static constexpr int off_q = 0;
  static constexpr int off_k = off_q + NQ * kQ;
  static constexpr int off_v = off_k + kStages * kK;
  static constexpr int off_p = off_v + kStages * kV;  // [query tile NQ][buffer 2]
  static constexpr int off_bar = off_p + 2 * NQ * kP;
  static constexpr int off_qmx = off_bar + 256;  // fused Q: granule maxima [query tile 2][granule 4][warp 2]
  // per softmax warp, two bias buffers of one key tile: [half 0: 64 floats]
  // [16 bytes of padding][half 1: 64 floats] (the padding puts the halves'
  // 16-byte chunks in different bank groups)
  static constexpr int kBiasBuf = 528;
  static constexpr int off_bias = off_bar + 512;
  static constexpr int bytes = off_bias + (RING ? 2 * 8 * NQ * kBiasBuf : 0);
  static constexpr int alloc = bytes + 1024;  // room to align the base to 1024
};

struct AttnArgs {
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  const float* bias;  // null unless smooth_q
  const float* q_mean;  // fused Q with smooth_q: the per-channel Q means
  void* out;
  int* err;
  int N, Npad, causal, num_qblocks;     // query rows (padded), causal flag, CTAs per slice
  int Nk, Npad_k, koff;                 // keys (padded); causal: row i sees keys j <= i + koff
  int Hq, G;                            // query heads per batch, query heads per key/value head
  int grouped;  // grid (G, query blocks, B*H/G) instead of (query blocks, B*H)
  float c_log2, log2Pr;
};

// error codes: 0x100 | site
enum : int {
  kErrProducer = 0x101,
  kErrMma = 0x102,
  kErrSoftmax = 0x103,
  kErrDrain = 0x104,
  kErrProbe = 0x1FF
};

SAGE_DEV float lo_half_to_float(uint32_t u) { return __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu))); }


// The CTA's query slice and its key/value slice, read from the special
// registers each time (volatile: recomputed where used rather than held in
// registers across the key-tile loop).
SAGE_DEV int query_slice(const AttnArgs& a) {
  uint32_t x, y, z, nx;
  asm volatile("mov.u32 %0, %%ctaid.x;" : "=r"(x));
  asm volatile("mov.u32 %0, %%ctaid.y;" : "=r"(y));
  asm volatile("mov.u32 %0, %%ctaid.z;" : "=r"(z));
  asm volatile("mov.u32 %0, %%nctaid.x;" : "=r"(nx));
  return a.grouped ? (int)(z * nx + x) : (int)y;
}
SAGE_DEV int kv_slice(const AttnArgs& a, int bh) {
  return a.G == 1 ? bh : (bh / a.Hq) * (a.Hq / a.G) + (bh % a.Hq) / a.G;
}

}  // namespace

// BIAS: 0 none; 1 one bias row per slice ([BH][Npad_k]); 2 one row per
// 128-row query tile (Q smoothed per block), stored key-tile-major
// ([BH][Npad/128 key tiles][Npad/128 query tiles][128]) so that the CTAs
// of a slice, which walk the key tiles together, read neighbouring bytes.
template <int D, typename OutT, int BIAS, bool F16ACC, bool FUSED_Q>
__global__ void __launch_bounds__(Roles<F16ACC>::kThreads, 1)
    attn_i8f8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  static_assert(BIAS >= 0 && BIAS <= 2 && !(BIAS == 2 && FUSED_Q), "per-tile bias rows: two-step path only");
  constexpr bool HAS_BIAS = BIAS != 0, kTileBias = BIAS == 2;
  using R = Roles<F16ACC>;
  constexpr int kNQ = R::kNQ;
  constexpr int kSoftmaxWarps = R::kSoftmaxWarps, kProducerWarp = R::kProducerWarp, kMmaWarp = R::kMmaWarp;
  using L = Smem<D, kNQ, HAS_BIAS>;
  // TMEM columns: S_q, O_q, and (FP16 accumulator) the two 64-key chunk partials H_c
  constexpr uint32_t kColO = F16ACC ? 128u : 256u;
  constexpr uint32_t kColH = 128u + D;
  constexpr int kHalfD = D / 2;  // O columns (channels) each thread of a row rescales and stores
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + L::off_bar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 1 + kStages;
  uint64_t* v_full = bars + 1 + 2 * kStages;
  uint64_t* v_empty = bars + 1 + 3 * kStages;
  uint64_t* s_full = bars + 1 + 4 * kStages;  // [2]
  uint64_t* s_free = s_full + 2;              // [2]
  uint64_t* p_full = s_full + 4;              // [2]
  uint64_t* o_done = s_full + 6;              // [2]
  uint64_t* mma_fin = s_full + 8;
  uint64_t* q_ready = s_full + 9;             // [2] fused Q: the tile's codes are in place
  uint32_t* tmem_slot = (uint32_t*)(s_full + 11);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Grid (query blocks, B*H): one slice's CTAs launch together and share its
  // K and V in L2; causal blocks launch longest-first within the slice.
  // Grouped (causal, few CTAs per SM): (G, query blocks, B*H/G), the blocks of
  // G slices longest-first across those slices (see causal_slice_group).
  // (written so that the slice and block indices rematerialize cheaply: a
  // variant that kept them live spilled registers and ran 2 % slower)
  const int qb = a.causal ? (a.num_qblocks - 1 - (int)(a.grouped ? blockIdx.y : blockIdx.x)) : (int)blockIdx.x;
  const int bh = a.grouped ? (int)(blockIdx.z * gridDim.x + blockIdx.x) : (int)blockIdx.y;
  const int n_ktiles = a.Npad_k / 128;
  int nt[kNQ];
  int T = 0;
#pragma unroll
  for (int q = 0; q < kNQ; ++q) {
    const int qt = kNQ * qb + q;
    // causal: up to the key tile of the last visible key of the tile's last real row
    nt[q] = qt * 128 >= a.N ? 0 : (a.causal ? min(n_ktiles, (min(qt * 128 + 127, a.N - 1) + a.koff) / 128 + 1)
                                            : n_ktiles);
    T = max(T, nt[q]);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int q = 0; q < kNQ; ++q) {
      mbar_init(&s_full[q], 1);
      mbar_init(&s_free[q], 8);   // 8 softmax warps per query tile
      mbar_init(&p_full[q], 8);
      mbar_init(&o_done[q], 1);
      mbar_init(&q_ready[q], 8);
    }
    mbar_init(mma_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t qbytes = 0;
      for (int q = 0; q < kNQ; ++q) qbytes += nt[q] > 0 ? (FUSED_Q ? 2 * L::kQ : L::kQ) : 0;
      mbar_arrive_expect_tx(q_full, qbytes);
      for (int q = 0; q < kNQ; ++q) {
        if (nt[q] == 0) continue;
        if (FUSED_Q) {
          // the raw 16-bit Q tile, 128 rows x 2d bytes, into this query tile's P~
          // buffers (free until its first P~): boxes of 128 bytes x 128 rows, 128B swizzle
#pragma unroll
          for (int x = 0; x < 2 * D / 128; ++x)
            tma_load_3d(smem + L::off_p + 2 * q * L::kP + x * 128 * 128, &tm_q, q_full, x * 128, (kNQ * qb + q) * 128,
                        bh);
        } else {
          tma_load_3d(smem + L::off_q + q * L::kQ, &tm_q, q_full, 0, (kNQ * qb + q) * 128, bh);
        }
      }
      // the key/value slice of this query head
      const int bkv = kv_slice(a, bh);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % kStages, n = j / kStages;
        if (j >= kStages && !mbar_wait(&k_empty[s], (n - 1) & 1, abort_flag)) {
          fail(abort_flag, a.err, kErrProducer);
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], L::kK);
        tma_load_5d(smem + L::off_k + s * L::kK, &tm_k, &k_full[s], 0, 0, 0, j, bkv);
        issued_k = j + 1;
        if (j >= kStages && !mbar_wait(&v_empty[s], (n - 1) & 1, abort_flag)) {
          fail(abort_flag, a.err, kErrProducer);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kV);
        tma_load_4d(smem + L::off_v + s * L::kV, &tm_v, &v_full[s], j * 128, 0, 0, bkv);
        issued_v = j + 1;
      }
      // Drain: every load issued into shared memory must land before exit.
      volatile int no_abort = 0;
      if (!mbar_wait(q_full, 0, &no_abort)) atomicCAS(a.err, 0, kErrDrain);
      for (int j = max(0, issued_k - kStages); j < issued_k; ++j)
        if (!mbar_wait(&k_full[j % kStages], (j / kStages) & 1, &no_abort)) atomicCAS(a.err, 0, kErrDrain);
      for (int j = max(0, issued_v - kStages); j < issued_v; ++j)
        if (!mbar_wait(&v_full[j % kStages], (j / kStages) & 1, &no_abort)) atomicCAS(a.err, 0, kErrDrain);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(2u, 1u, 1u, 128, 128);  // s32 <- s8 x s8
      // P~V: f32 <- e4m3 x e4m3, or f16 <- e4m3 x e4m3 per 64-key chunk
      constexpr uint32_t idesc_pv = idesc_make(F16ACC ? 0u : 1u, 0u, 0u, 128, D);
      const uint32_t q_base = smem_u32(smem + L::off_q), k_base = smem_u32(smem + L::off_k);
      const uint32_t v_base = smem_u32(smem + L::off_v), p_base = smem_u32(smem + L::off_p);
      bool ok = true;
      if (FUSED_Q) {
        // the softmax warps quantize the Q tiles
        for (int q = 0; q < kNQ && ok; ++q)
          if (nt[q] > 0) ok = mbar_wait(&q_ready[q], 0, abort_flag);
      } else {
        ok = mbar_wait(q_full, 0, abort_flag);
      }
      auto issue_s = [&](int q, int j) {
        const uint32_t qa = q_base + q * L::kQ, kb = k_base + (j % kStages) * L::kK;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8(tmem + q * 128, kmajor_desc(qa + kk * 32, D), kmajor_desc(kb + kk * 32, D), idesc_s, kk > 0);
        tc_commit(&s_full[q]);
      };
      auto issue_pv = [&](int q, int j) {
        const uint32_t pa = p_base + (2 * q + (j & 1)) * L::kP, vb = v_base + (j % kStages) * L::kV;
        if (F16ACC) {
          // keys [64c, 64c + 64) into H_c: two k = 32 steps accumulated in f16
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8(tmem + kColH + (kk >> 1) * D, kmajor_desc(pa + kk * 32, 128), kmajor_desc(vb + kk * 32, 128),
                   idesc_pv, kk & 1);
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8(tmem + kColO + q * D, kmajor_desc(pa + kk * 32, 128), kmajor_desc(vb + kk * 32, 128), idesc_pv,
                   (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&o_done[q]);
      };
      if (ok) ok = mbar_wait(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int q = 0; q < kNQ; ++q)
          if (nt[q] > 0) issue_s(q, 0);
        tc_commit(&k_empty[0]);
      }
      for (int j = 0; ok && j < T; ++j) {
        const bool next_k = j + 1 < T;
        if (next_k) {
          const int s1 = (j + 1) % kStages;
          if (!(ok = mbar_wait(&k_full[s1], ((j + 1) / kStages) & 1, abort_flag))) break;
          tc_fence_after();
        }
        // next S tiles first (they need only the S buffers back), then P~V
        for (int q = 0; q < kNQ && ok; ++q) {
          if (j + 1 < nt[q]) {
            if (!(ok = mbar_wait(&s_free[q], j & 1, abort_flag))) break;
            tc_fence_after();
            issue_s(q, j + 1);
          }
        }
        if (!ok) break;
        if (next_k) tc_commit(&k_empty[(j + 1) % kStages]);
        if (!(ok = mbar_wait(&v_full[j % kStages], (j / kStages) & 1, abort_flag))) break;
        tc_fence_after();
        for (int q = 0; q < kNQ && ok; ++q) {
          if (j < nt[q]) {
            if (!(ok = mbar_wait(&p_full[q], j & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(q, j);
          }
        }
        if (!ok) break;
        tc_commit(&v_empty[j % kStages]);
      }
      if (!ok) fail(abort_flag, a.err, kErrMma);
      // Every MMA issued so far must complete before the CTA frees TMEM.
      tc_commit(mma_fin);
      volatile int no_abort = 0;
      if (!mbar_wait(mma_fin, 0, &no_abort)) atomicCAS(a.err, 0, kErrDrain);
    }
  } else if (warp < kSoftmaxWarps) {
    // ------------------------------------------------------------ softmax
    const int q = warp >> 3;                // query tile
    const int wq = warp & 7;
    const int h = (lane >> 1) & 1;          // key half and channel half of this thread
    const int r = 32 * (wq & 3) + 16 * (wq >> 2) + (lane >> 2) + 8 * (lane & 1);
    const uint32_t lane_off = (uint32_t)(32 * (wq & 3) + 16 * (wq >> 2)) << 16;
    if (nt[q] > 0) {
      const int qt = kNQ * qb + q;
      const int row = qt * 128 + r;
      float sq;
      bool ok = true;
      if (!FUSED_Q) {
        sq = a.q_scale[(size_t)bh * (a.Npad / 32) + (row >> 5)];
      } else {
        // Q quantized here (SageAttention2++ summary Sec. 2.1: per-block Q
        // scales), with the steps of the quantization pass: x~ = x - mean_q
        // (smooth_q), granule of 32 rows: a = max |x~| over valid rows, scale
        // a / 127, code = rint_even(x~ * (127 / a)); rows past N give 0.
        ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag));
        float x[kHalfD];
        float am = 0.f;
        if (ok) {
          const uint8_t* raw = smem + L::off_p + 2 * q * L::kP;
#pragma unroll
          for (int k = 0; k < kHalfD / 8; ++k) {
            // 16-byte chunk k of this half row: byte b = 2 (d/2) h + 16 k of the row
            const int b = h * D + 16 * k;
            const uint4 u = *reinterpret_cast<const uint4*>(raw + (b >> 7) * (128 * 128) + r * 128 +
                                                            ((((b >> 4) & 7) ^ (r & 7)) << 4));
            const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float lo, hi;
              if constexpr (sizeof(OutT) == 2 && std::is_same<OutT, __half>::value) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&uu[e]));
                lo = f.x;
                hi = f.y;
              } else {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uu[e]));
                lo = f.x;
                hi = f.y;
              }
              x[8 * k + 2 * e] = lo;
              x[8 * k + 2 * e + 1] = hi;
            }
          }
          if (HAS_BIAS) {
            const float* mq = a.q_mean + (size_t)bh * D + h * kHalfD;
#pragma unroll
            for (int c = 0; c < kHalfD; ++c) x[c] = __fsub_rn(x[c], __ldg(mq + c));
          }
          if (row < a.N) {
#pragma unroll
            for (int c = 0; c < kHalfD; ++c) am = fmaxf(am, fabsf(x[c]));
          }
        }
        // granule maximum: this warp's 16 rows, then the other warp of the granule
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        float* qmx = (float*)(smem + L::off_qmx) + q * 8 + (wq & 3) * 2;
        if (lane == 0) qmx[wq >> 2] = am;
        named_bar_sync(1 + q * 4 + (wq & 3), 64);
        const float ag = fmaxf(qmx[0], qmx[1]);
        sq = ag > 0.f ? __fdiv_rn(ag, 127.0f) : 0.f;
        const float inv = ag > 0.f ? __fdiv_rn(127.0f, ag) : 0.f;
        // codes into the Q operand tile (K-major, d-byte rows in the d-byte swizzle)
        uint8_t* qrow = smem + L::off_q + q * L::kQ + r * D;
#pragma unroll
        for (int k = 0; k < kHalfD / 16; ++k) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float z[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) z[i] = __fadd_rn(__fmul_rn(x[16 * k + 4 * e + i], inv), 12582912.0f);
            const uint32_t lo = __byte_perm(__float_as_uint(z[0]), __float_as_uint(z[1]), 0x0040);
            const uint32_t hi = __byte_perm(__float_as_uint(z[2]), __float_as_uint(z[3]), 0x0040);
            w4[e] = row < a.N ? __byte_perm(lo, hi, 0x5410) : 0u;
          }
          const int c = (D / 32) * h + k;  // 16-byte chunk of the code row
          const int sw = D == 128 ? (c ^ (r & 7)) : (c ^ ((r >> 1) & 3));
          *reinterpret_cast<uint4*>(qrow + (sw << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_ready[q]);
      }
      // S columns [0, 128) of this query tile (two loads of 64), O columns of this
      // tile, H_0 (H_1 is D columns further)
      const uint32_t t_s = tmem + lane_off + q * 128;
      const uint32_t t_o = tmem + lane_off + kColO + q * D;
      const uint32_t t_h = tmem + lane_off + kColH;
      uint8_t* prow0 = smem + L::off_p + 2 * q * L::kP + r * 128;  // buffer 0; buffer 1 is kP further
      const float* ksc = a.k_scale + (size_t)kv_slice(a, bh) * (a.Npad_k / 64);
      const float* bvec = !HAS_BIAS ? nullptr
                          : a.bias + (kTileBias ? ((size_t)bh * (a.Npad / 128) * a.Npad + qt * 128) : (size_t)bh * a.Npad_k) +
                                h * 64;
      // floats between the bias values of consecutive key tiles
      const int bstride = kTileBias ? a.Npad : 128;
      // m: running row max of the logits (log2 units); l: this half's running
      // sum of p' = p * Pr.
      float m = -INFINITY, l = 0.f;
      float alpha_prev = 0.f;  // FP16 accumulator: rescale factor of the tile whose partials are pending
      // FP16 accumulator, after P~V(jt) completed: acc = (alpha_jt * acc + h_0) + h_1
      // over this thread's O columns (the first tile starts from acc = 0).
      auto fold_partials = [&](int jt, float alpha_t) {
#pragma unroll 1
        for (int i = 0; i < D / 32; ++i) {
          uint32_t o[16], h0[16], h1[16];
          tmem_ld16x64b_x16(t_h + 32 * i, h0);
          tmem_ld16x64b_x16(t_h + D + 32 * i, h1);
          if (jt > 0) tmem_ld16x64b_x16(t_o + 32 * i, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float2 acc = jt > 0 ? __fmul2_rn(make_float2(u2f(o[e]), u2f(o[e + 1])), make_float2(alpha_t, alpha_t))
                                : make_float2(0.f, 0.f);
            acc = __fadd2_rn(__fadd2_rn(acc, make_float2(lo_half_to_float(h0[e]), lo_half_to_float(h0[e + 1]))),
                             make_float2(lo_half_to_float(h1[e]), lo_half_to_float(h1[e + 1])));
            o[e] = f2u(acc.x);
            o[e + 1] = f2u(acc.y);
          }
          tmem_st16x64b_x16(t_o + 32 * i, o);
        }
        tmem_st_wait();
      };
      // K scales of both 64-key granules of the tile, loaded one tile ahead
      float2 ks_next = *reinterpret_cast<const float2*>(ksc);
      // A bias row of its own per query tile (Q smoothed per block) is read
      // by this CTA alone, from DRAM: its lines (two per key half and tile)
      // are prefetched into L2 two tiles ahead.  A row shared by the slice
      // stays in L2.
      // Each softmax warp copies the next tile's 128 bias values (512 bytes,
      // 16 per lane) into its own shared-memory buffer while it works on the
      // current tile, and reads them from there.
      constexpr bool bias_prefetch = kTileBias;
      constexpr bool kBiasRing = HAS_BIAS;
      // lane's 16 bytes of key tile jj's bias values (which start at bvec - h * 64)
      // into this warp's buffer jj & 1
      auto bias_copy = [&](int jj) {
        const uint32_t ring = smem_u32(smem + L::off_bias) + (uint32_t)warp * 2 * L::kBiasBuf;
        cp_async16(ring + (jj & 1) * L::kBiasBuf + 16 * lane + (lane >= 16 ? 16 : 0),
                   bvec - h * 64 + (size_t)jj * bstride + 4 * lane);
      };
      if (bias_prefetch) {
        prefetch_l2(bvec + 32 * (lane & 1));
        if (nt[q] > 1) prefetch_l2(bvec + bstride + 32 * (lane & 1));
      }
      if constexpr (kBiasRing) {
        bias_copy(0);
        cp_async_commit();
      }
      for (int j = 0; ok && j < nt[q]; ++j) {
        const float2 ks = ks_next;
        if (j + 1 < nt[q]) ks_next = *reinterpret_cast<const float2*>(ksc + 2 * (j + 1));
        if (bias_prefetch && j + 2 < nt[q]) prefetch_l2(bvec + (size_t)(j + 2) * bstride + 32 * (lane & 1));
        if constexpr (kBiasRing) {
          // buffer (j + 1) & 1 was last read for tile j - 1, by this warp
          __syncwarp();
          if (j + 1 < nt[q]) bias_copy(j + 1);
          cp_async_commit();  // (an empty group on the last tile keeps the count)
        }
        const int kbase = j * 128 + h * 64;
        // visible keys of this row among the half's 64 form the prefix c < lim
        int lim = 64;
        if (kbase + 63 >= a.Nk || (a.causal && kbase + 63 > row + a.koff)) {
          lim = min(lim, a.Nk - kbase);
          if (a.causal) lim = min(lim, row + a.koff - kbase + 1);
        }
        // warp-uniform outcome: tcgen05.ld below is a warp-collective instruction
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[q], j & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // sr[c] = S of key 64 h + c (int32, then as float)
        uint32_t sr[64];
        tmem_ld16x64b_x32(t_s, sr);
        tmem_ld16x64b_x32(t_s + 64, sr + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[q]);

        // Logits:
        //   kf = (sq * sk) * log2(e)/sqrt(d) for this half's 64-key granule,
        //   x  = float(S) (exact: |S| <= 128 * 127^2 < 2^24),
        //   t  = x * kf  (or fma(x, kf, bias * log2(e)/sqrt(d))),
        //   m' = max - log2(Pr),  d = fma(x, kf, -m')  (or t - m'),
        //   p' = 2^d = p * Pr on the special-function unit, P~ = e4m3(p').
        // Masked keys become -inf: out of the max, and 2^-inf = +0.  (A zero
        // scale -- an all-zero granule -- is raised to the smallest normal
        // float so that masked keys stay at -inf instead of NaN.)
        const float kf = fmaxf(__fmul_rn(__fmul_rn(sq, h ? ks.y : ks.x), a.c_log2), 1.17549435e-38f);
#pragma unroll
        for (int c = 0; c < 64; ++c) sr[c] = f2u(__int2float_rn((int)sr[c]));
        if (lim < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= lim) sr[c] = 0xFF800000u;
        }
        float mt;
        if (!HAS_BIAS) {
          float ga = -INFINITY, gb = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            ga = fmax3(ga, u2f(sr[c]), u2f(sr[c + 1]));
            gb = fmax3(gb, u2f(sr[c + 2]), u2f(sr[c + 3]));
          }
          // a half with no visible key gives -inf
          mt = __fmul_rn(fmaxf(ga, gb), kf);
        } else {
          const float2 cl2 = make_float2(a.c_log2, a.c_log2);
          float ma = -INFINITY, mb = -INFINITY;
          const uint32_t bbuf = smem_u32(smem + L::off_bias) + (uint32_t)warp * 2 * L::kBiasBuf + (j & 1) * L::kBiasBuf;
          if constexpr (kBiasRing) {
            // this tile's copies (all but the group just committed) have landed
            cp_async_wait<1>();
            if constexpr (kTileBias) {
              // each lane turns its own 16 bytes into bias * log2(e)/sqrt(d)
              // (the same rounded products the loop below would form), once
              // for the warp (measured: 2 % faster with the per-tile rows,
              // 1.5 % slower with the shared row, whose loop keeps the multiply)
              const uint32_t mine = bbuf + 16 * lane + (lane >= 16 ? 16 : 0);
              const float4 b = lds_f4(mine);
              const float2 lo = __fmul2_rn(make_float2(b.x, b.y), cl2), hi = __fmul2_rn(make_float2(b.z, b.w), cl2);
              sts_f4(mine, make_float4(lo.x, lo.y, hi.x, hi.y));
            }
            __syncwarp();
          }
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const int c = 4 * c4;
            float2 bl, bh;  // bias * log2(e)/sqrt(d) of keys c .. c + 3
            const float4 bw = lds_f4(bbuf + h * 272 + 16 * c4);
            if constexpr (kTileBias) {
              bl = make_float2(bw.x, bw.y);
              bh = make_float2(bw.z, bw.w);
            } else {
              bl = __fmul2_rn(make_float2(bw.x, bw.y), cl2);
              bh = __fmul2_rn(make_float2(bw.z, bw.w), cl2);
            }
            const float2 ta = __ffma2_rn(make_float2(u2f(sr[c]), u2f(sr[c + 1])), make_float2(kf, kf), bl);
            const float2 tb = __ffma2_rn(make_float2(u2f(sr[c + 2]), u2f(sr[c + 3])), make_float2(kf, kf), bh);
            sr[c] = f2u(ta.x);
            sr[c + 1] = f2u(ta.y);
            sr[c + 2] = f2u(tb.x);
            sr[c + 3] = f2u(tb.y);
            // masked keys carry -inf
            ma = fmax3(ma, ta.x, ta.y);
            mb = fmax3(mb, tb.x, tb.y);
          }
          mt = fmaxf(ma, mb);
        }
        // the row max: the other half of the row is lane ^ 2 of this warp
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
        const float m_new = fmaxf(m, mt);
        const float alpha = ex2(__fadd_rn(m, -m_new));  // +0 on the first tile (m = -inf), 1 if the max stays
        const float mp = __fadd_rn(m_new, -a.log2Pr);
        const float2 nmp = make_float2(-mp, -mp), kf2 = make_float2(kf, kf);

        // p' = p * Pr for the 64 keys, P~ = e4m3(p') packed 4 per word and
        // stored 16 keys at a time into this tile's P buffer (the buffer was
        // last read by the P~V two tiles back, which completed before the
        // previous tile's rescale), and the sum of p'
        uint8_t* prow = prow0 + (j & 1) * L::kP;
        float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 16 * cc + 4 * e;
            const float2 ya = make_float2(u2f(sr[c]), u2f(sr[c + 1])), yb = make_float2(u2f(sr[c + 2]), u2f(sr[c + 3]));
            // d = t - m' (one rounding of x * kf - m' without bias)
            const float2 da = HAS_BIAS ? __fadd2_rn(ya, nmp) : __ffma2_rn(ya, kf2, nmp);
            const float2 db = HAS_BIAS ? __fadd2_rn(yb, nmp) : __ffma2_rn(yb, kf2, nmp);
            // FP16 mode: 2 of every 8 pairs take the polynomial, the rest the
            // special-function unit (measured: the best split with two
            // softmax warps per SM sub-partition; the FP32 mode, with four,
            // is bound by instruction issue and keeps all on the unit)
            constexpr int kPolyPairs = F16ACC ? 2 : 0;
            const float2 pa = (2 * e) < kPolyPairs ? ex2_poly2(da) : make_float2(ex2(da.x), ex2(da.y));
            const float2 pb = (2 * e + 1) < kPolyPairs ? ex2_poly2(db) : make_float2(ex2(db.x), ex2(db.y));
            sa = __fadd2_rn(sa, pa);
            sb = __fadd2_rn(sb, pb);
            pw[e] = e4m3x4(pa, pb);
          }
          *reinterpret_cast<uint4*>(prow + (((4 * h + cc) ^ (r & 7)) << 4)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
        fence_proxy_async_smem();
        if (j > 0) {
          // P~V of the previous tile must be done before its O rows are
          // rescaled (and before the next tile reuses that P buffer).
          if (!__all_sync(0xffffffffu, mbar_wait(&o_done[q], (j - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (F16ACC) {
            // fold the previous tile's FP16 partials into the FP32 accumulator
            // before this tile's P~V overwrites them
            fold_partials(j - 1, alpha_prev);
          } else if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
            for (int i = 0; i < D / 64; ++i) {
              uint32_t o[32];
              tmem_ld16x64b_x32(t_o + 64 * i, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 v2 = __fmul2_rn(make_float2(u2f(o[e]), u2f(o[e + 1])), make_float2(alpha, alpha));
                o[e] = f2u(v2.x);
                o[e + 1] = f2u(v2.y);
              }
              tmem_st16x64b_x32(t_o + 64 * i, o);
            }
            tmem_st_wait();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[q]);
        l = __fadd_rn(__fmul_rn(alpha, l), (sa.x + sa.y) + (sb.x + sb.y));
        m = m_new;
        alpha_prev = alpha;
      }
      if constexpr (kBiasRing) cp_async_wait<0>();  // no copy into this warp's buffers outlives the loop
      if (ok && !__all_sync(0xffffffffu, mbar_wait(&o_done[q], (nt[q] - 1) & 1, abort_flag))) ok = false;
      if (ok && F16ACC) {
        tc_fence_after();
        fold_partials(nt[q] - 1, alpha_prev);
      }
      // the row sum is the sum of both halves' sums (l_0 + l_1 in both threads)
      const float l_other = __shfl_xor_sync(0xffffffffu, l, 2);
      l = h == 0 ? __fadd_rn(l, l_other) : __fadd_rn(l_other, l);
      if (!ok) {
        fail(abort_flag, a.err, kErrSoftmax);
      } else {
        tc_fence_after();
        const float inv_l = __fdiv_rn(1.0f, l);
        const int bh_e = query_slice(a);
        const float* vs = a.v_scale + (size_t)kv_slice(a, bh_e) * D + h * kHalfD;
        OutT* orow = (OutT*)a.out + ((size_t)bh_e * a.N + row) * D + h * kHalfD;
#pragma unroll 1
        for (int i = 0; i < D / 64; ++i) {
          // o[e] = channel h d/2 + 32 i + e of this row
          uint32_t o[32];
          tmem_ld16x64b_x32(t_o + 64 * i, o);
          tmem_ld_wait();
          if (row < a.N) {
            uint32_t hh[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = 32 * i + 2 * e;
              hh[e] = pack2<OutT>(div_by(__fmul_rn(u2f(o[2 * e]), __ldg(vs + c)), l, inv_l),
                                  div_by(__fmul_rn(u2f(o[2 * e + 1]), __ldg(vs + c + 1)), l, inv_l));
            }
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              *reinterpret_cast<uint4*>(orow + 32 * i + 8 * v4) =
                  make_uint4(hh[4 * v4], hh[4 * v4 + 1], hh[4 * v4 + 2], hh[4 * v4 + 3]);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // The MMA thread has waited for its last MMA and the producer for its last
  // load, so no asynchronous write targets this CTA's TMEM or shared memory.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kProducerWarp) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ debug
// One 128x128 INT32 tile S = Q^ K^T through the same TMA + kind::i8 + TMEM
// path as the attention kernel.  128 threads; out row = query.
template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, int bh,
                    int q_tile, int k_tile, int32_t* out, int* err) {
  __shared__ __align__(1024) uint8_t sq[128 * D];
  __shared__ __align__(1024) uint8_t sk[128 * D];
  __shared__ uint64_t bar_load, bar_mma;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar_load, 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int no_abort = 0;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar_load, 2 * 128 * D);
    tma_load_3d(sq, &tm_q, &bar_load, 0, q_tile * 128, bh);
    tma_load_3d(sk, &tm_k, &bar_load, 0, k_tile * 128, bh);
    if (mbar_wait(&bar_load, 0, &no_abort)) {
      tc_fence_after();
      constexpr uint32_t idesc_s = idesc_make(2u, 1u, 1u, 128, 128);
      const uint32_t qa = smem_u32(sq), kb = smem_u32(sk);
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        mma_i8(tmem, kmajor_desc(qa + kk * 32, D), kmajor_desc(kb + kk * 32, D), idesc_s, kk > 0);
    } else {
      abort_flag = 1;
      atomicCAS(err, 0, kErrProducer);
    }
    tc_commit(&bar_mma);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_mma, 0, &no_abort));
  tc_fence_after();
  if (!ok) atomicCAS(err, 0, kErrMma);
  if (ok && !abort_flag) {
    const uint32_t t = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = warp * 32 + lane;
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      uint32_t r[32];
      tmem_ld32(t + 32 * i, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) out[row * 128 + 32 * i + e] = (int32_t)r[e];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ------------------------------------------------------------------ timeout probe
// Waits on an mbarrier that nothing arrives at: the bounded wait runs out,
// the error word is set and the kernel returns (exercises the failure path
// without a fault or a hang).
__global__ void timeout_probe_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, &abort_flag)) atomicCAS(err, 0, kErrProbe);
  }
}

// ------------------------------------------------------------------ launchers
// Q tiles (and the debug tile's K) in row order.
static bool make_maps(const WsPtrs& w, const Problem& pb, CUtensorMap* mq, CUtensorMap* mk) {
  return make_tmap_u8_3d(mq, w.q_codes, pb.d, pb.Npad, pb.BH, pb.d, 128) &&
         make_tmap_u8_3d(mk, w.k_codes, pb.d, pb.Npad, pb.BH, pb.d, 128);
}

// The attention kernel's K and V^T tiles in pair order: shared-memory row
// 2i + e holds key 64e + i of the 128-key tile (K), channel (d/2) e + i (V^T).
//   K   [BHkv][Npk][d]: dims (d, e = 2, i = 64, tile, bh), box (d, 2, 64, 1, 1)
//   V^T [BHkv][d][Npk]: dims (Npk, e = 2, i = d/2, bh), box (128, 2, d/2, 1)
static bool make_pair_maps(const WsPtrs& w, const Problem& pb, CUtensorMap* mk, CUtensorMap* mv) {
  const uint64_t D = (uint64_t)pb.d, Np = (uint64_t)pb.npk();
  const uint64_t kd[5] = {D, 2, 64, Np / 128, (uint64_t)pb.bh_kv()};
  const uint64_t ks[4] = {64 * D, D, 128 * D, Np * D};
  const uint32_t kb[5] = {(uint32_t)D, 2, 64, 1, 1};
  const uint64_t vd[4] = {Np, 2, D / 2, (uint64_t)pb.bh_kv()};
  const uint64_t vs[3] = {(D / 2) * Np, Np, D * Np};
  const uint32_t vb[4] = {128, 2, (uint32_t)(D / 2), 1};
  return make_tmap_u8_nd(mk, w.k_codes, 5, kd, ks, kb, (int)D) && make_tmap_u8_nd(mv, w.vt_codes, 4, vd, vs, vb, 128);
}

template <int D, typename OutT, int BIAS, bool F16ACC, bool FUSED_Q>
static cudaError_t run_attn(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnArgs& a,
                            int BH, cudaStream_t s) {
  auto kern = attn_i8f8_kernel<D, OutT, BIAS, F16ACC, FUSED_Q>;
  using L = Smem<D, Roles<F16ACC>::kNQ, BIAS != 0>;
  // set on every launch: the attribute is per device, and a cached flag would
  // be shared by host threads and devices
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::alloc);
  if (e != cudaSuccess) return e;
  const int G = causal_slice_group(BH, 2.0 * a.Npad_k * D, 80e6);
  const dim3 grid = a.grouped ? dim3(G, a.num_qblocks, BH / G) : dim3(a.num_qblocks, BH);
  kern<<<grid, Roles<F16ACC>::kThreads, L::alloc, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

// q_raw: null, or the caller's 16-bit Q [BH, N, d] for the fused variant
// (then mq maps it as bytes: rows of 2d bytes, boxes of 128 bytes x 128 rows).
static cudaError_t launch_attn(const WsPtrs& w, const void* q_raw, void* out, const Problem& pb, float Pr,
                               cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const bool fused = q_raw != nullptr;
  const bool qmap = fused ? make_tmap_u8_3d(&mq, q_raw, 2 * (uint64_t)pb.d, pb.N, pb.BH, 128, 128)
                          : make_tmap_u8_3d(&mq, w.q_codes, pb.d, pb.Npad, pb.BH, pb.d, 128);
  if (!qmap || !make_pair_maps(w, pb, &mk, &mv)) return cudaErrorInvalidValue;
  AttnArgs a;
  a.q_scale = w.q_scale;
  a.k_scale = w.k_scale;
  a.v_scale = w.v_scale;
  a.bias = pb.smooth_q ? w.q_bias : nullptr;
  a.q_mean = w.q_mean;
  a.out = out;
  a.err = w.error;
  a.N = pb.N;
  a.Npad = pb.Npad;
  a.Nk = pb.nk();
  a.Npad_k = pb.npk();
  a.koff = pb.nk() - pb.N;
  a.Hq = pb.hq();
  a.G = pb.G;
  a.causal = pb.causal;
  const bool f16 = pb.mode == 1;
  const int nq = f16 ? 1 : 2;
  a.num_qblocks = (pb.Npad / 128 + nq - 1) / nq;
  // Causal CTAs differ in length (1 to num_qblocks tile pairs).  When the
  // longest is a sizeable share of one SM's work -- 2 * num_qblocks * 148 over
  // B*H * num_qblocks * (num_qblocks + 1) above 5 % -- launch longest-first
  // across slices (measured: llm_prefill B1 H32 N8192 0.570 -> 0.511 ms);
  // with many CTAs per SM the per-slice order keeps K and V shared in L2.
  a.grouped = pb.causal && (double)pb.BH * (a.num_qblocks + 1) < 5920.0;
  a.c_log2 = (float)(1.4426950408889634 / sqrt((double)pb.d));
  a.log2Pr = (float)log2((double)Pr);
  const bool bias = a.bias != nullptr;
  if (pb.q_blocks && (fused || !bias)) return cudaErrorInvalidValue;
#define SAGE_RUN(DD, TT, BB, FF, QQ) run_attn<DD, TT, BB, FF, QQ>(mq, mk, mv, a, pb.BH, s)
#define SAGE_RUN_Q(DD, TT, BB, FF) (fused ? SAGE_RUN(DD, TT, BB, FF, true) : SAGE_RUN(DD, TT, BB, FF, false))
#define SAGE_RUN_F(DD, TT, BB) (f16 ? SAGE_RUN_Q(DD, TT, BB, true) : SAGE_RUN_Q(DD, TT, BB, false))
  // per-tile bias rows: the two-step path only (the fused Q prologue subtracts one mean per slice)
#define SAGE_RUN_T(DD, TT) (f16 ? SAGE_RUN(DD, TT, 2, true, false) : SAGE_RUN(DD, TT, 2, false, false))
#define SAGE_RUN_B(DD, TT) (!bias ? SAGE_RUN_F(DD, TT, 0) : pb.q_blocks ? SAGE_RUN_T(DD, TT) : SAGE_RUN_F(DD, TT, 1))
  if (pb.d == 128) return pb.dtype == 0 ? SAGE_RUN_B(128, __half) : SAGE_RUN_B(128, __nv_bfloat16);
  return pb.dtype == 0 ? SAGE_RUN_B(64, __half) : SAGE_RUN_B(64, __nv_bfloat16);
#undef SAGE_RUN_B
#undef SAGE_RUN_T
#undef SAGE_RUN_F
#undef SAGE_RUN_Q
#undef SAGE_RUN
}

cudaError_t launch_attn_i8f8(const WsPtrs& w, void* out, const Problem& pb, float Pr, cudaStream_t s) {
  return launch_attn(w, nullptr, out, pb, Pr, s);
}

cudaError_t launch_attn_i8f8_fused_q(const WsPtrs& w, const void* q_raw, void* out, const Problem& pb, float Pr,
                                     cudaStream_t s) {
  return launch_attn(w, q_raw, out, pb, Pr, s);
}

cudaError_t launch_timeout_probe(const WsPtrs& w, cudaStream_t s) {
  timeout_probe_kernel<<<1, 32, 0, s>>>(w.error);
  return cudaGetLastError();
}

cudaError_t launch_debug_qk(const WsPtrs& w, const Problem& pb, int bh, int q_tile, int k_tile, int32_t* out,
                            cudaStream_t s) {
  CUtensorMap mq, mk;
  if (!make_maps(w, pb, &mq, &mk)) return cudaErrorInvalidValue;
  if (pb.d == 128)
    debug_qk_kernel<128><<<1, 128, 0, s>>>(mq, mk, bh, q_tile, k_tile, out, w.error);
  else
    debug_qk_kernel<64><<<1, 128, 0, s>>>(mq, mk, bh, q_tile, k_tile, out, w.error);
  return cudaGetLastError();
}

}  // namespace sage
