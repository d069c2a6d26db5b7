// attn_fp4.cu -- the NVFP4 mode's tensor-core path (SageAttention3 abstract:
// microscaling FP4 attention on Blackwell FP4 tensor cores).
//
// Operands in shared memory: e2m1 codes packed two per byte, K-major rows of
// 64 bytes (d = 128) in the 64-byte TMA swizzle.  Block scales (ue4m3, one
// per 16 elements along the contraction axis) come from the workspace in the
// 512-byte atoms tcgen05.cp copies into TMEM (32x128b, broadcast to the four
// lane quadrants); tcgen05.mma kind::mxf4nvf4 (K = 64 per instruction) reads
// them from TMEM and accumulates in FP32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_internal.h"
#include "sage_ptx.cuh"
#include "sage_softmax.cuh"

namespace sage {

using namespace sm;

namespace {

constexpr int kErrFp4Load = 0x301;  // a debug tile load did not land in time
constexpr int kErrFp4Mma = 0x302;   // a debug MMA did not complete in time

// One S tile (128 queries x 128 keys) of one slice, d = 128: the raw
// block-scaled dot products sum_c (q_c sq_c)(k_c sk_c), in FP32.
__global__ void __launch_bounds__(128)
    debug_fp4_s_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const uint8_t* __restrict__ sfq_atoms, const uint8_t* __restrict__ sfk_atoms, int bh,
                       int tiles, int q_tile, int k_tile, float* out, int* err) {
  __shared__ __align__(1024) uint8_t sq[128 * 64];
  __shared__ __align__(1024) uint8_t sk[128 * 64];
  __shared__ __align__(128) uint8_t sfq[2 * 512];
  __shared__ __align__(128) uint8_t sfk[2 * 512];
  __shared__ __align__(8) uint64_t bar_load, bar_mma;
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
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  constexpr uint32_t kColSfq = 128, kColSfk = 136;
  volatile int no_abort = 0;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar_load, 2 * 128 * 64 + 2 * 1024);
    tma_load_3d(sq, &tm_q, &bar_load, 0, q_tile * 128, bh);
    tma_load_3d(sk, &tm_k, &bar_load, 0, k_tile * 128, bh);
    bulk_load(sfq, sfq_atoms + ((size_t)bh * tiles + q_tile) * 1024, 1024, &bar_load);
    bulk_load(sfk, sfk_atoms + ((size_t)bh * tiles + k_tile) * 1024, 1024, &bar_load);
    if (mbar_wait(&bar_load, 0, &no_abort)) {
      tc_fence_after();
      for (int ka = 0; ka < 2; ++ka) {
        tmem_cp_sf(tmem + kColSfq + 4 * ka, sf_atom_desc(smem_u32(sfq + 512 * ka)));
        tmem_cp_sf(tmem + kColSfk + 4 * ka, sf_atom_desc(smem_u32(sfk + 512 * ka)));
      }
      constexpr uint32_t idesc = idesc_fp4(128, 128);
      const uint32_t qa = smem_u32(sq), kb = smem_u32(sk);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
        mma_fp4(tmem, kmajor_desc(qa + kk * 32, 64), kmajor_desc(kb + kk * 32, 64), idesc, tmem + kColSfq + 4 * kk,
                tmem + kColSfk + 4 * kk, kk > 0);
    } else {
      abort_flag = 1;
      atomicCAS(err, 0, kErrFp4Load);
    }
    tc_commit(&bar_mma);
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_mma, 0, &no_abort));
  tc_fence_after();
  if (!ok) atomicCAS(err, 0, kErrFp4Mma);
  if (ok && !abort_flag) {
    const uint32_t t = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = warp * 32 + lane;
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      uint32_t r[32];
      tmem_ld32(t + 32 * i, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) out[row * 128 + 32 * i + e] = __uint_as_float(r[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}


// ------------------------------------------------------------------ attention
// One CTA owns one 128-query tile of one (b, h) slice (d = 128) and walks the
// key tiles of 128 in order.  Warp roles (320 threads, 10 warps):
//   warps 0-7   softmax: warpgroup h = warp / 4 handles key half h (keys
//               [64h, 64h + 64) of every tile = one K = 64 MMA step);
//               thread <-> row <-> TMEM lane
//   warp 8      TMA producer (Q once, then a 3-stage ring of K and V^T tiles,
//               each with its block-scale atoms); owns the TMEM allocation
//   warp 9      MMA issuer (one thread): copies scale atoms into TMEM
//               (tcgen05.cp), S = Q K^T and O += P~ V with kind::mxf4nvf4
// TMEM (256 columns, two CTAs per SM): S [0,64) holds one 64-key half of a
// tile at a time (S = Q K_h^T, N = 64: the half's threads load it into
// registers and free it for the other half), O [64,192), block scales from
// 192: Q, K and V (two slots each, alternating by tile), P~ (per buffer).
// The K scales of half h are the copied atom's columns 2h, 2h+1.
// Per key tile j, the two threads of row i (one per key half):
//   load their 64 S values, take the half's logit max, exchange it,
//   m_new = max(m, both halves' max), alpha = exp2(m - m_new),
//   p = exp2(t - m_new) on the special-function unit (the argument in the
//   INT8 mode's steps), l_h = alpha l_h + sum p,
//   per 16 keys: bs = ue4m3(max p / (6 g_p)) (an FMA-corrected quotient),
//   r = 1 / (g_p dec(bs)) (from a table of the 128 scale codes),
//   P~ = e2m1(p r): 32 bytes of codes into the 64-byte swizzled P~ row and
//   one 32-bit word of four scales into TMEM (tcgen05.st),
//   wait for the previous P~V, multiply their half of the O row by alpha.
// At the end l = l_0 + l_1 and O = acc * (g_p g_v) / l (one reciprocal of l
// per row and an FMA correction per output).
// Every wait is bounded; a timeout records an error code in the workspace,
// makes the other roles stop, and the CTA frees its TMEM.
constexpr int kStagesF = 3;
constexpr int kSoftmaxWarpsF = 8, kProducerWarpF = 8, kMmaWarpF = 9;
constexpr int kThreadsF = 320;
constexpr uint32_t kTmemColsF = 256;
constexpr uint32_t kColS = 0, kColO = 64, kColSfq = 192, kColSfk = 200, kColSfv = 216, kColSfp = 232;

struct SmemF {
  static constexpr int kTile = 128 * 64;  // 128 rows x 64 bytes (d = 128 or 128 keys of e2m1)
  static constexpr int kSf = 1024;        // two scale atoms
  static constexpr int off_q = 0;
  static constexpr int off_sfq = off_q + kTile;
  static constexpr int off_k = off_sfq + kSf;  // 1024-aligned
  static constexpr int off_sfk = off_k + kStagesF * kTile;
  static constexpr int off_v = off_sfk + kStagesF * kSf;
  static constexpr int off_sfv = off_v + kStagesF * kTile;
  static constexpr int off_p = off_sfv + kStagesF * kSf;  // [buffer 2]
  static constexpr int off_bar = off_p + 2 * kTile;
  static constexpr int off_x = off_bar + 256;  // [parity 2][half 2][row 128] floats
  static constexpr int off_rtab = off_x + 2 * 2 * 128 * 4;  // [128] P~ block reciprocals
  static constexpr int off_bias = off_rtab + 128 * 4;         // [softmax warp 8][buffer 2][64 floats]
  static constexpr int bytes = off_bias + 8 * 2 * 256;
  static constexpr int alloc = bytes + 1024;
};
static_assert(SmemF::off_k % 1024 == 0 && SmemF::off_v % 1024 == 0 && SmemF::off_p % 1024 == 0, "tile alignment");

struct AttnF4Args {
  const uint8_t* sfq;  // scale atoms, 1024 bytes per (slice, 128-row tile)
  const uint8_t* sfk;
  const uint8_t* sfv;
  const float* gscale;  // [BH][4]
  const float* bias;    // null unless smooth_q
  void* out;
  int* err;
  int N, Npad, causal;
  int grouped;  // grid (G, query tiles, B*H/G) instead of (query tiles, B*H)
  float c_log2;
};

enum : int { kErrProducerF = 0x311, kErrMmaF = 0x312, kErrSoftmaxF = 0x313, kErrDrainF = 0x314 };

template <typename OutT, bool HAS_BIAS>
__global__ void __launch_bounds__(kThreadsF, 2)
    attn_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnF4Args a) {
  using L = SmemF;
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + L::off_bar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStagesF;
  uint64_t* v_full = k_full + 2 * kStagesF;
  uint64_t* v_empty = k_full + 3 * kStagesF;
  uint64_t* s_full = k_full + 4 * kStagesF;  // [half 2]
  uint64_t* s_free = s_full + 2;             // [half 2]
  uint64_t* p_full = s_full + 4;             // [2]
  uint64_t* o_done = s_full + 6;
  uint64_t* x_bar = s_full + 7;  // [2 parities]
  uint64_t* mma_fin = s_full + 9;
  uint32_t* tmem_slot = (uint32_t*)(s_full + 10);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* xch = (float*)(smem + L::off_x);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_ktiles = a.Npad / 128;
  // Grid (query tiles, B*H): one slice's CTAs together (K and V in L2),
  // causal tiles longest-first within the slice; grouped (G, query tiles,
  // B*H/G): longest-first across G slices at a time (see causal_slice_group).
  const int qi = a.grouped ? (int)blockIdx.y : (int)blockIdx.x;
  const int qt = a.causal ? (n_ktiles - 1 - qi) : qi;
  const int bh = a.grouped ? (int)(blockIdx.z * gridDim.x + blockIdx.x) : (int)blockIdx.y;
  const int T = a.causal ? qt + 1 : n_ktiles;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStagesF; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoftmaxWarpsF / 2);  // the four warps of one half
      mbar_init(&p_full[b], kSoftmaxWarpsF);
      mbar_init(&x_bar[b], 256);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 128) {
    // P~ block reciprocal for every non-negative ue4m3 scale code b:
    // RN(1 / RN(g_p * dec(b))), 0 for a zero scale (all 16 p of the block 0)
    const float sd = e4m3_to_f32(threadIdx.x);
    reinterpret_cast<float*>(smem + L::off_rtab)[threadIdx.x] =
        sd > 0.f ? __fdiv_rn(1.0f, __fmul_rn(__fdiv_rn(1.0f, 2688.0f), sd)) : 0.f;
  }
  if (warp == kProducerWarpF) {
    tmem_alloc(tmem_slot, kTmemColsF);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarpF) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const size_t tile0 = (size_t)bh * n_ktiles;  // scale atoms of this slice
      mbar_arrive_expect_tx(q_full, L::kTile + L::kSf);
      tma_load_3d(smem + L::off_q, &tm_q, q_full, 0, qt * 128, bh);
      bulk_load(smem + L::off_sfq, a.sfq + (tile0 + qt) * L::kSf, L::kSf, q_full);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % kStagesF, n = j / kStagesF;
        if (j >= kStagesF && !mbar_wait(&k_empty[s], (n - 1) & 1, abort_flag)) {
          fail(abort_flag, a.err, kErrProducerF);
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], L::kTile + L::kSf);
        tma_load_3d(smem + L::off_k + s * L::kTile, &tm_k, &k_full[s], 0, j * 128, bh);
        bulk_load(smem + L::off_sfk + s * L::kSf, a.sfk + (tile0 + j) * L::kSf, L::kSf, &k_full[s]);
        issued_k = j + 1;
        if (j >= kStagesF && !mbar_wait(&v_empty[s], (n - 1) & 1, abort_flag)) {
          fail(abort_flag, a.err, kErrProducerF);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kTile + L::kSf);
        tma_load_3d(smem + L::off_v + s * L::kTile, &tm_v, &v_full[s], j * 64, 0, bh);
        bulk_load(smem + L::off_sfv + s * L::kSf, a.sfv + (tile0 + j) * L::kSf, L::kSf, &v_full[s]);
        issued_v = j + 1;
      }
      // Drain: every load issued into shared memory must land before exit.
      volatile int no_abort = 0;
      if (!mbar_wait(q_full, 0, &no_abort)) atomicCAS(a.err, 0, kErrDrainF);
      for (int j = max(0, issued_k - kStagesF); j < issued_k; ++j)
        if (!mbar_wait(&k_full[j % kStagesF], (j / kStagesF) & 1, &no_abort)) atomicCAS(a.err, 0, kErrDrainF);
      for (int j = max(0, issued_v - kStagesF); j < issued_v; ++j)
        if (!mbar_wait(&v_full[j % kStagesF], (j / kStagesF) & 1, &no_abort)) atomicCAS(a.err, 0, kErrDrainF);
    }
  } else if (warp == kMmaWarpF) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_fp4(128, 64);   // one 64-key half of S
      constexpr uint32_t idesc_pv = idesc_fp4(128, 128);  // O += P~ V, N = d
      const uint32_t q_base = smem_u32(smem + L::off_q), k_base = smem_u32(smem + L::off_k);
      const uint32_t v_base = smem_u32(smem + L::off_v), p_base = smem_u32(smem + L::off_p);
      const uint32_t sfk_base = smem_u32(smem + L::off_sfk), sfv_base = smem_u32(smem + L::off_sfv);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int ka = 0; ka < 2; ++ka)
          tmem_cp_sf(tmem + kColSfq + 4 * ka, sf_atom_desc(smem_u32(smem + L::off_sfq) + 512 * ka));
      }
      // S(j) half h: keys [64h, 64h + 64) of tile j (rows 64h.. of the K tile;
      // their scales are columns 2h, 2h+1 of the copied atoms)
      auto issue_s = [&](int j, int h) {
        const int s = j % kStagesF;
        const uint32_t kb = k_base + s * L::kTile + h * 64 * 64, sfk = kColSfk + 8 * (j & 1);
        if (h == 0)
          for (int ka = 0; ka < 2; ++ka)
            tmem_cp_sf(tmem + sfk + 4 * ka, sf_atom_desc(sfk_base + s * L::kSf + 512 * ka));
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_fp4(tmem + kColS, kmajor_desc(q_base + kk * 32, 64), kmajor_desc(kb + kk * 32, 64), idesc_s,
                  tmem + kColSfq + 4 * kk, tmem + sfk + 4 * kk + 2 * h, kk > 0);
        tc_commit(&s_full[h]);
      };
      auto issue_pv = [&](int j) {
        const int s = j % kStagesF;
        const uint32_t pa = p_base + (j & 1) * L::kTile, vb = v_base + s * L::kTile, sfv = kColSfv + 8 * (j & 1);
        for (int ka = 0; ka < 2; ++ka)
          tmem_cp_sf(tmem + sfv + 4 * ka, sf_atom_desc(sfv_base + s * L::kSf + 512 * ka));
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_fp4(tmem + kColO, kmajor_desc(pa + kk * 32, 64), kmajor_desc(vb + kk * 32, 64), idesc_pv,
                  tmem + kColSfp + 8 * (j & 1) + 4 * kk, tmem + sfv + 4 * kk, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(o_done);
      };
      // the S buffer passes S(j)_0 -> S(j)_1 -> S(j+1)_0 -> ..., each issued
      // once the previous half has been loaded by its threads
      if (ok) ok = mbar_wait(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if ((ok = mbar_wait(&s_free[0], 0, abort_flag))) {
          tc_fence_after();
          issue_s(0, 1);
          tc_commit(&k_empty[0]);
        }
      }
      for (int j = 0; ok && j < T; ++j) {
        const bool next = j + 1 < T;
        const int s1 = (j + 1) % kStagesF;
        if (next) {
          if (!(ok = mbar_wait(&k_full[s1], ((j + 1) / kStagesF) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&s_free[1], j & 1, abort_flag))) break;  // S(j)_1 loaded
          tc_fence_after();
          issue_s(j + 1, 0);
        }
        if (!(ok = mbar_wait(&v_full[j % kStagesF], (j / kStagesF) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        issue_pv(j);
        tc_commit(&v_empty[j % kStagesF]);
        if (next) {
          if (!(ok = mbar_wait(&s_free[0], (j + 1) & 1, abort_flag))) break;  // S(j+1)_0 loaded
          tc_fence_after();
          issue_s(j + 1, 1);
          tc_commit(&k_empty[s1]);
        }
      }
      if (!ok) fail(abort_flag, a.err, kErrMmaF);
      // Every MMA issued so far must complete before the CTA frees TMEM.
      tc_commit(mma_fin);
      volatile int no_abort = 0;
      if (!mbar_wait(mma_fin, 0, &no_abort)) atomicCAS(a.err, 0, kErrDrainF);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int h = warp >> 2, w4 = warp & 3;
    const int r = threadIdx.x & 127;
    const int row = qt * 128 + r;
    const uint32_t lane_off = (uint32_t)(w4 * 32) << 16;
    const uint32_t t_o = tmem + lane_off + kColO + h * 64;
    uint8_t* prow0 = smem + L::off_p + r * 64;  // buffer 0; buffer 1 is kTile further
    const float* bvec = HAS_BIAS ? a.bias + (size_t)bh * a.Npad + h * 64 : nullptr;
    const float4 gsc = *reinterpret_cast<const float4*>(a.gscale + (size_t)bh * 4);  // g_q, g_k, g_v, 0
    // (a zero global scale -- an all-zero Q or K slice -- is raised to the
    // smallest normal float so that masked keys stay at -inf instead of NaN)
    const float kf = fmaxf(__fmul_rn(__fmul_rn(gsc.x, gsc.y), a.c_log2), 1.17549435e-38f);
    const float gp = __fdiv_rn(1.0f, 2688.0f);  // P~ global scale 1 / (6 * 448)
    const float six_gp = __fmul_rn(6.0f, gp);
    const float inv_six_gp = __fdiv_rn(1.0f, six_gp);
    const float* rtab = reinterpret_cast<const float*>(smem + L::off_rtab);
    const int swz = (r >> 1) & 3;  // 64-byte swizzle of this row's 16-byte chunks
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // With Q smoothing each softmax warp copies the next key tile's 64 bias
    // values of its key half (256 bytes, 16 per lane of the first 16) into
    // its own shared-memory buffer while it works on the current tile.
    const uint32_t bring = smem_u32(smem + L::off_bias) + (uint32_t)warp * 512;
    if constexpr (HAS_BIAS) {
      if (lane < 16) cp_async16(bring + 16 * lane, bvec + 4 * lane);
      cp_async_commit();
    }
    for (int j = 0; j < T; ++j) {
      if constexpr (HAS_BIAS) {
        __syncwarp();  // buffer (j + 1) & 1 was last read for tile j - 1
        if (j + 1 < T && lane < 16) cp_async16(bring + ((j + 1) & 1) * 256 + 16 * lane, bvec + (j + 1) * 128 + 4 * lane);
        cp_async_commit();
      }
      const int kbase = j * 128 + h * 64;
      int lim = 64;
      if (kbase + 63 >= a.N || (a.causal && j == qt)) {
        lim = min(lim, a.N - kbase);
        if (a.causal) lim = min(lim, row - kbase + 1);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[h], j & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[64];
      const uint32_t t_s = tmem + lane_off + kColS;
      tmem_ld32(t_s, sr);
      tmem_ld32(t_s + 32, sr + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[h]);

      // t = x kf (or fma(x, kf, bias log2(e)/sqrt(d))), the INT8 mode's steps
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
        mt = __fmul_rn(fmaxf(ga, gb), kf);
      } else {
        // this tile's copies (all but the group just committed) have landed
        cp_async_wait<1>();
        __syncwarp();
        const uint32_t bsm = bring + (j & 1) * 256;
        const float2 cl2 = make_float2(a.c_log2, a.c_log2);
        float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 bv = lds_f4(bsm + 16 * c4);
          const int c = 4 * c4;
          const float2 ta = __ffma2_rn(make_float2(u2f(sr[c]), u2f(sr[c + 1])), make_float2(kf, kf),
                                       __fmul2_rn(make_float2(bv.x, bv.y), cl2));
          const float2 tb = __ffma2_rn(make_float2(u2f(sr[c + 2]), u2f(sr[c + 3])), make_float2(kf, kf),
                                       __fmul2_rn(make_float2(bv.z, bv.w), cl2));
          sr[c] = f2u(ta.x);
          sr[c + 1] = f2u(ta.y);
          sr[c + 2] = f2u(tb.x);
          sr[c + 3] = f2u(tb.y);
          ma = fmax3(ma, ta.x, ta.y);
          mb = fmax3(mb, tb.x, tb.y);
        }
        mt = fmaxf(ma, mb);
      }
      float* xs = xch + (j & 1) * 256;
      xs[h * 128 + r] = mt;
      mbar_arrive(&x_bar[j & 1]);
      if (!__all_sync(0xffffffffu, mbar_wait(&x_bar[j & 1], (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      mt = fmaxf(mt, xs[(h ^ 1) * 128 + r]);
      const float m_new = fmaxf(m, mt);
      const float alpha = ex2(__fadd_rn(m, -m_new));
      const float2 nm2 = make_float2(-m_new, -m_new), kf2 = make_float2(kf, kf);

      // p for the 64 keys, then per 16 keys the FP4 block: P~ codes into this
      // tile's P buffer (last read by the P~V two tiles back, complete before
      // the previous tile's rescale) and the four scales into TMEM
      uint8_t* prow = prow0 + (j & 1) * L::kTile;
      float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
      uint32_t cw[4];
      uint32_t sfw = 0;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float p[16];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 16 * cc + 4 * e;
          // d = t - m_new (without bias in one rounding: fma(x, kf, -m_new))
          const float2 xa = make_float2(u2f(sr[c]), u2f(sr[c + 1])), xb = make_float2(u2f(sr[c + 2]), u2f(sr[c + 3]));
          const float2 da = HAS_BIAS ? __fadd2_rn(xa, nm2) : __ffma2_rn(xa, kf2, nm2);
          const float2 db = HAS_BIAS ? __fadd2_rn(xb, nm2) : __ffma2_rn(xb, kf2, nm2);
          const float2 pa = make_float2(ex2(da.x), ex2(da.y)), pb = make_float2(ex2(db.x), ex2(db.y));
          sa = __fadd2_rn(sa, pa);
          sb = __fadd2_rn(sb, pb);
          p[4 * e] = pa.x;
          p[4 * e + 1] = pa.y;
          p[4 * e + 2] = pb.x;
          p[4 * e + 3] = pb.y;
        }
        float am = 0.f;
#pragma unroll
        for (int e = 0; e < 16; e += 2) am = fmax3(am, p[e], p[e + 1]);
        // bs = ue4m3(am / (6 g_p)).  The quotient is formed as q0 = am * RN(1/c)
        // with one FMA correction (Markstein's division by a correctly rounded
        // reciprocal); over every float am in [0, 1] (p <= 1) it gives the same
        // e4m3 code as the correctly rounded quotient (exhaustive check; the
        // quotients differ only below the e4m3 range, for subnormal am).
        const float q0 = __fmul_rn(am, inv_six_gp);
        const float qd = __fmaf_rn(__fmaf_rn(-six_gp, q0, am), inv_six_gp, q0);
        const uint32_t bs = e4m3x2(qd, 0.f) & 0xFFu;
        const float rr = rtab[bs & 0x7Fu];  // p >= 0: bs is a non-negative code
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 v = __fmul2_rn(make_float2(p[e], p[e + 1]), make_float2(rr, rr));
          p[e] = v.x;
          p[e + 1] = v.y;
        }
        cw[2 * (cc & 1)] = e2m1x8(p);
        cw[2 * (cc & 1) + 1] = e2m1x8(p + 8);
        sfw |= bs << (8 * cc);
        if (cc & 1)  // a 16-byte chunk (32 keys) is complete
          *reinterpret_cast<uint4*>(prow + (((2 * h + (cc >> 1)) ^ swz) << 4)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      }
      tmem_st1(tmem + lane_off + kColSfp + 8 * (j & 1) + 4 * h + w4, sfw);
      fence_proxy_async_smem();
      if (j > 0) {
        // P~V of the previous tile must be done before its O rows are rescaled
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int i = 0; i < 2; ++i) {
            uint32_t o[32];
            tmem_ld32(t_o + 32 * i, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v2 = __fmul2_rn(make_float2(u2f(o[e]), u2f(o[e + 1])), make_float2(alpha, alpha));
              o[e] = f2u(v2.x);
              o[e + 1] = f2u(v2.y);
            }
            tmem_st32(t_o + 32 * i, o);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
      l = __fadd_rn(__fmul_rn(alpha, l), (sa.x + sa.y) + (sb.x + sb.y));
      m = m_new;
    }
    if constexpr (HAS_BIAS) cp_async_wait<0>();  // no copy into this warp's buffers outlives the loop
    if (ok && !__all_sync(0xffffffffu, mbar_wait(o_done, (T - 1) & 1, abort_flag))) ok = false;
    if (ok) {
      const int jx = T;
      float* xs = xch + (jx & 1) * 256;
      xs[h * 128 + r] = l;
      mbar_arrive(&x_bar[jx & 1]);
      if (!__all_sync(0xffffffffu, mbar_wait(&x_bar[jx & 1], (jx >> 1) & 1, abort_flag))) ok = false;
      else l = h == 0 ? __fadd_rn(l, xs[128 + r]) : __fadd_rn(xs[r], l);
    }
    if (!ok) {
      fail(abort_flag, a.err, kErrSoftmaxF);
    } else {
      tc_fence_after();
      const float gpv = __fmul_rn(gp, gsc.z);
      const float inv_l = __fdiv_rn(1.0f, l);
      OutT* orow = (OutT*)a.out + ((size_t)bh * a.N + row) * D + h * 64;
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {
        uint32_t o[32];
        tmem_ld32(t_o + 32 * i, o);
        tmem_ld_wait();
        if (row < a.N) {
          uint32_t hh[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            hh[e] = pack2<OutT>(div_by(__fmul_rn(u2f(o[2 * e]), gpv), l, inv_l),
                                div_by(__fmul_rn(u2f(o[2 * e + 1]), gpv), l, inv_l));
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            *reinterpret_cast<uint4*>(orow + 32 * i + 8 * v4) =
                make_uint4(hh[4 * v4], hh[4 * v4 + 1], hh[4 * v4 + 2], hh[4 * v4 + 3]);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kProducerWarpF) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemColsF);
  }
}

template <typename OutT, bool HAS_BIAS>
cudaError_t run_attn_fp4(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const AttnF4Args& a,
                         int BH, int ntiles, cudaStream_t s) {
  auto kern = attn_fp4_kernel<OutT, HAS_BIAS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SmemF::alloc);
  if (e != cudaSuccess) return e;
  // packed K and V codes: 64 + 64 bytes per token of a slice
  const int G = causal_slice_group(BH, 128.0 * a.Npad, 80e6);
  const dim3 grid = a.grouped ? dim3(G, ntiles, BH / G) : dim3(ntiles, BH);
  kern<<<grid, kThreadsF, SmemF::alloc, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fp4(const WsPtrs& w, void* out, const Problem& pb, cudaStream_t s) {
  if (pb.d != 128) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  // packed codes: Q, K [BH][Npad][64 bytes]; V^T [BH][128][Npad/2 bytes]; boxes 64 bytes x 128 rows
  if (!make_tmap_u8_3d(&mq, w.q_codes, 64, pb.Npad, pb.BH, 64, 128) ||
      !make_tmap_u8_3d(&mk, w.k_codes, 64, pb.Npad, pb.BH, 64, 128) ||
      !make_tmap_u8_3d(&mv, w.vt_codes, pb.Npad / 2, 128, pb.BH, 64, 128))
    return cudaErrorInvalidValue;
  AttnF4Args a;
  a.sfq = reinterpret_cast<const uint8_t*>(w.q_scale);
  a.sfk = reinterpret_cast<const uint8_t*>(w.k_scale);
  a.sfv = reinterpret_cast<const uint8_t*>(w.v_scale);
  a.gscale = w.global_scale;
  a.bias = pb.smooth_q ? w.q_bias : nullptr;
  a.out = out;
  a.err = w.error;
  a.N = pb.N;
  a.Npad = pb.Npad;
  a.causal = pb.causal;
  // causal: longest-first across slices when the longest CTA is a sizeable
  // share of one SM's work (two CTAs per SM; as for the INT8/FP8 kernel)
  a.grouped = pb.causal && (double)pb.BH * (pb.Npad / 128 + 1) < 11840.0;
  a.c_log2 = (float)(1.4426950408889634 / sqrt((double)pb.d));
  const int ntiles = pb.Npad / 128;
  const bool bias = a.bias != nullptr;
  if (pb.dtype == 0)
    return bias ? run_attn_fp4<__half, true>(mq, mk, mv, a, pb.BH, ntiles, s)
                : run_attn_fp4<__half, false>(mq, mk, mv, a, pb.BH, ntiles, s);
  return bias ? run_attn_fp4<__nv_bfloat16, true>(mq, mk, mv, a, pb.BH, ntiles, s)
              : run_attn_fp4<__nv_bfloat16, false>(mq, mk, mv, a, pb.BH, ntiles, s);
}

cudaError_t launch_debug_fp4_s(const WsPtrs& w, const Problem& pb, int bh, int q_tile, int k_tile, float* out,
                               cudaStream_t s) {
  CUtensorMap mq, mk;
  // packed codes [BH][Npad][64 bytes], boxes of 64 bytes x 128 rows (64-byte swizzle)
  if (!make_tmap_u8_3d(&mq, w.q_codes, 64, pb.Npad, pb.BH, 64, 128) ||
      !make_tmap_u8_3d(&mk, w.k_codes, 64, pb.Npad, pb.BH, 64, 128))
    return cudaErrorInvalidValue;
  debug_fp4_s_kernel<<<1, 128, 0, s>>>(mq, mk, reinterpret_cast<const uint8_t*>(w.q_scale),
                                       reinterpret_cast<const uint8_t*>(w.k_scale), bh, pb.Npad / 128, q_tile,
                                       k_tile, out, w.error);
  return cudaGetLastError();
}

}  // namespace sage
