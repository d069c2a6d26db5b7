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

namespace sage {

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

}  // namespace

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
