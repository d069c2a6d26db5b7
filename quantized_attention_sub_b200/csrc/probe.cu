// probe.cu -- tensor-core rate probe: back-to-back tcgen05.mma on operand
// tiles resident in shared memory, one CTA per SM, for each instruction kind
// the attention kernels issue.  It measures the denominators of the roofline
// fractions the library reports: the dense INT8, FP8 (FP32 and FP16
// accumulator), BF16 and block-scaled FP4 rates of this GPU, and the ratio of
// the FP16-accumulator FP8 rate to the FP32-accumulator one, which the
// SageAttention2++ summary (Sec. 2.2, Table 1) gives as 2x on the GPUs it
// targets.
//
// Shape: M = 128, N = 256 per instruction (cta_group::1), four K steps of 32
// bytes each per iteration (K = 128 INT8/FP8 elements, 64 BF16, 256 FP4), the
// accumulator in TMEM columns [0, 256).  N = 256 keeps the shared-memory
// operand traffic (12 KB per instruction) below the read bandwidth at the
// nominal 8-bit rate.  The operand bytes are a fixed pattern that is a valid,
// finite value in every format; block scales (FP4) are 1.0.
#include "sage_internal.h"
#include "sage_ptx.cuh"

namespace sage {

namespace {

constexpr int kProbeN = 256;
constexpr uint32_t kProbeCols = 512;  // D [0, 256), FP4 scales of A at 256, of B at 264
constexpr uint32_t kColSfa = 256, kColSfb = 264;

// D[tmem] (+)= A * B^T, BF16 x BF16 -> FP32 (kind::f16).
SAGE_DEV void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int KIND>
__device__ __forceinline__ void issue(uint32_t tmem, uint64_t ad, uint64_t bd, uint32_t acc) {
  if constexpr (KIND == kProbeI8) {
    mma_i8(tmem, ad, bd, idesc_make(2u, 1u, 1u, 128, kProbeN), acc);
  } else if constexpr (KIND == kProbeF8F32) {
    mma_f8(tmem, ad, bd, idesc_make(1u, 0u, 0u, 128, kProbeN), acc);
  } else if constexpr (KIND == kProbeF8F16) {
    mma_f8(tmem, ad, bd, idesc_make(0u, 0u, 0u, 128, kProbeN), acc);
  } else if constexpr (KIND == kProbeBF16) {
    mma_bf16(tmem, ad, bd, idesc_make(1u, 1u, 1u, 128, kProbeN), acc);
  } else {
    mma_fp4(tmem, ad, bd, idesc_fp4(128, kProbeN), tmem + kColSfa, tmem + kColSfb, acc);
  }
}

}  // namespace

// A (16 KB), B (32 KB), room to align to 1024; requested as 120 KB so that
// one CTA fits per SM (each takes the SM's 512 TMEM columns)
constexpr int kProbeSmem = 120 * 1024;
static_assert(128 * 128 + kProbeN * 128 + 1024 <= kProbeSmem, "probe tiles exceed the shared memory request");

template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sa = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sb = sa + 128 * 128;
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  // 0x22: INT8 34, e4m3 0.15625, bf16 pair 0x2222 (a small normal), e2m1 pair 1.0
  const uint4 pattern = make_uint4(0x22222222u, 0x22222222u, 0x22222222u, 0x22222222u);
  for (int i = threadIdx.x; i < 128 * 128 / 16; i += blockDim.x) reinterpret_cast<uint4*>(sa)[i] = pattern;
  for (int i = threadIdx.x; i < kProbeN * 128 / 16; i += blockDim.x) reinterpret_cast<uint4*>(sb)[i] = pattern;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kProbeCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (KIND == kProbeFP4) {
    // ue4m3 1.0 (0x38) in every scale byte of A (columns 256..259) and B
    // (264..271), each warp writing its own 32-lane quadrant
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (uint32_t c = 0; c < 16; ++c) tmem_st1(tmem + lane_off + kColSfa + c, 0x38383838u);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        issue<KIND>(tmem, kmajor_desc(a0 + 32 * kk, 128), kmajor_desc(b0 + 32 * kk, 128), (it | kk) ? 1u : 0u);
    }
    tc_commit(&bar);
    volatile int no_abort = 0;
    if (!mbar_wait(&bar, 0, &no_abort)) atomicCAS(err, 0, 0x1F0 | KIND);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kProbeCols);
}

template <int KIND>
static cudaError_t run_rate(int ctas, int iters, int* err, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
  if (e != cudaSuccess) return e;
  mma_rate_kernel<KIND><<<ctas, 128, kProbeSmem, s>>>(iters, err);
  return cudaGetLastError();
}

cudaError_t launch_mma_rate(int kind, int ctas, int iters, int* err, cudaStream_t s) {
  switch (kind) {
    case kProbeI8: return run_rate<kProbeI8>(ctas, iters, err, s);
    case kProbeF8F32: return run_rate<kProbeF8F32>(ctas, iters, err, s);
    case kProbeF8F16: return run_rate<kProbeF8F16>(ctas, iters, err, s);
    case kProbeBF16: return run_rate<kProbeBF16>(ctas, iters, err, s);
    case kProbeFP4: return run_rate<kProbeFP4>(ctas, iters, err, s);
    default: return cudaErrorInvalidValue;
  }
}

double mma_rate_ops(int kind, int ctas, int iters) {
  // K elements per instruction: 32 bytes of K per step
  const double k = kind == kProbeBF16 ? 16.0 : (kind == kProbeFP4 ? 64.0 : 32.0);
  return 2.0 * 128.0 * kProbeN * k * 4.0 * (double)iters * (double)ctas;
}

}  // namespace sage
