// quant_static.cu -- sage_quantize_qkv_static: the quantization pass for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not
// wanted -- inside a CUDA-graph capture that must not grow the memory pool,
// plugins whose host framework owns every allocation, or real-time loops that
// may not call the allocator.  Such a caller can still hand over its inputs
// and one output buffer, but not the statistics scratch area the regular
// entry point expects inside the workspace.  Here that scratch lives in a
// file-scope device array instead, of a fixed maximum size, which every GPU
// that loads this part of the library keeps until the process exits.
#include <mutex>

#include "sage_internal.h"

namespace sage {

// 16 MiB of statistics partials: 3 * BH * (Npad/64) * d + BH * d floats.
constexpr size_t kStaticScratchFloats = (size_t)4 << 20;

static __device__ __align__(256) float g_static_scratch[kStaticScratchFloats];

// Device address of g_static_scratch, looked up once per device.
static float* static_scratch_ptr(int device, cudaError_t* err) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static float* ptrs[kMaxDevices] = {};
  if (device < 0 || device >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[device]) {
    void* p = nullptr;
    // the calling thread's current device is `device`
    *err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    ptrs[device] = (float*)p;
  }
  *err = cudaSuccess;
  return ptrs[device];
}

size_t static_scratch_floats() { return kStaticScratchFloats; }

cudaError_t launch_quant_static(const void* q, const void* k, const void* v, const Problem& pb, float Vr,
                                WsPtrs w, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  float* scratch = static_scratch_ptr(dev, &e);
  if (!scratch) return e;
  w.scratch = scratch;
  return launch_quant_int8_fp8(q, k, v, pb, Vr, w, s);
}

}  // namespace sage
