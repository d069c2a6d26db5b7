// sage_softmax.cuh -- device helpers shared by the attention kernels: the
// method's exp2 (the same definition the CPU reference computation uses),
// saturating fma, packed conversions and TMEM access shapes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sage_ptx.cuh"

namespace sage {
namespace sm {

// Give up: tell the CTA's other roles to stop and record the first error code.
SAGE_DEV void fail(volatile int* abort_flag, int* err, int code) {
  *abort_flag = 1;
  atomicCAS(err, 0, code);
}

// 1.5 * 2^23: for |S| < 2^22 the bits (S + kMagicI) read as a float equal
// kMagicF + S exactly (|S| <= 128 * 127^2 < 2^21 here).
constexpr uint32_t kMagicI = 0x4B400000u;
constexpr float kMagicF = 12582912.0f;

SAGE_DEV float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2 of the method, the same definition the CPU reference computation uses.
// The argument is carried as g = (d + 127) / 256 saturated to [0, 1]; then
// k = floor(256 g) (the round-down fma with 1.5*2^23 gives 1.5*2^23 + k
// exactly, so k sits in the low byte of its bits), f = 256 g - k, 2^f by a
// degree-3 polynomial with constant term 1 (Remez fit of the relative error,
// max 8.6e-5; its values lie in [1, 2), so its exponent field is 127), and
// the exponent field replaced by k: 2^f * 2^(k - 127).  Exact at integer d;
// d <= -127 gives +0.  Every caller keeps d < 129 (k <= 255).
// Two equivalent ways to set that exponent are kept, since they schedule
// differently: a bit-field insert of k (y = 1.5*2^23 + k), or adding
// (k - 127) << 23 to the bits of 2^f (y = 1.5*2^23 - 127 + k); the kernels
// pick per instantiation whichever measured faster.
constexpr float kE1 = 0x1.63e658p-1f, kE2 = 0x1.d2378ap-3f, kE3 = 0x1.3baaa6p-4f;
constexpr float kMg = 12582912.0f;
constexpr float kMgAdd = 12582912.0f - 127.0f;

// r with its exponent field (bits 23..30) replaced by the low byte of y's bits.
SAGE_DEV float set_exponent(float r, float y) {
  uint32_t d;
  asm("bfi.b32 %0, %1, %2, 23, 8;" : "=r"(d) : "r"(__float_as_uint(y)), "r"(__float_as_uint(r)));
  return __uint_as_float(d);
}

SAGE_DEV float sat_fma(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

SAGE_DEV float exp2g(float g) {
  const float y = __fmaf_rd(g, 256.0f, kMg);
  const float f = __fmaf_rn(g, 256.0f, -__fadd_rn(y, -kMg));
  float r = __fmaf_rn(kE3, f, kE2);
  r = __fmaf_rn(r, f, kE1);
  r = __fmaf_rn(r, f, 1.0f);
  return set_exponent(r, y);
}

// exp2 of a plain argument d (used for the rescale factor alpha).
SAGE_DEV float exp2m(float d) { return exp2g(__saturatef(__fmul_rn(__fadd_rn(d, 127.0f), 0x1p-8f))); }

// The same as exp2g on a pair, with the packed f32x2 ALU operations; BFI
// selects the exponent insertion (the results are identical).
template <bool BFI = true>
SAGE_DEV float2 exp2g2(float2 g) {
  constexpr float M = BFI ? kMg : kMgAdd;
  const float2 y = __ffma2_rd(g, make_float2(256.0f, 256.0f), make_float2(M, M));
  const float2 k = __fadd2_rn(y, make_float2(-M, -M));
  const float2 f = __ffma2_rn(g, make_float2(256.0f, 256.0f), make_float2(-k.x, -k.y));
  float2 r = __ffma2_rn(make_float2(kE3, kE3), f, make_float2(kE2, kE2));
  r = __ffma2_rn(r, f, make_float2(kE1, kE1));
  r = __ffma2_rn(r, f, make_float2(1.0f, 1.0f));
  if (BFI) return make_float2(set_exponent(r.x, y.x), set_exponent(r.y, y.y));
  return make_float2(__uint_as_float(__float_as_uint(r.x) + (__float_as_uint(y.x) << 23)),
                     __uint_as_float(__float_as_uint(r.y) + (__float_as_uint(y.y) << 23)));
}

// Four floats -> four e4m3 codes in one word (round to nearest even,
// saturate to +-448); a.x lands in the low byte.
SAGE_DEV uint32_t e4m3x4(float2 a, float2 b) {
  uint32_t w;
  asm("{\n\t.reg .b16 lo, hi;\n\tcvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\tmov.b32 %0, {lo, hi};\n\t}"
      : "=r"(w)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return w;
}

// 32 lanes x 32 columns whose 32-bit cells each hold one f16 accumulator in
// the low half: thread t gets 16 registers, register i = columns (2i, 2i+1).
SAGE_DEV void tmem_ld16_pack16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.pack::16b.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
SAGE_DEV float2 h2f2(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}

SAGE_DEV float u2f(uint32_t u) { return __uint_as_float(u); }
SAGE_DEV uint32_t f2u(float f) { return __float_as_uint(f); }

template <typename OutT>
SAGE_DEV uint32_t pack2(float a, float b);
template <>
SAGE_DEV uint32_t pack2<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
SAGE_DEV uint32_t pack2<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}


}  // namespace sm
}  // namespace sage
