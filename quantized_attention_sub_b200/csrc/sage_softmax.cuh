// sage_softmax.cuh -- device helpers shared by the attention kernels: the
// softmax exponential on the special-function unit, packed conversions, TMEM
// access shapes and the abort helper.
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

// 2^x on the special-function unit (ex2.approx, subnormal results flushed to 0).
SAGE_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

// 2^d for two arguments on the FMA and ALU pipes, to share the softmax's
// exponentials with the special-function unit.  d is clamped to -127 (masked
// keys, d = -inf, give +0), split as d = n + f with n = rint(d) (adding
// 1.5 * 2^23 leaves n in the low bits) and f in [-1/2, 1/2]; 2^f is a degree-5
// polynomial with p(0) = 1 fitted by Remez exchange for least relative error
// on [-1/2, 1/2] (at most 4.9e-7 evaluated in fp32, comparable to ex2.approx),
// and n is added to the exponent field.  For d >= -127 the result is 2^d to
// that accuracy (a denormal or +0 below 2^-126); d is at most 2^9 here.
SAGE_DEV float2 ex2_poly2(float2 d) {
  const float2 lo = make_float2(fmaxf(d.x, -127.0f), fmaxf(d.y, -127.0f));
  const float2 t = __fadd2_rn(lo, make_float2(kMagicF, kMagicF));
  const float2 f = __fadd2_rn(lo, __fadd2_rn(make_float2(kMagicF, kMagicF), make_float2(-t.x, -t.y)));
  float2 q = __ffma2_rn(f, make_float2(0x1.23a604p-10f, 0x1.23a604p-10f), make_float2(0x1.3cbea8p-7f, 0x1.3cbea8p-7f));
  q = __ffma2_rn(q, f, make_float2(0x1.c74322p-5f, 0x1.c74322p-5f));
  q = __ffma2_rn(q, f, make_float2(0x1.ebfa4ep-3f, 0x1.ebfa4ep-3f));
  q = __ffma2_rn(q, f, make_float2(0x1.62e39ep-1f, 0x1.62e39ep-1f));
  const float2 p = __ffma2_rn(q, f, make_float2(1.0f, 1.0f));
  // the bits of t are kMagicI + n: shifted left by 23 only n << 23 remains
  return make_float2(u2f(f2u(p.x) + (f2u(t.x) << 23)), u2f(f2u(p.y) + (f2u(t.y) << 23)));
}

// a / b from a correctly rounded reciprocal inv = RN(1/b): q = a * inv, then
// one FMA correction (Markstein's division).  The correctly rounded quotient
// while the residual a - b q does not underflow; a last-bit difference at
// worst below that.
SAGE_DEV float div_by(float a, float b, float inv) {
  const float q = __fmul_rn(a, inv);
  return __fmaf_rn(__fmaf_rn(-b, q, a), inv, q);
}

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
