// Softmax arithmetic of the tcgen05 attention kernel: MUFU exp2, bf16
// packing, the packed two-lane fp32 instructions of sm_100, and a software
// exp2 on the FMA pipe.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace bsa {
namespace smx {

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Packed two-lane fp32 arithmetic of sm_100 (one instruction for both lanes).
__device__ __forceinline__ uint64_t f2_bits(float2 a) { return *reinterpret_cast<uint64_t*>(&a); }
__device__ __forceinline__ float2 bits_f2(uint64_t b) { return *reinterpret_cast<float2*>(&b); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
// acc + the two bf16 halves of w (exact bf16 values, fp32 sums).
__device__ __forceinline__ float add_bf16x2(float acc, uint32_t w) {
  unsigned short lo, hi;
  asm("mov.b32 {%0, %1}, %2;\n" : "=h"(lo), "=h"(hi) : "r"(w));
  asm("add.rn.f32.bf16 %0, %1, %0;\n" : "+f"(acc) : "h"(lo));
  asm("add.rn.f32.bf16 %0, %1, %0;\n" : "+f"(acc) : "h"(hi));
  return acc;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for two lanes on the FMA pipe, keeping the MUFU pipe free for the
// others.  Cody-Waite range reduction x = n + f, n = rint(x), |f| <= 1/2
// (rint by adding and subtracting 1.5 * 2^23), then a cubic in f fitted for
// minimal relative error on [-1/2, 1/2] (7.5e-5; exp2_poly_fit.py next to this
// file), and n added to the exponent field.  x is clamped below at -125 so
// the result stays a normal float (2^-125 instead of a smaller value: far
// below what one bf16 weight of a row can resolve).  Inputs here are <= 8.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 n = fsub2(t, make_float2(kRound, kRound));
  const float2 f = fsub2(x, n);
  float2 p = ffma2(f, make_float2(0.05517132207751274f, 0.05517132207751274f),
                   make_float2(0.24261054396629333f, 0.24261054396629333f));
  p = ffma2(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
  p = ffma2(p, f, make_float2(0.9999281167984009f, 0.9999281167984009f));
  // the low bits of t hold n (two's complement): shifted into the exponent
  const uint32_t e0 = __float_as_uint(t.x) << 23, e1 = __float_as_uint(t.y) << 23;
  return make_float2(__uint_as_float(__float_as_uint(p.x) + e0), __uint_as_float(__float_as_uint(p.y) + e1));
}

}  // namespace smx
}  // namespace bsa
