// Softmax arithmetic of the tcgen05 attention kernel: MUFU exp2, an FMA-pipe
// exp2, bf16 packing and the packed two-lane fp32 arithmetic of sm_100.
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

// 2^x for two lanes on the FMA pipe (keeping the MUFU pipe for the other
// scores): x = n + f with n = round(x) (adding and subtracting 1.5 * 2^23
// leaves n in the low mantissa bits) and f in [-1/2, 1/2], 2^f by the cubic
// of minimax relative error 7.5e-5 (coefficients from exp2_poly_fit.py next
// to this file, far below the 2^-9 of the bf16 weights it feeds), and n added
// to the exponent field.  x is clamped at -126 so the result stays a normal
// float; below that the weight is negligible beside the row's largest (2^-126
// instead of a smaller value).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 j = fadd2(x, make_float2(kRound, kRound));
  const float2 n = fsub2(j, make_float2(kRound, kRound));
  const float2 f = fsub2(x, n);
  float2 p = ffma2(f, make_float2(0.05517149344086647f, 0.05517149344086647f),
                   make_float2(0.24261093139648438f, 0.24261093139648438f));
  p = ffma2(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
  p = ffma2(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(j.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(j.y) << 23)));
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

}  // namespace smx
}  // namespace bsa
