// Softmax arithmetic of the tcgen05 attention kernel: MUFU exp2, bf16
// packing and the packed two-lane fp32 FMA of sm_100.
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
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
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

}  // namespace smx
}  // namespace bsa
