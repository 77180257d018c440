// Fractal token reorder and its inverse (NABLA summary, Metodologia 1).
//
// Pure data movement, HBM bound: every token row (d bf16 = 128 or 256 bytes)
// is read once and written once with 16-byte vector accesses.  A CTA moves
// kRows consecutive positions p of one (b, head); threads of a row cover its
// 16-byte vectors, so both the gathered source rows and the contiguous
// destination run are full 128-byte lines.
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 64;

template <bool kInverse>
__global__ void __launch_bounds__(kThreads) reorder_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           Dims g) {
  const int vec = g.d / 8;                    // 16-byte vectors per row
  const int rows_per_pass = kThreads / vec;
  // heads fastest: CTAs that run together move the same positions of every
  // head, i.e. adjacent rows of the same model-order tokens
  const int head = blockIdx.x % g.heads;
  const int b = blockIdx.y;
  const int c = threadIdx.x % vec;
  const int p0 = (blockIdx.x / g.heads) * kRows;
  const size_t bh = (size_t)b * g.heads + head;
#pragma unroll 4
  for (int r = threadIdx.x / vec; r < kRows; r += rows_per_pass) {
    const int p = p0 + r;
    if (p >= g.Npad) break;
    const size_t kidx = (bh * g.Npad + p) * vec + c;                        // kernel-order vector
    if (p < g.N) {
      const int n = fractal_token(p, g.H, g.W, g.P);
      const size_t midx = (((size_t)b * g.N + n) * g.heads + head) * vec + c;  // model-order vector
      if (kInverse) {
        dst[midx] = __ldcs(src + kidx);
      } else {
        dst[kidx] = __ldcs(src + midx);
      }
    } else if (!kInverse) {
      dst[kidx] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace

cudaError_t launch_reorder(const Dims& g, const void* x_bnhd, void* y_bhnd, cudaStream_t st) {
  dim3 grid((unsigned)(g.heads * ((g.Npad + kRows - 1) / kRows)), g.B);
  reorder_kernel<false><<<grid, kThreads, 0, st>>>((const uint4*)x_bnhd, (uint4*)y_bhnd, g);
  return cudaGetLastError();
}

cudaError_t launch_inverse_reorder(const Dims& g, const void* y_bhnd, void* x_bnhd, cudaStream_t st) {
  dim3 grid((unsigned)(g.heads * ((g.Npad + kRows - 1) / kRows)), g.B);
  reorder_kernel<true><<<grid, kThreads, 0, st>>>((const uint4*)y_bhnd, (uint4*)x_bnhd, g);
  return cudaGetLastError();
}

}  // namespace bsa
