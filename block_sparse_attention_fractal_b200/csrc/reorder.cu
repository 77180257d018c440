// Fractal token reorder and its inverse (NABLA summary, Metodologia 1), and
// the reorder of Q and K fused with their block mean-pooling (Metodologia 2,
// "Submuestreo").
//
// Pure data movement, HBM bound: every token row (d bf16 = 128 or 256 bytes)
// is read once and written once with 16-byte vector accesses.  One CTA moves
// one block of `BS` consecutive kernel-order positions of one (tensor, b,
// head); threads of a row cover its 16-byte vectors, so both the gathered
// model-order rows and the contiguous kernel-order run are whole 128-byte
// lines.  The block's token indices are computed once per row into shared
// memory, and every thread issues all its loads before its first store, so
// each SM keeps BS * d * 2 bytes per resident CTA in flight (the latency of
// one load is paid once per block, not once per row).  CTAs are numbered heads
// fastest: the CTAs that run together move the same positions of every head,
// i.e. the neighbouring rows of the same model-order tokens.
//
// Any other order of the tokens (a position -> token table, e.g. the Hilbert
// curve of order.cu) runs through the same kernels in place of the fractal
// formula.
//
// The pooled variant also sums each column of the block's valid rows in
// double (exact for bf16 inputs: no rounding unless a block mixes values more
// than 2^38 apart) and writes the block mean: qbar [bh][I][d] row-major for
// Q, kbar transposed [bh][d][I] for K (the layouts the mask kernel reads).
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 256;

struct Tensors {
  const uint4* src[2];
  uint4* dst[2];
  double* mean[2];   // block means (pooled variant): [0] row-major, [1] transposed
  int n;             // tensors in this launch (1 or 2)
  const int32_t* order;   // position -> token table, or null for the fractal order
};

template <int D, int BS, bool kInverse, bool kPool>
__global__ void __launch_bounds__(kThreads) reorder_kernel(Tensors a, Dims g) {
  constexpr int VEC = D / 8;                 // 16-byte vectors of a row
  constexpr int RPP = kThreads / VEC;        // rows per pass of the CTA
  constexpr int VPT = BS / RPP;              // vectors (rows) per thread
  static_assert(BS % RPP == 0, "block rows split evenly over the passes");
  // unit = ((I * n + tensor) * B + b) * heads + head
  unsigned u = blockIdx.x;
  const int head = u % g.heads;
  u /= g.heads;
  const int b = u % g.B;
  u /= g.B;
  const int t = u % a.n;
  const int I = u / a.n;
  const size_t bh = (size_t)b * g.heads + head;
  const int c = threadIdx.x % VEC;
  const int r0 = threadIdx.x / VEC;
  // (selects, not an indexed load: the parameter struct stays in registers)
  const uint4* __restrict__ src = t ? a.src[1] : a.src[0];
  uint4* __restrict__ dst = t ? a.dst[1] : a.dst[0];

  // The block's token indices, computed once per row (the integer divisions
  // of the fractal order would otherwise run in each of the row's VEC
  // threads and dominate the kernel's instruction count).
  __shared__ int tok[BS];
  if (threadIdx.x < BS) {
    const int p = I * BS + threadIdx.x;
    tok[threadIdx.x] = (p >= g.N) ? -1 : (a.order != nullptr ? a.order[p] : fractal_token(p, g.H, g.W, g.P));
  }
  __syncthreads();

  uint4 v[VPT];
  int n[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int p = I * BS + r0 + j * RPP;
    n[j] = tok[r0 + j * RPP];
    const size_t kidx = (bh * g.Npad + p) * VEC + c;                                   // kernel order
    const size_t midx = (((size_t)b * g.N + (n[j] < 0 ? 0 : n[j])) * g.heads + head) * VEC + c;  // model order
    if (kInverse) v[j] = __ldcs(src + kidx);
    else v[j] = (n[j] >= 0) ? __ldcs(src + midx) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int p = I * BS + r0 + j * RPP;
    if (kInverse) {
      if (n[j] >= 0) dst[(((size_t)b * g.N + n[j]) * g.heads + head) * VEC + c] = v[j];
    } else {
      dst[(bh * g.Npad + p) * VEC + c] = v[j];   // padded positions get zeros
    }
  }

  if constexpr (kPool) {
    // column sums of this thread's rows (its 8 columns), then over the rows
    // of the warp (lanes c, c + VEC, ...) and over the warps
    __shared__ double part[kThreads / 32][VEC][8];
    double s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = 0.0;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      const uint32_t w4[4] = {v[j].x, v[j].y, v[j].z, v[j].w};   // padded rows are zero
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[2 * e] += (double)__uint_as_float(w4[e] << 16);
        s[2 * e + 1] += (double)__uint_as_float(w4[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int o = VEC; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) s[e] += __shfl_xor_sync(0xffffffffu, s[e], o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane < VEC)
#pragma unroll
      for (int e = 0; e < 8; ++e) part[warp][lane][e] = s[e];
    __syncthreads();
    if (threadIdx.x < D) {
      const int col = threadIdx.x;
      double sum = 0.0;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) sum += part[w][col / 8][col % 8];
      const int cnt = min(BS, g.N - I * BS);
      const double mean = sum / (double)cnt;
      if (t == 0) a.mean[0][(bh * g.nb + I) * D + col] = mean;
      else a.mean[1][(bh * D + col) * g.nb + I] = mean;   // k: transposed
    }
  }
}

template <int D, int BS, bool kInverse, bool kPool>
cudaError_t launch_t(const Tensors& a, const Dims& g, cudaStream_t st) {
  const size_t units = (size_t)g.nb * a.n * g.B * g.heads;
  if (units > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  reorder_kernel<D, BS, kInverse, kPool><<<(unsigned)units, kThreads, 0, st>>>(a, g);
  return cudaGetLastError();
}

template <bool kInverse, bool kPool>
cudaError_t launch(const Tensors& a, const Dims& g, cudaStream_t st) {
  if (g.d == 128 && g.bs == 64) return launch_t<128, 64, kInverse, kPool>(a, g, st);
  if (g.d == 128 && g.bs == 128) return launch_t<128, 128, kInverse, kPool>(a, g, st);
  if (g.d == 64 && g.bs == 64) return launch_t<64, 64, kInverse, kPool>(a, g, st);
  return launch_t<64, 128, kInverse, kPool>(a, g, st);
}

}  // namespace

cudaError_t launch_reorder(const Dims& g, const void* x_bnhd, void* y_bhnd, cudaStream_t st) {
  return launch_reorder_perm(g, nullptr, x_bnhd, y_bhnd, st);
}

cudaError_t launch_inverse_reorder(const Dims& g, const void* y_bhnd, void* x_bnhd, cudaStream_t st) {
  return launch_inverse_reorder_perm(g, nullptr, y_bhnd, x_bnhd, st);
}

cudaError_t launch_reorder_qk_pool(const Dims& g, const void* q_bnhd, const void* k_bnhd, void* q_bhnd,
                                   void* k_bhnd, double* qbar, double* kbar, cudaStream_t st) {
  return launch_reorder_qk_pool_perm(g, nullptr, q_bnhd, k_bnhd, q_bhnd, k_bhnd, qbar, kbar, st);
}

cudaError_t launch_reorder_perm(const Dims& g, const int32_t* order, const void* x_bnhd, void* y_bhnd,
                                cudaStream_t st) {
  Tensors a = {{(const uint4*)x_bnhd, nullptr}, {(uint4*)y_bhnd, nullptr}, {nullptr, nullptr}, 1, order};
  return launch<false, false>(a, g, st);
}

cudaError_t launch_inverse_reorder_perm(const Dims& g, const int32_t* order, const void* y_bhnd, void* x_bnhd,
                                        cudaStream_t st) {
  Tensors a = {{(const uint4*)y_bhnd, nullptr}, {(uint4*)x_bnhd, nullptr}, {nullptr, nullptr}, 1, order};
  return launch<true, false>(a, g, st);
}

cudaError_t launch_reorder_qk_pool_perm(const Dims& g, const int32_t* order, const void* q_bnhd,
                                        const void* k_bnhd, void* q_bhnd, void* k_bhnd, double* qbar, double* kbar,
                                        cudaStream_t st) {
  Tensors a = {{(const uint4*)q_bnhd, (const uint4*)k_bnhd}, {(uint4*)q_bhnd, (uint4*)k_bhnd}, {qbar, kbar}, 2,
               order};
  return launch<false, true>(a, g, st);
}

}  // namespace bsa
