// Token-radius block masks (TRA summary, section 2, "El Pipeline de TRA"):
// entropy -> token budget -> radius -> block mask, in the KV-list format the
// attention kernels walk.
//
// The entropy of each query row comes from a dense warm-up pass of the
// attention kernel (bsa_attn_fwd_entropy over dense lists, dense_lists_kernel
// here).  Then, per query token i at (t_i, h_i, w_i):
//   budget_i = clamp(tau * exp(H_i), 1, N) keys
//   r_i      = sqrt(budget_i / (pi * sum_t phi(|t - t_i|)^2)),  phi(d) = exp(-gamma d)
// so that the 2-D disks of radius r_i phi(|t - t_i|) in every frame t hold the
// budget in area; key token j is in i's support when
//   (h_j - h_i)^2 + (w_j - w_i)^2 <= (r_i phi(|t_j - t_i|))^2,
// a query token votes for a key block when the block holds a key of its
// support, and block I keeps block J when at least `vote` of I's valid query
// tokens vote for J.
//
// radius_mask_kernel: one CTA per (b, head, query block I).  The block's query
// tokens, their radii (double) and bounding box go to shared memory; each
// warp takes key blocks J in turn, skips J when the gap between the two
// blocks' bounding boxes already exceeds the largest radius of I at that
// frame distance, and otherwise counts the voting query tokens exactly
// (every query token against every key token of J).  The kept blocks are
// written as an ascending list.
#include <cfloat>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kRadThreads = 256;
constexpr int kRadWarps = kRadThreads / 32;
constexpr int kMaxFrames = 1024;

__global__ void dense_lists_kernel(Dims g, int32_t* __restrict__ kv_count, int32_t* __restrict__ kv_idx) {
  const size_t row = blockIdx.x;   // (b, head, I)
  for (int J = threadIdx.x; J < g.nb; J += blockDim.x) kv_idx[row * g.nb + J] = J;
  if (threadIdx.x == 0) kv_count[row] = g.nb;
}

__device__ __forceinline__ void coords(int p, const Dims& g, int& t, int& h, int& w) {
  const int n = fractal_token(p, g.H, g.W, g.P);
  const int HW = g.H * g.W;
  t = n / HW;
  const int r = n - t * HW;
  h = r / g.W;
  w = r - h * g.W;
}

template <int BS>
__global__ void __launch_bounds__(kRadThreads) radius_mask_kernel(const float* __restrict__ entropy, Dims g,
                                                                  double tau, double gamma, int vote,
                                                                  int32_t* __restrict__ kv_count,
                                                                  int32_t* __restrict__ kv_idx,
                                                                  uint8_t* __restrict__ mask) {
  __shared__ int qt[BS], qh[BS], qw[BS];
  __shared__ double qr[BS];
  __shared__ double phi[kMaxFrames];
  __shared__ int kt[kRadWarps][BS], kh[kRadWarps][BS], kw[kRadWarps][BS];
  __shared__ uint32_t keep_bits[BSA_MAX_BLOCKS / 32];
  __shared__ int box[6];          // tmin, tmax, hmin, hmax, wmin, wmax of block I
  __shared__ double rmax_s;
  const int nb = g.nb;
  const size_t row = blockIdx.x;  // (b, head, I)
  const size_t bh = row / nb;
  const int I = (int)(row % nb);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nq = min(BS, g.N - I * BS);          // valid query tokens of I

  for (int d = threadIdx.x; d < g.T; d += kRadThreads) phi[d] = exp(-gamma * (double)d);
  for (int i = threadIdx.x; i < BSA_MAX_BLOCKS / 32; i += kRadThreads) keep_bits[i] = 0u;
  if (threadIdx.x == 0) {
    box[0] = box[2] = box[4] = INT_MAX;
    box[1] = box[3] = box[5] = INT_MIN;
    rmax_s = 0.0;
  }
  __syncthreads();
  if (threadIdx.x < nq) {
    const int i = threadIdx.x, p = I * BS + i;
    int t, h, w;
    coords(p, g, t, h, w);
    qt[i] = t;
    qh[i] = h;
    qw[i] = w;
    // budget (keys) and base radius, in the order the definition states
    const double H = (double)entropy[bh * g.Npad + p];
    const double budget = fmin(fmax(tau * exp(H), 1.0), (double)g.N);
    double area = 0.0;
    for (int tt = 0; tt < g.T; ++tt) area += M_PI * exp(-2.0 * gamma * (double)abs(tt - t));
    const double r = sqrt(budget / area);
    qr[i] = r;
    atomicMin(&box[0], t);
    atomicMax(&box[1], t);
    atomicMin(&box[2], h);
    atomicMax(&box[3], h);
    atomicMin(&box[4], w);
    atomicMax(&box[5], w);
  }
  __syncthreads();
  if (wid == 0) {
    double rm = 0.0;
    for (int i = lane; i < nq; i += 32) rm = fmax(rm, qr[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rm = fmax(rm, __shfl_xor_sync(0xffffffffu, rm, o));
    if (lane == 0) rmax_s = rm;
  }
  __syncthreads();
  const double rmax = rmax_s;

  for (int J = wid; J < nb; J += kRadWarps) {
    const int nk = min(BS, g.N - J * BS);
    int tmin = INT_MAX, tmax = INT_MIN, hmin = INT_MAX, hmax = INT_MIN, wmin = INT_MAX, wmax = INT_MIN;
    for (int j = lane; j < nk; j += 32) {
      int t, h, w;
      coords(J * BS + j, g, t, h, w);
      kt[wid][j] = t;
      kh[wid][j] = h;
      kw[wid][j] = w;
      tmin = min(tmin, t);
      tmax = max(tmax, t);
      hmin = min(hmin, h);
      hmax = max(hmax, h);
      wmin = min(wmin, w);
      wmax = max(wmax, w);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tmin = min(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
      tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      hmin = min(hmin, __shfl_xor_sync(0xffffffffu, hmin, o));
      hmax = max(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
      wmin = min(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
      wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    }
    __syncwarp();
    // lower bounds of the frame distance and of the 2-D gap between the boxes
    const int dt = max(0, max(tmin - box[1], box[0] - tmax));
    const int dh = max(0, max(hmin - box[3], box[2] - hmax));
    const int dw = max(0, max(wmin - box[5], box[4] - wmax));
    const double reach = rmax * phi[dt];
    bool kept = false;
    if ((double)(dh * dh + dw * dw) <= reach * reach * (1.0 + 1e-12)) {
      int votes = 0;
      for (int i0 = 0; i0 < nq; i0 += 32) {
        const int i = i0 + lane;
        bool hit = false;
        if (i < nq) {
          const int ti = qt[i], hi = qh[i], wi = qw[i];
          const double ri = qr[i];
          for (int j = 0; j < nk && !hit; ++j) {
            const double rad = ri * phi[abs(kt[wid][j] - ti)];
            const int eh = kh[wid][j] - hi, ew = kw[wid][j] - wi;
            hit = (double)(eh * eh + ew * ew) <= rad * rad;
          }
        }
        votes += __popc(__ballot_sync(0xffffffffu, hit));
      }
      kept = votes >= vote;
    }
    if (lane == 0 && kept) atomicOr(&keep_bits[J >> 5], 1u << (J & 31));
    __syncwarp();   // kt/kh/kw are rewritten for the warp's next J
  }
  __syncthreads();

  // ascending list of the kept blocks (warp 0), and the optional u8 mask
  if (wid == 0) {
    const int nw = (nb + 31) >> 5;
    int base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int wi = w0 + lane;
      uint32_t u = (wi < nw) ? keep_bits[wi] : 0u;
      const int n = __popc(u);
      int incl = n;
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += t;
      }
      int pos = base + incl - n;
      while (u != 0u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        kv_idx[row * nb + pos++] = wi * 32 + bit;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) kv_count[row] = base;
  }
  if (mask != nullptr)
    for (int J = threadIdx.x; J < nb; J += kRadThreads) mask[row * nb + J] = (keep_bits[J >> 5] >> (J & 31)) & 1u;
}

}  // namespace

cudaError_t launch_dense_lists(const Dims& g, int32_t* kv_count, int32_t* kv_idx, cudaStream_t st) {
  const size_t rows = (size_t)g.B * g.heads * g.nb;
  dense_lists_kernel<<<(unsigned)rows, 256, 0, st>>>(g, kv_count, kv_idx);
  return cudaGetLastError();
}

cudaError_t launch_radius_mask(const Dims& g, const float* entropy, double tau, double gamma, int vote,
                               int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  if (g.T > kMaxFrames) return cudaErrorInvalidValue;
  const size_t rows = (size_t)g.B * g.heads * g.nb;
  if (g.bs == 64)
    radius_mask_kernel<64><<<(unsigned)rows, kRadThreads, 0, st>>>(entropy, g, tau, gamma, vote, kv_count, kv_idx,
                                                                   mask);
  else
    radius_mask_kernel<128><<<(unsigned)rows, kRadThreads, 0, st>>>(entropy, g, tau, gamma, vote, kv_count, kv_idx,
                                                                    mask);
  return cudaGetLastError();
}

}  // namespace bsa
