// Adaptive block mask (NABLA summary, Metodologia 2 and 3):
//   pool_kernel: block means of Q and K ("Submuestreo"), double precision;
//   mask_kernel: reduced attention softmax(qbar kbar^T / sqrt(d)) per row
//                ("Atencion Reducida"), the CDF threshold ("Umbralizacion CDF"),
//                the optional STA union, and the ascending KV index lists that
//                the attention kernel walks ("Expansion").
//
// Precision: bf16 values summed in double are exact, so the block means equal
// the exact mean rounded once.  Dot products, exp and the probability masses
// are double, which keeps every threshold decision within ~1e-15 of the exact
// one; only rows whose prefix mass sits that close to 1 - thr can differ from
// an exact evaluation.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace bsa {

namespace {

// ---------------------------------------------------------------- pooling

constexpr int kPoolThreads = 256;
// block tiles in flight per CTA (64 KB of stages: several CTAs per SM)
template <int D, int BS>
constexpr int pool_stages() { return (BS * D * 2 <= 16384) ? 4 : 2; }
constexpr uint64_t kPoolWaitNs = 250ull * 1000ull * 1000ull;

// Persistent: CTA c pools the blocks c, c + gridDim.x, ... of all (tensor, b,
// head) in that order (item = ((which * B + b) * heads + head) * nb + I,
// which 0 = Q, 1 = K).  Each block tile (bs rows x d bf16, contiguous in
// kernel order) arrives by one bulk copy into a ring of kPoolStages shared
// memory stages, so several tiles per SM are in flight while earlier ones are
// reduced.  Thread t sums the column pair t mod (d/2) over every
// (256 / (d/2))-th valid row; the partial sums are combined through shared
// memory in double.  Sums of bf16 values in double are exact, so the means are
// the exact means rounded once.  A bulk copy that does not arrive in time sets
// BSA_ERR_TIMEOUT in the error word and the CTA stops.
template <int D, int BS>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            double* __restrict__ qbar, double* __restrict__ kbar,
                                                            Ctrl* ctrl, Dims g, uint32_t seq) {
  constexpr uint32_t kTileBytes = BS * D * 2;
  constexpr int kPoolStages = pool_stages<D, BS>();
  constexpr int kPairs = D / 2;                    // bf16 column pairs of a row
  constexpr int kRowGroups = kPoolThreads / kPairs;
  extern __shared__ __align__(128) uint8_t pool_smem[];
  uint8_t* tiles = pool_smem;                                             // [stages][tile]
  double* part = reinterpret_cast<double*>(pool_smem + kPoolStages * kTileBytes);  // [row groups][D]
  __shared__ uint64_t full[4];
  __shared__ int stop;

  const int total = 2 * g.B * g.heads * g.nb;
  const int G = gridDim.x;
  auto item_ptr = [&](int it) -> const __nv_bfloat16* {
    const int I = it % g.nb;
    const int rest = it / g.nb;                    // (which * B + b) * heads + head
    const int which = rest / (g.B * g.heads);
    const size_t bh = rest % (g.B * g.heads);
    const __nv_bfloat16* src = which ? k : q;
    return src + (bh * g.Npad + (size_t)I * BS) * D;
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPoolStages; ++s) sm100::mbar_init(&full[s], 1);
    stop = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  uint32_t armed = 0;   // stage loads issued (thread 0)
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPoolStages; ++s) {
      const int it = blockIdx.x + s * G;
      if (it >= total) break;
      ++armed;
      sm100::mbar_arrive_expect_tx(&full[s], kTileBytes);
      sm100::bulk_load(tiles + s * kTileBytes, item_ptr(it), kTileBytes, &full[s]);
    }
  }
  const int cp = threadIdx.x % kPairs;
  const int rg = threadIdx.x / kPairs;
  for (int n = 0;; ++n) {
    const int it = blockIdx.x + n * G;
    if (it >= total) break;
    const int s = n % kPoolStages;
    const bool ok = sm100::mbar_wait_ns(&full[s], (n / kPoolStages) & 1, kPoolWaitNs, &ctrl->abort_seq, seq);
    if (!ok) {
      if (threadIdx.x == 0) {
        report_error(ctrl, kErrTimeout, blockIdx.x, (uint32_t)it, 40u);
        atomicExch(&ctrl->abort_seq, seq);
      }
      stop = 1;
    }
    __syncthreads();
    if (stop) break;
    const int I = it % g.nb;
    const int cnt = min(BS, g.N - I * BS);
    const __nv_bfloat162* t2 = reinterpret_cast<const __nv_bfloat162*>(tiles + s * kTileBytes);
    double a0 = 0.0, a1 = 0.0;
#pragma unroll 4
    for (int r = rg; r < cnt; r += kRowGroups) {
      const float2 f = __bfloat1622float2(t2[r * kPairs + cp]);
      a0 += (double)f.x;
      a1 += (double)f.y;
    }
    part[rg * D + 2 * cp] = a0;
    part[rg * D + 2 * cp + 1] = a1;
    __syncthreads();   // the stage is read and the partial sums are in place
    if (threadIdx.x == 0 && it + kPoolStages * G < total) {
      ++armed;
      sm100::mbar_arrive_expect_tx(&full[s], kTileBytes);
      sm100::bulk_load(tiles + s * kTileBytes, item_ptr(it + kPoolStages * G), kTileBytes, &full[s]);
    }
    if (threadIdx.x < D) {
      const int col = threadIdx.x;
      double sum = 0.0;
#pragma unroll
      for (int i = 0; i < kRowGroups; ++i) sum += part[i * D + col];
      const int rest = it / g.nb;
      const int which = rest / (g.B * g.heads);
      const size_t bh = rest % (g.B * g.heads);
      // qbar row-major [bh][I][d]; kbar transposed [bh][d][I] (the mask kernel
      // reads it one column of d at a time)
      if (which) kbar[(bh * D + col) * g.nb + I] = sum / (double)cnt;
      else qbar[(bh * g.nb + I) * D + col] = sum / (double)cnt;
    }
    __syncthreads();   // part is rewritten by the next block
  }
  // no bulk copy of this CTA may still be in flight when it exits
  if (threadIdx.x == 0) sm100::mbar_drain_ring(full, kPoolStages, armed, kPoolWaitNs);
}

// ------------------------------------------------------------- mask rows

constexpr int kMaskRows = 16;                 // query-block rows per CTA (one warp each)
constexpr int kMaskThreads = 32 * kMaskRows;  // 512

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ unsigned long long warp_max(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

__device__ __forceinline__ void block_tile(int I, const Dims& g, int& t, int& th, int& tw) {
  const int n = fractal_token(I * g.bs, g.H, g.W, g.P);
  const int HW = g.H * g.W;
  t = n / HW;
  const int rem = n - t * HW;
  const int h = rem / g.W;
  th = h / g.P;
  tw = (rem - h * g.W) / g.P;
}

// Persistent grid: CTA c handles the groups of kMaskRows rows c, c + gridDim.x,
// ... of all (b, head).  Dynamic smem: qbar rows [kMaskRows][D] then scores
// [kMaskRows][nb], both double.  NJ = ceil(nb / 32) rounded up to a power of
// two: the values of a row that each lane holds in phase 2.
template <int D, int NJ>
__global__ void __launch_bounds__(kMaskThreads) mask_kernel(const double* __restrict__ qbar,
                                                            const double* __restrict__ kbar, Dims g, double thr,
                                                            double scale, int sta_t, int sta_h, int sta_w,
                                                            int32_t* __restrict__ kv_count,
                                                            int32_t* __restrict__ kv_idx, uint8_t* __restrict__ mask) {
  constexpr int kMaxJ = NJ;
  extern __shared__ __align__(16) double smem[];
  double* qs = smem;                       // [kMaskRows][D]
  double* sc = smem + kMaskRows * D;       // [kMaskRows][nb]
  const int nb = g.nb;
  const int groups = (nb + kMaskRows - 1) / kMaskRows;
  const int total = groups * g.B * g.heads;
  for (int grp = blockIdx.x; grp < total; grp += gridDim.x) {
  const size_t bh = (size_t)(grp / groups);
  const int I0 = (grp % groups) * kMaskRows;
  const int rows = min(kMaskRows, nb - I0);

  for (int i = threadIdx.x; i < kMaskRows * D; i += kMaskThreads) {
    const int r = i / D;
    qs[i] = (r < rows) ? qbar[(bh * nb + I0 + r) * D + (i % D)] : 0.0;
  }
  __syncthreads();

  // Phase 1: scores s[r][J] = scale * qbar_r . kbar_J on the fp64 tensor
  // cores (mma.sync m8n8k4, fp64 multiply-add): warp w computes both 8-row
  // halves of the CTA's rows against the 8-column tiles w, w + 16, ... of J.
  // A fragments (qbar rows) come from shared memory, B fragments from the
  // transposed kbar [bh][d][nb] in global memory (64 contiguous bytes per
  // fragment row).
  {
    constexpr int kWarps = kMaskThreads / 32;
    constexpr int NT = (NJ * 32 / 8 + kWarps - 1) / kWarps;   // 8-column tiles per warp
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int gq = lane >> 2, tq = lane & 3;                   // fragment row / column group
    const double* kt = kbar + bh * D * (size_t)nb;
    double acc[2][NT][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[mt][n][0] = acc[mt][n][1] = 0.0;
    // B fragments are loaded PD k-steps ahead of their use (a register ring),
    // so the L2 latency of kbar overlaps the MMAs of the steps in between.
    constexpr int PD = (NT <= 4) ? 4 : 2;
    constexpr int KS = D / 4;                                  // k-steps of 4
    double bq[PD][NT];
    auto load_b = [&](int ks, double (&dst)[NT]) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int J = (wid + n * kWarps) * 8 + gq;
        dst[n] = (J < nb) ? __ldg(kt + (size_t)(4 * ks + tq) * nb + J) : 0.0;
      }
    };
#pragma unroll
    for (int p = 0; p < PD; ++p) load_b(p, bq[p]);
#pragma unroll 1
    for (int ks0 = 0; ks0 < KS; ks0 += PD) {
#pragma unroll
      for (int p = 0; p < PD; ++p) {
        const int ks = ks0 + p;
        const double a0 = qs[gq * D + 4 * ks + tq];
        const double a1 = qs[(8 + gq) * D + 4 * ks + tq];
        double bv[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) bv[n] = bq[p][n];
        if (ks + PD < KS) load_b(ks + PD, bq[p]);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
                       : "+d"(acc[0][n][0]), "+d"(acc[0][n][1])
                       : "d"(a0), "d"(bv[n]));
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
                       : "+d"(acc[1][n][0]), "+d"(acc[1][n][1])
                       : "d"(a1), "d"(bv[n]));
        }
      }
    }
    // accumulator element (row gq + 8 mt, column 2 tq + e) of each tile
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int Jb = (wid + n * kWarps) * 8 + 2 * tq;
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (Jb + e < nb) sc[(mt * 8 + gq) * nb + Jb + e] = acc[mt][n][e] * scale;
      }
  }
  __syncthreads();

  // Phase 2: one warp per row.  Lane L holds J = L + 32 i.
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (warp < rows) {
  const int I = I0 + warp;
  const double* srow = sc + warp * nb;

  double a[kMaxJ];
  double mx = -DBL_MAX;
#pragma unroll
  for (int i = 0; i < kMaxJ; ++i) {
    const int J = lane + 32 * i;
    a[i] = (J < nb) ? srow[J] : -DBL_MAX;
    mx = fmax(mx, a[i]);
  }
  mx = warp_max(mx);
  double z = 0.0;
#pragma unroll
  for (int i = 0; i < kMaxJ; ++i) {
    const int J = lane + 32 * i;
    a[i] = (J < nb) ? exp(a[i] - mx) : 0.0;
    z += a[i];
  }
  z = warp_sum(z);
  const double rz = 1.0 / z;
#pragma unroll
  for (int i = 0; i < kMaxJ; ++i) a[i] *= rz;  // A = e / sum(e)

  // keep bits: bit i of `keep` <-> J = lane + 32 i
  uint32_t keep = 0u;
  const double target = 1.0 - thr;
  double total = 0.0;
#pragma unroll
  for (int i = 0; i < kMaxJ; ++i) total += a[i];
  total = warp_sum(total);
  if (thr == 0.0 || total < target) {
    // thr == 0 keeps every block; so does a row whose whole mass rounds below 1 - thr.
#pragma unroll
    for (int i = 0; i < kMaxJ; ++i)
      if (lane + 32 * i < nb) keep |= 1u << i;
  } else {
    // Largest key v (bit pattern of a non-negative double, monotone in value)
    // with mass(A >= v) >= target: the probability of the last kept block.
    // Bits above the largest key's highest set bit are 0 in v: the search
    // starts below them (every key is below hi = 2^(top + 1)).
    unsigned long long kmax = 0ull;
#pragma unroll
    for (int i = 0; i < kMaxJ; ++i) {
      const unsigned long long key = (unsigned long long)__double_as_longlong(a[i]);
      kmax = (lane + 32 * i < nb && key > kmax) ? key : kmax;
    }
    kmax = warp_max(kmax);
    const int top = 63 - __clzll((long long)kmax);
    unsigned long long lo = 0ull, hi = (top >= 63) ? ~0ull : (1ull << (top + 1));
    int cnt_lo = nb, cnt_hi = 0;
    bool unique = false;
    for (int bit = top; bit >= 0; --bit) {
      const unsigned long long cand = lo | (1ull << bit);
      double m = 0.0;
      int c = 0;
#pragma unroll
      for (int i = 0; i < kMaxJ; ++i) {
        const bool ge = (lane + 32 * i < nb) && (unsigned long long)__double_as_longlong(a[i]) >= cand;
        m += ge ? a[i] : 0.0;
        c += ge ? 1 : 0;
      }
      m = warp_sum(m);
      c = __reduce_add_sync(0xffffffffu, c);
      if (m >= target) {
        lo = cand;
        cnt_lo = c;
      } else {
        hi = cand;
        cnt_hi = c;
      }
      if (cnt_lo - cnt_hi == 1) {
        unique = true;
        break;
      }
    }
    unsigned long long vb = lo;
    if (unique) {  // the single block with lo <= key < hi
      unsigned long long best = 0ull;
#pragma unroll
      for (int i = 0; i < kMaxJ; ++i) {
        const unsigned long long key = (unsigned long long)__double_as_longlong(a[i]);
        if (lane + 32 * i < nb && key < hi && key > best) best = key;
      }
      vb = warp_max(best);
    }
    // Every block above the boundary value is kept; blocks equal to it are
    // added in ascending index order until the mass reaches the target.
    double run = 0.0;
#pragma unroll
    for (int i = 0; i < kMaxJ; ++i) {
      const unsigned long long key = (unsigned long long)__double_as_longlong(a[i]);
      if (lane + 32 * i < nb && key > vb) {
        keep |= 1u << i;
        run += a[i];
      }
    }
    run = warp_sum(run);
    const double vval = __longlong_as_double((long long)vb);
#pragma unroll
    for (int i = 0; i < kMaxJ; ++i) {
      if (run >= target) break;
      const unsigned long long key = (unsigned long long)__double_as_longlong(a[i]);
      uint32_t ties = __ballot_sync(0xffffffffu, (lane + 32 * i < nb) && key == vb);
      while (ties != 0u && run < target) {
        const int src = __ffs(ties) - 1;
        ties &= ties - 1u;
        if (lane == src) keep |= 1u << i;
        run += vval;
      }
    }
  }

  if (sta_t >= 0) {
    int ti, hi_, wi;
    block_tile(I, g, ti, hi_, wi);
#pragma unroll 1
    for (int i = 0; i < kMaxJ; ++i) {
      const int J = lane + 32 * i;
      if (J >= nb) break;
      int tj, hj, wj;
      block_tile(J, g, tj, hj, wj);
      if (abs(ti - tj) <= sta_t && abs(hi_ - hj) <= sta_h && abs(wi - wj) <= sta_w) keep |= 1u << i;
    }
  }

  const size_t row = bh * nb + I;
  int base = 0;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < kMaxJ; ++i) {
    const int J = lane + 32 * i;
    const bool k = (keep >> i) & 1u;
    const uint32_t bal = __ballot_sync(0xffffffffu, k);
    if (k) kv_idx[row * nb + base + __popc(bal & lt)] = J;
    if (mask != nullptr && J < nb) mask[row * nb + J] = k ? 1 : 0;
    base += __popc(bal);
  }
  if (lane == 0) kv_count[row] = base;
  }  // warp < rows
  __syncthreads();   // qs and sc are rewritten by the next group
  }  // groups
}

}  // namespace

template <int D, int BS>
cudaError_t launch_pool_t(const Dims& g, const void* q, const void* k, double* qbar, double* kbar, Ctrl* ctrl,
                          uint32_t seq, cudaStream_t st) {
  const size_t smem = (size_t)pool_stages<D, BS>() * BS * D * 2 + (size_t)(kPoolThreads / (D / 2)) * D * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(pool_kernel<D, BS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_kernel<D, BS>, kPoolThreads, smem)) !=
      cudaSuccess)
    return e;
  const int total = 2 * g.B * g.heads * g.nb;
  const int grid = std::max(1, std::min(total, sms * std::max(1, per_sm)));
  pool_kernel<D, BS><<<grid, kPoolThreads, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qbar,
                                                       kbar, ctrl, g, seq);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Dims& g, const void* q, const void* k, double* qbar, double* kbar, Ctrl* ctrl,
                        uint32_t seq, cudaStream_t st) {
  if (g.d == 128 && g.bs == 64) return launch_pool_t<128, 64>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 128 && g.bs == 128) return launch_pool_t<128, 128>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 64 && g.bs == 64) return launch_pool_t<64, 64>(g, q, k, qbar, kbar, ctrl, seq, st);
  return launch_pool_t<64, 128>(g, q, k, qbar, kbar, ctrl, seq, st);
}

template <int D, int NJ>
cudaError_t launch_mask_t(const Dims& g, const double* qbar, const double* kbar, double thr, int sta_t, int sta_h,
                          int sta_w, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  const size_t smem = (size_t)kMaskRows * (g.d + g.nb) * sizeof(double);
  const double scale = 1.0 / std::sqrt((double)g.d);
  cudaError_t e = cudaFuncSetAttribute(mask_kernel<D, NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mask_kernel<D, NJ>, kMaskThreads, smem)) !=
      cudaSuccess)
    return e;
  const int total = (g.nb + kMaskRows - 1) / kMaskRows * g.B * g.heads;
  const int grid = std::max(1, std::min(total, sms * std::max(1, per_sm)));
  mask_kernel<D, NJ><<<grid, kMaskThreads, smem, st>>>(qbar, kbar, g, thr, scale, sta_t, sta_h, sta_w, kv_count,
                                                       kv_idx, mask);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_mask_d(const Dims& g, const double* qbar, const double* kbar, double thr, int sta_t, int sta_h,
                          int sta_w, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  if (g.nb <= 128) return launch_mask_t<D, 4>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  if (g.nb <= 256) return launch_mask_t<D, 8>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  if (g.nb <= 512) return launch_mask_t<D, 16>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  return launch_mask_t<D, 32>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
}

cudaError_t launch_mask(const Dims& g, const double* qbar, const double* kbar, double thr, int sta_t, int sta_h,
                        int sta_w, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  if (g.d == 128) return launch_mask_d<128>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  return launch_mask_d<64>(g, qbar, kbar, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
}

}  // namespace bsa
