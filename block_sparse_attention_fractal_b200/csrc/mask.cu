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

constexpr int kMaskThreads = 256;             // 8 warps
constexpr int kMaskWarps = kMaskThreads / 32;
// Query-block rows per CTA: 16, or 8 when rows are longer than 512 blocks
// (the CTA's scores then stay at 64 KB of shared memory, two CTAs per SM).
template <int NJ>
constexpr int mask_rows() { return NJ <= 16 ? 16 : 8; }

__device__ __forceinline__ double warp_sum(double v) {
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
__device__ __forceinline__ unsigned long long warp_min(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w < v ? w : v;
  }
  return v;
}

// A probability in fixed point, units of 2^-52, in bits 11-63, and a count of
// one in bits 0-10: sums of up to 1024 of these add both fields at once
// without carrying from one into the other (the masses of a row sum to
// about 2^52 < 2^53).  Rounding each probability to 2^-53 moves a row's
// prefix masses by less than 1024 * 2^-53 = 1.1e-13, far inside the 1e-6
// window within which a threshold decision counts as ambiguous.
constexpr double kMassScale = 4503599627370496.0;   // 2^52
__device__ __forceinline__ unsigned long long packed_mass(double a) {
  return (__double2ull_rn(a * kMassScale) << 11) | 1ull;
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

// Persistent grid: CTA c handles the groups of R rows c, c + gridDim.x, ...
// of all (b, head).  Dynamic shared memory: qbar rows [R][D], scores [R][nb]
// (double), then a 256-bucket histogram per warp (uint64).  NJ = ceil(nb / 32)
// rounded up to a power of two: the values of a row that each lane holds.
template <int D, int NJ>
__global__ void __launch_bounds__(kMaskThreads, 2) mask_kernel(const double* __restrict__ qbar,
                                                               const double* __restrict__ kbar, Dims g, double thr,
                                                               double scale, int sta_t, int sta_h, int sta_w,
                                                               int32_t* __restrict__ kv_count,
                                                               int32_t* __restrict__ kv_idx,
                                                               uint8_t* __restrict__ mask) {
  constexpr int R = mask_rows<NJ>();
  constexpr int MT = R / 8;                                    // 8-row MMA tiles
  extern __shared__ __align__(16) double smem[];
  double* qs = smem;                                           // [R][D]
  double* sc = smem + R * D;                                   // [R][nb]
  const int nb = g.nb;
  unsigned long long* hist = reinterpret_cast<unsigned long long*>(sc + R * nb);   // [warps][256]
  const int groups = (nb + R - 1) / R;
  const int total = groups * g.B * g.heads;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned long long* my_hist = hist + wid * 256;
  const unsigned long long target = __double2ull_rn((1.0 - thr) * kMassScale);

  for (int grp = blockIdx.x; grp < total; grp += gridDim.x) {
    const size_t bh = (size_t)(grp / groups);
    const int I0 = (grp % groups) * R;
    const int rows = min(R, nb - I0);

    for (int i = threadIdx.x; i < R * D; i += kMaskThreads) {
      const int r = i / D;
      qs[i] = (r < rows) ? qbar[(bh * nb + I0 + r) * D + (i % D)] : 0.0;
    }
    __syncthreads();

    // Phase 1: scores s[r][J] = scale * qbar_r . kbar_J on the fp64 tensor
    // cores (mma.sync m8n8k4, fp64 multiply-add): warp w computes the R rows
    // against the 8-column tiles w, w + 8, ... of J.  A fragments (qbar rows)
    // come from shared memory, B fragments from the transposed kbar
    // [bh][d][nb] in global memory (64 contiguous bytes per fragment row),
    // loaded PD k-steps ahead of their use.
    // (in passes of at most 8 column tiles, so the accumulators and the B
    // prefetch fit in registers for long rows)
    {
      constexpr int NTW = NJ / 2;                                // 8-column tiles per warp
      constexpr int NT = NTW < 8 ? NTW : 8;                      // ... per pass
      const int gq = lane >> 2, tq = lane & 3;
      const double* kt = kbar + bh * D * (size_t)nb;
#pragma unroll 1
      for (int pass = 0; pass < NTW / NT; ++pass) {
        double acc[MT][NT][2];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int n = 0; n < NT; ++n) acc[mt][n][0] = acc[mt][n][1] = 0.0;
        constexpr int PD = 2;
        constexpr int KS = D / 4;
        double bq[PD][NT];
        auto load_b = [&](int ks, double (&dst)[NT]) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const int J = (wid + (pass * NT + n) * kMaskWarps) * 8 + gq;
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
            double av[MT];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) av[mt] = qs[(mt * 8 + gq) * D + 4 * ks + tq];
            double bv[NT];
#pragma unroll
            for (int n = 0; n < NT; ++n) bv[n] = bq[p][n];
            if (ks + PD < KS) load_b(ks + PD, bq[p]);
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
                asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
                             : "+d"(acc[mt][n][0]), "+d"(acc[mt][n][1])
                             : "d"(av[mt]), "d"(bv[n]));
          }
        }
        // accumulator element (row gq + 8 mt, column 2 tq + e) of each tile
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const int Jb = (wid + (pass * NT + n) * kMaskWarps) * 8 + 2 * tq;
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (Jb + e < nb) sc[(mt * 8 + gq) * nb + Jb + e] = acc[mt][n][e] * scale;
          }
      }
    }
    __syncthreads();

    // Phase 2: warp w takes rows w, w + 8, ...  Lane L owns J = L + 32 i of
    // the row; the probabilities replace the scores in shared memory (each
    // lane rereads only its own entries), so long rows need no registers.
    for (int rr = wid; rr < rows; rr += kMaskWarps) {
      const int I = I0 + rr;
      double* srow = sc + rr * nb;
      auto key_of = [&](int J) { return (unsigned long long)__double_as_longlong(srow[J]); };
      double mx = -DBL_MAX;
#pragma unroll
      for (int i = 0; i < NJ; ++i) {
        const int J = lane + 32 * i;
        if (J < nb) mx = fmax(mx, srow[J]);
      }
      mx = warp_max(mx);
      double z = 0.0;
#pragma unroll
      for (int i = 0; i < NJ; ++i) {
        const int J = lane + 32 * i;
        if (J < nb) {
          const double e = exp(srow[J] - mx);
          srow[J] = e;
          z += e;
        }
      }
      z = warp_sum(z);
      const double rz = 1.0 / z;
      unsigned long long tot = 0ull;
#pragma unroll
      for (int i = 0; i < NJ; ++i) {
        const int J = lane + 32 * i;
        if (J < nb) {
          const double pr = srow[J] * rz;   // A = e / sum(e)
          srow[J] = pr;
          tot += packed_mass(pr);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);

      // keep bits: bit i of `keep` <-> J = lane + 32 i
      uint32_t keep = 0u;
      if (thr == 0.0 || (tot >> 11) < target) {
        // thr == 0 keeps every block; so does a row whose whole mass rounds below 1 - thr.
#pragma unroll
        for (int i = 0; i < NJ; ++i)
          if (lane + 32 * i < nb) keep |= 1u << i;
      } else {
        // Radix select of the boundary probability vb: the smallest kept
        // value, i.e. the largest v whose mass(A >= v) reaches the target.
        // Keys are the bit patterns of the (non-negative) probabilities,
        // ordered like the values.  Each round histograms one 8-bit digit of
        // the candidates' keys (fixed-point mass and count per bucket), scans
        // the buckets from the top and keeps the bucket where the running
        // mass reaches the target; the keys above it are kept for sure.  The
        // search starts at the highest bit in which the keys differ and ends
        // when one candidate is left, or when all bits are fixed (ties).
        unsigned long long kmax = 0ull, kmin = ~0ull;
#pragma unroll
        for (int i = 0; i < NJ; ++i) {
          const int J = lane + 32 * i;
          if (J < nb) {
            const unsigned long long key = key_of(J);
            kmax = key > kmax ? key : kmax;
            kmin = key < kmin ? key : kmin;
          }
        }
        kmax = warp_max(kmax);
        kmin = warp_min(kmin);
        unsigned long long vb = kmax;      // the boundary key
        unsigned long long above = 0ull;   // packed mass of the keys above the candidates
        bool single = true;
        if (kmax != kmin) {
          int top = 63 - __clzll((long long)(kmax ^ kmin));   // highest bit in which keys differ (< 63)
          unsigned long long pref = kmax >> (top + 1);         // the bits above it, common to all keys
          int cnt = 0;
          int s = 0;
          for (;;) {
            const int w = min(8, top + 1);
            s = top + 1 - w;
#pragma unroll
            for (int k = 0; k < 8; ++k) my_hist[lane + 32 * k] = 0ull;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
              const int J = lane + 32 * i;
              if (J < nb) {
                const unsigned long long key = key_of(J);
                if ((key >> (top + 1)) == pref)
                  atomicAdd(&my_hist[(key >> s) & ((1u << w) - 1u)], packed_mass(srow[J]));
              }
            }
            __syncwarp();
            // lane L scans buckets 255 - 8 L down to 248 - 8 L
            unsigned long long loc[8], lsum = 0ull;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              loc[e] = my_hist[255 - 8 * lane - e];
              lsum += loc[e];
            }
            unsigned long long incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += t;
            }
            unsigned long long cum = above + (incl - lsum), before = 0ull;
            int found = -1;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const unsigned long long nc = cum + loc[e];
              if (found < 0 && (nc >> 11) >= target) {
                found = e;
                before = cum;
              }
              cum = nc;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, found >= 0);
            const int src = __ffs(bal) - 1;   // bal != 0: the candidates and `above` reach the target
            const int e_sel = __shfl_sync(0xffffffffu, found, src);
            above = __shfl_sync(0xffffffffu, before, src);
            const int d_sel = 255 - 8 * src - e_sel;
            cnt = (int)(my_hist[d_sel] & 2047ull);
            pref = (pref << w) | (unsigned long long)d_sel;
            __syncwarp();   // the histogram is cleared by the next round
            if (cnt == 1 || s == 0) break;
            top = s - 1;
          }
          if (cnt == 1) {
            // the one key with these leading bits
            unsigned long long best = 0ull;
#pragma unroll
            for (int i = 0; i < NJ; ++i) {
              const int J = lane + 32 * i;
              if (J < nb && (key_of(J) >> s) == pref) best = key_of(J);
            }
            vb = warp_max(best);
          } else {
            vb = pref;          // all bits fixed: cnt equal keys
            single = false;
          }
        }
        // Every block above vb is kept.  With a single block at vb it is kept
        // too; equal keys at vb are added in ascending index order until the
        // mass reaches the target.
#pragma unroll
        for (int i = 0; i < NJ; ++i) {
          const int J = lane + 32 * i;
          if (J < nb) {
            const unsigned long long key = key_of(J);
            if (key > vb || (single && key == vb)) keep |= 1u << i;
          }
        }
        if (!single) {
          unsigned long long run = above >> 11;
          const unsigned long long mv = packed_mass(__longlong_as_double((long long)vb)) >> 11;
#pragma unroll
          for (int i = 0; i < NJ; ++i) {
            if (run >= target) break;
            const int J = lane + 32 * i;
            uint32_t ties = __ballot_sync(0xffffffffu, J < nb && key_of(J) == vb);
            while (ties != 0u && run < target) {
              const int srcl = __ffs(ties) - 1;
              ties &= ties - 1u;
              if (lane == srcl) keep |= 1u << i;
              run += mv;
            }
          }
        }
      }

      if (sta_t >= 0) {
        int ti, hi_, wi;
        block_tile(I, g, ti, hi_, wi);
#pragma unroll 1
        for (int i = 0; i < NJ; ++i) {
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
      for (int i = 0; i < NJ; ++i) {
        const int J = lane + 32 * i;
        const bool k = (keep >> i) & 1u;
        const uint32_t bal = __ballot_sync(0xffffffffu, k);
        if (k) kv_idx[row * nb + base + __popc(bal & lt)] = J;
        if (mask != nullptr && J < nb) mask[row * nb + J] = k ? 1 : 0;
        base += __popc(bal);
      }
      if (lane == 0) kv_count[row] = base;
    }  // rows of this warp
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
  constexpr int R = mask_rows<NJ>();
  const size_t smem = (size_t)R * (g.d + g.nb) * sizeof(double) + (size_t)kMaskWarps * 256 * sizeof(uint64_t);
  const double scale = 1.0 / std::sqrt((double)g.d);
  cudaError_t e = cudaFuncSetAttribute(mask_kernel<D, NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mask_kernel<D, NJ>, kMaskThreads, smem)) !=
      cudaSuccess)
    return e;
  const int total = (g.nb + R - 1) / R * g.B * g.heads;
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
