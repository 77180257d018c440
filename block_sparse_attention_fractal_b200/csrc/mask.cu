// Adaptive block mask (NABLA summary, Metodologia 2 and 3):
//   pool_kernel: block means of Q and K ("Submuestreo"), double precision;
//   scores_kernel: the reduced scores qbar kbar^T / sqrt(d) ("Atencion
//                Reducida") on the fp64 tensor cores, into the workspace;
//   select_kernel: per row, the softmax, the CDF threshold ("Umbralizacion
//                CDF"), the optional STA union, and the ascending KV index
//                lists that the attention kernel walks ("Expansion").
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

using sm100::cp_async16;
using sm100::cp_async8;
using sm100::cp_async_commit;
using sm100::cp_async_wait;

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

// ------------------------------------------------------- reduced scores

// scores_kernel: S[bh][I][J] = scale * qbar_I . kbar_J for one 32 x 64 tile of
// one (b, head) per CTA, on the fp64 tensor cores (mma.sync m8n8k4, fp64
// multiply-add).  The head dimension is walked in chunks of 32: each chunk's
// qbar rows and kbar columns are copied to shared memory with cp.async (two
// buffers, the next chunk in flight while the current one is multiplied),
// with rows padded so the fragment loads of a half-warp hit 16 different
// banks.  Each of the 4 warps computes 32 rows x 16 columns.
constexpr int kScoreRows = 32, kScoreCols = 64, kScoreThreads = 128;
constexpr int kKC = 32;                       // head-dimension chunk
constexpr int kAStride = kKC + 4;             // doubles per staged qbar row
constexpr int kBStride = kScoreCols + 4;      // doubles per staged kbar row
constexpr int kStageDoubles = kScoreRows * kAStride + kKC * kBStride;

template <int D>
__global__ void __launch_bounds__(kScoreThreads) scores_kernel(const double* __restrict__ qbar,
                                                               const double* __restrict__ kbar, Dims g,
                                                               double scale, double* __restrict__ scores) {
  extern __shared__ __align__(16) double sm[];
  const int nb = g.nb;
  const int tiles_i = (nb + kScoreRows - 1) / kScoreRows, tiles_j = (nb + kScoreCols - 1) / kScoreCols;
  const int tj = blockIdx.x % tiles_j;
  const int ti = (blockIdx.x / tiles_j) % tiles_i;
  const size_t bh = blockIdx.x / ((unsigned)tiles_j * tiles_i);
  const int I0 = ti * kScoreRows, J0 = tj * kScoreCols;
  const double* qsrc = qbar + (bh * nb) * D;
  const double* ksrc = kbar + bh * D * (size_t)nb;
  // chunk kc into buffer buf: 32 x 32 of qbar (16-byte pieces), 32 x 64 of
  // kbar (8-byte pieces); pieces past the matrix are zero-filled (their
  // source address is clamped to the matrix start, never read)
  auto stage = [&](int kc, int buf) {
    double* As = sm + buf * kStageDoubles;
    double* Bs = As + kScoreRows * kAStride;
    for (int i = threadIdx.x; i < kScoreRows * kKC / 2; i += kScoreThreads) {
      const int r = i / (kKC / 2), c2 = i % (kKC / 2);
      const bool ok = I0 + r < nb;
      cp_async16(As + r * kAStride + 2 * c2, ok ? qsrc + (size_t)(I0 + r) * D + kc * kKC + 2 * c2 : qsrc, ok);
    }
    // kbar rows are nb doubles long (nb may be odd): 8-byte pieces
    for (int i = threadIdx.x; i < kKC * kScoreCols; i += kScoreThreads) {
      const int k = i / kScoreCols, c = i % kScoreCols;
      const bool ok = J0 + c < nb;
      cp_async8(Bs + k * kBStride + c, ok ? ksrc + (size_t)(kc * kKC + k) * nb + J0 + c : ksrc, ok);
    }
    cp_async_commit();
  };
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  double acc[4][2][2];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int n = 0; n < 2; ++n) acc[mt][n][0] = acc[mt][n][1] = 0.0;
  constexpr int NC = D / kKC;
  stage(0, 0);
#pragma unroll 1
  for (int kc = 0; kc < NC; ++kc) {
    if (kc + 1 < NC) {
      stage(kc + 1, (kc + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const double* As = sm + (kc & 1) * kStageDoubles;
    const double* Bs = As + kScoreRows * kAStride;
#pragma unroll
    for (int ks = 0; ks < kKC / 4; ++ks) {
      double av[4], bv[2];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) av[mt] = As[(mt * 8 + gq) * kAStride + 4 * ks + tq];
#pragma unroll
      for (int n = 0; n < 2; ++n) bv[n] = Bs[(4 * ks + tq) * kBStride + wid * 16 + n * 8 + gq];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int n = 0; n < 2; ++n)
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
                       : "+d"(acc[mt][n][0]), "+d"(acc[mt][n][1])
                       : "d"(av[mt]), "d"(bv[n]));
    }
    __syncthreads();   // the buffer is refilled two chunks on
  }
  // accumulator element (row gq + 8 mt, column 2 tq + e) of each 8 x 8 tile
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    const int I = I0 + mt * 8 + gq;
    if (I >= nb) continue;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      const int J = J0 + wid * 16 + n * 8 + 2 * tq;
      double* dst = scores + (bh * nb + I) * (size_t)nb + J;
      if (J + 1 < nb) {
        dst[0] = acc[mt][n][0] * scale;
        dst[1] = acc[mt][n][1] * scale;
      } else if (J < nb) {
        dst[0] = acc[mt][n][0] * scale;
      }
    }
  }
}

// --------------------------------------------------------- selection rows

constexpr int kSelThreads = 256;             // 8 warps, one row each at a time
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kHistSlots = 256 + 32;
__device__ __forceinline__ int hslot(int b) { return b + (b >> 3); }

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
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

// select_kernel: one warp per row of the reduced map (grid-stride over all
// rows of all (b, head)).  The row's scores are copied to the warp's slice of
// shared memory, turned into probabilities in place (fp64 softmax), and the
// CDF threshold picks the kept blocks (radix select below); the optional STA
// union is added and the ascending KV list written.  Lane L owns J = L + 32 i.
template <int NJ, bool kProbs>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const double* __restrict__ scores, Dims g, double thr,
                                                             int sta_t, int sta_h, int sta_w,
                                                             int32_t* __restrict__ kv_count,
                                                             int32_t* __restrict__ kv_idx,
                                                             uint8_t* __restrict__ mask) {
  extern __shared__ __align__(16) double ssm[];
  const int nb = g.nb;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double* srow = ssm + wid * (NJ * 32);                                     // this warp's row
  // histogram of 256 buckets, bucket b at b + b / 8 (the scan's lanes read 8
  // consecutive buckets each: the padding spreads them over the banks)
  unsigned long long* my_hist =
      reinterpret_cast<unsigned long long*>(ssm + kSelWarps * NJ * 32) + wid * kHistSlots;
  const unsigned long long target = __double2ull_rn((1.0 - thr) * kMassScale);
  const size_t total_rows = (size_t)g.B * g.heads * nb;

  for (size_t row = (size_t)blockIdx.x * kSelWarps + wid; row < total_rows; row += (size_t)gridDim.x * kSelWarps) {
    const int I = (int)(row % nb);
    const double* src = scores + row * nb;
    // the row into shared memory, its largest and smallest value on the way
    // (scores, or with kProbs the probabilities themselves)
    double mx = -DBL_MAX, mn = DBL_MAX;
#pragma unroll
    for (int i = 0; i < NJ; ++i) {
      const int J = lane + 32 * i;
      if (J < nb) {
        const double v = src[J];
        srow[J] = v;
        mx = fmax(mx, v);
        mn = fmin(mn, v);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    unsigned long long kmax, kmin;
    if (kProbs) {
      kmax = (unsigned long long)__double_as_longlong(mx);
      kmin = (unsigned long long)__double_as_longlong(mn);
    } else {
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
#pragma unroll
      for (int i = 0; i < NJ; ++i) {
        const int J = lane + 32 * i;
        if (J < nb) srow[J] *= rz;        // A = e / sum(e)
      }
      // The largest and smallest probabilities, by the same arithmetic as the
      // row's own entries (exp(0) = 1 exactly): their bit patterns bound the
      // keys of the radix select.
      kmax = (unsigned long long)__double_as_longlong(1.0 * rz);
      kmin = (unsigned long long)__double_as_longlong(exp(mn - mx) * rz);
    }
    auto key_of = [&](int J) { return (unsigned long long)__double_as_longlong(srow[J]); };

    // keep bits: bit i of `keep` <-> J = lane + 32 i
    uint32_t keep = 0u;
    bool keep_all = (thr == 0.0);       // thr == 0 keeps every block
    if (!keep_all) {
      // Radix select of the boundary probability vb: the smallest kept
      // value, i.e. the largest v whose mass(A >= v) reaches the target.
      // Keys are the bit patterns of the (non-negative) probabilities,
      // ordered like the values.  Each round histograms one 8-bit digit of
      // the candidates' keys (fixed-point mass and count per bucket, shared
      // memory atomics), scans the buckets from the top and keeps the bucket
      // where the running mass reaches the target; the keys above it are kept
      // for sure.  The search starts at the highest bit in which the keys
      // differ and ends when one candidate is left, or when all bits are
      // fixed (equal keys: ties).  A row whose whole mass rounds below the
      // target keeps every block.
      unsigned long long vb = kmax;      // the boundary key
      unsigned long long above = 0ull;   // packed mass of the keys above the candidates
      bool single = true;
      if (kmax == kmin) {
        // all probabilities equal: ties from the first block on
        unsigned long long tot = 0ull;
#pragma unroll
        for (int i = 0; i < NJ; ++i)
          if (lane + 32 * i < nb) tot += packed_mass(srow[lane + 32 * i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        keep_all = (tot >> 11) < target;
        single = false;
      } else {
        int top = 63 - __clzll((long long)(kmax ^ kmin));   // highest bit in which keys differ (< 63)
        unsigned long long pref = kmax >> (top + 1);         // the bits above it, common to all keys
        int cnt = 0, s = 0;
        bool first = true;
        for (;;) {
          const int w = min(8, top + 1);
          s = top + 1 - w;
#pragma unroll
          for (int k = 0; k < kHistSlots / 32; ++k) my_hist[lane + 32 * k] = 0ull;
          __syncwarp();
#pragma unroll
          for (int i = 0; i < NJ; ++i) {
            const int J = lane + 32 * i;
            if (J < nb) {
              const unsigned long long key = key_of(J);
              if ((key >> (top + 1)) == pref)
                atomicAdd(&my_hist[hslot((int)((key >> s) & ((1u << w) - 1u)))], packed_mass(srow[J]));
            }
          }
          __syncwarp();
          // lane L scans buckets 255 - 8 L down to 248 - 8 L
          unsigned long long loc[8], lsum = 0ull;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            loc[e] = my_hist[hslot(255 - 8 * lane - e)];
            lsum += loc[e];
          }
          unsigned long long incl = lsum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          if (first && (__shfl_sync(0xffffffffu, incl, 31) >> 11) < target) {
            keep_all = true;             // the whole row's mass rounds below 1 - thr
            break;
          }
          first = false;
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
          if (bal == 0u) {                // cannot happen: the candidates and `above` reach the target
            keep_all = true;
            break;
          }
          const int src_lane = __ffs(bal) - 1;
          const int e_sel = __shfl_sync(0xffffffffu, found, src_lane);
          above = __shfl_sync(0xffffffffu, before, src_lane);
          const int d_sel = 255 - 8 * src_lane - e_sel;
          cnt = (int)(my_hist[hslot(d_sel)] & 2047ull);
          pref = (pref << w) | (unsigned long long)d_sel;
          __syncwarp();   // the histogram is cleared by the next round
          if (cnt == 1 || s == 0) break;
          top = s - 1;
        }
        if (!keep_all) {
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
      }
      if (!keep_all) {
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
    }
    if (keep_all) {
#pragma unroll
      for (int i = 0; i < NJ; ++i)
        if (lane + 32 * i < nb) keep |= 1u << i;
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
    __syncwarp();   // srow is rewritten by the warp's next row
  }
}

// ----------------------------------------------------- sub-block scoring

// subblock_reduce_kernel: block importance from sub-block scores (DFSAttn
// explainer, section 2).  One warp per (b, head, query block I): for each of
// I's valid query sub-blocks a, the softmax over all valid key sub-blocks b of
// the scores S[a][b] (fp64), and the mass that falls on each key block J
// (the sum over J's sub-blocks); the masses are averaged over I's valid query
// sub-blocks.  M[bh][I][J] is written as a row of probabilities (it sums to 1)
// for the selection kernel.  `gs` describes the sub-block grid (nb = the
// number of valid sub-blocks), `g` the block grid; per = block / sub
// consecutive sub-blocks make a block.
template <int PER>
__global__ void __launch_bounds__(256) subblock_reduce_kernel(const double* __restrict__ S, Dims g, int ns,
                                                              double* __restrict__ M) {
  extern __shared__ __align__(16) double macc[];     // [8 warps][nb]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nb = g.nb;
  const size_t unit = (size_t)blockIdx.x * 8 + wid;  // bh * nb + I
  if (unit >= (size_t)g.B * g.heads * nb) return;
  const size_t bh = unit / nb;
  const int I = (int)(unit % nb);
  double* acc = macc + wid * nb;
  for (int J = lane; J < nb; J += 32) acc[J] = 0.0;
  __syncwarp();
  const int a0 = I * PER, a1 = min(a0 + PER, ns);
  for (int a = a0; a < a1; ++a) {
    const double* row = S + (bh * ns + a) * (size_t)ns;
    double mx = -DBL_MAX;
    for (int b = lane; b < ns; b += 32) mx = fmax(mx, row[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double z = 0.0;
    for (int b = lane; b < ns; b += 32) z += exp(row[b] - mx);
    z = warp_sum(z);
    const double rz = 1.0 / z;
    // per key block: the PER consecutive sub-blocks of a block sit in PER
    // consecutive lanes of one 32-wide slice (PER divides 32)
    for (int b0 = 0; b0 < ns; b0 += 32) {
      const int b = b0 + lane;
      double p = (b < ns) ? exp(row[b] - mx) * rz : 0.0;
#pragma unroll
      for (int o = PER / 2; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      if ((lane % PER) == 0 && b < ns) acc[b / PER] += p;
    }
    __syncwarp();
  }
  const double inv = 1.0 / (double)(a1 - a0);
  for (int J = lane; J < nb; J += 32) M[unit * nb + J] = acc[J] * inv;
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
  if (g.d == 128 && g.bs == 16) return launch_pool_t<128, 16>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 128 && g.bs == 32) return launch_pool_t<128, 32>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 64 && g.bs == 16) return launch_pool_t<64, 16>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 64 && g.bs == 32) return launch_pool_t<64, 32>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 128 && g.bs == 64) return launch_pool_t<128, 64>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 128 && g.bs == 128) return launch_pool_t<128, 128>(g, q, k, qbar, kbar, ctrl, seq, st);
  if (g.d == 64 && g.bs == 64) return launch_pool_t<64, 64>(g, q, k, qbar, kbar, ctrl, seq, st);
  return launch_pool_t<64, 128>(g, q, k, qbar, kbar, ctrl, seq, st);
}

size_t mask_scores_bytes(const Dims& g) { return (size_t)g.B * g.heads * g.nb * g.nb * sizeof(double); }

template <int NJ, bool kProbs>
cudaError_t launch_select_t(const Dims& g, const double* scores, double thr, int sta_t, int sta_h, int sta_w,
                            int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  const size_t smem = (size_t)kSelWarps * (NJ * 32 * sizeof(double) + kHistSlots * sizeof(uint64_t));
  cudaError_t e = cudaFuncSetAttribute(select_kernel<NJ, kProbs>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel<NJ, kProbs>, kSelThreads, smem)) !=
      cudaSuccess)
    return e;
  const size_t rows = (size_t)g.B * g.heads * g.nb;
  const size_t need = (rows + kSelWarps - 1) / kSelWarps;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>(need, (size_t)sms * std::max(1, per_sm)));
  select_kernel<NJ, kProbs><<<grid, kSelThreads, smem, st>>>(scores, g, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask);
  return cudaGetLastError();
}

template <bool kProbs>
cudaError_t launch_select(const Dims& g, const double* scores, double thr, int sta_t, int sta_h, int sta_w,
                          int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st) {
  if (g.nb <= 128) return launch_select_t<4, kProbs>(g, scores, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  if (g.nb <= 256) return launch_select_t<8, kProbs>(g, scores, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  if (g.nb <= 512)
    return launch_select_t<16, kProbs>(g, scores, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
  return launch_select_t<32, kProbs>(g, scores, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
}

template <int D>
cudaError_t launch_scores_t(const Dims& g, const double* qbar, const double* kbar, double* scores, cudaStream_t st) {
  const size_t smem = 2 * (size_t)kStageDoubles * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const size_t tiles = (size_t)((g.nb + kScoreRows - 1) / kScoreRows) * ((g.nb + kScoreCols - 1) / kScoreCols) *
                       g.B * g.heads;
  if (tiles > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  scores_kernel<D><<<(unsigned)tiles, kScoreThreads, smem, st>>>(qbar, kbar, g, 1.0 / std::sqrt((double)D), scores);
  return cudaGetLastError();
}

cudaError_t launch_mask(const Dims& g, const double* qbar, const double* kbar, double* scores, double thr,
                        int sta_t, int sta_h, int sta_w, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask,
                        cudaStream_t st) {
  cudaError_t e = (g.d == 128) ? launch_scores_t<128>(g, qbar, kbar, scores, st)
                               : launch_scores_t<64>(g, qbar, kbar, scores, st);
  if (e != cudaSuccess) return e;
  return launch_select<false>(g, scores, thr, sta_t, sta_h, sta_w, kv_count, kv_idx, mask, st);
}

SubblockLayout subblock_layout(const Dims& g, int sub) {
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  SubblockLayout L;
  L.ns = (g.N + sub - 1) / sub;
  const size_t bh = (size_t)g.B * g.heads;
  L.qbar = sizeof(Ctrl);
  L.kbar = L.qbar + a256(bh * L.ns * g.d * sizeof(double));
  L.scores = L.kbar + a256(bh * L.ns * g.d * sizeof(double));
  L.M = L.scores + a256(bh * L.ns * (size_t)L.ns * sizeof(double));
  L.total = L.M + a256(bh * g.nb * (size_t)g.nb * sizeof(double));
  return L;
}

cudaError_t launch_mask_subblock(const Dims& g, int sub, const void* q, const void* k, double thr,
                                 int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, void* workspace, uint32_t seq,
                                 cudaStream_t st) {
  const SubblockLayout L = subblock_layout(g, sub);
  char* ws = (char*)workspace;
  double* qbar = (double*)(ws + L.qbar);
  double* kbar = (double*)(ws + L.kbar);
  double* S = (double*)(ws + L.scores);
  double* M = (double*)(ws + L.M);
  // the sub-block grid: `sub` tokens per block, only the sub-blocks holding a valid token
  Dims gs = g;
  gs.bs = sub;
  gs.nb = L.ns;
  cudaError_t e = launch_pool(gs, q, k, qbar, kbar, (Ctrl*)workspace, seq, st);
  if (e != cudaSuccess) return e;
  e = (g.d == 128) ? launch_scores_t<128>(gs, qbar, kbar, S, st) : launch_scores_t<64>(gs, qbar, kbar, S, st);
  if (e != cudaSuccess) return e;
  const size_t units = (size_t)g.B * g.heads * g.nb;
  const size_t smem = 8 * (size_t)g.nb * sizeof(double);
  const unsigned grid = (unsigned)((units + 7) / 8);
  auto run = [&](auto kernel) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r != cudaSuccess) return r;
    kernel<<<grid, 256, smem, st>>>(S, g, L.ns, M);
    return cudaGetLastError();
  };
  switch (g.bs / sub) {
    case 1: e = run(subblock_reduce_kernel<1>); break;
    case 2: e = run(subblock_reduce_kernel<2>); break;
    case 4: e = run(subblock_reduce_kernel<4>); break;
    case 8: e = run(subblock_reduce_kernel<8>); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_select<true>(g, M, thr, -1, -1, -1, kv_count, kv_idx, mask, st);
}

}  // namespace bsa
