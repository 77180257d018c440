// Work plan of the attention kernel: which query blocks share a 128-row tile,
// and in which order the tiles are launched.
//
// The tensor cores run M=128 x N=128 tiles at full rate but M=64 or N=64 tiles
// at about half rate, so with 64-token blocks two query blocks share one
// 128-row tile and walk the union of their KV lists.  Work that only one of
// the two needs is wasted on the other half, so blocks are paired to maximise
// the overlap of their lists: a few rounds of mutual-best-partner matching
// among blocks at most kWindow positions apart in the fractal order (where
// spatial and temporal neighbours of a video block sit), weighted by the number
// of shared KV blocks; blocks left unmatched are paired in index order.  With
// 128-token blocks every tile is one block.
//
// Tiles of each (batch, head) are then ordered by decreasing union size, so the
// longest tiles start first and short ones fill the tail of the grid.
// Pairing and order change only the schedule, never the result.
//
// Two kernels (64-token blocks):
//   overlap_kernel  many CTAs: each builds the kept-block bitmaps of 64 rows
//                   from the lists (coalesced reads) and writes, for its 32
//                   rows, the overlap with each of the next kWindow rows and
//                   the row's own distinct-block count;
//   match_kernel    one CTA per (batch, head): matching rounds over those
//                   weights, then the ordered tile list.
// With 128-token blocks only match_kernel runs, keyed by the list counts.
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kWindow = 32;          // partner candidates: rows r - kWindow .. r + kWindow
constexpr int kRounds = 6;
constexpr int kOverlapRows = 32;     // rows whose weights one overlap CTA writes
constexpr int kOverlapThreads = kOverlapRows * kWindow;  // 1024
constexpr int kMatchThreads = 1024;
static_assert(kMatchThreads >= BSA_MAX_BLOCKS, "match_kernel handles one block row per thread");
static_assert(kWindow % 2 == 0 && kMatchThreads % 64 == 0, "two lanes per row split the window in halves");

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// match_kernel keeps the weights transposed in shared memory, [offset][row]
// with this row stride (uint16 units): a warp's 32 rows read 32 neighbouring
// entries of one offset, free of bank conflicts.
__host__ __device__ inline int wts_stride(int nb) { return nb + (nb & 1) + 2; }

// Plan region of the workspace: items | weights | counts (the last two only
// with 64-token blocks).
struct PlanRegion {
  size_t items, weights, counts, counter, total;
};

PlanRegion plan_region(const Dims& g) {
  const size_t bh = (size_t)g.B * g.heads;
  const int qb = 128 / g.bs;
  PlanRegion R;
  R.items = 0;
  const size_t items_bytes = bh * ((g.nb + qb - 1) / qb) * sizeof(int2);
  R.weights = align256(items_bytes);
  const size_t w_bytes = (qb == 2) ? bh * g.nb * kWindow * sizeof(uint16_t) : 0;
  R.counts = R.weights + align256(w_bytes);
  const size_t c_bytes = (qb == 2) ? bh * g.nb * sizeof(int32_t) : 0;
  R.counter = R.counts + align256(c_bytes);  // work counter of the persistent attention kernel
  R.total = R.counter + 256;
  return R;
}

// grid (ceil(nb / 32), B*heads), 1024 threads.  Shared memory: bitmaps of
// rows [r0, r0 + 64) with a padded stride (conflict-free by row).
__global__ void __launch_bounds__(kOverlapThreads) overlap_kernel(const int32_t* __restrict__ kv_count,
                                                                  const int32_t* __restrict__ kv_idx, Dims g,
                                                                  uint16_t* __restrict__ weights,
                                                                  int32_t* __restrict__ counts) {
  constexpr int kRowsHeld = kOverlapRows + kWindow;
  constexpr int kStride = BSA_MAX_BLOCKS / 32 + 1;
  __shared__ uint32_t bm[kRowsHeld * kStride];
  const int nb = g.nb;
  const int nw = (nb + 31) >> 5;
  const size_t bh = blockIdx.y;
  const int r0 = blockIdx.x * kOverlapRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < kRowsHeld * kStride; i += kOverlapThreads) bm[i] = 0u;
  __syncthreads();
  for (int lr = warp; lr < kRowsHeld; lr += kOverlapThreads / 32) {
    const int r = r0 + lr;
    if (r >= nb) break;
    const size_t row = bh * nb + r;
    int cnt = kv_count[row];
    cnt = cnt < 0 ? 0 : (cnt > nb ? nb : cnt);
    const int32_t* list = kv_idx + row * nb;
    for (int e = lane; e < cnt; e += 32) {
      const int J = list[e];
      if (J >= 0 && J < nb) atomicOr(&bm[lr * kStride + (J >> 5)], 1u << (J & 31));
    }
  }
  __syncthreads();

  const int lr = threadIdx.x / kWindow;
  const int off = threadIdx.x % kWindow + 1;
  const int r = r0 + lr;
  if (r >= nb) return;
  int w = 0;
  if (r + off < nb) {
    const uint32_t* a = bm + lr * kStride;
    const uint32_t* b = bm + (lr + off) * kStride;
    for (int i = 0; i < nw; ++i) w += __popc(a[i] & b[i]);
  }
  weights[(bh * nb + r) * kWindow + (off - 1)] = (uint16_t)w;
  if (off == 1) {
    int c = 0;
    for (int i = 0; i < nw; ++i) c += __popc(bm[lr * kStride + i]);
    counts[bh * nb + r] = c;
  }
}

// grid B*heads, 1024 threads.  QB = 2: pairs rows by the weights; QB = 1:
// every row is its own tile.  Both then sort the tiles by decreasing size.
template <int QB>
__global__ void __launch_bounds__(kMatchThreads) match_kernel(const int32_t* __restrict__ kv_count,
                                                              const uint16_t* __restrict__ weights,
                                                              const int32_t* __restrict__ counts, Dims g,
                                                              int2* __restrict__ items, int* __restrict__ work) {
  __shared__ int partner[BSA_MAX_BLOCKS];
  __shared__ int choice[BSA_MAX_BLOCKS];
  __shared__ int cnt_s[BSA_MAX_BLOCKS];
  __shared__ int unm[BSA_MAX_BLOCKS];     // unmatched rows, ascending
  __shared__ int bin[BSA_MAX_BLOCKS];      // tiles per union size (bin nb - size), then their first slot
  __shared__ int wsum[32];
  __shared__ int n_unm;
  extern __shared__ uint16_t wts[];   // [kWindow][S]: weight of rows (r, r + off) at (off - 1) * S + r (QB == 2)
  const int nb = g.nb;
  const size_t bh = blockIdx.x;
  const int n_items = (nb + QB - 1) / QB;

  if (threadIdx.x == 0 && blockIdx.x == 0) *work = 0;
  for (int r = threadIdx.x; r < nb; r += kMatchThreads) {
    int c;
    if (QB == 2) {
      c = counts[bh * nb + r];
    } else {
      c = kv_count[bh * nb + r];
      c = c < 0 ? 0 : (c > nb ? nb : c);
    }
    cnt_s[r] = c;
    partner[r] = (QB == 2) ? -1 : r;
  }
  const int S = wts_stride(nb);
  if (QB == 2) {
    const uint16_t* src = weights + bh * nb * kWindow;
    for (int i = threadIdx.x; i < nb * kWindow; i += kMatchThreads) wts[(i % kWindow) * S + i / kWindow] = src[i];
  }
  __syncthreads();

  if (QB == 2) {
    // Each unmatched row's heaviest free partner within the window, offsets
    // scanned nearest first (lower index first at equal offset), a strictly
    // heavier weight replacing the pick: ties keep the nearer, then the
    // lower, index.  Up to kMatchThreads / 2 rows, two adjacent lanes scan
    // half the offsets each and the far half's pick wins only when strictly
    // heavier, which is the same rule.
    const bool split = nb <= kMatchThreads / 2;
    auto scan = [&](int r, int off0, int off1, int& best, int& bestw) {
      for (int off = off0; off <= off1; ++off) {
        const int lo = r - off, hi = r + off;
        if (lo >= 0 && partner[lo] < 0) {
          const int w = wts[(off - 1) * S + lo];
          if (w > bestw) { bestw = w; best = lo; }
        }
        if (hi < nb && partner[hi] < 0) {
          const int w = wts[(off - 1) * S + r];
          if (w > bestw) { bestw = w; best = hi; }
        }
      }
    };
    for (int round = 0; round < kRounds; ++round) {
      if (split) {
        const int r = threadIdx.x >> 1, part = threadIdx.x & 1;
        int best = -1, bestw = -1;
        if (r < nb && partner[r] < 0) scan(r, 1 + part * (kWindow / 2), (part + 1) * (kWindow / 2), best, bestw);
        const int far_w = __shfl_down_sync(0xffffffffu, bestw, 1);
        const int far_b = __shfl_down_sync(0xffffffffu, best, 1);
        if (part == 0 && r < nb) choice[r] = (far_w > bestw) ? far_b : best;
      } else {
        for (int r = threadIdx.x; r < nb; r += kMatchThreads) {
          int best = -1, bestw = -1;
          if (partner[r] < 0) scan(r, 1, kWindow, best, bestw);
          choice[r] = best;
        }
      }
      __syncthreads();
      int formed = 0;
      for (int r = threadIdx.x; r < nb; r += kMatchThreads) {
        const int J = choice[r];
        if (partner[r] < 0 && J >= 0 && choice[J] == r) {  // mutual: both sides set it
          partner[r] = J;
          formed = 1;
        }
      }
      if (!__syncthreads_or(formed)) break;
    }
    // The rest, paired in index order: rank of each unmatched row by a
    // block-wide prefix count, then pairs (rank 2k, rank 2k + 1).
    {
      const int r = threadIdx.x;   // nb <= kMatchThreads: one row per thread
      const bool un = r < nb && partner[r] < 0;
      const int lane = r & 31, wid = r >> 5;
      const uint32_t bal = __ballot_sync(0xffffffffu, un);
      if (lane == 0) wsum[wid] = __popc(bal);
      __syncthreads();
      if (wid == 0) {
        const int v = wsum[lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        wsum[lane] = incl - v;                       // exclusive prefix of warp totals
        if (lane == 31) n_unm = incl;
      }
      __syncthreads();
      if (un) unm[wsum[wid] + __popc(bal & ((1u << lane) - 1u))] = r;
      __syncthreads();
      const int n = n_unm;
      for (int k = threadIdx.x; 2 * k < n; k += kMatchThreads) {
        const int a = unm[2 * k];
        const int b2 = (2 * k + 1 < n) ? unm[2 * k + 1] : a;   // an odd one out is a single block
        partner[a] = b2;
        partner[b2] = a;
      }
    }
    __syncthreads();
  }

  // Tiles (the lower block of each pair) in decreasing union size: a counting
  // sort on the size (at most nb), ties in any order (only the launch order of
  // equal tiles depends on it, never the result).
  for (int i = threadIdx.x; i < nb; i += kMatchThreads) bin[i] = 0;
  __syncthreads();
  int usz = -1, ur = -1, up = -1;
  {
    const int r = threadIdx.x;
    if (r < nb) {
      const int p = partner[r];
      if (p >= r) {
        int u = cnt_s[r];
        if (QB == 2 && p != r) {
          u += cnt_s[p];
          if (p - r <= kWindow) u -= wts[(p - r - 1) * S + r];
        }
        usz = min(max(u, 1), nb);
        ur = r;
        up = p;
        atomicAdd(&bin[nb - usz], 1);   // bin 0 = largest size
      }
    }
  }
  __syncthreads();
  {  // exclusive prefix over the nb bins (one per thread)
    const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
    const int v = (t < nb) ? bin[t] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int wv = wsum[lane];
      int wi = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += x;
      }
      wsum[lane] = wi - wv;
    }
    __syncthreads();
    if (t < nb) bin[t] = wsum[wid] + incl - v;
  }
  __syncthreads();
  if (usz >= 0) {
    const int slot = atomicAdd(&bin[nb - usz], 1);
    if (slot < n_items) items[bh * n_items + slot] = make_int2(ur, (QB == 2 && up != ur) ? up : -1);
  }
}

}  // namespace

size_t plan_region_bytes(const Dims& g) { return plan_region(g).total; }

int* plan_work_counter(const Dims& g, int2* items) { return (int*)((char*)items + plan_region(g).counter); }

cudaError_t launch_plan(const Dims& g, const int32_t* kv_count, const int32_t* kv_idx, int2* items,
                        cudaStream_t st) {
  const PlanRegion R = plan_region(g);
  const int bh = g.B * g.heads;
  cudaError_t e;
  if (g.bs == 64) {
    uint16_t* weights = (uint16_t*)((char*)items + R.weights);
    int32_t* counts = (int32_t*)((char*)items + R.counts);
    const dim3 grid((g.nb + kOverlapRows - 1) / kOverlapRows, bh);
    overlap_kernel<<<grid, kOverlapThreads, 0, st>>>(kv_count, kv_idx, g, weights, counts);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = (size_t)wts_stride(g.nb) * kWindow * sizeof(uint16_t);
    e = cudaFuncSetAttribute(match_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    match_kernel<2><<<bh, kMatchThreads, smem, st>>>(kv_count, weights, counts, g, items,
                                                     plan_work_counter(g, items));
  } else {
    match_kernel<1><<<bh, kMatchThreads, 0, st>>>(kv_count, nullptr, nullptr, g, items, plan_work_counter(g, items));
  }
  return cudaGetLastError();
}

}  // namespace bsa
