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
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kWindow = 32;
constexpr int kRounds = 6;

__device__ __forceinline__ int overlap(const uint32_t* a, const uint32_t* b, int nw) {
  int s = 0;
  for (int w = 0; w < nw; ++w) s += __popc(a[w] & b[w]);
  return s;
}

struct PlanLayout {
  int nw, stride, n_items, pow2;
  size_t off_partner, off_choice, off_key;  // in 32-bit words
  size_t bytes;
};

__host__ __device__ inline PlanLayout plan_layout(int nb, int qb) {
  PlanLayout L;
  L.nw = (nb + 31) >> 5;
  L.stride = L.nw + 1;  // padded rows: conflict-free access by row
  L.n_items = (nb + qb - 1) / qb;
  L.pow2 = 1;
  while (L.pow2 < L.n_items) L.pow2 <<= 1;
  L.off_partner = (size_t)nb * L.stride;
  L.off_choice = L.off_partner + nb;
  L.off_key = (L.off_choice + nb + 1) & ~(size_t)1;  // 8-byte aligned
  L.bytes = L.off_key * 4 + (size_t)L.pow2 * 8;
  return L;
}

// grid: B*heads CTAs.  Shared memory (PlanLayout): kept bitmaps [nb][nw + 1]
// words, partner [nb], choice [nb], item keys [pow2] (64-bit).
template <int QB>
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ kv_count,
                                                            const int32_t* __restrict__ kv_idx, Dims g,
                                                            int2* __restrict__ items) {
  extern __shared__ __align__(16) uint32_t psm[];
  __shared__ int n_keys;
  const int nb = g.nb;
  const PlanLayout L = plan_layout(nb, QB);
  const int nw = L.nw, stride = L.stride;
  uint32_t* bm = psm;
  int* partner = reinterpret_cast<int*>(psm + L.off_partner);
  int* choice = reinterpret_cast<int*>(psm + L.off_choice);
  unsigned long long* key = reinterpret_cast<unsigned long long*>(psm + L.off_key);
  const size_t bh = blockIdx.x;

  for (int i = threadIdx.x; i < nb * stride; i += blockDim.x) bm[i] = 0u;
  if (threadIdx.x == 0) n_keys = 0;
  __syncthreads();
  for (int r = threadIdx.x; r < nb; r += blockDim.x) {
    const size_t row = bh * nb + r;
    int cnt = kv_count[row];
    cnt = cnt < 0 ? 0 : (cnt > nb ? nb : cnt);
    const int32_t* list = kv_idx + row * nb;
    for (int i = 0; i < cnt; ++i) {
      const int J = list[i];
      if (J >= 0 && J < nb) bm[r * stride + (J >> 5)] |= 1u << (J & 31);
    }
    partner[r] = (QB == 2) ? -1 : r;
  }
  __syncthreads();

  if (QB == 2) {
    for (int round = 0; round < kRounds; ++round) {
      for (int r = threadIdx.x; r < nb; r += blockDim.x) {
        int best = -1, bestw = -1;
        if (partner[r] < 0) {
          for (int off = 1; off <= kWindow; ++off) {
#pragma unroll
            for (int sgn = 0; sgn < 2; ++sgn) {
              const int J = sgn ? r + off : r - off;
              if (J < 0 || J >= nb || partner[J] >= 0) continue;
              const int w = overlap(bm + r * stride, bm + J * stride, nw);
              if (w > bestw) {  // ties keep the nearer, then the lower, index
                bestw = w;
                best = J;
              }
            }
          }
        }
        choice[r] = best;
      }
      __syncthreads();
      for (int r = threadIdx.x; r < nb; r += blockDim.x) {
        const int J = choice[r];
        if (partner[r] < 0 && J >= 0 && choice[J] == r) partner[r] = J;  // mutual: both sides set it
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) {  // the rest, in index order
      int pending = -1;
      for (int r = 0; r < nb; ++r) {
        if (partner[r] >= 0) continue;
        if (pending < 0) {
          pending = r;
        } else {
          partner[pending] = r;
          partner[r] = pending;
          pending = -1;
        }
      }
      if (pending >= 0) partner[pending] = pending;  // a single block
    }
    __syncthreads();
  }

  // One key per tile (the lower block of each pair): descending union size,
  // then ascending block index.
  for (int r = threadIdx.x; r < nb; r += blockDim.x) {
    const int p = partner[r];
    if (p < r) continue;
    int u = 0;
    for (int w = 0; w < nw; ++w) u += __popc(bm[r * stride + w] | bm[p * stride + w]);
    const int slot = atomicAdd(&n_keys, 1);
    key[slot] = ((unsigned long long)(0xFFFFu - (unsigned)u) << 32) | ((unsigned long long)r << 16) |
                (unsigned long long)(p & 0xFFFF);
  }
  __syncthreads();
  for (int i = n_keys + threadIdx.x; i < L.pow2; i += blockDim.x) key[i] = ~0ull;
  __syncthreads();
  // bitonic sort of the keys, ascending
  for (int k = 2; k <= L.pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < L.pow2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = key[i], b = key[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            key[i] = b;
            key[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < L.n_items; i += blockDim.x) {
    const unsigned long long kk = key[i];
    const int r = (int)((kk >> 16) & 0xFFFFu);
    const int p = (int)(kk & 0xFFFFu);
    items[bh * L.n_items + i] = make_int2(r, (QB == 2 && p != r) ? p : -1);
  }
}

}  // namespace

size_t plan_smem_bytes(const Dims& g) { return plan_layout(g.nb, 128 / g.bs).bytes; }

size_t plan_items_bytes(const Dims& g) {
  const int qb = 128 / g.bs;
  return (size_t)g.B * g.heads * ((g.nb + qb - 1) / qb) * sizeof(int2);
}

cudaError_t launch_plan(const Dims& g, const int32_t* kv_count, const int32_t* kv_idx, int2* items,
                        cudaStream_t st) {
  const size_t smem = plan_smem_bytes(g);
  cudaError_t e;
  if (g.bs == 64) {
    e = cudaFuncSetAttribute(plan_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    plan_kernel<2><<<g.B * g.heads, kPlanThreads, smem, st>>>(kv_count, kv_idx, g, items);
  } else {
    e = cudaFuncSetAttribute(plan_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    plan_kernel<1><<<g.B * g.heads, kPlanThreads, smem, st>>>(kv_count, kv_idx, g, items);
  }
  return cudaGetLastError();
}

}  // namespace bsa
