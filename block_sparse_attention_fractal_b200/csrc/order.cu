// Hilbert-curve token order (DFSAttn explainer, section 1, "El barajado de la
// Curva de Hilbert"): tokens are ordered along a 3-D Hilbert curve so that
// neighbours in the sequence are neighbours in space and time.
//
// The curve is J. Skilling's construction ("Programming the Hilbert curve",
// AIP Conf. Proc. 707, 2004), axes (t, h, w), over the smallest power-of-two
// cube that holds the T x H x W grid; grid points keep the cube's order and
// the points outside the grid are skipped.  The position of token n is the
// number of grid points with a smaller curve index, found without a sort:
//   hilbert_mark_kernel    each token's index; its bit set in a bitmap over
//                          the cube (one bit per curve position)
//   popc_blocks_kernel     popcount of each 64-word block of the bitmap
//   scan_blocks_kernel     exclusive prefix over the blocks (one CTA)
//   rank_kernel            rank = prefix of the token's block + popcounts of
//                          the words before it in the block + the bits below
//                          it in its word; order[rank] = n
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kWordsPerBlock = 64;   // bitmap words per block (summed by one warp of popc_blocks_kernel)

// Curve index of (x0, x1, x2) on the cube of side 2^bits: the coordinates
// become the "transposed" index by undoing the excess work of the reflected
// Gray code from the top bit level down (an axis whose bit q is set flips the
// lower bits of axis 0; otherwise axes 0 and i exchange their lower bits),
// then a Gray encoding across the axes and a final fix-up of the lower bits;
// the index interleaves the three words from the top bit down, axis 0 first.
__device__ __forceinline__ uint32_t hilbert_index3(uint32_t x0, uint32_t x1, uint32_t x2, int bits) {
  uint32_t x[3] = {x0, x1, x2};
  const uint32_t top = 1u << (bits - 1);
  for (uint32_t q = top; q > 1u; q >>= 1) {
    const uint32_t low = q - 1u;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (x[i] & q) {
        x[0] ^= low;
      } else {
        const uint32_t t = (x[0] ^ x[i]) & low;
        x[0] ^= t;
        x[i] ^= t;
      }
    }
  }
  x[1] ^= x[0];
  x[2] ^= x[1];
  uint32_t fix = 0u;
  for (uint32_t q = top; q > 1u; q >>= 1)
    if (x[2] & q) fix ^= q - 1u;
  x[0] ^= fix;
  x[1] ^= fix;
  x[2] ^= fix;
  uint32_t h = 0u;
  for (int b = bits - 1; b >= 0; --b) {
    h = (h << 1) | ((x[0] >> b) & 1u);
    h = (h << 1) | ((x[1] >> b) & 1u);
    h = (h << 1) | ((x[2] >> b) & 1u);
  }
  return h;
}

__global__ void hilbert_mark_kernel(Dims g, int bits, uint32_t* __restrict__ keys, uint32_t* __restrict__ bitmap) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= g.N) return;
  const int HW = g.H * g.W;
  const int t = n / HW, r = n - t * HW;
  const int h = r / g.W, w = r - h * g.W;
  const uint32_t key = hilbert_index3((uint32_t)t, (uint32_t)h, (uint32_t)w, bits);
  keys[n] = key;
  atomicOr(&bitmap[key >> 5], 1u << (key & 31u));
}

__global__ void __launch_bounds__(256) popc_blocks_kernel(const uint32_t* __restrict__ bitmap, size_t words,
                                                          size_t blocks, uint32_t* __restrict__ block_sums) {
  const size_t blk = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // one warp per block
  if (blk >= blocks) return;
  const int lane = threadIdx.x & 31;
  const size_t w0 = blk * kWordsPerBlock;
  uint32_t s = 0u;
#pragma unroll
  for (int i = 0; i < kWordsPerBlock / 32; ++i)
    if (w0 + lane + 32 * i < words) s += __popc(bitmap[w0 + lane + 32 * i]);
  s = __reduce_add_sync(0xffffffffu, s);
  if (lane == 0) block_sums[blk] = s;
}

// Exclusive prefix over `n` block sums, in place (one CTA of 1024 threads,
// 1024 sums per round).
__global__ void __launch_bounds__(1024) scan_blocks_kernel(uint32_t* __restrict__ sums, int n) {
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t carry;
  if (threadIdx.x == 0) carry = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const uint32_t v = (i < n) ? sums[i] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const uint32_t x = wsum[lane];
      uint32_t xi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += t;
      }
      wsum[lane] = xi - x;   // exclusive prefix of the warp totals
    }
    __syncthreads();
    const uint32_t c0 = carry;
    if (i < n) sums[i] = c0 + wsum[wid] + incl - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry = c0 + wsum[31] + incl;
    __syncthreads();
  }
}

__global__ void rank_kernel(Dims g, const uint32_t* __restrict__ keys, const uint32_t* __restrict__ bitmap,
                            const uint32_t* __restrict__ block_prefix, int32_t* __restrict__ order) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= g.N) return;
  const uint32_t key = keys[n];
  const size_t word = key >> 5;
  const size_t blk = word / kWordsPerBlock;
  uint32_t rank = block_prefix[blk];
  for (size_t w = blk * kWordsPerBlock; w < word; ++w) rank += __popc(bitmap[w]);
  rank += __popc(bitmap[word] & ((1u << (key & 31u)) - 1u));
  order[rank] = n;
}

}  // namespace

int hilbert_bits(const Dims& g) {
  const int m = max(g.T, max(g.H, g.W));
  int b = 1;
  while ((1 << b) < m) ++b;
  return b;
}

HilbertLayout hilbert_layout(const Dims& g) {
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const int bits = hilbert_bits(g);
  HilbertLayout L;
  L.bits = bits;
  L.words = ((size_t)1 << (3 * bits)) / 32 + 1;
  L.blocks = (L.words + kWordsPerBlock - 1) / kWordsPerBlock;
  L.keys = 0;
  L.bitmap = a256((size_t)g.N * sizeof(uint32_t));
  L.block_sums = L.bitmap + a256(L.words * sizeof(uint32_t));
  L.total = L.block_sums + a256(L.blocks * sizeof(uint32_t));
  return L;
}

cudaError_t launch_hilbert_order(const Dims& g, int32_t* order, void* scratch, cudaStream_t st) {
  const HilbertLayout L = hilbert_layout(g);
  char* base = (char*)scratch;
  uint32_t* keys = (uint32_t*)(base + L.keys);
  uint32_t* bitmap = (uint32_t*)(base + L.bitmap);
  uint32_t* sums = (uint32_t*)(base + L.block_sums);
  cudaError_t e = cudaMemsetAsync(bitmap, 0, L.words * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const unsigned tok_grid = (unsigned)((g.N + 255) / 256);
  hilbert_mark_kernel<<<tok_grid, 256, 0, st>>>(g, L.bits, keys, bitmap);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  popc_blocks_kernel<<<(unsigned)((L.blocks + 7) / 8), 256, 0, st>>>(bitmap, L.words, L.blocks, sums);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  scan_blocks_kernel<<<1, 1024, 0, st>>>(sums, (int)L.blocks);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  rank_kernel<<<tok_grid, 256, 0, st>>>(g, keys, bitmap, sums, order);
  return cudaGetLastError();
}

}  // namespace bsa
