// Block-sparse attention forward on the legacy warp-level tensor-core path
// (mma.sync.m16n8k16 bf16 -> fp32).  NABLA summary, Metodologia 2
// "Expansion": only the listed N x N tiles are computed.
//
// Baseline kernel.  One CTA (4 warps) owns 64 query rows of one query block;
// each warp owns 16 rows.  Keys and values stream through a double-buffered
// shared-memory ring in sub-tiles of 64 keys (cp.async), taken in list order.
// Scores, the online softmax (base-2, running max and sum per row) and the
// output accumulator stay in registers; P is re-used as the A operand of the
// P.V product without leaving registers.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

constexpr int kThreads = 128;
constexpr int kBM = 64;  // query rows per CTA
constexpr int kBN = 64;  // keys per sub-tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Element offset of (row, 16-byte chunk) in a [rows][D] bf16 tile whose chunks
// are XOR-swizzled by the row (conflict-free ldmatrix and cp.async).
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}


// Copies a [64][D] tile starting at global row `row0` of a [rows][D] matrix.
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16* s, const __nv_bfloat16* gsrc, size_t row0) {
  constexpr int kChunks = D / 8;
#pragma unroll
  for (int i = 0; i < (64 * kChunks) / kThreads; ++i) {
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kChunks;
    const int c = idx % kChunks;
    cp_async16(smem_u32(s + swz<D>(r, c)), gsrc + (row0 + r) * D + c * 8);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_mma_kernel(const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v,
                                                            const int32_t* __restrict__ kv_count,
                                                            const int32_t* __restrict__ kv_idx, float scale_log2,
                                                            __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                            Ctrl* ctrl, Dims g) {
  extern __shared__ __align__(128) __nv_bfloat16 sm[];
  __nv_bfloat16* Qs = sm;                  // [64][D]
  __nv_bfloat16* Ks = sm + kBM * D;        // [2][64][D]
  __nv_bfloat16* Vs = Ks + 2 * kBN * D;    // [2][64][D]

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int q0 = blockIdx.x * kBM;             // first query row of this CTA
  const int I = q0 / g.bs;                     // its query block
  const int parts = g.bs / kBN;                // 64-key sub-tiles per block
  const size_t bh = (size_t)b * g.heads + head;
  const size_t rowbase = bh * (size_t)g.Npad;
  const size_t lrow = bh * g.nb + I;

  int cnt = kv_count[lrow];
  if (cnt < 1 || cnt > g.nb) {
    if (tid == 0) report_error(ctrl, kErrCount, (uint32_t)lrow, (uint32_t)cnt, 1u);
    cnt = cnt < 0 ? 0 : (cnt > g.nb ? g.nb : cnt);
  }
  const int32_t* list = kv_idx + lrow * g.nb;
  const int nsub = cnt * parts;

  // key block of sub-tile st, or -1 when the listed index is out of range
  auto sub_block = [&](int st) -> int {
    const int J = list[st / parts];
    return (J >= 0 && J < g.nb) ? J : -1;
  };
  auto issue_sub = [&](int st, int buf) {
    int J = sub_block(st);
    if (J < 0) J = 0;  // load something harmless; every key of it is masked
    const size_t r0 = rowbase + (size_t)J * g.bs + (st % parts) * kBN;
    load_tile<D>(Ks + buf * kBN * D, k, r0);
    load_tile<D>(Vs + buf * kBN * D, v, r0);
  };

  load_tile<D>(Qs, q, rowbase + q0);
  if (nsub > 0) issue_sub(0, 0);
  cp_async_commit();

  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f}, lx[2] = {0.f, 0.f};
  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  uint32_t qf[D / 16][4];

  for (int st = 0; st < nsub; ++st) {
    const int buf = st & 1;
    if (st + 1 < nsub) {
      issue_sub(st + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (st == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int c = 2 * kk + (lane >> 4);
        ldsm_x4(smem_u32(Qs + swz<D>(r, c)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const __nv_bfloat16* Kb = Ks + buf * kBN * D;
    const __nv_bfloat16* Vb = Vs + buf * kBN * D;

    // S = Q K^T for this warp's 16 rows x 64 keys
    float sacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(Kb + swz<D>(key, c)), b0, b1, b2, b3);
        mma_bf16(sacc[2 * np], qf[kk], b0, b1);
        mma_bf16(sacc[2 * np + 1], qf[kk], b2, b3);
      }
    }

    // mask keys that are padding or belong to an out-of-range list entry
    const int J = sub_block(st);
    if (J < 0 && tid == 0 && (st % parts) == 0)
      report_error(ctrl, kErrIndex, (uint32_t)lrow, (uint32_t)list[st / parts], 2u);
    const int key0 = (J < 0) ? g.N : J * g.bs + (st % parts) * kBN;
    const int kvalid = g.N - key0;  // keys [key0, key0 + kvalid) are real
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kl = j * 8 + 2 * (lane & 3) + (e & 1);
        const float x = (kl < kvalid) ? sacc[j][e] * scale_log2 : -INFINITY;
        sacc[j][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    }
    float alpha[2], msafe[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
      mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      const float mn = fmaxf(m[h], mx[h]);
      msafe[h] = (mn == -INFINITY) ? 0.f : mn;
      alpha[h] = ex2(m[h] - msafe[h]);
      m[h] = mn;
    }
    float rs[2] = {0.f, 0.f}, rx[2] = {0.f, 0.f};
    uint32_t pf[4][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = ex2(sacc[j][0] - msafe[0]);
      const float p1 = ex2(sacc[j][1] - msafe[0]);
      const float p2 = ex2(sacc[j][2] - msafe[1]);
      const float p3 = ex2(sacc[j][3] - msafe[1]);
      const uint32_t w01 = pack_bf16(p0, p1);
      const uint32_t w23 = pack_bf16(p2, p3);
      pf[j >> 1][(j & 1) * 2 + 0] = w01;
      pf[j >> 1][(j & 1) * 2 + 1] = w23;
      // O is normalised by the sum of the rounded weights the P.V product
      // uses; the LSE by the sum of the unrounded ones
      rs[0] += __uint_as_float(w01 << 16) + __uint_as_float(w01 & 0xFFFF0000u);
      rs[1] += __uint_as_float(w23 << 16) + __uint_as_float(w23 & 0xFFFF0000u);
      rx[0] += p0 + p1;
      rx[1] += p2 + p3;
    }
    l[0] = l[0] * alpha[0] + rs[0];
    l[1] = l[1] * alpha[1] + rs[1];
    lx[0] = lx[0] * alpha[0] + rx[0];
    lx[1] = lx[1] * alpha[1] + rx[1];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      oacc[i][0] *= alpha[0];
      oacc[i][1] *= alpha[0];
      oacc[i][2] *= alpha[1];
      oacc[i][3] *= alpha[1];
    }

    // O += P V
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t a[4] = {pf[t][0], pf[t][1], pf[t][2], pf[t][3]};
#pragma unroll
      for (int u = 0; u < D / 16; ++u) {
        const int key = t * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int c = 2 * u + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(Vb + swz<D>(key, c)), b0, b1, b2, b3);
        mma_bf16(oacc[2 * u], a, b0, b1);
        mma_bf16(oacc[2 * u + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

  // epilogue: normalise, write bf16 rows (0 for padded rows) and the LSE
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    lx[h] += __shfl_xor_sync(0xffffffffu, lx[h], 1);
    lx[h] += __shfl_xor_sync(0xffffffffu, lx[h], 2);
  }
  const float kLn2 = 0.69314718055994531f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = q0 + warp * 16 + (lane >> 2) + h * 8;
    const bool real = row < g.N && l[h] > 0.f;
    const float inv = real ? 1.f / l[h] : 0.f;
    __nv_bfloat16* orow = o + (rowbase + row) * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const int col = i * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(orow + col) = pack_bf16(oacc[i][2 * h] * inv, oacc[i][2 * h + 1] * inv);
    }
    if (lse != nullptr && (lane & 3) == 0) lse[rowbase + row] = real ? (m[h] + log2f(lx[h])) * kLn2 : 0.f;
  }
}

}  // namespace

cudaError_t launch_attn_mma(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                            const int32_t* kv_idx, float scale, void* o, float* lse, Ctrl* ctrl, cudaStream_t st) {
  dim3 grid(g.Npad / kBM, g.heads, g.B);
  const float scale_log2 = scale * 1.4426950408889634f;
  const size_t smem = (size_t)(kBM + 4 * kBN) * g.d * sizeof(__nv_bfloat16);
  cudaError_t e;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(attn_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_mma_kernel<128><<<grid, kThreads, smem, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, kv_count, kv_idx, scale_log2,
        (__nv_bfloat16*)o, lse, ctrl, g);
  } else {
    e = cudaFuncSetAttribute(attn_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_mma_kernel<64><<<grid, kThreads, smem, st>>>(
        (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, kv_count, kv_idx, scale_log2,
        (__nv_bfloat16*)o, lse, ctrl, g);
  }
  return cudaGetLastError();
}

}  // namespace bsa
