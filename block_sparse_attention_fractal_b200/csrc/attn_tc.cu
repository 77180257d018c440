// Block-sparse attention forward on the sm_100a tensor cores (tcgen05 + TMEM,
// TMA-staged tiles).  NABLA summary, Metodologia 2 "Expansion": only the
// listed N x N tiles are computed.
//
// One CTA owns a query tile of 128 rows: one query block (block 128) or two
// consecutive query blocks (block 64; rows 0-63 and 64-127).  It walks the
// union of the tile's KV lists in tiles of 128 keys (one entry of 128 keys,
// or two entries of 64) and, per KV tile:
//   S = Q K^T     tcgen05.mma, A = Q and B = K from shared memory, S in TMEM
//   softmax       one thread per query row reads its S row from TMEM, masks
//                 the keys its query block does not keep (and padding), keeps
//                 a running base-2 max (rescaling O only when the max grows
//                 by more than 8) and writes P = 2^(s - m) as bf16 back into
//                 the S columns of TMEM; O is normalised by the sum of the
//                 rounded weights, the LSE uses the unrounded ones
//   O += P V      tcgen05.mma with A = P from TMEM and B = V (MN-major) from
//                 shared memory, O in TMEM
// Roles: warp 0 issues TMA loads, warp 1 issues MMAs (one elected thread),
// warps 2-5 run the softmax and the epilogue.  Two CTAs share an SM (TMEM
// 256 columns each), so one CTA's softmax overlaps the other's MMAs.
// Every mbarrier wait is bounded; on expiry the CTA records BSA_ERR_TIMEOUT
// in the workspace error word and leaves.
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "softmax_math.cuh"
#include "tma_host.h"

namespace bsa {

namespace {

using namespace sm100;
using namespace smx;

constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 250ull * 1000ull * 1000ull;  // 250 ms: far beyond any legitimate wait
constexpr uint32_t kTmemCols = 256;
// One pair of scores in kPolyEvery takes the software exp2 (0 = none).
constexpr int kPolyEvery = 0;

struct Ctl {
  uint64_t q_full, k_full, k_empty, v_full, v_empty, s_full, p_full, pv_done;
  uint32_t tmem_base;
  int n_ent;
  int pad[2];
  uint32_t bm[2][BSA_MAX_BLOCKS / 32];  // kept blocks of each query block of the tile
  uint16_t ent[BSA_MAX_BLOCKS];         // union of the lists, ascending
  uint8_t mem[BSA_MAX_BLOCKS];          // bit h: entry kept by query block h
};

__device__ __forceinline__ void timeout(Ctrl* ctrl, uint32_t site) {
  report_error(ctrl, kErrTimeout, blockIdx.x, threadIdx.x, site);
}

// Bounded wait; gives up early once any CTA of the launch has timed out.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl) {
  return mbar_wait_ns(bar, parity, kWaitNs, &ctrl->error, kErrTimeout);
}

// Same, with one verdict for the whole warp (tcgen05.ld/st that follow are
// warp-collective and must not run in a partial warp).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Ctrl* ctrl) {
  const bool ok = wait(bar, parity, ctrl);
  return __all_sync(0xffffffffu, ok);
}

template <int D, int BS, bool WITH_LSE>
__global__ void __launch_bounds__(kThreads, 2) attn_tc_kernel(const __grid_constant__ CUtensorMap mq,
                                                              const __grid_constant__ CUtensorMap mk,
                                                              const __grid_constant__ CUtensorMap mv,
                                                              const int32_t* __restrict__ kv_count,
                                                              const int32_t* __restrict__ kv_idx,
                                                              const int2* __restrict__ items, float scale_log2,
                                                              __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                              Ctrl* ctrl, Dims g, int items_per_bh) {
  constexpr int QB = 128 / BS;          // query blocks per tile
  constexpr int E = 128 / BS;           // list entries per KV tile
  constexpr int CH = D / 64;            // 64-column (128-byte) chunks of a row
  constexpr uint32_t kTile = 128u * D * 2u;
  constexpr uint32_t kChunk = 128u * 128u;  // bytes of one chunk of a 128-row tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = base + kTile;
  uint8_t* sV = base + 2 * kTile;
  Ctl& c = *reinterpret_cast<Ctl*>(base + 3 * kTile);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int item = blockIdx.x % items_per_bh;
  const int bh = blockIdx.x / items_per_bh;
  const int nb = g.nb;
  const int nw = (nb + 31) >> 5;

  // the tile's query blocks, from the plan (second block -1 when single)
  const int2 it = items[(size_t)bh * items_per_bh + item];
  int qblk[QB];
  bool qval[QB];
  qblk[0] = it.x;
  qval[0] = it.x >= 0 && it.x < nb;
  if (QB == 2) {
    qblk[QB - 1] = it.y;
    qval[QB - 1] = it.y >= 0 && it.y < nb;
  }
  if (!qval[0]) {  // a corrupt plan: compute nothing for this tile
    qblk[0] = 0;
  }

  if (tid == 0) {
    mbar_init(&c.q_full, 1);
    mbar_init(&c.k_full, 1);
    mbar_init(&c.k_empty, 1);
    mbar_init(&c.v_full, 1);
    mbar_init(&c.v_empty, 1);
    mbar_init(&c.s_full, 1);
    mbar_init(&c.p_full, 128);
    mbar_init(&c.pv_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  for (int i = tid; i < 2 * (BSA_MAX_BLOCKS / 32); i += kThreads) (&c.bm[0][0])[i] = 0u;
  __syncthreads();

  // Kept-block bitmaps of the tile's query blocks (duplicates collapse).
#pragma unroll
  for (int h = 0; h < QB; ++h) {
    if (!qval[h]) continue;
    const size_t row = (size_t)bh * nb + qblk[h];
    int cnt = kv_count[row];
    if (cnt < 1 || cnt > nb) {
      if (tid == 0) report_error(ctrl, kErrCount, (uint32_t)row, (uint32_t)cnt, 3u);
      cnt = cnt < 0 ? 0 : (cnt > nb ? nb : cnt);
    }
    const int32_t* list = kv_idx + row * nb;
    for (int i = tid; i < cnt; i += kThreads) {
      const int J = list[i];
      if (J >= 0 && J < nb) atomicOr(&c.bm[h][J >> 5], 1u << (J & 31));
      else report_error(ctrl, kErrIndex, (uint32_t)row, (uint32_t)J, 4u);
    }
  }
  __syncthreads();

  // Union list in ascending order (warp 0): ballot-free compaction by words.
  if (warp == 0) {
    int off = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int wi = w0 + lane;
      const uint32_t b0 = (wi < nw) ? c.bm[0][wi] : 0u;
      const uint32_t b1 = (QB > 1 && wi < nw) ? c.bm[1][wi] : 0u;
      uint32_t u = b0 | b1;
      const int n = __popc(u);
      int incl = n;
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += t;
      }
      int pos = off + incl - n;
      while (u != 0u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1u;
        c.ent[pos] = (uint16_t)(wi * 32 + bit);
        c.mem[pos] = (uint8_t)(((b0 >> bit) & 1u) | (((b1 >> bit) & 1u) << 1));
        ++pos;
      }
      off += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) c.n_ent = off;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = c.tmem_base;
  const int n_ent = c.n_ent;
  const int n_tiles = (n_ent + E - 1) / E;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      mbar_arrive_expect_tx(&c.q_full, kTile);
#pragma unroll
      for (int ch = 0; ch < CH; ++ch) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int row0;
          if (QB == 2) row0 = (qval[h & (QB - 1)] ? qblk[h & (QB - 1)] : qblk[0]) * 64;
          else row0 = qblk[0] * 128 + 64 * h;
          tma_load_3d(sQ + ch * kChunk + h * (kChunk / 2), &mq, &c.q_full, ch * 64, row0, bh);
        }
      }
      for (int j = 0; j < n_tiles; ++j) {
        int krow[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (E == 2) {
            const int idx = (2 * j + h < n_ent) ? 2 * j + h : 2 * j;
            krow[h] = (int)c.ent[idx] * 64;
          } else {
            krow[h] = (int)c.ent[j] * 128 + 64 * h;
          }
        }
        if (j > 0 && !wait(&c.k_empty, (j - 1) & 1, ctrl)) { timeout(ctrl, 10); break; }
        mbar_arrive_expect_tx(&c.k_full, kTile);
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sK + ch * kChunk + h * (kChunk / 2), &mk, &c.k_full, ch * 64, krow[h], bh);
        if (j > 0 && !wait(&c.v_empty, (j - 1) & 1, ctrl)) { timeout(ctrl, 11); break; }
        mbar_arrive_expect_tx(&c.v_full, kTile);
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sV + ch * kChunk + h * (kChunk / 2), &mv, &c.v_full, ch * 64, krow[h], bh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t tS = tmem, tO = tmem + 128;
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
      bool ok = wait(&c.q_full, 0, ctrl);
      if (!ok) timeout(ctrl, 20);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (!wait(&c.k_full, j & 1, ctrl)) { timeout(ctrl, 21); break; }
        if (j > 0 && !wait(&c.pv_done, (j - 1) & 1, ctrl)) { timeout(ctrl, 22); break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          mma_ss(tS, smem_desc_sw128(aQ + off, 16, 1024), smem_desc_sw128(aK + off, 16, 1024), idS, kk > 0);
        }
        mma_commit(&c.s_full);
        mma_commit(&c.k_empty);
        if (!wait(&c.p_full, j & 1, ctrl)) { timeout(ctrl, 23); break; }
        if (!wait(&c.v_full, j & 1, ctrl)) { timeout(ctrl, 24); break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tO, tS + kk * 8, smem_desc_sw128(aV + kk * 2048, kChunk, 1024), idO, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&c.pv_done);
        mma_commit(&c.v_empty);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;                         // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;                    // query row of the tile
    const int half = (QB == 2) ? (r >> 6) : 0;
    const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
    float m = -INFINITY;
    float l = 0.f, lx = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      int lim[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        int key0, kept;
        if (E == 2) {
          const int idx = 2 * j + h;
          kept = (idx < n_ent) ? ((c.mem[idx] >> half) & 1) : 0;
          key0 = (idx < n_ent) ? (int)c.ent[idx] * 64 : 0;
        } else {
          kept = 1;
          key0 = (int)c.ent[j] * 128 + 64 * h;
        }
        lim[h] = kept ? max(0, min(64, g.N - key0)) : 0;
      }
      if (!wait_warp(&c.s_full, j & 1, ctrl)) { timeout(ctrl, 30); ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(trow + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(trow + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(trow + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(trow + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      const float* x = reinterpret_cast<const float*>(sr);
      // Row max of the raw scores over the kept, real keys (scale > 0 keeps
      // the order), then in the base-2 domain.
      float mx = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (lim[h] == 64) {
#pragma unroll
          for (int i = 0; i < 64; i += 2) mx = fmax3(mx, x[h * 64 + i], x[h * 64 + i + 1]);
        } else if (lim[h] > 0) {
#pragma unroll
          for (int i = 0; i < 64; ++i) mx = (i < lim[h]) ? fmaxf(mx, x[h * 64 + i]) : mx;
        }
      }
      const float mnew = fmaxf(m, mx * scale_log2);
      // The running max moves only when it grows by more than 8 (a factor 256
      // in p), or when it is set for the first time.  The O rescale that goes
      // with it uses warp-collective TMEM accesses, so the whole warp takes it
      // when any lane needs it; lanes whose max did not move use alpha = 1.
      const bool grow = mnew > m + 8.0f;
      if (__any_sync(0xffffffffu, grow && m != -INFINITY)) {
        // O is stable: S of tile j was issued after the P.V product of tile j-1 completed.
        const float alpha = (grow && m != -INFINITY) ? ex2f(m - mnew) : 1.0f;
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t ov[32];
          tmem_ld32(trow + 128 + cc, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(trow + 128 + cc, ov);
        }
        tmem_wait_st();
        l *= alpha;
        lx *= alpha;
      }
      if (grow) m = mnew;
      const float nm = (m == -INFINITY) ? 0.f : -m;
      // p = 2^(s * scale_log2 - m): one packed FFMA per two scores, then the
      // MUFU ex2 for most pairs and the FMA-pipe polynomial for one pair in
      // kPolyEvery.  O is normalised by the sum of the bf16-rounded weights
      // the P.V product uses (an exact convex combination of V rows up to
      // accumulation rounding); the LSE, when asked for, uses the fp32 sum of
      // the unrounded ones.  Halves the row's query block does not keep cost
      // nothing.
      const float2 sl2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(nm, nm);
      float rs[2] = {0.f, 0.f};
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {   // 32 keys -> 16 packed columns at a time
          uint32_t pk[16];
          if (lim[h] > 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = qq * 32 + 2 * i;  // key within the half
              const float2 y = ffma2(make_float2(x[h * 64 + c], x[h * 64 + c + 1]), sl2, nm2);
              float2 p;
              if (kPolyEvery > 0 && (i % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
                p = exp2_poly2(y);
              } else {
                p.x = ex2f(y.x);
                p.y = ex2f(y.y);
              }
              if (lim[h] < 64) {
                p.x = (c < lim[h]) ? p.x : 0.f;
                p.y = (c + 1 < lim[h]) ? p.y : 0.f;
              }
              pk[i] = pack_bf16(p.x, p.y);
              rs[i & 1] = add_bf16x2(rs[i & 1], pk[i]);
              if (WITH_LSE) acc = fadd2(acc, p);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
          // keys [64h + 32qq, +32) -> bf16 pairs in TMEM columns [32h + 16qq, +16)
          // (those S columns are already in registers)
          tmem_st16(trow + 32 * h + 16 * qq, pk);
        }
      }
      l += rs[0] + rs[1];
      if (WITH_LSE) lx += acc.x + acc.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&c.p_full);
    }

    // epilogue: O / l -> bf16 rows, LSE
    if (ok && n_tiles > 0) {
      if (!wait_warp(&c.pv_done, (n_tiles - 1) & 1, ctrl)) { timeout(ctrl, 31); ok = false; }
      tc_fence_after();
    }
    int grow;
    if (QB == 2) grow = qval[half] ? qblk[half] * 64 + (r & 63) : -1;
    else grow = qval[0] ? qblk[0] * 128 + r : -1;
    if (grow >= 0 && grow < g.Npad) {
      const bool real = ok && n_tiles > 0 && grow < g.N && l > 0.f;
      const float inv = real ? 1.f / l : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(o + ((size_t)bh * g.Npad + grow) * D);
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t ov[32];
        if (ok && n_tiles > 0) {
          tmem_ld32(trow + 128 + cc, ov);
          tmem_wait_ld();
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = real ? pack_bf16(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv) : 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) orow[cc / 8 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
      if (WITH_LSE)
        lse[(size_t)bh * g.Npad + grow] = real ? (m + __log2f(lx)) * 0.69314718055994531f : 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int BS, bool WITH_LSE>
cudaError_t launch_tc(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                      const int32_t* kv_idx, const int2* items, float scale, void* o, float* lse, Ctrl* ctrl,
                      cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)g.Npad, bhs = (uint64_t)g.B * g.heads;
  if (!make_map_bf16_3d(&mq, q, D, rows, bhs, 64, 64) || !make_map_bf16_3d(&mk, k, D, rows, bhs, 64, 64) ||
      !make_map_bf16_3d(&mv, v, D, rows, bhs, 64, 64))
    return cudaErrorInvalidValue;
  const int n_items = (BS == 64) ? (g.nb + 1) / 2 : g.nb;
  const size_t smem = 3u * 128u * D * 2u + sizeof(Ctl) + 1024u;
  cudaError_t e =
      cudaFuncSetAttribute(attn_tc_kernel<D, BS, WITH_LSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(bhs * n_items));
  attn_tc_kernel<D, BS, WITH_LSE><<<grid, kThreads, smem, st>>>(mq, mk, mv, kv_count, kv_idx, items,
                                                      scale * 1.4426950408889634f, (__nv_bfloat16*)o, lse, ctrl, g,
                                                      n_items);
  return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_tc_lse(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                          const int32_t* kv_idx, const int2* items, float scale, void* o, float* lse, Ctrl* ctrl,
                          cudaStream_t st) {
  if (lse != nullptr) return launch_tc<D, BS, true>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
  return launch_tc<D, BS, false>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
}

}  // namespace

cudaError_t launch_attn_tc(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                           const int32_t* kv_idx, const int2* items, float scale, void* o, float* lse, Ctrl* ctrl,
                           cudaStream_t st) {
  if (g.d == 128 && g.bs == 64)
    return launch_tc_lse<128, 64>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
  if (g.d == 128 && g.bs == 128)
    return launch_tc_lse<128, 128>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
  if (g.d == 64 && g.bs == 64)
    return launch_tc_lse<64, 64>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
  return launch_tc_lse<64, 128>(g, q, k, v, kv_count, kv_idx, items, scale, o, lse, ctrl, st);
}

}  // namespace bsa
