// Block-sparse attention forward on the sm_100a tensor cores, with P in
// tensor memory: persistent, one CTA per SM.  NABLA summary, Metodologia 2
// "Expansion": only the listed N x N tiles are computed.
//
// Work: the plan's 128-row query tiles (one block of 128, or two blocks of 64,
// rows 0-63 and 64-127), fetched one at a time from a work counter in the
// plan's order (longest first within each head).  A tile walks the union of
// its KV lists in KV tiles of 128 keys (one entry of 128, or two of 64); KV
// tile j belongs to softmax group w = j mod 2:
//   S = Q K^T      tcgen05.mma (M=128, N=128), A = Q and B = K from shared
//                  memory, into TMEM S buffer w
//   softmax        one thread per query row (group w: warps 4 + 4w .. 7 + 4w):
//                  masks keys its row's block does not keep (and padding),
//                  keeps a running base-2 max (O_w rescaled only when it grows
//                  by more than 8) and writes P = 2^(s - m) as bf16 into the
//                  first 64 columns of the same TMEM buffer (tcgen05.st)
//   O_w += P V     tcgen05.mma with A = P from TMEM and B = V (MN-major) from
//                  shared memory, O_w in TMEM
// Shared memory then carries only the TMA tiles and the MMA reads of Q, K and
// V, and one thread issues every MMA: staging P in shared memory instead
// (written by the softmax, read by the MMA from there) measured the same speed
// with a second issuer and 64 KB more shared-memory traffic per KV tile.
//
// One thread issues every MMA of the CTA, in this order: S(0), S(1), then for
// each j: O_w += P(j) V(j), S(j + 2) into the same buffer w.  tcgen05.mma
// operations of one thread execute in issue order, so S(j + 2) overwrites the
// P(j) columns only after the P.V product has read them; and the commit that
// reports S(j + 2) complete covers every earlier MMA of the thread, so a
// softmax that has seen its S knows that its group's previous P.V product is
// done (O_w can be rescaled, P can be rewritten).  TMEM holds S_0, S_1, O_0,
// O_1 (4 x 128 columns).  The epilogue merges the two groups' partial results
// of each row exactly.  K and V have two stages in shared memory, each loaded
// by its own producer warp.  O is normalised by the sum of the bf16-rounded
// weights the P.V product uses (an exact convex combination of V rows up to
// accumulation rounding); the LSE uses the fp32 sum of the unrounded ones.
//
// Roles: warps 0 and 2 issue TMA loads (Q and K; V), warp 1 issues the MMAs
// (one elected thread), warps 4-11 run the softmax and the epilogue (warp w
// reads TMEM lanes 32 (w mod 4) .. +31).  Every mbarrier wait is bounded; on
// expiry the CTA records BSA_ERR_TIMEOUT in the workspace error word, tells
// the launch's other CTAs to give up (its own launch sequence number in the
// control block), waits (bounded) for the copies and MMAs it has already
// issued, frees its TMEM and leaves.
#include <cmath>
#include <cstdlib>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "softmax_math.cuh"
#include "tma_host.h"

namespace bsa {

namespace {

using namespace sm100;
using namespace smx;

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kGroupThreads = 128;   // threads of one softmax group
constexpr uint64_t kWaitNs = 250ull * 1000ull * 1000ull;  // 250 ms: far beyond any legitimate wait
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;     // O_0 at 256, O_1 at 384; S_0 at 0, S_1 at 128

struct Ctl {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];   // per softmax group
  uint64_t drain;      // final commit of the MMA issuer before TMEM is freed
  uint32_t tmem_base;
  int n_ent;
  int item;
  int abort;
  uint32_t bm[2][BSA_MAX_BLOCKS / 32];  // kept blocks of each query block of the tile
  // union of the lists, ascending: block index in bits 0-11, bit 12 + h set
  // when query block h of the tile keeps the entry
  uint16_t ent[BSA_MAX_BLOCKS];
};
constexpr uint16_t kEntBlock = 0x0FFFu;

__device__ __forceinline__ void timeout(Ctrl* ctrl, Ctl& c, uint32_t seq, uint32_t site) {
  report_error(ctrl, kErrTimeout, blockIdx.x, threadIdx.x, site);
  atomicExch(&ctrl->abort_seq, seq);
  c.abort = 1;
}

// Bounded wait; gives up early once a CTA of this launch (sequence number
// `seq`) has timed out.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  return mbar_wait_ns(bar, parity, kWaitNs, &ctrl->abort_seq, seq);
}

// Same, with one verdict for the whole warp (the tcgen05.ld/st that follow
// are warp-collective and must not run in a partial warp).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  const bool ok = wait(bar, parity, ctrl, seq);
  return __all_sync(0xffffffffu, ok);
}

// Barrier of the two softmax warps that share TMEM lane quarter q4; returns
// the AND of `ok` over both warps, so the pair leaves its loop together (a
// named barrier has no time limit: both warps must always reach it).
__device__ __forceinline__ bool pair_sync(int q4, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n"
      ".reg .pred p, q;\n"
      "setp.ne.u32 q, %1, 0;\n"
      "bar.red.and.pred p, %2, 64, q;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(1 + q4)
      : "memory");
  return r != 0u;
}

// O_w *= alpha for this thread's row, 32 columns at a time (warp-collective
// TMEM accesses: every lane of the warp calls it).
template <int D>
__device__ __forceinline__ void rescale_o_cols(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int cc = 0; cc < D; cc += 32) {
    uint32_t ov[32];
    tmem_ld32(tO + cc, ov);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
    tmem_st32(tO + cc, ov);
  }
  tmem_wait_st();
}

// MODE 0: O only; 1: O and the LSE; 2: O, the LSE and the entropy of each
// row's attention distribution.
template <int D, int BS, int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ CUtensorMap mq,
                                                               const __grid_constant__ CUtensorMap mk,
                                                               const __grid_constant__ CUtensorMap mv,
                                                               const int32_t* __restrict__ kv_count,
                                                               const int32_t* __restrict__ kv_idx,
                                                               const int2* __restrict__ items, int* work,
                                                               float scale_log2, __nv_bfloat16* __restrict__ o,
                                                               float* __restrict__ lse, float* __restrict__ ent,
                                                               Ctrl* ctrl, Dims g,
                                                               int items_per_bh, int n_items, uint32_t seq,
                                                               int force_timeout) {
  constexpr bool WITH_LSE = MODE >= 1;
  constexpr bool WITH_ENT = MODE == 2;
  constexpr int QB = 128 / BS;          // query blocks per tile
  constexpr int E = 128 / BS;           // list entries per KV tile
  constexpr int CH = D / 64;            // 64-column (128-byte) chunks of a row
  constexpr uint32_t kTile = 128u * D * 2u;
  constexpr uint32_t kChunk = 128u * 128u;  // bytes of one chunk of a 128-row tile

  // 128-byte swizzled tiles need 1024-byte aligned shared memory; the layout
  // fills the 227 KB of a CTA at D = 128, so there is no room to realign.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report_error(ctrl, kErrLayout, blockIdx.x, 0u, 2u);
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sK = sQ + kTile;            // two stages
  uint8_t* sV = sQ + 3 * kTile;        // two stages
  Ctl& c = *reinterpret_cast<Ctl*>(sQ + 5 * kTile);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int nb = g.nb;
  const int nw = (nb + 31) >> 5;

  if (tid == 0) {
    mbar_init(&c.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c.k_full[s], 1);
      mbar_init(&c.k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c.v_full[s], 1);
      mbar_init(&c.v_empty[s], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&c.s_full[w], 1);
      mbar_init(&c.p_full[w], kGroupThreads);
      mbar_init(&c.pv_done[w], 1);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mq);
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;

  // Test hook of the failure path: one bounded wait (2 ms) on an mbarrier
  // that nothing arrives on, before any copy or MMA is issued; it records
  // BSA_ERR_TIMEOUT and the CTA does no work.
  if (force_timeout) {
    if (tid == 0 && !mbar_wait_ns(&c.q_full, 0, 2ull * 1000ull * 1000ull, nullptr, 0u)) timeout(ctrl, c, seq, 1);
    __syncthreads();
  }

  uint32_t jbase = 0;  // KV tiles this CTA has run so far (phase counter of the K/V stages)
  uint32_t gbase[2] = {0u, 0u};  // KV tiles each softmax group has run so far
  uint32_t nq = 0;     // Q loads so far (phase of q_full)
  uint32_t armed = 0;  // K (warp 0) or V (warp 2) stage loads this producer thread has issued

  for (;;) {
    if (tid == 0) c.item = atomicAdd(work, 1);
    for (int i = tid; i < 2 * (BSA_MAX_BLOCKS / 32); i += kThreads) (&c.bm[0][0])[i] = 0u;
    __syncthreads();
    const int item = c.item;
    if (item >= n_items || c.abort) break;
    const int bh = item / items_per_bh;

    // the tile's query blocks, from the plan (second block -1 when single)
    const int2 it = items[item];
    int qblk[QB];
    bool qval[QB];
    qblk[0] = it.x;
    qval[0] = it.x >= 0 && it.x < nb;
    if (QB == 2) {
      qblk[QB - 1] = it.y;
      qval[QB - 1] = it.y >= 0 && it.y < nb;
    }
    if (!qval[0]) qblk[0] = 0;  // a corrupt plan: compute nothing for this tile

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

    // Union list in ascending order (warp 0).
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
          c.ent[pos] = (uint16_t)((wi * 32 + bit) | (((b0 >> bit) & 1u) << 12) | (((b1 >> bit) & 1u) << 13));
          ++pos;
        }
        off += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) c.n_ent = off;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int n_ent = c.n_ent;
    const int n_tiles = (n_ent + E - 1) / E;

    if (warp == 0 || warp == 2) {
      // ---------------------------------------------------------- TMA producers
      // warp 0: Q, then K of every KV tile; warp 2: V (two stages each), so
      // a V wait never holds back the next K.
      const bool is_k = warp == 0;
      if (lane == 0 && n_tiles > 0) {
        if (is_k) {
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
        }
        for (int j = 0; j < n_tiles; ++j) {
          const uint32_t jg = jbase + j;
          int krow[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (E == 2) {
              const int idx = (2 * j + h < n_ent) ? 2 * j + h : 2 * j;
              krow[h] = (int)(c.ent[idx] & kEntBlock) * 64;
            } else {
              krow[h] = (int)(c.ent[j] & kEntBlock) * 128 + 64 * h;
            }
          }
          if (is_k) {
            const uint32_t s = jg & 1;
            if (jg >= 2 && !wait(&c.k_empty[s], ((jg - 2) >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 10); break; }
            mbar_arrive_expect_tx(&c.k_full[s], kTile);
            ++armed;
            uint8_t* dk = sK + s * kTile;
#pragma unroll
            for (int ch = 0; ch < CH; ++ch)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_3d(dk + ch * kChunk + h * (kChunk / 2), &mk, &c.k_full[s], ch * 64, krow[h], bh);
          } else {
            const uint32_t s = jg & 1;
            if (jg >= 2 && !wait(&c.v_empty[s], ((jg - 2) >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 11); break; }
            mbar_arrive_expect_tx(&c.v_full[s], kTile);
            ++armed;
            uint8_t* dv = sV + s * kTile;
#pragma unroll
            for (int ch = 0; ch < CH; ++ch)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_3d(dv + ch * kChunk + h * (kChunk / 2), &mv, &c.v_full[s], ch * 64, krow[h], bh);
          }
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // S(0), S(1), then for each KV tile j: O_w += P(j) V(j) once group w
      // has written P(j) and V(j) has landed, followed by S(j + 2) into the
      // same TMEM buffer (in issue order: it overwrites P(j) only after the
      // P.V product has read it).
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
        const uint64_t dQ = smem_desc_sw128(smem_addr(sQ), 16, 1024);
        const uint32_t aK = smem_addr(sK), aV = smem_addr(sV);
        // S(jj) into buffer jj mod 2; false on a timeout
        auto issue_s = [&](int jj) -> bool {
          const uint32_t jg = jbase + jj, ks = jg & 1;
          const int w = jj & 1;
          if (!wait(&c.k_full[ks], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 21); return false; }
          tc_fence_after();
          // descriptors built once per tile: two adds per MMA
          const uint64_t dK = smem_desc_sw128(aK + ks * kTile, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(tmem + 128 * w, smem_desc_add(dQ, off), smem_desc_add(dK, off), idS, kk > 0);
          }
          mma_commit(&c.s_full[w]);
          mma_commit(&c.k_empty[ks]);
          return true;
        };
        bool go = true;
        if (!wait(&c.q_full, nq & 1, ctrl, seq)) {
          timeout(ctrl, c, seq, 20);
          go = false;
        }
        for (int jj = 0; go && jj < 2 && jj < n_tiles; ++jj) go = issue_s(jj);
        for (int j = 0; go && j < n_tiles; ++j) {
          const uint32_t jg = jbase + j, vs = jg & 1;
          const int w = j & 1;
          const uint32_t gw = gbase[w] + (j >> 1);
          if (!wait(&c.p_full[w], gw & 1, ctrl, seq)) { timeout(ctrl, c, seq, 23); break; }
          if (!wait(&c.v_full[vs], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 24); break; }
          tc_fence_after();
          const uint64_t dV = smem_desc_sw128(aV + vs * kTile, kChunk, 1024);
          const uint32_t acc0 = (j >= 2) ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kTmemO + 128 * w, tmem + 128 * w + 8 * kk, smem_desc_add(dV, kk * 2048), idO,
                   kk > 0 ? 1u : acc0);
          mma_commit(&c.pv_done[w]);
          mma_commit(&c.v_empty[vs]);
          if (j + 2 < n_tiles) go = issue_s(j + 2);
        }
      }
    } else if (warp >= kSoftmaxWarp0) {
      // ---------------------------------------------------------- softmax + epilogue
      const int q4 = warp & 3;                         // TMEM lane quarter of this warp
      const int w = (warp - kSoftmaxWarp0) >> 2;       // softmax group: KV tiles j = w mod 2
      const int r = q4 * 32 + lane;                    // query row of the tile
      const int half = (QB == 2) ? (r >> 6) : 0;       // query block of the row
      const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
      const uint32_t tS = trow + 128 * w, tOw = trow + kTmemO + 128 * w;
      float m = -INFINITY;
      float l = 0.f, lx = 0.f;
      // entropy: vx = sum of p (y - m) over the row's weights p = 2^(y - m),
      // y the base-2 logits, relative to the current running max m
      float vx = 0.f;
      bool ok = true;
      int mine = 0;   // KV tiles this group ran in this item
      auto rescale_o = [&](uint32_t tO, float alpha) { rescale_o_cols<D>(tO, alpha); };
      for (int j = w; j < n_tiles; j += 2, ++mine) {
        const uint32_t gw = gbase[w] + (j >> 1);
        int lim[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int key0, kept;
          if (E == 2) {
            const int idx = 2 * j + h;
            kept = (idx < n_ent) ? ((c.ent[idx] >> (12 + half)) & 1) : 0;
            key0 = (idx < n_ent) ? (int)(c.ent[idx] & kEntBlock) * 64 : 0;
          } else {
            kept = 1;
            key0 = (int)(c.ent[j] & kEntBlock) * 128 + 64 * h;
          }
          lim[h] = kept ? max(0, min(64, g.N - key0)) : 0;
        }
        // S(j) complete: the commit behind it also covers this group's
        // previous P.V product, so O_w and the P columns are free as well
        if (!wait_warp(&c.s_full[w], gw & 1, ctrl, seq)) { timeout(ctrl, c, seq, 30); ok = false; break; }
        tc_fence_after();
        // The row max is needed only to keep 2^(y - m) in range: bf16 P and
        // the fp32 sums and accumulators hold weights far beyond 2^64.  So the
        // max pass runs only while a row of the warp has no max yet (its
        // first kept tile); later tiles use the running max as it stands and
        // check each chunk's weights before storing them (below).
        const bool need_max = __any_sync(0xffffffffu, m == -INFINITY);
        if (need_max) {
          // Pass 1: row max of the raw scores over the kept, real keys (scale
          // > 0 keeps the order), 64 columns at a time.
          float mh[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sr[64];
            tmem_ld32(tS + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tS + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            const float* xh = reinterpret_cast<const float*>(sr);
            if (lim[h] == 64) {
              float m0 = xh[0], m1 = xh[1], m2 = xh[2], m3 = xh[3];
#pragma unroll
              for (int i = 4; i < 64; i += 8) {
                m0 = fmax3(m0, xh[i], xh[i + 1]);
                m1 = fmax3(m1, xh[i + 2], xh[i + 3]);
                m2 = fmax3(m2, xh[i + 4], xh[i + 5]);
                m3 = fmax3(m3, xh[i + 6], xh[i + 7]);
              }
              mh[h] = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
            } else {
              float mm = -INFINITY;
              if (lim[h] > 0) {
#pragma unroll
                for (int i = 0; i < 64; ++i) mm = (i < lim[h]) ? fmaxf(mm, xh[i]) : mm;
              }
              mh[h] = mm;
            }
          }
          const float mnew = fmaxf(m, fmaxf(mh[0], mh[1]) * scale_log2);
          // The running max moves only when it grows by more than 8 (a factor
          // 256 in p), or when it is set for the first time.  The O rescale
          // uses warp-collective TMEM accesses, so the whole warp takes it
          // when any lane needs it (lanes whose max did not move use alpha =
          // 1).  O_w is stable: its last P.V product has completed (waited
          // above).
          const bool grow = mnew > m + 8.0f;
          if (__any_sync(0xffffffffu, grow && m != -INFINITY)) {
            const float alpha = (grow && m != -INFINITY) ? ex2f(m - mnew) : 1.0f;
            rescale_o(tOw, alpha);
            if (WITH_ENT && grow && m != -INFINITY) vx = alpha * (vx + (m - mnew) * lx);
            l *= alpha;
            lx *= alpha;
          }
          if (grow) m = mnew;
        }
        float nm = (m == -INFINITY) ? 0.f : -m;
        // p = 2^(s * scale_log2 - m): one FFMA and one MUFU ex2 per score.  O is
        // normalised by the sum of the bf16-rounded weights the P.V product
        // uses (an exact convex combination of V rows up to accumulation
        // rounding); the LSE, when asked for, uses the fp32 sum of the
        // unrounded ones.  Halves the row's query block does not keep cost
        // nothing.
        // Pass 2, 32 keys at a time (the next chunk's load in flight): their
        // bf16 weights, two per 32-bit column, go to columns [16 c, 16 c + 16)
        // of the same TMEM buffer -- columns whose scores this pass has
        // already read into registers.
        float rs[2] = {0.f, 0.f};
        float rx = 0.f, ry = 0.f;
        float rx_ok = 0.f, ry_ok = 0.f;   // the LSE and entropy sums of the chunks stored so far
        const float2 sc2 = make_float2(scale_log2, scale_log2);
        // one chunk's weights from its scores x: pk, and the sums
        auto exp_chunk = [&](const float* x, int cl, float nmv, uint32_t (&pk)[16]) {
          const float2 nm2 = make_float2(nmv, nmv);
          auto exp_pair = [&](int i, bool masked) {
            // both arguments in one fma.rn.f32x2 (half the issue slots)
            const float2 yy = ffma2(make_float2(x[2 * i], x[2 * i + 1]), sc2, nm2);
            const float y0 = yy.x, y1 = yy.y;
            float2 p;
            p.x = ex2f(y0);
            p.y = ex2f(y1);
            if (masked) {
              p.x = (2 * i < cl) ? p.x : 0.f;
              p.y = (2 * i + 1 < cl) ? p.y : 0.f;
            }
            pk[i] = pack_bf16(p.x, p.y);
            rs[i & 1] = add_bf16x2(rs[i & 1], pk[i]);
            if (WITH_LSE) rx += p.x + p.y;
            if (WITH_ENT) ry = fmaf(p.x, y0, fmaf(p.y, y1, ry));
          };
          // valid keys of the chunk: all 32 (the common case, no per-key
          // test in the loop), some, or none
          if (cl == 32) {
#pragma unroll
            for (int i = 0; i < 16; ++i) exp_pair(i, false);
          } else if (cl > 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i) exp_pair(i, true);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
        };
        int c_fail = 4;
        uint32_t sc[2][32];
        tmem_ld32(tS, sc[0]);
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          const int h = cch >> 1;
          tmem_wait_ld();
          if (cch < 3) tmem_ld32(tS + 32 * (cch + 1), sc[(cch + 1) & 1]);
          uint32_t pk[16];
          exp_chunk(reinterpret_cast<const float*>(sc[cch & 1]), min(32, max(0, lim[h] - (cch & 1) * 32)), nm, pk);
          // Without the max pass, a weight of 2^64 or more means this tile's
          // scores exceed the running max by 64 or more: nothing of this
          // chunk is stored, and the tile goes on below with a new max.
          if (!need_max && __any_sync(0xffffffffu, !(rs[0] + rs[1] < 0x1p64f))) {
            c_fail = cch;
            break;
          }
          tmem_st16(tS + 16 * cch, pk);
          rx_ok = rx;
          ry_ok = ry;
        }
        if (c_fail < 4) {
          // Rare: the running max moves by 64 or more within a tile.  The new
          // max comes from the scores of chunks c_fail..3 (columns the P
          // stores have not reached); O, the row sums and the weights of the
          // chunks already stored are rescaled by alpha = 2^(m - m_new) (the
          // stored bf16 weights re-rounded, their sum recomputed from them);
          // chunks c_fail..3 are then redone with the new max.
          tmem_wait_ld();                     // the prefetch in flight
          float mx = -INFINITY;
#pragma unroll 1
          for (int cc = c_fail; cc < 4; ++cc) {
            uint32_t t[32];
            tmem_ld32(tS + 32 * cc, t);
            tmem_wait_ld();
            const int cl = min(32, max(0, lim[cc >> 1] - (cc & 1) * 32));
#pragma unroll
            for (int i = 0; i < 32; ++i) mx = (i < cl) ? fmaxf(mx, __uint_as_float(t[i])) : mx;
          }
          const float mnew = fmaxf(m, mx * scale_log2);
          const float alpha = ex2f(m - mnew);   // m is finite here: the max pass ran on an earlier tile
          rescale_o(tOw, alpha);
          if (WITH_ENT) vx = alpha * (vx + (m - mnew) * lx);
          l *= alpha;
          lx *= alpha;
          rs[0] = rs[1] = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < c_fail; ++cc) {
            uint32_t pv[16];
            tmem_ld16(tS + 16 * cc, pv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              pv[i] = pack_bf16(__uint_as_float(pv[i] << 16) * alpha, __uint_as_float(pv[i] & 0xFFFF0000u) * alpha);
              rs[i & 1] = add_bf16x2(rs[i & 1], pv[i]);
            }
            tmem_st16(tS + 16 * cc, pv);
          }
          if (WITH_ENT) ry = alpha * (ry_ok + (m - mnew) * rx_ok);
          rx = alpha * rx_ok;
          m = mnew;
          nm = -m;
#pragma unroll 1
          for (int cc = c_fail; cc < 4; ++cc) {
            uint32_t t[32];
            tmem_ld32(tS + 32 * cc, t);
            tmem_wait_ld();
            uint32_t pk[16];
            exp_chunk(reinterpret_cast<const float*>(t), min(32, max(0, lim[cc >> 1] - (cc & 1) * 32)), nm, pk);
            tmem_st16(tS + 16 * cc, pk);
          }
        }
        l += rs[0] + rs[1];
        if (WITH_LSE) lx += rx;
        if (WITH_ENT) vx += ry;
        tmem_wait_st();             // the P stores, complete before the tensor core reads them
        tc_fence_before();
        mbar_arrive(&c.p_full[w]);
      }

      // epilogue: the two groups' partial results of row r are merged,
      // O = (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / (l_0 2^(m_0 - m) + l_1 2^(m_1 - m));
      // group w writes the columns [w D / 2, (w + 1) D / 2) of the row.
      // This thread reads both groups' O accumulators: wait for the last P.V
      // product of each group that ran a tile.
      const int cnt0 = (n_tiles + 1) / 2, cnt1 = n_tiles / 2;
      const bool has0 = cnt0 > 0, has1 = cnt1 > 0;
      // The pv_done parity waits protect this group's own accumulator; the
      // other group's is covered by its own wait, ordered before this
      // thread's reads by the pair barrier below (and the fence after it).
      if (ok && has0 && !wait_warp(&c.pv_done[0], (gbase[0] + cnt0 - 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 31); ok = false; }
      if (ok && has1 && !wait_warp(&c.pv_done[1], (gbase[1] + cnt1 - 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 31); ok = false; }
      tc_fence_after();
      // The merge goes through the K stages: every S of the item has completed
      // (its softmax ran) and the next item's K loads start after the item.
      float* xm = reinterpret_cast<float*>(sK);   // [group][row]: running max
      float* xl = xm + 2 * 128;                   // [group][sum kind][row]: row sums
      float* xv = xl + 4 * 128;                   // [group][row]: entropy sums
      xm[w * 128 + r] = (mine > 0) ? m : -INFINITY;
      xl[(2 * w + 0) * 128 + r] = l;
      xl[(2 * w + 1) * 128 + r] = lx;
      if (WITH_ENT) xv[w * 128 + r] = vx;
      tc_fence_before();
      ok = pair_sync(q4, ok);
      tc_fence_after();
      const float m0 = xm[r], m1 = xm[128 + r];
      const float mt = fmaxf(m0, m1);
      const float a0 = (has0 && m0 != -INFINITY) ? ex2f(m0 - mt) : 0.f;
      const float a1 = (has1 && m1 != -INFINITY) ? ex2f(m1 - mt) : 0.f;
      const float lt = xl[r] * a0 + xl[2 * 128 + r] * a1;
      const float lxt = xl[128 + r] * a0 + xl[3 * 128 + r] * a1;
      int grow;
      if (QB == 2) grow = qval[half] ? qblk[half] * 64 + (r & 63) : -1;
      else grow = qval[0] ? qblk[0] * 128 + r : -1;
      const bool store = grow >= 0 && grow < g.Npad;
      const bool real = ok && store && grow < g.N && lt > 0.f;
      const float inv = real ? 1.f / lt : 0.f;
      const float s0 = a0 * inv, s1 = a1 * inv;
      uint4* orow = reinterpret_cast<uint4*>(o + ((size_t)bh * g.Npad + (store ? grow : 0)) * D + w * (D / 2));
      // The TMEM loads are warp-collective: their conditions (ok, has0, has1)
      // are the same in every lane; only the stores depend on the row.
#pragma unroll 1
      for (int cc = 0; cc < D / 2; cc += 16) {
        const int col = w * (D / 2) + cc;
        uint32_t o0[16], o1[16];
        if (ok && has0) tmem_ld16(trow + kTmemO + col, o0);
        if (ok && has1) tmem_ld16(trow + kTmemO + 128 + col, o1);
        if (ok && (has0 || has1)) tmem_wait_ld();
        uint32_t pw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v0 = 0.f, v1 = 0.f;
          if (has0) {
            v0 = __uint_as_float(o0[2 * i]) * s0;
            v1 = __uint_as_float(o0[2 * i + 1]) * s0;
          }
          if (has1) {
            v0 = fmaf(__uint_as_float(o1[2 * i]), s1, v0);
            v1 = fmaf(__uint_as_float(o1[2 * i + 1]), s1, v1);
          }
          pw[i] = real ? pack_bf16(v0, v1) : 0u;
        }
        if (store) {
#pragma unroll
          for (int i = 0; i < 2; ++i)
            orow[cc / 8 + i] = make_uint4(pw[4 * i], pw[4 * i + 1], pw[4 * i + 2], pw[4 * i + 3]);
        }
      }
      if (WITH_LSE && w == 0 && store)
        lse[(size_t)bh * g.Npad + grow] = real ? (mt + __log2f(lxt)) * 0.69314718055994531f : 0.f;
      if (WITH_ENT && w == 0 && store) {
        // H = -sum p ln p with p = 2^(y - mt) / lxt: ln 2 (log2 lxt - sum 2^(y - mt) (y - mt) / lxt)
        float vt = 0.f;
        if (has0 && m0 != -INFINITY) vt += a0 * (xv[r] + (m0 - mt) * xl[128 + r]);
        if (has1 && m1 != -INFINITY) vt += a1 * (xv[128 + r] + (m1 - mt) * xl[3 * 128 + r]);
        ent[(size_t)bh * g.Npad + grow] = real ? (__log2f(lxt) - vt / lxt) * 0.69314718055994531f : 0.f;
      }
      fence_proxy_async_smem();   // the merge's accesses, ordered before the next K loads
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    jbase += n_tiles;
    gbase[0] += (n_tiles + 1) / 2;
    gbase[1] += n_tiles / 2;
    if (n_tiles > 0) ++nq;
  }

  // Drain: every copy and MMA this CTA issued completes before its TMEM is
  // freed and it exits (after a timeout some may still be in flight).  In a
  // normal exit all of them have completed already and these waits return
  // at once.
  if (lane == 0) {
    if (warp == 0) {
      mbar_drain_ring(&c.q_full, 1, nq, kWaitNs);
      mbar_drain_ring(c.k_full, 2, armed, kWaitNs);
    } else if (warp == 2) {
      mbar_drain_ring(c.v_full, 2, armed, kWaitNs);
    } else if (warp == 1) {
      mma_commit(&c.drain);
      mbar_wait_ns(&c.drain, 0, kWaitNs, nullptr, 0u);
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

template <int D, int BS, int MODE>
cudaError_t launch_fwd(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                       const int32_t* kv_idx, const int2* items, int* work, float scale, void* o, float* lse,
                       float* ent, Ctrl* ctrl, uint32_t seq, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)g.Npad, bhs = (uint64_t)g.B * g.heads;
  if (!make_map_bf16_3d(&mq, q, D, rows, bhs, 64, 64) || !make_map_bf16_3d(&mk, k, D, rows, bhs, 64, 64) ||
      !make_map_bf16_3d(&mv, v, D, rows, bhs, 64, 64))
    return cudaErrorInvalidValue;
  const int items_per_bh = (BS == 64) ? (g.nb + 1) / 2 : g.nb;
  const int n_items = (int)(bhs * items_per_bh);
  const size_t smem = 5u * 128u * D * 2u + sizeof(Ctl);
  static_assert(5u * 128u * 128u * 2u + sizeof(Ctl) <= 227u * 1024u, "shared memory layout");
  cudaError_t e =
      cudaFuncSetAttribute(attn_fwd_kernel<D, BS, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = n_items < num_sms() ? n_items : num_sms();
  attn_fwd_kernel<D, BS, MODE><<<grid, kThreads, smem, st>>>(mq, mk, mv, kv_count, kv_idx, items, work,
                                                                 scale * 1.4426950408889634f, (__nv_bfloat16*)o, lse,
                                                                 ent, ctrl, g, items_per_bh, n_items, seq,
                                                                 force_timeout_requested());
  return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_fwd_mode(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                           const int32_t* kv_idx, const int2* items, int* work, float scale, void* o, float* lse,
                           float* ent, Ctrl* ctrl, uint32_t seq, cudaStream_t st) {
  if (ent != nullptr)
    return launch_fwd<D, BS, 2>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
  if (lse != nullptr)
    return launch_fwd<D, BS, 1>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
  return launch_fwd<D, BS, 0>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
}

}  // namespace

int force_timeout_requested() {
  const char* v = std::getenv("BSA_TEST_FORCE_TIMEOUT");
  return (v != nullptr && v[0] == '1') ? 1 : 0;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

cudaError_t launch_attn(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                        const int32_t* kv_idx, const int2* items, int* work, float scale, void* o, float* lse,
                        float* ent, Ctrl* ctrl, uint32_t seq, cudaStream_t st) {
  if (g.d == 128 && g.bs == 64)
    return launch_fwd_mode<128, 64>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
  if (g.d == 128 && g.bs == 128)
    return launch_fwd_mode<128, 128>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
  if (g.d == 64 && g.bs == 64)
    return launch_fwd_mode<64, 64>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
  return launch_fwd_mode<64, 128>(g, q, k, v, kv_count, kv_idx, items, work, scale, o, lse, ent, ctrl, seq, st);
}

}  // namespace bsa
