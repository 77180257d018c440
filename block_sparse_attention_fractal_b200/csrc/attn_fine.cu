// Attention over fine-grained KV selections on the sm_100a tensor cores
// (AB-Attention article, "Los tres recursos": the fine selection on coarse
// hardware, and SIP's inclusion-probability weights).
//
// Each 128-row query block I of head (b, h) has its own list of KV blocks of
// only 4 tokens (CSR: entries sel_offsets[r] .. sel_offsets[r + 1] of sel_idx,
// r = (b * heads + h) * nq + I), each with an optional weight w > 0 (the
// inverse of its inclusion probability).  Every run of 32 list entries is
// gathered by index into one full 128-key tile of K and of V in shared
// memory, so the tensor cores see the same 128 x 128 tiles as in the
// block-sparse kernel; the weight enters as the logit shift log2 w of the
// block's 4 keys (numerator and normalisation alike, so the result is the
// Horvitz-Thompson estimate with no extra pass):
//   O[q] = sum_k w_k 2^(s_qk) V[k] / sum_k w_k 2^(s_qk),  s = scale log2(e) q.k
//
// Roles (384 threads, persistent, one CTA per SM, query blocks from a work
// counter):
//   warps 0 and 3  gather K into three stages: each thread copies 16-byte
//                  pieces of the tile's rows with cp.async into the 128-byte
//                  swizzled layout the MMA descriptors expect (zero-filled past
//                  the list's end and for keys >= N).  It issues tile j's
//                  copies before it waits for its own copies of tile j - 1,
//                  so two tiles are in flight; once those have landed it
//                  orders them for the tensor core (proxy fence) and arrives
//                  on the stage's barrier.  Lane 0 of warp 0 also loads Q by TMA
//   warp 2         gathers V the same way
//   warp 1         issues the MMAs (one elected thread): S(0), S(1), then
//                  O_w += P(j) V(j) and S(j + 2) into the same TMEM buffer,
//                  as in the block-sparse kernel
//   warps 4-11     softmax (two groups on alternating KV tiles) and epilogue;
//                  the first warp of each group turns the tile's 32 entries
//                  into 128 column shifts (log2 w, or -inf for a missing key)
//                  in one of the group's two shared-memory slots, loaded one
//                  tile ahead, and a named barrier of the group's 128 threads
//                  (which also carries the group's abort verdict) hands them
//                  to the other three warps
// Every mbarrier wait is bounded, with the same abort and drain sequence as
// the block-sparse kernel.
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

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kGroupThreads = 128;
constexpr uint64_t kWaitNs = 250ull * 1000ull * 1000ull;   // 250 ms
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;   // O_0 at 256, O_1 at 384; S_0 at 0, S_1 at 128
constexpr int kKeyBlock = 4;       // tokens of a KV block
constexpr int kEntries = 128 / kKeyBlock;   // list entries per 128-key tile (one per lane)
constexpr int kKThreads = 64;      // K gather: warps 0 and 3
constexpr int kVThreads = 32;      // V gather: warp 2
constexpr uint32_t kStages = 3;    // K and V stages in shared memory

struct Ctl {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int item;
  int len;          // list entries of the current query block
  int abort;
  long long off;    // its first entry
  // per softmax group, two slots (tiles j with (j / 2) mod 2 = 0, 1): base-2
  // logit shift of each key column of the tile
  alignas(16) float shift[2][2][128];
};

struct FineArgs {
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const long long* sel_offsets;
  const int32_t* sel_idx;
  const float* sel_w;      // null: every weight 1
  long long n_sel;         // entries of sel_idx (and sel_w)
  __nv_bfloat16* o;
  float* lse;
  Ctrl* ctrl;
  int* work;
  float scale_log2;
  int N, Npad, nq, nkb;    // tokens, padded rows, query blocks and 4-token KV blocks per head
  int n_items;             // B * heads * nq
  uint32_t seq;
  int force_timeout;
};

__device__ __forceinline__ void timeout(Ctrl* ctrl, Ctl& c, uint32_t seq, uint32_t site) {
  report_error(ctrl, kErrTimeout, blockIdx.x, threadIdx.x, site);
  atomicExch(&ctrl->abort_seq, seq);
  c.abort = 1;
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  return mbar_wait_ns(bar, parity, kWaitNs, &ctrl->abort_seq, seq);
}

// One verdict for the whole warp (warp-collective instructions follow).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  const bool ok = wait(bar, parity, ctrl, seq);
  return __all_sync(0xffffffffu, ok);
}

// Barrier of the two softmax warps that share TMEM lane quarter q4 (AND of ok).
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

// Named barrier of the 128 threads of softmax group w; returns the AND of
// `ok` over them (the group leaves its loop together).
__device__ __forceinline__ bool group_sync(int w, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n"
      ".reg .pred p, q;\n"
      "setp.ne.u32 q, %1, 0;\n"
      "bar.red.and.pred p, %2, 128, q;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(5 + w)
      : "memory");
  return r != 0u;
}

// List entry `lane` of KV tile j: its block index (-1 past the list's end or
// when out of range, which is reported) and weight.
__device__ __forceinline__ int entry_block(const FineArgs& a, long long off, int len, int j, int lane, bool report) {
  const int e = j * kEntries + lane;
  if (e >= len) return -1;
  const int blk = __ldg(a.sel_idx + off + e);
  if (blk < 0 || blk >= a.nkb) {
    if (report) report_error(a.ctrl, kErrIndex, (uint32_t)(off + e), (uint32_t)blk, 40u);
    return -1;
  }
  return blk;
}

// This thread's share of one 128-key tile: rows r = sub, sub + RS, ... (key
// 4 e + (r mod 4) of entry e = r / 4, whose block index lane e of the warp
// holds), 16-byte piece pc of each row, into the 128-byte swizzled layout
// (64-column chunks of 128 rows x 128 bytes; piece c of row r at
// ((c ^ (r mod 8)) * 16) within the row).
template <int D, int NT>
__device__ __forceinline__ void gather_tile(uint32_t stage, const __nv_bfloat16* __restrict__ base, int blk_lane,
                                            int t, int N) {
  constexpr int PR = D / 8;       // 16-byte pieces per row
  constexpr int RS = NT / PR;     // rows per step of the NT threads
  static_assert(NT % PR == 0 && 128 % RS == 0, "tile rows split evenly");
  const int sub = t / PR, pc = t % PR;
  const uint32_t col = (uint32_t)(pc >> 3) * (128u * 128u);
  const uint32_t cc = (uint32_t)(pc & 7);
#pragma unroll 8
  for (int r0 = 0; r0 < 128; r0 += RS) {
    const int row = r0 + sub;
    const int blk = __shfl_sync(0xffffffffu, blk_lane, row >> 2);
    const int key = blk * kKeyBlock + (row & 3);
    const bool ok = blk >= 0 && key < N;
    const __nv_bfloat16* src = base + (ok ? (size_t)key * D + pc * 8 : 0);
    cp_async16(stage + col + (uint32_t)row * 128u + ((cc ^ (uint32_t)(row & 7)) << 4), src, ok);
  }
}

template <int D, bool WITH_LSE>
__global__ void __launch_bounds__(kThreads, 1) attn_fine_kernel(const __grid_constant__ CUtensorMap mq,
                                                                const FineArgs a) {
  constexpr int CH = D / 64;
  constexpr uint32_t kTile = 128u * D * 2u;
  constexpr uint32_t kChunk = 128u * 128u;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report_error(a.ctrl, kErrLayout, blockIdx.x, 0u, 2u);
    return;
  }
  uint8_t* sQ = smem_raw;
  uint8_t* sK = sQ + kTile;                     // kStages stages
  uint8_t* sV = sK + kStages * kTile;           // kStages stages
  Ctl& c = *reinterpret_cast<Ctl*>(sV + kStages * kTile);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  Ctrl* ctrl = a.ctrl;
  const uint32_t seq = a.seq;

  if (tid == 0) {
    mbar_init(&c.q_full, 1);
    for (uint32_t s = 0; s < kStages; ++s) {
      mbar_init(&c.k_full[s], kKThreads);
      mbar_init(&c.k_empty[s], 1);
      mbar_init(&c.v_full[s], kVThreads);
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
  if (warp == 0 && lane == 0) tma_prefetch_desc(&mq);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;

  // Test hook of the failure path (as in the block-sparse kernel).
  if (a.force_timeout) {
    if (tid == 0 && !mbar_wait_ns(&c.q_full, 0, 2ull * 1000ull * 1000ull, nullptr, 0u)) timeout(ctrl, c, seq, 1);
    __syncthreads();
  }

  uint32_t jbase = 0;
  uint32_t gbase[2] = {0u, 0u};
  uint32_t nq = 0;

  for (;;) {
    if (tid == 0) {
      const int item = atomicAdd(a.work, 1);
      c.item = item;
      if (item < a.n_items) {
        long long o0 = a.sel_offsets[item], o1 = a.sel_offsets[item + 1];
        if (o0 < 0 || o1 < o0 || o1 > a.n_sel || o1 - o0 > 0x7FFFFFFFll) {
          report_error(ctrl, kErrCount, (uint32_t)item, (uint32_t)(o1 - o0), 41u);
          o0 = o1 = 0;
        }
        c.off = o0;
        c.len = (int)(o1 - o0);
      }
    }
    __syncthreads();
    const int item = c.item;
    if (item >= a.n_items || c.abort) break;
    const int bh = item / a.nq;
    const int I = item - bh * a.nq;
    const long long off = c.off;
    const int len = c.len;
    const int n_tiles = (len + kEntries - 1) / kEntries;

    if (warp == 0 || warp == 2 || warp == 3) {
      // ---------------------------------------------------------- gathers
      const bool is_k = warp != 2;
      if (warp == 0 && lane == 0 && n_tiles > 0) {
        mbar_arrive_expect_tx(&c.q_full, kTile);
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sQ + ch * kChunk + h * (kChunk / 2), &mq, &c.q_full, ch * 64, I * 128 + 64 * h, bh);
      }
      const __nv_bfloat16* base = (is_k ? a.k : a.v) + (size_t)bh * a.Npad * D;
      const uint32_t s0 = smem_addr(is_k ? sK : sV);
      uint64_t* full = is_k ? c.k_full : c.v_full;
      uint64_t* empty = is_k ? c.k_empty : c.v_empty;
      int blk = (n_tiles > 0) ? entry_block(a, off, len, 0, lane, warp == 0) : -1;
      int issued = 0;   // tiles of this item whose copies this thread has issued
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t jg = jbase + j, s = jg % kStages;
        if (jg >= kStages && !wait_warp(&empty[s], ((jg - kStages) / kStages) & 1, ctrl, seq)) {
          if (lane == 0) timeout(ctrl, c, seq, is_k ? 10 : 11);
          break;
        }
        if (is_k) gather_tile<D, kKThreads>(s0 + s * kTile, base, blk, (warp == 0 ? 0 : 32) + lane, a.N);
        else gather_tile<D, kVThreads>(s0 + s * kTile, base, blk, lane, a.N);
        cp_async_commit();
        ++issued;
        // the next tile's entries, in flight while these copies land
        blk = (j + 1 < n_tiles) ? entry_block(a, off, len, j + 1, lane, warp == 0) : -1;
        if (j > 0) {
          // tile j - 1 has landed once at most one group (tile j) is in flight
          cp_async_wait<1>();
          fence_proxy_async_smem();   // the copies, ordered before the tensor core reads them
          mbar_arrive(&full[(jg - 1) % kStages]);
        }
      }
      // the last tile issued; after a timeout only the wait (nothing may be
      // left in flight when the item ends)
      cp_async_wait<0>();
      if (issued == n_tiles && n_tiles > 0) {
        fence_proxy_async_smem();
        mbar_arrive(&full[(jbase + n_tiles - 1) % kStages]);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
        const uint64_t dQ = smem_desc_sw128(smem_addr(sQ), 16, 1024);
        const uint32_t aK = smem_addr(sK), aV = smem_addr(sV);
        auto issue_s = [&](int jj) -> bool {
          const uint32_t jg = jbase + jj, ks = jg % kStages;
          const int w = jj & 1;
          if (!wait(&c.k_full[ks], (jg / kStages) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 21); return false; }
          tc_fence_after();
          const uint64_t dK = smem_desc_sw128(aK + ks * kTile, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t offb = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(tmem + 128 * w, smem_desc_add(dQ, offb), smem_desc_add(dK, offb), idS, kk > 0);
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
          const uint32_t jg = jbase + j, vs = jg % kStages;
          const int w = j & 1;
          const uint32_t gw = gbase[w] + (j >> 1);
          if (!wait(&c.p_full[w], gw & 1, ctrl, seq)) { timeout(ctrl, c, seq, 23); break; }
          if (!wait(&c.v_full[vs], (jg / kStages) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 24); break; }
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
    } else {
      // ---------------------------------------------------------- softmax + epilogue
      const int q4 = warp & 3;
      const int w = (warp - kSoftmaxWarp0) >> 2;
      const int r = q4 * 32 + lane;
      const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
      const uint32_t tS = trow + 128 * w, tOw = trow + kTmemO + 128 * w;
      const bool writer = q4 == 0;   // the group's first warp writes its shifts
      float m = -INFINITY;
      float l = 0.f, lx = 0.f;
      bool ok = true;
      int mine = 0;
      // entries of this group's first tile; each later tile's are loaded one
      // tile ahead
      int blk = -1;
      float wt = 1.f;
      if (writer && w < n_tiles) {
        blk = entry_block(a, off, len, w, lane, false);
        if (a.sel_w != nullptr && w * kEntries + lane < len) wt = __ldg(a.sel_w + off + w * kEntries + lane);
      }
      for (int j = w; j < n_tiles; j += 2, ++mine) {
        const uint32_t gw = gbase[w] + (j >> 1);
        float* shs = c.shift[w][(j >> 1) & 1];
        if (writer) {
          // column shifts of tile j: log2 w for the block's valid keys, -inf
          // for keys >= N, missing entries and invalid weights (reported).
          // The slot was last read for tile j - 4, before the group barrier
          // of tile j - 2.
          float sh = -INFINITY;
          int nv = 0;
          if (blk >= 0) {
            nv = min(kKeyBlock, a.N - blk * kKeyBlock);
            if (a.sel_w == nullptr) {
              sh = 0.f;
            } else if (wt > 0.f && wt <= 3.0e38f) {
              sh = log2f(wt);
            } else {
              report_error(ctrl, kErrWeight, (uint32_t)(off + j * kEntries + lane), __float_as_uint(wt), 42u);
              nv = 0;
            }
          }
          reinterpret_cast<float4*>(shs)[lane] = make_float4(nv > 0 ? sh : -INFINITY, nv > 1 ? sh : -INFINITY,
                                                             nv > 2 ? sh : -INFINITY, nv > 3 ? sh : -INFINITY);
          const int jn = j + 2;
          blk = -1;
          wt = 1.f;
          if (jn < n_tiles) {
            blk = entry_block(a, off, len, jn, lane, false);
            if (a.sel_w != nullptr && jn * kEntries + lane < len) wt = __ldg(a.sel_w + off + jn * kEntries + lane);
          }
        }
        // the shifts, visible to the whole group; a warp that timed out on
        // the previous tile makes the whole group leave here
        ok = group_sync(w, ok);
        if (!ok) break;
        const float4* shw4 = reinterpret_cast<const float4*>(shs);
        if (!wait_warp(&c.s_full[w], gw & 1, ctrl, seq)) {
          timeout(ctrl, c, seq, 30);
          ok = false;
          continue;   // to the next group barrier (or the end of the loop)
        }
        tc_fence_after();
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
        auto rescale_o = [&](float alpha) {
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t ov[32];
            tmem_ld32(tOw + cc, ov);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(tOw + cc, ov);
          }
          tmem_wait_st();
        };
        // As in the block-sparse kernel: the max pass runs only while a row
        // of the warp has no max yet; later tiles check each chunk's weights.
        const bool need_max = __any_sync(0xffffffffu, m == -INFINITY);
        if (need_max) {
          // Pass 1: row max of y = s * scale_log2 + shift over the 128 columns.
          float mh[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sr[64];
            tmem_ld32(tS + 64 * h, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld32(tS + 64 * h + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_wait_ld();
            const float* xh = reinterpret_cast<const float*>(sr);
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float4 s4 = shw4[16 * h + i];
              const float2 ya = ffma2(make_float2(xh[4 * i], xh[4 * i + 1]), sc2, make_float2(s4.x, s4.y));
              const float2 yb = ffma2(make_float2(xh[4 * i + 2], xh[4 * i + 3]), sc2, make_float2(s4.z, s4.w));
              m0 = fmax3(m0, ya.x, ya.y);
              m1 = fmax3(m1, yb.x, yb.y);
            }
            mh[h] = fmaxf(m0, m1);
          }
          const float mnew = fmaxf(m, fmaxf(mh[0], mh[1]));
          // Lazy rescale: the running max moves only when it grows by more
          // than 8 (or is set for the first time).
          const bool grow = mnew > m + 8.0f;
          if (__any_sync(0xffffffffu, grow && m != -INFINITY)) {
            const float alpha = (grow && m != -INFINITY) ? ex2f(m - mnew) : 1.0f;
            rescale_o(alpha);
            l *= alpha;
            lx *= alpha;
          }
          if (grow) m = mnew;
        }
        float nm = (m == -INFINITY) ? 0.f : -m;
        // Pass 2: p = 2^(s * scale_log2 + shift - m), 32 keys at a time; the
        // bf16 weights go to columns [16 c, 16 c + 16) of the same buffer.
        float rs[2] = {0.f, 0.f};
        float rx = 0.f, rx_ok = 0.f;
        const float2 one2 = make_float2(1.f, 1.f);
        auto exp_chunk = [&](const float* x, int cch, float nmv, uint32_t (&pk)[16]) {
          const float2 nm2 = make_float2(nmv, nmv);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 s4 = shw4[8 * cch + i];
            const float2 ca = ffma2(make_float2(s4.x, s4.y), one2, nm2);   // shift - m
            const float2 cb = ffma2(make_float2(s4.z, s4.w), one2, nm2);
            const float2 ya = ffma2(make_float2(x[4 * i], x[4 * i + 1]), sc2, ca);
            const float2 yb = ffma2(make_float2(x[4 * i + 2], x[4 * i + 3]), sc2, cb);
            const float p0 = ex2f(ya.x), p1 = ex2f(ya.y), p2 = ex2f(yb.x), p3 = ex2f(yb.y);
            pk[2 * i] = pack_bf16(p0, p1);
            pk[2 * i + 1] = pack_bf16(p2, p3);
            rs[0] = add_bf16x2(rs[0], pk[2 * i]);
            rs[1] = add_bf16x2(rs[1], pk[2 * i + 1]);
            if (WITH_LSE) rx += (p0 + p1) + (p2 + p3);
          }
        };
        int c_fail = 4;
        uint32_t sc[2][32];
        tmem_ld32(tS, sc[0]);
#pragma unroll
        for (int cch = 0; cch < 4; ++cch) {
          tmem_wait_ld();
          if (cch < 3) tmem_ld32(tS + 32 * (cch + 1), sc[(cch + 1) & 1]);
          uint32_t pk[16];
          exp_chunk(reinterpret_cast<const float*>(sc[cch & 1]), cch, nm, pk);
          // a weight of 2^64 or more: this tile's logits exceed the running
          // max by 64 or more; nothing of this chunk is stored
          if (!need_max && __any_sync(0xffffffffu, !(rs[0] + rs[1] < 0x1p64f))) {
            c_fail = cch;
            break;
          }
          tmem_st16(tS + 16 * cch, pk);
          rx_ok = rx;
        }
        if (c_fail < 4) {
          // Rare: a new max from the logits of chunks c_fail..3, O, the sums
          // and the stored weights rescaled, chunks c_fail..3 redone (as in
          // the block-sparse kernel).
          tmem_wait_ld();
          float mx = -INFINITY;
#pragma unroll 1
          for (int cc = c_fail; cc < 4; ++cc) {
            uint32_t t[32];
            tmem_ld32(tS + 32 * cc, t);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 s4 = shw4[8 * cc + i];
              mx = fmax3(mx, fmaf(__uint_as_float(t[4 * i]), a.scale_log2, s4.x),
                         fmaf(__uint_as_float(t[4 * i + 1]), a.scale_log2, s4.y));
              mx = fmax3(mx, fmaf(__uint_as_float(t[4 * i + 2]), a.scale_log2, s4.z),
                         fmaf(__uint_as_float(t[4 * i + 3]), a.scale_log2, s4.w));
            }
          }
          const float mnew = fmaxf(m, mx);
          const float alpha = ex2f(m - mnew);   // m is finite: the max pass ran on an earlier tile
          rescale_o(alpha);
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
          rx = alpha * rx_ok;
          m = mnew;
          nm = -m;
#pragma unroll 1
          for (int cc = c_fail; cc < 4; ++cc) {
            uint32_t t[32];
            tmem_ld32(tS + 32 * cc, t);
            tmem_wait_ld();
            uint32_t pk[16];
            exp_chunk(reinterpret_cast<const float*>(t), cc, nm, pk);
            tmem_st16(tS + 16 * cc, pk);
          }
        }
        l += rs[0] + rs[1];
        if (WITH_LSE) lx += rx;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&c.p_full[w]);
      }

      // epilogue: merge of the two groups' partial results (as in the
      // block-sparse kernel); group w writes columns [w D / 2, (w + 1) D / 2).
      const int cnt0 = (n_tiles + 1) / 2, cnt1 = n_tiles / 2;
      const bool has0 = cnt0 > 0, has1 = cnt1 > 0;
      if (ok && has0 && !wait_warp(&c.pv_done[0], (gbase[0] + cnt0 - 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 31); ok = false; }
      if (ok && has1 && !wait_warp(&c.pv_done[1], (gbase[1] + cnt1 - 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 31); ok = false; }
      tc_fence_after();
      // The merge goes through the K stages: every S of the item has
      // completed and the next item's K gathers start after the item.
      float* xm = reinterpret_cast<float*>(sK);
      float* xl = xm + 2 * 128;
      xm[w * 128 + r] = (mine > 0) ? m : -INFINITY;
      xl[(2 * w + 0) * 128 + r] = l;
      xl[(2 * w + 1) * 128 + r] = lx;
      tc_fence_before();
      ok = pair_sync(q4, ok);
      tc_fence_after();
      const float m0 = xm[r], m1 = xm[128 + r];
      const float mt = fmaxf(m0, m1);
      const float a0 = (has0 && m0 != -INFINITY) ? ex2f(m0 - mt) : 0.f;
      const float a1 = (has1 && m1 != -INFINITY) ? ex2f(m1 - mt) : 0.f;
      const float lt = xl[r] * a0 + xl[2 * 128 + r] * a1;
      const float lxt = xl[128 + r] * a0 + xl[3 * 128 + r] * a1;
      const int qrow = I * 128 + r;
      const bool real = ok && qrow < a.N && lt > 0.f;
      const float inv = real ? 1.f / lt : 0.f;
      const float s0 = a0 * inv, s1 = a1 * inv;
      uint4* orow = reinterpret_cast<uint4*>(a.o + ((size_t)bh * a.Npad + qrow) * D + w * (D / 2));
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
#pragma unroll
        for (int i = 0; i < 2; ++i)
          orow[cc / 8 + i] = make_uint4(pw[4 * i], pw[4 * i + 1], pw[4 * i + 2], pw[4 * i + 3]);
      }
      if (WITH_LSE && w == 0)
        a.lse[(size_t)bh * a.Npad + qrow] = real ? (mt + __log2f(lxt)) * 0.69314718055994531f : 0.f;
      fence_proxy_async_smem();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    jbase += n_tiles;
    gbase[0] += (n_tiles + 1) / 2;
    gbase[1] += n_tiles / 2;
    if (n_tiles > 0) ++nq;
  }

  // Drain: the gathers wait for their own copies before arriving, so only the
  // Q loads and the MMAs can still be in flight after a timeout.
  if (lane == 0) {
    if (warp == 0) {
      mbar_drain_ring(&c.q_full, 1, nq, kWaitNs);
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

template <int D, bool WITH_LSE>
cudaError_t launch_fine_t(const FineArgs& a, const void* q, uint64_t bhs, cudaStream_t st) {
  CUtensorMap mq;
  if (!make_map_bf16_3d(&mq, q, D, (uint64_t)a.Npad, bhs, 64, 64)) return cudaErrorInvalidValue;
  const size_t smem = (1u + 2u * kStages) * 128u * D * 2u + sizeof(Ctl);
  static_assert((1u + 2u * kStages) * 128u * 128u * 2u + sizeof(Ctl) <= 227u * 1024u, "shared memory layout");
  cudaError_t e =
      cudaFuncSetAttribute(attn_fine_kernel<D, WITH_LSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms() ? a.n_items : num_sms();
  attn_fine_kernel<D, WITH_LSE><<<grid, kThreads, smem, st>>>(mq, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fine(const Dims& g, const void* q, const void* k, const void* v, const int64_t* sel_offsets,
                             const int32_t* sel_idx, const float* sel_w, int64_t n_sel, float scale, void* o,
                             float* lse, Ctrl* ctrl, int* work, uint32_t seq, cudaStream_t st) {
  FineArgs a;
  a.k = (const __nv_bfloat16*)k;
  a.v = (const __nv_bfloat16*)v;
  a.sel_offsets = (const long long*)sel_offsets;
  a.sel_idx = sel_idx;
  a.sel_w = sel_w;
  a.n_sel = (long long)n_sel;
  a.o = (__nv_bfloat16*)o;
  a.lse = lse;
  a.ctrl = ctrl;
  a.work = work;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.N = g.N;
  a.Npad = g.Npad;
  a.nq = g.Npad / 128;
  a.nkb = (g.N + kKeyBlock - 1) / kKeyBlock;
  const uint64_t bhs = (uint64_t)g.B * g.heads;
  if (bhs * (uint64_t)a.nq > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  a.n_items = (int)(bhs * a.nq);
  a.seq = seq;
  a.force_timeout = force_timeout_requested();
  cudaError_t e = cudaMemsetAsync(work, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  if (g.d == 128)
    return lse != nullptr ? launch_fine_t<128, true>(a, q, bhs, st) : launch_fine_t<128, false>(a, q, bhs, st);
  return lse != nullptr ? launch_fine_t<64, true>(a, q, bhs, st) : launch_fine_t<64, false>(a, q, bhs, st);
}

}  // namespace bsa
