// Backward pass of the block-sparse attention on the sm_100a tensor cores.
// NABLA summary, "Contribuciones Clave" ("Aceleracion de Doble Fase"): the
// adaptive block-sparse attention also runs in pre-training and fine-tuning,
// so its gradients follow the same block mask.  For a query row q of block I
// and the valid keys k of the blocks I keeps (scale s, the forward pass's
// log-sum-exp L_q):
//   P[q,k]  = exp(s Q_q . K_k - L_q)
//   dV_k   += sum_q P[q,k] dO_q
//   dP[q,k] = dO_q . V_k
//   dS[q,k] = P[q,k] (dP[q,k] - D_q),   D_q = dO_q . O_q
//   dQ_q    = s sum_k dS[q,k] K_k,       dK_k = s sum_q dS[q,k] Q_q
//
// Two persistent kernels, so that no gradient needs atomics:
//   dq kernel    the forward's 128-row query tiles (the same plan), walking
//                the union of their KV lists: S = Q K^T and dP = dO V^T into
//                TMEM, P and dS by the softmax warps (dS written as bf16 over
//                the S columns), dQ += dS K with A = dS from TMEM;
//   dkdv kernel  128-key tiles (one block of 128, or two blocks of 64 paired
//                by the same planner run on the transposed lists), walking the
//                union of the query blocks that keep them: S^T = K Q^T and
//                dP^T = V dO^T into TMEM, P^T and dS^T written as bf16 over
//                their own columns, dV += P^T dO and dK += dS^T Q with A from
//                TMEM.
// tcgen05.mma operations of one thread execute in issue order: a product
// that overwrites the bf16 operand of an earlier product runs after it.
// The dq kernel keeps S in two TMEM buffers and writes dS over the S it was
// computed from, so the next tile's dP (one fixed buffer, free once the
// softmax warps have read it) is issued as soon as they finish a tile, ahead
// of that tile's dQ product and the S of the tile after next.  Its softmax
// warps work in two phases: fp32 P in place over S (S is in TMEM a tile
// ahead), then dS once dP is there, so only the dP product's wait sits
// between two tiles' softmax work, and the exponentials overlap it.  The dkdv kernel has no TMEM
// to spare (S, dP and two accumulators fill it); its softmax warps work in two
// phases instead: P^T from S^T alone (the exponentials), then dS^T from the
// bf16 P^T kept in registers once dP^T is there.  dV and the next S^T run
// after the first phase, dK and the next dP^T after the second, so the next
// tile's exponentials overlap dK and dP^T.
//
// Small kernels before them: D = rowsum(dO * O) per row (fp32), and the
// transposed lists (for each KV block, the ascending list of query blocks
// that keep it) from the forward lists through a bit matrix.
//
// Every mbarrier wait is bounded (as in the forward kernels): on expiry the
// CTA records BSA_ERR_TIMEOUT, tells the launch's other CTAs to give up, waits
// (bounded) for what it has issued, frees its TMEM and leaves.
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

constexpr int kThreads = 256;            // warps: 0, 2 producers, 1 MMA issuer, 3 idle, 4-7 softmax
constexpr int kSoftmaxWarp0 = 4;
constexpr uint32_t kGroupThreads = 128;
constexpr uint64_t kWaitNs = 250ull * 1000ull * 1000ull;
constexpr uint32_t kTmemCols = 512;
// TMEM column bases.  dkdv: S^T (P^T over it), dP^T (dS^T over it), dV, dK.
// dq: S of even tiles, dP, S of odd tiles (dS over each S), dQ.
constexpr uint32_t kTS = 0, kTdP = 128, kTAcc0 = 256, kTAcc1 = 384;
constexpr uint32_t kTS1 = 256, kTdQ = 384;
constexpr uint16_t kEntBlock = 0x0FFFu;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------ small kernels

// D[bh][row] = sum_c dO[row][c] * O[row][c] (bf16 values, fp32 sum); D/8
// consecutive lanes per row, one 16-byte vector of O and of dO each.
template <int D>
__global__ void __launch_bounds__(256) bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         float* __restrict__ Dv, Dims g) {
  constexpr int VEC = D / 8;                       // 16-byte vectors per row
  const size_t rows = (size_t)g.B * g.heads * g.Npad;
  const size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) / VEC;
  const int c = threadIdx.x % VEC;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = reinterpret_cast<const uint4*>(o)[row * VEC + c];
    const uint4 b = reinterpret_cast<const uint4*>(dO)[row * VEC + c];
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc);
      acc = fmaf(__uint_as_float(aw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int off = VEC / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && c == 0) {
    const int p = (int)(row % g.Npad);
    Dv[row] = (p < g.N) ? acc : 0.f;
  }
}

// Bit matrix of the forward lists: bits[bh][I][J / 32] bit J % 32 set when
// block I keeps J (entries outside [0, nb) ignored).  One warp per row.
__global__ void __launch_bounds__(256) bwd_bits_kernel(const int32_t* __restrict__ kv_count,
                                                       const int32_t* __restrict__ kv_idx, Dims g,
                                                       uint32_t* __restrict__ bits) {
  __shared__ uint32_t sw[8][BSA_MAX_BLOCKS / 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nb = g.nb, nw = (nb + 31) >> 5;
  const size_t row = (size_t)blockIdx.x * 8 + wid;
  if (row >= (size_t)g.B * g.heads * nb) return;
  for (int i = lane; i < BSA_MAX_BLOCKS / 32; i += 32) sw[wid][i] = 0u;
  __syncwarp();
  int cnt = kv_count[row];
  cnt = cnt < 0 ? 0 : (cnt > nb ? nb : cnt);
  for (int e = lane; e < cnt; e += 32) {
    const int J = kv_idx[row * nb + e];
    if (J >= 0 && J < nb) atomicOr(&sw[wid][J >> 5], 1u << (J & 31));
  }
  __syncwarp();
  for (int i = lane; i < nw; i += 32) bits[row * nw + i] = sw[wid][i];
}

// Transposed lists: for KV block J of (b, head), q_count = the number of
// query blocks I that keep J, q_idx = those I in ascending order.  One warp
// per (bh, J): a column of the bit matrix, 32 rows at a time.
__global__ void __launch_bounds__(256) bwd_tlist_kernel(const uint32_t* __restrict__ bits, Dims g,
                                                        int32_t* __restrict__ q_count, int32_t* __restrict__ q_idx) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nb = g.nb, nw = (nb + 31) >> 5;
  const size_t col = (size_t)blockIdx.x * 8 + wid;        // bh * nb + J
  if (col >= (size_t)g.B * g.heads * nb) return;
  const size_t bh = col / nb;
  const int J = (int)(col % nb);
  const uint32_t* b = bits + bh * nb * nw;
  int n = 0;
  for (int I0 = 0; I0 < nb; I0 += 32) {
    const int I = I0 + lane;
    const bool kept = I < nb && ((b[(size_t)I * nw + (J >> 5)] >> (J & 31)) & 1u);
    const uint32_t bal = __ballot_sync(0xffffffffu, kept);
    if (kept) q_idx[col * nb + n + __popc(bal & ((1u << lane) - 1u))] = I;
    n += __popc(bal);
  }
  if (lane == 0) q_count[col] = n;
}

// ------------------------------------------------------- the main kernels

struct Ctl {
  uint64_t a_full[3], a_empty[3], b_full[2], b_empty[2];   // per-tile operand stages (a: three for dq)
  uint64_t fixed_full;                                      // the item's fixed operands
  uint64_t sdp_full, ds_full, acc_done, drain;
  uint64_t dp_full, p_full;                                 // dP (dP^T) in TMEM; dkdv: P^T written
  uint64_t s_full[2];                                       // dq: S in TMEM buffer 0 / 1
  uint32_t tmem_base;
  int n_ent;
  int item;
  int abort;
  uint32_t bm[2][BSA_MAX_BLOCKS / 32];
  uint16_t ent[BSA_MAX_BLOCKS];
};

__device__ __forceinline__ void timeout(Ctrl* ctrl, Ctl& c, uint32_t seq, uint32_t site) {
  report_error(ctrl, kErrTimeout, blockIdx.x, threadIdx.x, site);
  atomicExch(&ctrl->abort_seq, seq);
  c.abort = 1;
}
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  return mbar_wait_ns(bar, parity, kWaitNs, &ctrl->abort_seq, seq);
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Ctrl* ctrl, uint32_t seq) {
  const bool ok = wait(bar, parity, ctrl, seq);
  return __all_sync(0xffffffffu, ok);
}

// One kernel body for both passes.
//   DKDV = false (dq pass): fixed operands Q and dO (128 query rows), tile
//     operands K (stage a, three stages: S of a tile is issued a tile ahead)
//     and V (stage b) of each KV tile; S = Q K^T, dP = dO V^T; dQ += dS K.
//   DKDV = true (dkdv pass): fixed operands K and V (128 keys), tile operands
//     Q (a) and dO (b) of each query tile, plus that tile's L and D rows;
//     S^T = K Q^T, dP^T = V dO^T; acc0 = dV += P^T dO, acc1 = dK += dS^T Q.
// `lists` are the lists the tile walks (kv lists for dq, transposed lists for
// dkdv); `items` the planner's 128-row tiles of the fixed side.
template <int D, int BS, bool DKDV>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_kernel(
    const __grid_constant__ CUtensorMap mfix0, const __grid_constant__ CUtensorMap mfix1,
    const __grid_constant__ CUtensorMap mtile0, const __grid_constant__ CUtensorMap mtile1,
    const int32_t* __restrict__ l_count, const int32_t* __restrict__ l_idx, const int2* __restrict__ items,
    int* work, const float* __restrict__ lse, const float* __restrict__ Dv, float scale_log2, float scale,
    __nv_bfloat16* __restrict__ out0, __nv_bfloat16* __restrict__ out1, Ctrl* ctrl, Dims g, int items_per_bh,
    int n_items, uint32_t seq) {
  constexpr int QB = 128 / BS;          // blocks per 128-row tile (fixed side and walked side alike)
  constexpr int CH = D / 64;            // 128-byte chunks of a row
  constexpr uint32_t kTile = 128u * D * 2u;
  constexpr uint32_t kChunk = 128u * 128u;
  constexpr uint32_t NA = DKDV ? 2u : 3u;   // stages of tile operand a
  constexpr uint32_t kRowBytes = DKDV ? 2u * 256u * sizeof(float) : 0u;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_addr(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report_error(ctrl, kErrLayout, blockIdx.x, 0u, 5u);
    return;
  }
  uint8_t* sF0 = smem_raw;              // fixed operand 0 (Q or K)
  uint8_t* sF1 = sF0 + kTile;           // fixed operand 1 (dO or V)
  uint8_t* sA = sF0 + 2 * kTile;        // NA stages of tile operand a (K or Q)
  uint8_t* sB = sA + NA * kTile;        // two stages of tile operand b (V or dO)
  float* sRow = reinterpret_cast<float*>(sB + 2 * kTile);   // dkdv: [stage][L 128 | D 128]
  Ctl& c = *reinterpret_cast<Ctl*>(sB + 2 * kTile + kRowBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = g.nb, nw = (nb + 31) >> 5;

  if (tid == 0) {
    for (int s = 0; s < (int)NA; ++s) {
      mbar_init(&c.a_full[s], 1);
      mbar_init(&c.a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&c.b_full[s], 1);
      mbar_init(&c.b_empty[s], 1);
    }
    mbar_init(&c.fixed_full, 1);
    mbar_init(&c.sdp_full, 1);
    mbar_init(&c.ds_full, kGroupThreads);
    mbar_init(&c.dp_full, 1);
    mbar_init(&c.p_full, kGroupThreads);
    mbar_init(&c.s_full[0], 1);
    mbar_init(&c.s_full[1], 1);
    mbar_init(&c.acc_done, 1);
    mbar_init(&c.drain, 1);
    c.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mfix0);
    tma_prefetch_desc(&mfix1);
    tma_prefetch_desc(&mtile0);
    tma_prefetch_desc(&mtile1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;

  uint32_t jbase = 0;   // walked tiles so far (phase counter of the a/b stages and of sdp/ds/acc)
  uint32_t nfix = 0;    // fixed loads so far
  uint32_t armed = 0;   // stage loads this producer thread has issued

  for (;;) {
    if (tid == 0) c.item = atomicAdd(work, 1);
    for (int i = tid; i < 2 * (BSA_MAX_BLOCKS / 32); i += kThreads) (&c.bm[0][0])[i] = 0u;
    __syncthreads();
    const int item = c.item;
    if (item >= n_items || c.abort) break;
    const int bh = item / items_per_bh;
    const int2 it = items[item];
    int fblk[QB];
    bool fval[QB];
    fblk[0] = it.x;
    fval[0] = it.x >= 0 && it.x < nb;
    if (QB == 2) {
      fblk[QB - 1] = it.y;
      fval[QB - 1] = it.y >= 0 && it.y < nb;
    }
    if (!fval[0]) fblk[0] = 0;

    // the walked lists of the tile's fixed blocks, as bitmaps, then their
    // ascending union with membership bits (bit 12 + h: fixed block h lists it)
#pragma unroll
    for (int h = 0; h < QB; ++h) {
      if (!fval[h]) continue;
      const size_t row = (size_t)bh * nb + fblk[h];
      int cnt = l_count[row];
      if (cnt < 0 || cnt > nb) {
        if (tid == 0) report_error(ctrl, kErrCount, (uint32_t)row, (uint32_t)cnt, 6u);
        cnt = cnt < 0 ? 0 : nb;
      }
      const int32_t* list = l_idx + row * nb;
      for (int i = tid; i < cnt; i += kThreads) {
        const int J = list[i];
        if (J >= 0 && J < nb) atomicOr(&c.bm[h][J >> 5], 1u << (J & 31));
        else report_error(ctrl, kErrIndex, (uint32_t)row, (uint32_t)J, 7u);
      }
    }
    __syncthreads();
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
    const int n_tiles = (n_ent + QB - 1) / QB;

    // global row of 64-row half h of walked tile j (64-aligned)
    auto walked_row0 = [&](int j, int h) -> int {
      if (QB == 2) {
        const int idx = (2 * j + h < n_ent) ? 2 * j + h : 2 * j;
        return (int)(c.ent[idx] & kEntBlock) * 64;
      }
      return (int)(c.ent[j] & kEntBlock) * 128 + 64 * h;
    };
    auto fixed_row0 = [&](int h) -> int {
      if (QB == 2) return (fval[h & (QB - 1)] ? fblk[h & (QB - 1)] : fblk[0]) * 64;
      return fblk[0] * 128 + 64 * h;
    };

    if (warp == 0 || warp == 2) {
      // ------------------------------------------------------------ producers
      // warp 0: the fixed operands, then operand a of every walked tile;
      // warp 2: operand b of every walked tile (and, dkdv, its L and D rows).
      const bool is_a = warp == 0;
      if (lane == 0 && n_tiles > 0) {
        if (is_a) {
          mbar_arrive_expect_tx(&c.fixed_full, 2 * kTile);
#pragma unroll
          for (int ch = 0; ch < CH; ++ch)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tma_load_3d(sF0 + ch * kChunk + h * (kChunk / 2), &mfix0, &c.fixed_full, ch * 64, fixed_row0(h), bh);
              tma_load_3d(sF1 + ch * kChunk + h * (kChunk / 2), &mfix1, &c.fixed_full, ch * 64, fixed_row0(h), bh);
            }
        }
        const uint32_t ns = is_a ? NA : 2u;
        for (int j = 0; j < n_tiles; ++j) {
          const uint32_t jg = jbase + j, s = jg % ns;
          uint64_t* full = is_a ? &c.a_full[s] : &c.b_full[s];
          uint64_t* empty = is_a ? &c.a_empty[s] : &c.b_empty[s];
          if (jg >= ns && !wait(empty, ((jg / ns) - 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 10); break; }
          const uint32_t extra = (!is_a && DKDV) ? 2u * 128u * sizeof(float) : 0u;
          mbar_arrive_expect_tx(full, kTile + extra);
          ++armed;
          uint8_t* dst = (is_a ? sA : sB) + s * kTile;
          const CUtensorMap* m = is_a ? &mtile0 : &mtile1;
#pragma unroll
          for (int ch = 0; ch < CH; ++ch)
#pragma unroll
            for (int h = 0; h < 2; ++h) tma_load_3d(dst + ch * kChunk + h * (kChunk / 2), m, full, ch * 64, walked_row0(j, h), bh);
          if (!is_a && DKDV) {
            float* rows = sRow + s * 256;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const size_t r0 = (size_t)bh * g.Npad + walked_row0(j, h);
              bulk_load(rows + 64 * h, lse + r0, 64 * sizeof(float), full);
              bulk_load(rows + 128 + 64 * h, Dv + r0, 64 * sizeof(float), full);
            }
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
        const uint64_t dF0 = smem_desc_sw128(smem_addr(sF0), 16, 1024);
        const uint64_t dF1 = smem_desc_sw128(smem_addr(sF1), 16, 1024);
        const uint32_t aA = smem_addr(sA), aB = smem_addr(sB);
        bool go = wait(&c.fixed_full, nfix & 1, ctrl, seq);
        if (!go) timeout(ctrl, c, seq, 20);
        if (!DKDV) {
          // dq, per walked tile j: S_j = Q K_j^T into the S buffer of j's
          // parity (each buffer with a barrier of its own), issued a tile
          // ahead; dP_j = dO V_j^T as soon as the softmax warps are done with
          // tile j - 1 (its dP is read); then dQ += dS_{j-1} K_{j-1} and
          // S_{j+1} over dS_{j-1}.
          auto issue_s = [&](uint32_t jg) -> bool {
            const uint32_t sa = jg % NA;
            if (!wait(&c.a_full[sa], (jg / NA) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 21); return false; }
            tc_fence_after();
            const uint64_t dA = smem_desc_sw128(aA + sa * kTile, 16, 1024);
            const uint32_t col = (jg & 1) ? kTS1 : kTS;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
              mma_ss(tmem + col, smem_desc_add(dF0, off), smem_desc_add(dA, off), idS, kk > 0);
            }
            mma_commit(&c.s_full[jg & 1]);
            return true;
          };
          auto issue_dp = [&](uint32_t jg) -> bool {
            const uint32_t sb = jg & 1;
            if (!wait(&c.b_full[sb], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 22); return false; }
            tc_fence_after();
            const uint64_t dB = smem_desc_sw128(aB + sb * kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
              mma_ss(tmem + kTdP, smem_desc_add(dF1, off), smem_desc_add(dB, off), idS, kk > 0);
            }
            mma_commit(&c.dp_full);
            mma_commit(&c.b_empty[sb]); // V_j is read by dP_j alone
            return true;
          };
          go = go && issue_s(jbase);
          go = go && (n_tiles < 2 || issue_s(jbase + 1));
          go = go && issue_dp(jbase);
          for (int j = 0; go && j < n_tiles; ++j) {
            const uint32_t jg = jbase + j, sa = jg % NA;
            if (!wait(&c.ds_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 23); break; }
            tc_fence_after();
            if (j + 1 < n_tiles && !issue_dp(jg + 1)) break;
            // dQ += dS K: A = dS (bf16 over the S columns), B = K (MN-major)
            const uint32_t col = (jg & 1) ? kTS1 : kTS;
            const uint64_t dK = smem_desc_sw128(aA + sa * kTile, kChunk, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + kTdQ, tmem + col + 8 * kk, smem_desc_add(dK, kk * 2048), idO, (kk > 0 || j > 0) ? 1u : 0u);
            mma_commit(&c.a_empty[sa]);
            if (j == n_tiles - 1) mma_commit(&c.acc_done);
            if (j + 2 < n_tiles && !issue_s(jg + 2)) break;
          }
        } else {
          // dkdv, per walked tile j: S^T_j = K Q_j^T, then dP^T_j = V dO_j^T,
          // each on a barrier of its own; once the softmax warps have written
          // P^T_j over S^T_j, dV += P^T dO and S^T_{j+1} over it; once they
          // have written dS^T_j over dP^T_j, dK += dS^T Q and dP^T_{j+1}.
          // The softmax warps compute P^T_{j+1} while dK and dP^T_{j+1} run.
          auto issue_s = [&](uint32_t jg) -> bool {
            const uint32_t s = jg & 1;
            if (!wait(&c.a_full[s], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 21); return false; }
            tc_fence_after();
            const uint64_t dA = smem_desc_sw128(aA + s * kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
              mma_ss(tmem + kTS, smem_desc_add(dF0, off), smem_desc_add(dA, off), idS, kk > 0);
            }
            mma_commit(&c.sdp_full);
            return true;
          };
          auto issue_dp = [&](uint32_t jg) -> bool {
            const uint32_t s = jg & 1;
            if (!wait(&c.b_full[s], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 22); return false; }
            tc_fence_after();
            const uint64_t dB = smem_desc_sw128(aB + s * kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
              mma_ss(tmem + kTdP, smem_desc_add(dF1, off), smem_desc_add(dB, off), idS, kk > 0);
            }
            mma_commit(&c.dp_full);
            return true;
          };
          go = go && issue_s(jbase) && issue_dp(jbase);
          for (int j = 0; go && j < n_tiles; ++j) {
            const uint32_t jg = jbase + j, s = jg & 1;
            const uint32_t acc = (j > 0) ? 1u : 0u;
            if (!wait(&c.p_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 23); break; }
            tc_fence_after();
            // dV += P^T dO: A = P^T (bf16 over the S columns), B = dO (MN-major)
            const uint64_t dOt = smem_desc_sw128(aB + s * kTile, kChunk, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + kTAcc0, tmem + kTS + 8 * kk, smem_desc_add(dOt, kk * 2048), idO, kk > 0 ? 1u : acc);
            if (j + 1 < n_tiles && !issue_s(jg + 1)) break;
            if (!wait(&c.ds_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 24); break; }
            tc_fence_after();
            // dK += dS^T Q: A = dS^T (bf16 over the dP columns), B = Q (MN-major)
            const uint64_t dQt = smem_desc_sw128(aA + s * kTile, kChunk, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + kTAcc1, tmem + kTdP + 8 * kk, smem_desc_add(dQt, kk * 2048), idO, kk > 0 ? 1u : acc);
            // the stages (and this tile's L and D rows) are free once dK has read Q
            mma_commit(&c.a_empty[s]);
            mma_commit(&c.b_empty[s]);
            if (j == n_tiles - 1) mma_commit(&c.acc_done);
            if (j + 1 < n_tiles && !issue_dp(jg + 1)) break;
          }
        }
      }
    } else if (warp >= kSoftmaxWarp0) {
      // ------------------------------------------------------------ softmax warps
      // Thread = TMEM lane = row r of the fixed side (a query row for dq, a
      // key row for dkdv); columns = the walked tile's 128 keys (dq) or
      // queries (dkdv), 64 per half.
      const int q4 = warp & 3;
      const int r = q4 * 32 + lane;
      const int fhalf = (QB == 2) ? (r >> 6) : 0;        // fixed block of the row
      const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
      int frow;                                           // global row of r on the fixed side
      if (QB == 2) frow = fval[fhalf] ? fblk[fhalf] * 64 + (r & 63) : -1;
      else frow = fval[0] ? fblk[0] * 128 + r : -1;
      const bool frow_ok = frow >= 0 && frow < g.N;
      // dq: this row's log-sum-exp (base 2) and D
      float lse2 = 0.f, drow = 0.f;
      if (!DKDV && frow_ok) {
        lse2 = lse[(size_t)bh * g.Npad + frow] * kLog2e;
        drow = Dv[(size_t)bh * g.Npad + frow];
      }
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const uint32_t jg = jbase + j, s = jg & 1;
        // valid columns of each 64-column half: kept by this row's block, real rows/keys
        int lim[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          int col0, kept;
          if (QB == 2) {
            const int idx = 2 * j + h;
            kept = (idx < n_ent) ? ((c.ent[idx] >> (12 + fhalf)) & 1) : 0;
            col0 = (idx < n_ent) ? (int)(c.ent[idx] & kEntBlock) * 64 : 0;
          } else {
            kept = 1;
            col0 = (int)(c.ent[j] & kEntBlock) * 128 + 64 * h;
          }
          lim[h] = (kept && frow_ok) ? max(0, min(64, g.N - col0)) : 0;
        }
        const float2 sl2 = make_float2(scale_log2, scale_log2);
        if (!DKDV) {
          // dq phase 1, S alone (in TMEM a tile ahead): per pair of columns
          // p = 2^(x scale log2 e - L log2 e) in packed two-lane arithmetic,
          // written as fp32 over the S just read.  Two buffers: the next
          // chunk's scores load while this one is computed.
          if (!wait_warp(&c.s_full[jg & 1], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 30); ok = false; break; }
          tc_fence_after();
          const uint32_t tS = trow + ((jg & 1) ? kTS1 : kTS);
          {
            const float2 nl = make_float2(-lse2, -lse2);
            uint32_t sv2[2][32];
            tmem_ld32(tS, sv2[0]);
#pragma unroll
            for (int cch = 0; cch < 4; ++cch) {
              tmem_wait_ld();
              if (cch < 3) tmem_ld32(tS + 32 * (cch + 1), sv2[(cch + 1) & 1]);
              uint32_t* sv = sv2[cch & 1];
              // valid columns of this chunk: all 32 (no per-column test in
              // the loop, the common case), some, or none (stored as they
              // are: phase 2 writes zeros there).  cl differs between the
              // lanes of a warp at the ragged end, so the warp-collective
              // TMEM store below runs in every case.
              const int cl = min(32, max(0, lim[cch >> 1] - 32 * (cch & 1)));
              auto pair = [&](int i, bool masked) {
                const float2 y = ffma2(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2, nl);
                float2 p = make_float2(ex2f(y.x), ex2f(y.y));
                if (masked) {
                  p.x = (2 * i < cl) ? p.x : 0.f;
                  p.y = (2 * i + 1 < cl) ? p.y : 0.f;
                }
                sv[2 * i] = __float_as_uint(p.x);
                sv[2 * i + 1] = __float_as_uint(p.y);
              };
              if (cl == 32) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pair(i, false);
              } else if (cl > 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pair(i, true);
              }
              tmem_st32(tS + 32 * cch, sv2[cch & 1]);
            }
          }
          tmem_wait_st();
          // phase 2, once dP is in TMEM: dS = p (dP - D) from the fp32 p,
          // as bf16 over the columns already read (dP is then free for the
          // next tile's product)
          if (!wait_warp(&c.dp_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 34); ok = false; break; }
          tc_fence_after();
          const float2 dd = make_float2(drow, drow);
          uint32_t pv2[2][32], dv2[2][32];
          tmem_ld32(tS, pv2[0]);
          tmem_ld32(trow + kTdP, dv2[0]);
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            tmem_wait_ld();
            if (cch < 3) {
              tmem_ld32(tS + 32 * (cch + 1), pv2[(cch + 1) & 1]);
              tmem_ld32(trow + kTdP + 32 * (cch + 1), dv2[(cch + 1) & 1]);
            }
            const uint32_t* pv = pv2[cch & 1];
            const uint32_t* dv = dv2[cch & 1];
            const int cl = min(32, max(0, lim[cch >> 1] - 32 * (cch & 1)));
            uint32_t dk[16];
            if (cl > 0) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 ds = fmul2(make_float2(__uint_as_float(pv[2 * i]), __uint_as_float(pv[2 * i + 1])),
                                        fsub2(make_float2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])), dd));
                dk[i] = pack_bf16(ds.x, ds.y);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) dk[i] = 0u;
            }
            tmem_st16(tS + 16 * cch, dk);
          }
        } else {
          if (!wait_warp(&c.sdp_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 30); ok = false; break; }
          tc_fence_after();
          // dkdv phase 1, S^T alone: P^T = 2^(x scale log2 e - L log2 e) per
          // pair of columns, as bf16 over the S^T columns already read and
          // kept in registers; then the dV product may run.
          // L and D of the tile's 128 query columns land with its dO stage,
          // which S^T does not wait for
          if (!wait_warp(&c.b_full[s], (jg >> 1) & 1, ctrl, seq)) { timeout(ctrl, c, seq, 33); ok = false; break; }
          const float* rowL = sRow + s * 256;
          const float2 nlg2 = make_float2(-kLog2e, -kLog2e);
          uint32_t pk[4][16];
          {
            uint32_t sv2[2][32];
            tmem_ld32(trow + kTS, sv2[0]);
#pragma unroll
            for (int cch = 0; cch < 4; ++cch) {
              tmem_wait_ld();
              if (cch < 3) tmem_ld32(trow + kTS + 32 * (cch + 1), sv2[(cch + 1) & 1]);
              const uint32_t* sv = sv2[cch & 1];
              const int cl = min(32, max(0, lim[cch >> 1] - 32 * (cch & 1)));
              auto pair = [&](int i, bool masked) {
                const float2 nl = fmul2(*reinterpret_cast<const float2*>(rowL + 32 * cch + 2 * i), nlg2);
                const float2 y = ffma2(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2, nl);
                float2 p = make_float2(ex2f(y.x), ex2f(y.y));
                if (masked) {
                  p.x = (2 * i < cl) ? p.x : 0.f;
                  p.y = (2 * i + 1 < cl) ? p.y : 0.f;
                }
                pk[cch][i] = pack_bf16(p.x, p.y);
              };
              if (cl == 32) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pair(i, false);
              } else if (cl > 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) pair(i, true);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[cch][i] = 0u;
              }
              tmem_st16(trow + kTS + 16 * cch, pk[cch]);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&c.p_full);
          // phase 2, once dP^T is in TMEM: dS^T = P^T (dP^T - D) from the
          // bf16 P^T (the operand dV uses), as bf16 over the dP^T columns
          if (!wait_warp(&c.dp_full, jg & 1, ctrl, seq)) { timeout(ctrl, c, seq, 32); ok = false; break; }
          tc_fence_after();
          uint32_t dv2[2][32];
          tmem_ld32(trow + kTdP, dv2[0]);
#pragma unroll
          for (int cch = 0; cch < 4; ++cch) {
            tmem_wait_ld();
            if (cch < 3) tmem_ld32(trow + kTdP + 32 * (cch + 1), dv2[(cch + 1) & 1]);
            const uint32_t* dv = dv2[cch & 1];
            uint32_t dk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 p = make_float2(__uint_as_float(pk[cch][i] << 16), __uint_as_float(pk[cch][i] & 0xFFFF0000u));
              const float2 dd = *reinterpret_cast<const float2*>(rowL + 128 + 32 * cch + 2 * i);
              const float2 ds = fmul2(p, fsub2(make_float2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])), dd));
              dk[i] = pack_bf16(ds.x, ds.y);
            }
            tmem_st16(trow + kTdP + 16 * cch, dk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&c.ds_full);
      }

      // epilogue: the accumulators of this item, scaled, as bf16 rows
      if (ok && n_tiles > 0 && !wait_warp(&c.acc_done, nfix & 1, ctrl, seq)) { timeout(ctrl, c, seq, 31); ok = false; }
      tc_fence_after();
      const bool store = frow >= 0 && frow < g.Npad;
      const bool real = ok && n_tiles > 0 && frow_ok;
#pragma unroll 1
      for (int a = 0; a < (DKDV ? 2 : 1); ++a) {
        // dq: out0 = dQ (scaled); dkdv: out0 = dV (acc0), out1 = dK (acc1, scaled)
        __nv_bfloat16* dst = (a == 0) ? out0 : out1;
        const float mul = (DKDV && a == 0) ? 1.f : scale;
        const uint32_t tacc = trow + (DKDV ? (a == 0 ? kTAcc0 : kTAcc1) : kTdQ);
        uint4* orow = reinterpret_cast<uint4*>(dst + ((size_t)bh * g.Npad + (store ? frow : 0)) * D);
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 16) {
          uint32_t v[16];
          if (ok && n_tiles > 0) {
            tmem_ld16(tacc + cc, v);
            tmem_wait_ld();
          }
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = real ? pack_bf16(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul) : 0u;
          if (store) {
            orow[cc / 8] = make_uint4(w[0], w[1], w[2], w[3]);
            orow[cc / 8 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
      }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    jbase += n_tiles;
    if (n_tiles > 0) ++nfix;
  }

  // Drain: every copy and MMA this CTA issued completes before TMEM is freed.
  if (lane == 0) {
    if (warp == 0) {
      mbar_drain_ring(&c.fixed_full, 1, nfix, kWaitNs);
      mbar_drain_ring(c.a_full, NA, armed, kWaitNs);
    } else if (warp == 2) {
      mbar_drain_ring(c.b_full, 2, armed, kWaitNs);
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

template <int D, int BS, bool DKDV>
cudaError_t launch_pass(const Dims& g, const void* fix0, const void* fix1, const void* tile0, const void* tile1,
                        const int32_t* l_count, const int32_t* l_idx, const int2* items, int* work,
                        const float* lse, const float* Dv, float scale, void* out0, void* out1, Ctrl* ctrl,
                        uint32_t seq, cudaStream_t st) {
  CUtensorMap m0, m1, m2, m3;
  const uint64_t rows = (uint64_t)g.Npad, bhs = (uint64_t)g.B * g.heads;
  if (!make_map_bf16_3d(&m0, fix0, D, rows, bhs, 64, 64) || !make_map_bf16_3d(&m1, fix1, D, rows, bhs, 64, 64) ||
      !make_map_bf16_3d(&m2, tile0, D, rows, bhs, 64, 64) || !make_map_bf16_3d(&m3, tile1, D, rows, bhs, 64, 64))
    return cudaErrorInvalidValue;
  const int items_per_bh = (BS == 64) ? (g.nb + 1) / 2 : g.nb;
  const int n_items = (int)(bhs * items_per_bh);
  // Q/K and dO/V, the stages of a (three for dq, two for dkdv) and of b, the
  // dkdv L and D rows, the control block
  const size_t smem = (DKDV ? 6u : 7u) * 128u * D * 2u + (DKDV ? 2u * 256u * sizeof(float) : 0u) + sizeof(Ctl);
  static_assert(6u * 128u * 128u * 2u + 2u * 256u * sizeof(float) + sizeof(Ctl) <= 227u * 1024u, "smem layout");
  static_assert(7u * 128u * 128u * 2u + sizeof(Ctl) <= 227u * 1024u, "smem layout");
  cudaError_t e =
      cudaFuncSetAttribute(attn_bwd_kernel<D, BS, DKDV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = n_items < num_sms() ? n_items : num_sms();
  attn_bwd_kernel<D, BS, DKDV><<<grid, kThreads, smem, st>>>(
      m0, m1, m2, m3, l_count, l_idx, items, work, lse, Dv, scale * 1.4426950408889634f, scale,
      (__nv_bfloat16*)out0, (__nv_bfloat16*)out1, ctrl, g, items_per_bh, n_items, seq);
  return cudaGetLastError();
}

template <int D, int BS>
cudaError_t launch_bwd_t(const Dims& g, const BwdArgs& a, cudaStream_t st) {
  cudaError_t e;
  // dq pass: fixed Q, dO; walked K (a), V (b) over the forward lists
  e = launch_pass<D, BS, false>(g, a.q, a.dO, a.k, a.v, a.kv_count, a.kv_idx, a.items_q, a.work_q, a.lse, a.Dv,
                                a.scale, a.dq, nullptr, a.ctrl, a.seq, st);
  if (e != cudaSuccess) return e;
  // dkdv pass: fixed K, V; walked Q (a), dO (b) over the transposed lists
  return launch_pass<D, BS, true>(g, a.k, a.v, a.q, a.dO, a.q_count, a.q_idx, a.items_kv, a.work_kv, a.lse, a.Dv,
                                  a.scale, a.dv, a.dk, a.ctrl, a.seq, st);
}

}  // namespace

cudaError_t launch_bwd_prep(const Dims& g, const void* o, const void* dO, const int32_t* kv_count,
                            const int32_t* kv_idx, float* Dv, uint32_t* bits, int32_t* q_count, int32_t* q_idx,
                            cudaStream_t st) {
  const size_t rows = (size_t)g.B * g.heads * g.Npad;
  const size_t threads = rows * (g.d / 8);
  const unsigned grid_rows = (unsigned)((threads + 255) / 256);
  if (g.d == 128)
    bwd_rowdot_kernel<128><<<grid_rows, 256, 0, st>>>((const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, Dv, g);
  else
    bwd_rowdot_kernel<64><<<grid_rows, 256, 0, st>>>((const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, Dv, g);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t block_rows = (size_t)g.B * g.heads * g.nb;
  const unsigned grid_b = (unsigned)((block_rows + 7) / 8);
  bwd_bits_kernel<<<grid_b, 256, 0, st>>>(kv_count, kv_idx, g, bits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_tlist_kernel<<<grid_b, 256, 0, st>>>(bits, g, q_count, q_idx);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const Dims& g, const BwdArgs& a, cudaStream_t st) {
  if (g.d == 128 && g.bs == 64) return launch_bwd_t<128, 64>(g, a, st);
  if (g.d == 128 && g.bs == 128) return launch_bwd_t<128, 128>(g, a, st);
  if (g.d == 64 && g.bs == 64) return launch_bwd_t<64, 64>(g, a, st);
  return launch_bwd_t<64, 128>(g, a, st);
}

}  // namespace bsa
