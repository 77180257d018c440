// C ABI of libbsa (declared in include/bsa.h): argument checking, workspace
// layout and kernel launches.  No entry point allocates, frees or
// synchronises, except bsa_check_device_status.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using bsa::Ctrl;
using bsa::Dims;

namespace bsa {

uint32_t next_launch_seq() {
  static std::atomic<uint32_t> counter{0};
  uint32_t s;
  do {
    s = counter.fetch_add(1, std::memory_order_relaxed) + 1u;
  } while (s == 0u);
  return s;
}

}  // namespace bsa

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bsa_status check_shape(const bsa_shape* s, Dims* out) {
  if (s == nullptr) return BSA_ERR_INVALID_ARG;
  if (s->B < 1 || s->T < 1 || s->H < 1 || s->W < 1 || s->heads < 1 || s->patch < 1) return BSA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return BSA_ERR_INVALID_ARG;
  if (s->block != 64 && s->block != 128) return BSA_ERR_INVALID_ARG;
  const int64_t N = (int64_t)s->T * s->H * s->W;
  if (N > (int64_t)1 << 30) return BSA_ERR_UNSUPPORTED;
  const int64_t Npad = (N + s->block - 1) / s->block * s->block;
  const int64_t elems = (int64_t)s->B * s->heads * Npad * s->d;
  if (elems > ((int64_t)1 << 40)) return BSA_ERR_UNSUPPORTED;
  if ((int64_t)s->B * s->heads > 65535 * 64 || s->heads > 65535 || s->B > 65535) return BSA_ERR_UNSUPPORTED;
  if (out != nullptr) {
    out->B = s->B;
    out->T = s->T;
    out->H = s->H;
    out->W = s->W;
    out->heads = s->heads;
    out->d = s->d;
    out->bs = s->block;
    out->P = s->patch;
    out->N = (int)N;
    out->Npad = (int)Npad;
    out->nb = (int)(Npad / s->block);
  }
  return BSA_OK;
}

size_t pooled_bytes(const Dims& g) { return (size_t)g.B * g.heads * g.nb * g.d * sizeof(double); }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace: control block | qbar | kbar | reduced scores | attention plan region.
size_t scores_offset(const Dims& g) { return sizeof(Ctrl) + align256(2 * pooled_bytes(g)); }
size_t plan_offset(const Dims& g) { return scores_offset(g) + align256(bsa::mask_scores_bytes(g)); }

size_t workspace_bytes(const Dims& g) { return plan_offset(g) + align256(bsa::plan_region_bytes(g)); }

bsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

// Hilbert order: cubes up to side 2^9 (bitmap of 2^27 bits, 16 MiB).
constexpr int kMaxHilbertBits = 9;

// Sub-block size: 16 or 32 tokens, dividing the block, or the block itself.
bool subblock_ok(const Dims& g, int sub) {
  return (sub == 16 || sub == 32 || sub == g.bs) && sub <= g.bs && g.bs % sub == 0;
}

}  // namespace

extern "C" {

bsa_status bsa_validate_shape(const bsa_shape* s) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

int64_t bsa_seq_len(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? g.N : -1;
}

int64_t bsa_padded_len(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? g.Npad : -1;
}

int64_t bsa_num_blocks(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? g.nb : -1;
}

size_t bsa_workspace_bytes(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? workspace_bytes(g) : 0;
}

int64_t bsa_plan_items_offset(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? (int64_t)plan_offset(g) : -1;
}

bsa_status bsa_workspace_init(void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (workspace == nullptr || !aligned16(workspace) || ws_bytes < sizeof(Ctrl)) return BSA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(workspace, 0, sizeof(Ctrl), (cudaStream_t)stream));
}

bsa_status bsa_reorder(const bsa_shape* s, const void* x_bnhd, void* y_bhnd, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (x_bnhd == nullptr || y_bhnd == nullptr || !aligned16(x_bnhd) || !aligned16(y_bhnd) || x_bnhd == y_bhnd)
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_reorder(g, x_bnhd, y_bhnd, (cudaStream_t)stream));
}

bsa_status bsa_inverse_reorder(const bsa_shape* s, const void* y_bhnd, void* x_bnhd, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (x_bnhd == nullptr || y_bhnd == nullptr || !aligned16(x_bnhd) || !aligned16(y_bhnd) || x_bnhd == y_bhnd)
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_inverse_reorder(g, y_bhnd, x_bnhd, (cudaStream_t)stream));
}

bsa_status bsa_reorder_qk_pooled(const bsa_shape* s, const void* q_bnhd, const void* k_bnhd, void* q_bhnd,
                                 void* k_bhnd, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  const void* ptrs[5] = {q_bnhd, k_bnhd, q_bhnd, k_bhnd, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return BSA_ERR_INVALID_ARG;
  if (q_bnhd == q_bhnd || k_bnhd == k_bhnd || q_bhnd == k_bhnd) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(g)) return BSA_ERR_INVALID_ARG;
  double* qbar = (double*)((char*)workspace + sizeof(Ctrl));
  double* kbar = qbar + pooled_bytes(g) / sizeof(double);
  return from_cuda(bsa::launch_reorder_qk_pool(g, q_bnhd, k_bnhd, q_bhnd, k_bhnd, qbar, kbar, (cudaStream_t)stream));
}

bsa_status bsa_build_block_mask_pooled(const bsa_shape* s, float thr, int32_t sta_t, int32_t sta_h, int32_t sta_w,
                                       int32_t* kv_count, int32_t* kv_idx, uint8_t* mask_or_null, void* workspace,
                                       size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  if (!(thr >= 0.0f && thr < 1.0f)) return BSA_ERR_INVALID_ARG;
  if (kv_count == nullptr || kv_idx == nullptr || workspace == nullptr) return BSA_ERR_INVALID_ARG;
  if (!aligned16(kv_count) || !aligned16(kv_idx) || !aligned16(workspace)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(g)) return BSA_ERR_INVALID_ARG;
  const bool sta = sta_t >= 0 && sta_h >= 0 && sta_w >= 0;
  double* qbar = (double*)((char*)workspace + sizeof(Ctrl));
  double* kbar = qbar + pooled_bytes(g) / sizeof(double);
  double* scores = (double*)((char*)workspace + scores_offset(g));
  return from_cuda(bsa::launch_mask(g, qbar, kbar, scores, (double)thr, sta ? sta_t : -1, sta ? sta_h : -1,
                                    sta ? sta_w : -1, kv_count, kv_idx, mask_or_null, (cudaStream_t)stream));
}

bsa_status bsa_build_block_mask(const bsa_shape* s, const void* q_bhnd, const void* k_bhnd, float thr,
                                int32_t sta_t, int32_t sta_h, int32_t sta_w, int32_t* kv_count, int32_t* kv_idx,
                                uint8_t* mask_or_null, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  if (!(thr >= 0.0f && thr < 1.0f)) return BSA_ERR_INVALID_ARG;
  if (q_bhnd == nullptr || k_bhnd == nullptr || kv_count == nullptr || kv_idx == nullptr || workspace == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q_bhnd) || !aligned16(k_bhnd) || !aligned16(kv_count) || !aligned16(kv_idx) ||
      !aligned16(workspace))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(g)) return BSA_ERR_INVALID_ARG;
  const bool sta = sta_t >= 0 && sta_h >= 0 && sta_w >= 0;
  double* qbar = (double*)((char*)workspace + sizeof(Ctrl));
  double* kbar = qbar + pooled_bytes(g) / sizeof(double);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = bsa::launch_pool(g, q_bhnd, k_bhnd, qbar, kbar, (Ctrl*)workspace, bsa::next_launch_seq(), cs);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  double* scores = (double*)((char*)workspace + scores_offset(g));
  e = bsa::launch_mask(g, qbar, kbar, scores, (double)thr, sta ? sta_t : -1, sta ? sta_h : -1, sta ? sta_w : -1,
                       kv_count, kv_idx, mask_or_null, cs);
  return from_cuda(e);
}

}  // extern "C"

namespace {

bsa_status attn_common(const bsa_shape* s, const void* q, const void* k, const void* v, const int32_t* kv_count,
                       const int32_t* kv_idx, float scale, void* o, float* lse_or_null, float* ent_or_null,
                       void* workspace, size_t ws_bytes, bsa_stream_t stream, bool baseline) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || kv_count == nullptr || kv_idx == nullptr ||
      workspace == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(kv_count) ||
      !aligned16(kv_idx) || !aligned16(workspace) || (lse_or_null != nullptr && !aligned16(lse_or_null)) ||
      (ent_or_null != nullptr && !aligned16(ent_or_null)))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(g)) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return BSA_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = (float)(1.0 / std::sqrt((double)g.d));
  Ctrl* ctrl = (Ctrl*)workspace;
  if (baseline)
    return from_cuda(bsa::launch_attn_mma(g, q, k, v, kv_count, kv_idx, scale, o, lse_or_null, ctrl,
                                          (cudaStream_t)stream));
  int2* items = (int2*)((char*)workspace + plan_offset(g));
  cudaError_t e = bsa::launch_plan(g, kv_count, kv_idx, items, (cudaStream_t)stream);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  return from_cuda(bsa::launch_attn(g, q, k, v, kv_count, kv_idx, items, bsa::plan_work_counter(g, items), scale, o,
                                   lse_or_null, ent_or_null, ctrl, bsa::next_launch_seq(), (cudaStream_t)stream));
}

}  // namespace

extern "C" {

bsa_status bsa_attn_fwd(const bsa_shape* s, const void* q, const void* k, const void* v, const int32_t* kv_count,
                        const int32_t* kv_idx, float scale, void* o, float* lse_or_null, void* workspace,
                        size_t ws_bytes, bsa_stream_t stream) {
  return attn_common(s, q, k, v, kv_count, kv_idx, scale, o, lse_or_null, nullptr, workspace, ws_bytes, stream,
                     false);
}

bsa_status bsa_attn_fwd_entropy(const bsa_shape* s, const void* q, const void* k, const void* v,
                                const int32_t* kv_count, const int32_t* kv_idx, float scale, void* o, float* lse,
                                float* entropy, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  if (lse == nullptr || entropy == nullptr) return BSA_ERR_INVALID_ARG;
  return attn_common(s, q, k, v, kv_count, kv_idx, scale, o, lse, entropy, workspace, ws_bytes, stream, false);
}

bsa_status bsa_dense_lists(const bsa_shape* s, int32_t* kv_count, int32_t* kv_idx, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  if (kv_count == nullptr || kv_idx == nullptr || !aligned16(kv_count) || !aligned16(kv_idx))
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_dense_lists(g, kv_count, kv_idx, (cudaStream_t)stream));
}

bsa_status bsa_attn_fwd_baseline(const bsa_shape* s, const void* q, const void* k, const void* v,
                                 const int32_t* kv_count, const int32_t* kv_idx, float scale, void* o,
                                 float* lse_or_null, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  return attn_common(s, q, k, v, kv_count, kv_idx, scale, o, lse_or_null, nullptr, workspace, ws_bytes, stream,
                     true);
}

}  // extern "C"

namespace {

// Backward workspace: control block | D | bit matrix | transposed counts |
// transposed lists | planner region of the query tiles | of the KV tiles.
struct BwdLayout {
  size_t Dv, bits, q_count, q_idx, plan_q, plan_kv, total;
};

BwdLayout bwd_layout(const Dims& g) {
  const size_t bh = (size_t)g.B * g.heads;
  const size_t nw = (size_t)(g.nb + 31) / 32;
  BwdLayout L;
  L.Dv = sizeof(Ctrl);
  L.bits = L.Dv + align256(bh * g.Npad * sizeof(float));
  L.q_count = L.bits + align256(bh * g.nb * nw * sizeof(uint32_t));
  L.q_idx = L.q_count + align256(bh * g.nb * sizeof(int32_t));
  L.plan_q = L.q_idx + align256(bh * g.nb * g.nb * sizeof(int32_t));
  L.plan_kv = L.plan_q + align256(bsa::plan_region_bytes(g));
  L.total = L.plan_kv + align256(bsa::plan_region_bytes(g));
  return L;
}

}  // namespace

extern "C" {

size_t bsa_attn_bwd_workspace_bytes(const bsa_shape* s) {
  Dims g;
  return check_shape(s, &g) == BSA_OK ? bwd_layout(g).total : 0;
}

bsa_status bsa_attn_bwd(const bsa_shape* s, const void* q, const void* k, const void* v, const void* o,
                        const void* dO, const float* lse, const int32_t* kv_count, const int32_t* kv_idx, float scale,
                        void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  const void* ptrs[13] = {q, k, v, o, dO, lse, kv_count, kv_idx, dq, dk, dv, workspace, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return BSA_ERR_INVALID_ARG;
  if (dq == dk || dq == dv || dk == dv) return BSA_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(g);
  if (ws_bytes < L.total) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return BSA_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = (float)(1.0 / std::sqrt((double)g.d));
  char* ws = (char*)workspace;
  cudaStream_t cs = (cudaStream_t)stream;
  bsa::BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dO = dO;
  a.lse = lse;
  a.Dv = (const float*)(ws + L.Dv);
  a.kv_count = kv_count;
  a.kv_idx = kv_idx;
  a.q_count = (const int32_t*)(ws + L.q_count);
  a.q_idx = (const int32_t*)(ws + L.q_idx);
  int2* items_q = (int2*)(ws + L.plan_q);
  int2* items_kv = (int2*)(ws + L.plan_kv);
  a.items_q = items_q;
  a.items_kv = items_kv;
  a.work_q = bsa::plan_work_counter(g, items_q);
  a.work_kv = bsa::plan_work_counter(g, items_kv);
  a.scale = scale;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.ctrl = (Ctrl*)workspace;
  a.seq = bsa::next_launch_seq();
  cudaError_t e = bsa::launch_bwd_prep(g, o, dO, kv_count, kv_idx, (float*)(ws + L.Dv), (uint32_t*)(ws + L.bits),
                                       (int32_t*)(ws + L.q_count), (int32_t*)(ws + L.q_idx), cs);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  if (bsa::launch_plan(g, kv_count, kv_idx, items_q, cs) != cudaSuccess) return BSA_ERR_CUDA;
  if (bsa::launch_plan(g, a.q_count, a.q_idx, items_kv, cs) != cudaSuccess) return BSA_ERR_CUDA;
  return from_cuda(bsa::launch_attn_bwd(g, a, cs));
}

bsa_status bsa_build_block_mask_radius(const bsa_shape* s, const float* entropy, float tau, float gamma,
                                       int32_t vote, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask_or_null,
                                       bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS || g.T > 1024) return BSA_ERR_UNSUPPORTED;
  if (!(tau > 0.0f) || !std::isfinite(tau) || !(gamma >= 0.0f) || !std::isfinite(gamma) || vote < 1)
    return BSA_ERR_INVALID_ARG;
  if (entropy == nullptr || kv_count == nullptr || kv_idx == nullptr || !aligned16(entropy) || !aligned16(kv_count) ||
      !aligned16(kv_idx))
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_radius_mask(g, entropy, (double)tau, (double)gamma, vote, kv_count, kv_idx,
                                           mask_or_null, (cudaStream_t)stream));
}

size_t bsa_hilbert_workspace_bytes(const bsa_shape* s) {
  Dims g;
  if (check_shape(s, &g) != BSA_OK || bsa::hilbert_bits(g) > kMaxHilbertBits) return 0;
  return bsa::hilbert_layout(g).total;
}

bsa_status bsa_hilbert_order(const bsa_shape* s, int32_t* order, void* workspace, size_t ws_bytes,
                             bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (bsa::hilbert_bits(g) > kMaxHilbertBits) return BSA_ERR_UNSUPPORTED;
  if (order == nullptr || workspace == nullptr || !aligned16(order) || !aligned16(workspace))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa::hilbert_layout(g).total) return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_hilbert_order(g, order, workspace, (cudaStream_t)stream));
}

bsa_status bsa_reorder_perm(const bsa_shape* s, const int32_t* order, const void* x_bnhd, void* y_bhnd,
                            bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (order == nullptr || x_bnhd == nullptr || y_bhnd == nullptr || !aligned16(x_bnhd) || !aligned16(y_bhnd) ||
      x_bnhd == y_bhnd)
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_reorder_perm(g, order, x_bnhd, y_bhnd, (cudaStream_t)stream));
}

bsa_status bsa_inverse_reorder_perm(const bsa_shape* s, const int32_t* order, const void* y_bhnd, void* x_bnhd,
                                    bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (order == nullptr || x_bnhd == nullptr || y_bhnd == nullptr || !aligned16(x_bnhd) || !aligned16(y_bhnd) ||
      x_bnhd == y_bhnd)
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_inverse_reorder_perm(g, order, y_bhnd, x_bnhd, (cudaStream_t)stream));
}

bsa_status bsa_reorder_qk_pooled_perm(const bsa_shape* s, const int32_t* order, const void* q_bnhd,
                                      const void* k_bnhd, void* q_bhnd, void* k_bhnd, void* workspace,
                                      size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (order == nullptr) return BSA_ERR_INVALID_ARG;
  const void* ptrs[5] = {q_bnhd, k_bnhd, q_bhnd, k_bhnd, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return BSA_ERR_INVALID_ARG;
  if (q_bnhd == q_bhnd || k_bnhd == k_bhnd || q_bhnd == k_bhnd) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(g)) return BSA_ERR_INVALID_ARG;
  double* qbar = (double*)((char*)workspace + sizeof(Ctrl));
  double* kbar = qbar + pooled_bytes(g) / sizeof(double);
  return from_cuda(bsa::launch_reorder_qk_pool_perm(g, order, q_bnhd, k_bnhd, q_bhnd, k_bhnd, qbar, kbar,
                                                    (cudaStream_t)stream));
}

size_t bsa_subblock_workspace_bytes(const bsa_shape* s, int32_t sub) {
  Dims g;
  if (check_shape(s, &g) != BSA_OK || !subblock_ok(g, sub)) return 0;
  return bsa::subblock_layout(g, sub).total;
}

bsa_status bsa_build_block_mask_subblock(const bsa_shape* s, const void* q_bhnd, const void* k_bhnd, int32_t sub,
                                         float thr, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask_or_null,
                                         void* workspace, size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.nb > BSA_MAX_BLOCKS) return BSA_ERR_UNSUPPORTED;
  if (!subblock_ok(g, sub)) return BSA_ERR_INVALID_ARG;
  if (!(thr >= 0.0f && thr < 1.0f)) return BSA_ERR_INVALID_ARG;
  if (q_bhnd == nullptr || k_bhnd == nullptr || kv_count == nullptr || kv_idx == nullptr || workspace == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q_bhnd) || !aligned16(k_bhnd) || !aligned16(kv_count) || !aligned16(kv_idx) ||
      !aligned16(workspace))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa::subblock_layout(g, sub).total) return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_mask_subblock(g, sub, q_bhnd, k_bhnd, (double)thr, kv_count, kv_idx, mask_or_null,
                                             workspace, bsa::next_launch_seq(), (cudaStream_t)stream));
}

size_t bsa_attn_fine_workspace_bytes(const bsa_shape* s) {
  Dims g;
  if (check_shape(s, &g) != BSA_OK || g.bs != 128) return 0;
  return sizeof(Ctrl) + 256;
}

bsa_status bsa_attn_fwd_fine(const bsa_shape* s, const void* q, const void* k, const void* v,
                             const int64_t* sel_offsets, const int32_t* sel_idx, const float* sel_w_or_null,
                             int64_t n_sel, float scale, void* o, float* lse_or_null, void* workspace,
                             size_t ws_bytes, bsa_stream_t stream) {
  Dims g;
  bsa_status st = check_shape(s, &g);
  if (st != BSA_OK) return st;
  if (g.bs != 128) return BSA_ERR_UNSUPPORTED;
  const void* ptrs[6] = {q, k, v, o, sel_offsets, workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return BSA_ERR_INVALID_ARG;
  if (n_sel < 0 || (n_sel > 0 && sel_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  if ((sel_idx != nullptr && ((uintptr_t)sel_idx & 3u)) || (sel_w_or_null != nullptr && ((uintptr_t)sel_w_or_null & 3u)))
    return BSA_ERR_INVALID_ARG;
  if (lse_or_null != nullptr && !aligned16(lse_or_null)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < sizeof(Ctrl) + 256) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return BSA_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = (float)(1.0 / std::sqrt((double)g.d));
  int* work = (int*)((char*)workspace + sizeof(Ctrl));
  return from_cuda(bsa::launch_attn_fine(g, q, k, v, sel_offsets, sel_idx, sel_w_or_null, n_sel, scale, o,
                                         lse_or_null, (Ctrl*)workspace, work, bsa::next_launch_seq(),
                                         (cudaStream_t)stream));
}

bsa_status bsa_check_device_status(void* workspace, bsa_stream_t stream) {
  if (workspace == nullptr || !aligned16(workspace)) return BSA_ERR_INVALID_ARG;
  cudaStream_t cs = (cudaStream_t)stream;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return BSA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return BSA_ERR_CUDA;
  if (word != 0u) {
    if (cudaMemset(workspace, 0, sizeof(Ctrl)) != cudaSuccess) return BSA_ERR_CUDA;
  }
  if (word & bsa::kErrLayout) return BSA_ERR_CUDA;
  if (word & bsa::kErrTimeout) return BSA_ERR_TIMEOUT;
  if (word & (bsa::kErrIndex | bsa::kErrCount | bsa::kErrWeight)) return BSA_ERR_DEVICE_INDEX;
  return BSA_OK;
}

const char* bsa_status_string(bsa_status st) {
  switch (st) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_DEVICE_INDEX: return "BSA_ERR_DEVICE_INDEX";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
  }
  return "BSA_ERR_UNKNOWN";
}

}  // extern "C"
