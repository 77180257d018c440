// Internal launchers of libbsa (host side).  Argument checking happens in
// bsa_api.cu before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include "common.cuh"

namespace bsa {

// A fresh nonzero launch sequence number (host side, thread safe); kernels
// with bounded waits compare it with Ctrl::abort_seq.
uint32_t next_launch_seq();

// Multiprocessors of the current device (148 when the query fails).
int num_sms();

// 1 when BSA_TEST_FORCE_TIMEOUT=1 is set in the environment: the tcgen05
// attention kernels then take their bounded-wait failure path (tests of the
// device error word).
int force_timeout_requested();

cudaError_t launch_reorder(const Dims& g, const void* x_bnhd, void* y_bhnd, cudaStream_t st);
cudaError_t launch_inverse_reorder(const Dims& g, const void* y_bhnd, void* x_bnhd, cudaStream_t st);
// Q and K reordered in one launch, their block means written on the way:
// `qbar` [B, heads, nb, d], `kbar` transposed [B, heads, d, nb] (double).
cudaError_t launch_reorder_qk_pool(const Dims& g, const void* q_bnhd, const void* k_bnhd, void* q_bhnd,
                                   void* k_bhnd, double* qbar, double* kbar, cudaStream_t st);

// Block means of Q and K (double): `qbar` [B, heads, nb, d], `kbar`
// transposed [B, heads, d, nb].
cudaError_t launch_pool(const Dims& g, const void* q, const void* k, double* qbar, double* kbar, Ctrl* ctrl,
                        uint32_t seq, cudaStream_t st);

// Reduced attention + CDF threshold (+ STA union) -> KV lists: the fp64
// scores go through `scores` ([B, heads, nb, nb] double, mask_scores_bytes).
size_t mask_scores_bytes(const Dims& g);
cudaError_t launch_mask(const Dims& g, const double* qbar, const double* kbar, double* scores, double thr,
                        int sta_t, int sta_h, int sta_w, int32_t* kv_count, int32_t* kv_idx, uint8_t* mask,
                        cudaStream_t st);

// Block-sparse attention on the legacy warp-level mma.sync tensor-core path
// (baseline kernel; any supported shape).
cudaError_t launch_attn_mma(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                            const int32_t* kv_idx, float scale, void* o, float* lse, Ctrl* ctrl, cudaStream_t st);

// Work plan of the tcgen05 attention kernel: one int2 (first block, second
// block or -1) per 128-row tile of every (batch, head), in launch order, at
// the start of a plan region of plan_region_bytes(g) bytes (the rest is the
// matching scratch of 64-token blocks).
size_t plan_region_bytes(const Dims& g);
// Work counter of the persistent attention kernel inside the plan region
// (zeroed by launch_plan).
int* plan_work_counter(const Dims& g, int2* items);
cudaError_t launch_plan(const Dims& g, const int32_t* kv_count, const int32_t* kv_idx, int2* items, cudaStream_t st);

// Block-sparse attention on the tcgen05 tensor cores (TMEM accumulators,
// TMA-staged tiles, P in TMEM): persistent, one CTA per SM, two softmax
// groups on alternating KV tiles, query tiles fetched from the plan's work
// counter.  `lse` and `ent` (the entropy of each row's attention
// distribution, nats) are optional outputs.
cudaError_t launch_attn(const Dims& g, const void* q, const void* k, const void* v, const int32_t* kv_count,
                        const int32_t* kv_idx, const int2* items, int* work, float scale, void* o, float* lse,
                        float* ent, Ctrl* ctrl, uint32_t seq, cudaStream_t st);

// Attention over per-query-block lists of 4-token KV blocks with optional
// inclusion weights (attn_fine.cu); 128-row query blocks (g.bs == 128).
// `work` is a device int the launch zeroes and uses as its work counter.
cudaError_t launch_attn_fine(const Dims& g, const void* q, const void* k, const void* v, const int64_t* sel_offsets,
                             const int32_t* sel_idx, const float* sel_w, int64_t n_sel, float scale, void* o,
                             float* lse, Ctrl* ctrl, int* work, uint32_t seq, cudaStream_t st);

// Hilbert-curve token order (order.cu): order[p] = the token at position p.
// Scratch: the tokens' curve indices, a bitmap over the enclosing cube and
// the prefix counts of its 64-word blocks.
struct HilbertLayout {
  int bits;                        // bits per axis of the cube
  size_t words, blocks;            // bitmap words, 64-word blocks
  size_t keys, bitmap, block_sums, total;   // byte offsets in the scratch, total bytes
};
int hilbert_bits(const Dims& g);
HilbertLayout hilbert_layout(const Dims& g);
cudaError_t launch_hilbert_order(const Dims& g, int32_t* order, void* scratch, cudaStream_t st);

// Reorders with an explicit position -> token table instead of the fractal order.
cudaError_t launch_reorder_perm(const Dims& g, const int32_t* order, const void* x_bnhd, void* y_bhnd,
                                cudaStream_t st);
cudaError_t launch_inverse_reorder_perm(const Dims& g, const int32_t* order, const void* y_bhnd, void* x_bnhd,
                                        cudaStream_t st);
cudaError_t launch_reorder_qk_pool_perm(const Dims& g, const int32_t* order, const void* q_bnhd,
                                        const void* k_bnhd, void* q_bhnd, void* k_bhnd, double* qbar, double* kbar,
                                        cudaStream_t st);

// Sub-block scoring (mask.cu): block importance from the reduced attention
// of `sub`-token sub-blocks, then the CDF selection.  Workspace: control
// block | sub-block means of Q and K | sub-block scores | block importance.
struct SubblockLayout {
  int ns;                                  // sub-blocks holding a valid token
  size_t qbar, kbar, scores, M, total;     // byte offsets, total bytes
};
SubblockLayout subblock_layout(const Dims& g, int sub);
cudaError_t launch_mask_subblock(const Dims& g, int sub, const void* q, const void* k, double thr,
                                 int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, void* workspace, uint32_t seq,
                                 cudaStream_t st);

// Token-radius block masks (radius.cu): dense lists for the warm-up pass, and
// the mask from per-token entropies [B, heads, Npad].
cudaError_t launch_dense_lists(const Dims& g, int32_t* kv_count, int32_t* kv_idx, cudaStream_t st);
cudaError_t launch_radius_mask(const Dims& g, const float* entropy, double tau, double gamma, int vote,
                               int32_t* kv_count, int32_t* kv_idx, uint8_t* mask, cudaStream_t st);

// Backward pass (attn_bwd.cu).  Every pointer is device memory; the planner
// regions (items_q / items_kv with their work counters) are filled by
// launch_plan from the forward lists and from the transposed lists.
struct BwdArgs {
  const void *q, *k, *v, *dO;         // [B, heads, Npad, d] bf16, kernel order
  const float* lse;                   // [B, heads, Npad] natural-log LSE of the forward pass
  const float* Dv;                    // [B, heads, Npad] rowsum(dO * O) (launch_bwd_prep)
  const int32_t *kv_count, *kv_idx;   // forward lists
  const int32_t *q_count, *q_idx;     // transposed lists (launch_bwd_prep)
  const int2 *items_q, *items_kv;     // planner tiles of query blocks / of KV blocks
  int *work_q, *work_kv;              // their work counters
  float scale;
  void *dq, *dk, *dv;                 // [B, heads, Npad, d] bf16 outputs
  Ctrl* ctrl;
  uint32_t seq;
};
// D = rowsum(dO * O), the bit matrix of the forward lists (`bits`,
// [B, heads, nb, ceil(nb / 32)] uint32) and the transposed lists.
cudaError_t launch_bwd_prep(const Dims& g, const void* o, const void* dO, const int32_t* kv_count,
                            const int32_t* kv_idx, float* Dv, uint32_t* bits, int32_t* q_count, int32_t* q_idx,
                            cudaStream_t st);
cudaError_t launch_attn_bwd(const Dims& g, const BwdArgs& a, cudaStream_t st);

}  // namespace bsa
