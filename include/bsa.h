/*
 * bsa.h -- C ABI of the B200 block-sparse video attention library (libbsa.so).
 *
 * The library implements NABLA-style content-adaptive block-sparse
 * self-attention as described in the NABLA technical summary
 * ("NABLA - Atencion de Bloque Adaptativa al Vecindario para la Generacion
 * Eficiente de Video", gist.science/es/paper/2507.13546), section
 * "Metodologia":
 *   1. fractal P x P token reorder           -> bsa_reorder / bsa_inverse_reorder
 *   2. block mean-pooling of Q and K,
 *      reduced attention map, per-row CDF
 *      threshold (optionally united with a
 *      static sliding-tile window, item 3)  -> bsa_build_block_mask
 *   3. attention restricted to the kept
 *      N x N tiles ("Expansion")             -> bsa_attn_fwd
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Device pointers refer to memory of the current CUDA device; every call is
 *    asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream)
 *    and never synchronises, except bsa_check_device_status.
 *  - The caller owns every buffer.  The library never allocates or frees
 *    memory.  Buffers must be contiguous and 16-byte aligned.
 *  - Tensors are bf16 (IEEE-754 binary16 "brain float", __nv_bfloat16).
 *  - Layouts:  model order  [B, N, heads, d]     (token n = t*H*W + h*W + w)
 *              kernel order [B, heads, Npad, d]  (fractal order, zero tail)
 *    with N = T*H*W, Npad = ceil(N / block) * block, nb = Npad / block.
 *  - Argument errors are reported synchronously by the return value and
 *    launch nothing.  Errors found on the device (an out-of-range KV index or
 *    count, a bounded wait that expired) never trap: they set bits of an error
 *    word held in the workspace, which bsa_check_device_status reports
 *    (BSA_ERR_CUDA for a shared-memory layout the device did not honour).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* bsa_stream_t;

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,   /* bad shape, pointer, alignment, threshold or workspace size   */
  BSA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement (e.g. nb > max) */
  BSA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed                   */
  BSA_ERR_DEVICE_INDEX = 4,  /* device saw an invalid list: index, count, offsets or weight   */
  BSA_ERR_TIMEOUT = 5        /* a bounded device-side wait expired                           */
} bsa_status;

/* Problem shape.  d in {64, 128}; block in {64, 128}; patch >= 1. */
typedef struct bsa_shape {
  int32_t B;      /* batch                                  */
  int32_t T;      /* latent frames                          */
  int32_t H;      /* latent height                          */
  int32_t W;      /* latent width                           */
  int32_t heads;  /* attention heads                        */
  int32_t d;      /* head dimension                         */
  int32_t block;  /* block size (tokens per mask block)     */
  int32_t patch;  /* P of the fractal P x P reorder         */
} bsa_shape;

/* Largest nb (= Npad / block) that bsa_build_block_mask and bsa_attn_fwd accept. */
#define BSA_MAX_BLOCKS 1024

/* BSA_OK when the shape is one the kernels implement, else the reason. */
BSA_API bsa_status bsa_validate_shape(const bsa_shape* s);

/* N = T*H*W, Npad and nb of a shape (-1 for a NULL or invalid shape). */
BSA_API int64_t bsa_seq_len(const bsa_shape* s);
BSA_API int64_t bsa_padded_len(const bsa_shape* s);
BSA_API int64_t bsa_num_blocks(const bsa_shape* s);

/* Bytes of device workspace that bsa_build_block_mask and bsa_attn_fwd need
 * for this shape: a control block (device error word), the pooled block means
 * of Q and K (2 * B*heads*nb*d doubles), the reduced scores (B*heads*nb*nb
 * doubles) and the attention work plan (one int2 per 128-row query tile; with
 * 64-token blocks also 64 bytes of pairing weights and 4 bytes of counts per
 * block row; a work counter), each part rounded up to 256 bytes.  0 for an
 * invalid shape. */
BSA_API size_t bsa_workspace_bytes(const bsa_shape* s);

/* Byte offset, inside the workspace, of the work plan that bsa_attn_fwd
 * writes on every call (-1 for an invalid shape): one int2 per 128-row query
 * tile of every (batch, head), [B * heads][ceil(nb * block / 128)], in
 * launch order: the tile's first query block and its second (-1 when the tile
 * holds one block; blocks of 128 always hold one).  Read-only diagnostics
 * (e.g. the KV tiles a call runs: the union of each tile's lists). */
BSA_API int64_t bsa_plan_items_offset(const bsa_shape* s);

/* Clears the control block of a freshly allocated workspace (async memset).
 * Call once after allocation; bsa_check_device_status clears it again. */
BSA_API bsa_status bsa_workspace_init(void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* Fractal reorder plus layout change, NABLA summary, Metodologia 1
 * ("Reordenamiento de Tokens"): y[b, h, p, :] = x[b, pi(p), h, :] for p < N and
 * 0 for N <= p < Npad, where pi lists, frame by frame, the P x P spatial patches
 * in row-major order and the tokens of each patch in row-major order (edge
 * patches clipped to H and W).  Bit-exact data movement.
 *   x_bnhd: device, [B, N, heads, d] bf16, read only.
 *   y_bhnd: device, [B, heads, Npad, d] bf16, written; must not overlap x. */
BSA_API bsa_status bsa_reorder(const bsa_shape* s, const void* x_bnhd, void* y_bhnd, bsa_stream_t stream);

/* Inverse of bsa_reorder (the output returns to the model's token order):
 * x[b, pi(p), h, :] = y[b, h, p, :] for p < N; the padded tail is dropped.
 *   y_bhnd: device, [B, heads, Npad, d] bf16, read only.
 *   x_bnhd: device, [B, N, heads, d] bf16, written; must not overlap y. */
BSA_API bsa_status bsa_inverse_reorder(const bsa_shape* s, const void* y_bhnd, void* x_bnhd, bsa_stream_t stream);

/* Adaptive block mask, NABLA summary, Metodologia 2 (pooling, reduced
 * attention, CDF thresholding, expansion) and 3 (union with STA).
 *   q_bhnd, k_bhnd: device, [B, heads, Npad, d] bf16 in kernel order (output of
 *       bsa_reorder; the padded tail is ignored).
 *   thr: in [0, 1).  Per row I of softmax(qbar kbar^T / sqrt(d)) over blocks,
 *       the blocks taken in decreasing probability (ties: lower index first)
 *       up to and including the first whose cumulative mass reaches 1 - thr
 *       are kept; thr == 0 keeps every block.  Means, dot products and masses
 *       are computed in double precision.
 *   sta_t, sta_h, sta_w: half-widths of the static 3D window in block-tile
 *       units; block I sits at the tile (t, h / P, w / P) of its first token in
 *       fractal order.  Any negative value disables the union.
 *   kv_count: device, [B, heads, nb] int32, written: kept blocks per row.
 *   kv_idx:   device, [B, heads, nb, nb] int32, written: row (b, h, I) holds its
 *       kept block indices in ascending order in its first kv_count entries;
 *       later entries are left untouched.
 *   mask_or_null: device, [B, heads, nb, nb] uint8 (1 = kept) or NULL.
 *   workspace / ws_bytes: at least bsa_workspace_bytes(s), initialised once by
 *       bsa_workspace_init; the pooled means are scratch. */
BSA_API bsa_status bsa_build_block_mask(const bsa_shape* s, const void* q_bhnd, const void* k_bhnd, float thr,
                                int32_t sta_t, int32_t sta_h, int32_t sta_w,
                                int32_t* kv_count, int32_t* kv_idx, uint8_t* mask_or_null,
                                void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* Reorder of Q and K (as bsa_reorder, one launch for both) fused with the
 * first step of the adaptive mask, NABLA summary, Metodologia 2
 * "Submuestreo": on the way, the mean of the valid tokens of every block of Q
 * and of K is computed in double and kept in the workspace, where
 * bsa_build_block_mask_pooled reads it.  Q and K are then read from HBM once
 * for both the reorder and the pooling.
 *   q_bnhd, k_bnhd: device, [B, N, heads, d] bf16 model order, read only.
 *   q_bhnd, k_bhnd: device, [B, heads, Npad, d] bf16 kernel order, written
 *       (zero tail); neither may overlap an input or the other output.
 *   workspace / ws_bytes: at least bsa_workspace_bytes(s); its pooled-mean
 *       region is overwritten. */
BSA_API bsa_status bsa_reorder_qk_pooled(const bsa_shape* s, const void* q_bnhd, const void* k_bnhd, void* q_bhnd,
                                         void* k_bhnd, void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* bsa_build_block_mask from the block means that bsa_reorder_qk_pooled left
 * in `workspace` (same rule, arguments and outputs otherwise): the reduced
 * attention, the CDF threshold and the optional STA union, NABLA summary,
 * Metodologia 2 ("Atencion Reducida", "Umbralizacion CDF", "Expansion") and 3.
 * Must follow bsa_reorder_qk_pooled of the same shape on the same workspace
 * (stream order). */
BSA_API bsa_status bsa_build_block_mask_pooled(const bsa_shape* s, float thr, int32_t sta_t, int32_t sta_h,
                                               int32_t sta_w, int32_t* kv_count, int32_t* kv_idx,
                                               uint8_t* mask_or_null, void* workspace, size_t ws_bytes,
                                               bsa_stream_t stream);

/* Block-sparse attention forward, NABLA summary, Metodologia 2 "Expansion":
 * for every valid query row q of block I,
 *   O[q] = sum_k softmax_k(scale * Q[q] . K[k]) V[k],
 * with k over the valid keys (k < N) of the blocks listed for I.  fp32
 * accumulation and softmax, bf16 output (round to nearest even).  Any valid
 * lists are accepted (e.g. an externally computed mask).
 *   q, k, v: device, [B, heads, Npad, d] bf16 in kernel order.
 *   kv_count, kv_idx: as written by bsa_build_block_mask.  Indices outside
 *       [0, nb) are skipped and counts outside [1, nb] clamped; both set the
 *       device error word (BSA_ERR_DEVICE_INDEX).
 *   scale: softmax scale, >= 0; 0 selects 1/sqrt(d).
 *   o: device, [B, heads, Npad, d] bf16, written (padded rows are 0).
 *   lse_or_null: device, [B, heads, Npad] float32 natural-log sum-exp of the
 *       scaled scores per row (0 for padded rows), or NULL.
 *   workspace / ws_bytes: as for bsa_build_block_mask. */
BSA_API bsa_status bsa_attn_fwd(const bsa_shape* s, const void* q, const void* k, const void* v,
                        const int32_t* kv_count, const int32_t* kv_idx, float scale,
                        void* o, float* lse_or_null,
                        void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Token-radius masks (TRA summary, gist.science/es/paper/2608.02504, section
 * 2): entropy -> budget -> radius -> block mask, in the same list format.
 * ------------------------------------------------------------------------- */

/* bsa_attn_fwd that also writes, for every valid query row, the entropy (in
 * nats) of its attention distribution over the listed keys,
 * H = -sum_k p_k ln p_k, and its LSE (both required).  TRA summary, section 2
 * ("Entropia-a-Presupuesto"): the dense warm-up pass that measures each
 * query's entropy (with dense lists, see bsa_dense_lists).
 *   lse, entropy: device, [B, heads, Npad] float32, written (0 for padded rows).
 *   Other arguments and errors as for bsa_attn_fwd. */
BSA_API bsa_status bsa_attn_fwd_entropy(const bsa_shape* s, const void* q, const void* k, const void* v,
                                        const int32_t* kv_count, const int32_t* kv_idx, float scale, void* o,
                                        float* lse, float* entropy, void* workspace, size_t ws_bytes,
                                        bsa_stream_t stream);

/* Lists that keep every block (kv_count = nb, kv_idx[b, h, I, J] = J): the
 * dense attention of a warm-up pass. */
BSA_API bsa_status bsa_dense_lists(const bsa_shape* s, int32_t* kv_count, int32_t* kv_idx, bsa_stream_t stream);

/* Block mask from token radii, TRA summary, section 2 ("Presupuesto-a-Radio",
 * "Ejecucion Eficiente").  Per valid query token i at (t_i, h_i, w_i), with
 * phi(d) = exp(-gamma d):
 *   budget_i = clamp(tau * exp(entropy_i), 1, N) keys;
 *   r_i = sqrt(budget_i / (pi * sum_t phi(|t - t_i|)^2)) (the disks of radius
 *         r_i phi(|t - t_i|) in every frame hold the budget in area);
 *   key j is in i's support when (h_j-h_i)^2 + (w_j-w_i)^2 <= (r_i phi(|t_j-t_i|))^2;
 * query token i votes for key block J when J holds a key of its support, and
 * block I keeps J when at least `vote` of I's valid tokens vote for J.  Tokens
 * are in the fractal order (the tile-major layout the summary asks for).
 * Radii and comparisons in double precision.
 *   entropy: device, [B, heads, Npad] float32 (bsa_attn_fwd_entropy).
 *   tau > 0, gamma >= 0, vote >= 1; T <= 1024.
 *   kv_count, kv_idx, mask_or_null: as written by bsa_build_block_mask. */
BSA_API bsa_status bsa_build_block_mask_radius(const bsa_shape* s, const float* entropy, float tau, float gamma,
                                               int32_t vote, int32_t* kv_count, int32_t* kv_idx,
                                               uint8_t* mask_or_null, bsa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Alternative token order and block estimator (DFSAttn explainer,
 * gist.science/es/paper/2605.23445, sections 1 and 2): a 3-D Hilbert-curve
 * order of the tokens, and block importance from finer sub-block scores,
 * feeding the same CDF threshold.
 * ------------------------------------------------------------------------- */

/* Scratch bytes of bsa_hilbert_order (0 for an invalid shape or a grid whose
 * largest side exceeds 512). */
BSA_API size_t bsa_hilbert_workspace_bytes(const bsa_shape* s);

/* The 3-D Hilbert-curve order of the T x H x W tokens, DFSAttn explainer,
 * section 1 ("El barajado de la Curva de Hilbert"): order[p] = the token
 * n = t*H*W + h*W + w at position p, for p < N.  The curve is J. Skilling's
 * construction ("Programming the Hilbert curve", 2004) over the smallest
 * power-of-two cube holding the grid, axes (t, h, w); grid points keep the
 * cube's order, points outside the grid are skipped.
 *   order: device, [N] int32, written.
 *   workspace / ws_bytes: scratch of at least bsa_hilbert_workspace_bytes(s). */
BSA_API bsa_status bsa_hilbert_order(const bsa_shape* s, int32_t* order, void* workspace, size_t ws_bytes,
                                     bsa_stream_t stream);

/* bsa_reorder, bsa_inverse_reorder and bsa_reorder_qk_pooled with the token
 * order given as a table (e.g. from bsa_hilbert_order) instead of the fractal
 * order: y[b, h, p, :] = x[b, order[p], h, :] for p < N, zero tail.  `order`
 * (device, [N] int32) must be a permutation of 0..N-1.  The STA union of the
 * block-mask calls places blocks by the fractal order and does not apply to
 * other orders. */
BSA_API bsa_status bsa_reorder_perm(const bsa_shape* s, const int32_t* order, const void* x_bnhd, void* y_bhnd,
                                    bsa_stream_t stream);
BSA_API bsa_status bsa_inverse_reorder_perm(const bsa_shape* s, const int32_t* order, const void* y_bhnd,
                                            void* x_bnhd, bsa_stream_t stream);
BSA_API bsa_status bsa_reorder_qk_pooled_perm(const bsa_shape* s, const int32_t* order, const void* q_bnhd,
                                              const void* k_bnhd, void* q_bhnd, void* k_bhnd, void* workspace,
                                              size_t ws_bytes, bsa_stream_t stream);

/* Workspace bytes of bsa_build_block_mask_subblock (0 for an invalid shape or
 * sub-block size): a control block, the sub-block means of Q and K
 * (2 * B*heads*ns*d doubles, ns = ceil(N / sub)), the sub-block scores
 * (B*heads*ns*ns doubles) and the block importance (B*heads*nb*nb doubles). */
BSA_API size_t bsa_subblock_workspace_bytes(const bsa_shape* s, int32_t sub);

/* Block mask from sub-block scores, DFSAttn explainer, section 2 ("La
 * puntuacion de Sub-bloque"), with NABLA's CDF rule (bsa_build_block_mask):
 * Q and K are mean-pooled over sub-blocks of `sub` tokens (valid tokens only),
 * each query sub-block's softmax over all key sub-blocks (scale 1/sqrt(d)) is
 * summed over each key block's sub-blocks, and block I's importance for block
 * J is that mass averaged over I's query sub-blocks (rows sum to 1); the CDF
 * threshold then keeps the shortest most-important prefix of mass >= 1 - thr.
 * With sub == block this is NABLA's reduced map.  Double precision throughout.
 *   sub: 16 or 32 (dividing the block size), or the block size.
 *   Other arguments as for bsa_build_block_mask (no STA union);
 *   workspace / ws_bytes: at least bsa_subblock_workspace_bytes(s, sub). */
BSA_API bsa_status bsa_build_block_mask_subblock(const bsa_shape* s, const void* q_bhnd, const void* k_bhnd,
                                                 int32_t sub, float thr, int32_t* kv_count, int32_t* kv_idx,
                                                 uint8_t* mask_or_null, void* workspace, size_t ws_bytes,
                                                 bsa_stream_t stream);

/* Bytes of device workspace bsa_attn_bwd needs for this shape (0 for an
 * invalid shape): a control block (device error word), D = rowsum(dO * O)
 * (B*heads*Npad floats), a bit matrix of the block mask (B*heads*nb*
 * ceil(nb/32) words), the transposed lists (B*heads*nb*(nb+1) int32) and two
 * attention work plans, each part rounded up to 256 bytes.  Initialise the
 * control block once with bsa_workspace_init. */
BSA_API size_t bsa_attn_bwd_workspace_bytes(const bsa_shape* s);

/* Block-sparse attention backward: the gradients of bsa_attn_fwd with respect
 * to Q, K and V, following the same block mask.  NABLA summary, "Contribuciones
 * Clave" ("Aceleracion de Doble Fase": the block-sparse attention also runs in
 * pre-training and fine-tuning).  For every valid query row q of block I and
 * the valid keys k of the blocks I keeps, with P = exp(scale Q.K - lse):
 *   dV_k = sum_q P[q,k] dO_q,  dS = P (dO_q . V_k - dO_q . O_q),
 *   dQ_q = scale sum_k dS[q,k] K_k,  dK_k = scale sum_q dS[q,k] Q_q.
 * bf16 operands (P and dS rounded to bf16 for the products, as the forward
 * rounds P), fp32 accumulation, bf16 outputs.
 *   q, k, v, o, dO: device, [B, heads, Npad, d] bf16 in kernel order (o: the
 *       forward output, dO: the gradient of the loss with respect to it).
 *   lse: device, [B, heads, Npad] float32, the forward pass's lse_or_null.
 *   kv_count, kv_idx: the lists the forward pass used.
 *   scale: as for bsa_attn_fwd (0 selects 1/sqrt(d)).
 *   dq, dk, dv: device, [B, heads, Npad, d] bf16, written (padded rows 0);
 *       pairwise distinct.
 *   workspace / ws_bytes: at least bsa_attn_bwd_workspace_bytes(s).
 * Errors as for bsa_attn_fwd. */
BSA_API bsa_status bsa_attn_bwd(const bsa_shape* s, const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const int32_t* kv_count, const int32_t* kv_idx,
                                float scale, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                                bsa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Fine-grained KV selection (AB-Attention article, news.hamidun.com/es/news/
 * 14960, "Los tres recursos de AB-Attention": the fine selection on coarse
 * hardware, and SIP's inclusion-probability weights).
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace bsa_attn_fwd_fine needs (a control block and a
 * work counter); 0 for an invalid shape or one whose block is not 128. */
BSA_API size_t bsa_attn_fine_workspace_bytes(const bsa_shape* s);

/* Attention of each 128-row query block over its own list of KV blocks of 4
 * tokens, each optionally weighted by the inverse w of its inclusion
 * probability (the Horvitz-Thompson estimate of both the softmax numerator
 * and its normalisation, as a logit shift ln w):
 *   O[q] = sum_k w_b(k) exp(scale Q[q].K[k]) V[k] / sum_k w_b(k) exp(scale Q[q].K[k])
 * over the valid keys k < N of the listed blocks b (block b holds keys
 * 4b .. 4b + 3).  The chosen blocks are gathered by index into full 128-key
 * tiles of the tcgen05 tensor cores; fp32 softmax and accumulation, bf16
 * output.
 *   s: shape with block = 128 (the query block); BSA_ERR_UNSUPPORTED otherwise.
 *   q, k, v: device, [B, heads, Npad, d] bf16 (any token order: the lists
 *       index rows of k and v as given).
 *   sel_offsets: device, int64 [B * heads * Npad / 128 + 1], CSR offsets: the
 *       list of query block I of (b, h) is entries sel_offsets[r] ..
 *       sel_offsets[r + 1] - 1 of sel_idx, r = (b * heads + h) * (Npad / 128) + I.
 *   sel_idx: device, int32 [n_sel], 4-token block indices in [0, ceil(N / 4)),
 *       in any order (a repeated entry counts again); NULL when n_sel = 0.
 *   sel_w_or_null: device, float32 [n_sel] positive finite weights, or NULL
 *       (every weight 1: plain attention over the selected keys).
 *   n_sel: entries of sel_idx (and sel_w).
 *   scale: >= 0; 0 selects 1/sqrt(d).
 *   o: device, [B, heads, Npad, d] bf16, written; rows >= N, and rows whose
 *       list holds no valid key, are 0.
 *   lse_or_null: device, [B, heads, Npad] float32 natural-log sum of
 *       w exp(scale s) per row (0 where o is 0), or NULL.
 *   workspace / ws_bytes: at least bsa_attn_fine_workspace_bytes(s).
 * A list whose offsets decrease or leave [0, n_sel] is treated as empty, an
 * index outside [0, ceil(N / 4)) and a weight that is not positive and finite
 * are skipped; each sets the device error word (BSA_ERR_DEVICE_INDEX). */
BSA_API bsa_status bsa_attn_fwd_fine(const bsa_shape* s, const void* q, const void* k, const void* v,
                                     const int64_t* sel_offsets, const int32_t* sel_idx,
                                     const float* sel_w_or_null, int64_t n_sel, float scale, void* o,
                                     float* lse_or_null, void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* Same contract as bsa_attn_fwd, computed by the legacy warp-level
 * mma.sync tensor-core kernel instead of the tcgen05 one.  Kept as the measured
 * baseline the tcgen05 kernel is compared with. */
BSA_API bsa_status bsa_attn_fwd_baseline(const bsa_shape* s, const void* q, const void* k, const void* v,
                                         const int32_t* kv_count, const int32_t* kv_idx, float scale,
                                         void* o, float* lse_or_null,
                                         void* workspace, size_t ws_bytes, bsa_stream_t stream);

/* Size in bytes of the device array that bsa_attn_fwd_noalloc uses as its
 * scratch (4 MiB, reserved on every GPU that loads the library). */
#define BSA_NOALLOC_SCRATCH_BYTES (4u << 20)

/* bsa_attn_fwd for callers that cannot allocate device memory.  The NABLA
 * summary has no counterpart: this is a library convenience.
 *
 * Some callers cannot call cudaMalloc or any other allocator where they run
 * attention: code given a fixed memory budget up front, a plug-in inside a host
 * program that owns every allocation, or a path that must not take the
 * allocator's locks.  This entry point needs no workspace.  Its scratch (the
 * device error word and the work plan of the tensor-core kernel) lives in one
 * static device array of BSA_NOALLOC_SCRATCH_BYTES that the library holds on
 * every GPU until the process exits.  The entry point calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Arguments, layouts and results are those of bsa_attn_fwd.  There is no
 * workspace argument.  Instead:
 *   error_word_or_null: device, one uint32 (4-byte aligned), written at the end
 *       of the call with the device error bits of this call (0 = none,
 *       1 = a KV index outside [0, nb), 2 = a KV count outside [1, nb],
 *       4 = a bounded wait expired, 8 = the attention kernel found its
 *       shared memory not 1024-byte aligned and did nothing), or NULL to
 *       ignore them.
 *
 * Limits and errors: a shape whose scratch exceeds BSA_NOALLOC_SCRATCH_BYTES
 * is refused with
 * BSA_ERR_UNSUPPORTED before anything is launched.  The scratch is 256 bytes
 * plus the work plan: 8 bytes per 128-row query tile (B*heads*ceil(nb /
 * (128 / block)) tiles), with 64-token blocks 68 bytes per block row
 * (B*heads*nb rows), and a 256-byte work counter, each part rounded up to 256
 * bytes.  Argument errors are those of bsa_attn_fwd.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and remembers it with the
 * current CUDA context.  Make that first call before any stream capture.  A
 * device reset (cudaDeviceReset, or a context destroyed and created again)
 * gives the array a new address: the next call notices the new context and
 * looks the address up again, so it too must come before any capture.
 *
 * Sharing: every call on a device uses the same array.  The call clears the
 * error word at its start and rewrites the plan, so nothing carries over from
 * one call to the next.  Calls whose GPU work overlaps (other streams, other
 * host threads) race on the array: serialise them. */
BSA_API bsa_status bsa_attn_fwd_noalloc(const bsa_shape* s, const void* q, const void* k, const void* v,
                                        const int32_t* kv_count, const int32_t* kv_idx, float scale,
                                        void* o, float* lse_or_null, uint32_t* error_word_or_null,
                                        bsa_stream_t stream);

/* Synchronises `stream`, reads and clears the device error word of
 * `workspace`: BSA_OK, BSA_ERR_DEVICE_INDEX, BSA_ERR_TIMEOUT or BSA_ERR_CUDA
 * (a pending asynchronous CUDA error). */
BSA_API bsa_status bsa_check_device_status(void* workspace, bsa_stream_t stream);

/* Static string naming a status. */
BSA_API const char* bsa_status_string(bsa_status st);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */
