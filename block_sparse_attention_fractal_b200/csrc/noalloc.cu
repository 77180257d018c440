// bsa_attn_fwd_noalloc: the block-sparse attention forward of bsa_attn_fwd,
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run attention: code that runs under a fixed memory budget handed out
// up front, plugins inside a host application that owns every allocation, or
// paths that must not touch the allocator's locks.  bsa_attn_fwd needs a
// caller-provided workspace for its scratch (the control block with the device
// error word, and the work plan of the tensor-core kernel).  This variant keeps
// that scratch in one file-scope device array instead, so the caller passes
// only inputs and outputs.
//
// The array is a fixed BSA_NOALLOC_SCRATCH_BYTES on every GPU that loads the
// library, held until the process exits.  Every call shares it: calls whose
// work overlaps on the GPU (two streams, two host threads) race on it.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace {

using bsa::Ctrl;
using bsa::Dims;

constexpr int kMaxDevices = 64;

// The scratch: control block, then the attention work plan.
static __device__ __align__(256) uint8_t g_noalloc_scratch[BSA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch for each device ordinal (in host code the
// symbol itself is only a host-side stand-in, not a device address), with the
// context it was looked up in: a device reset (or a context destroyed and made
// again) loads the module anew, so an address from another context is stale
// and is looked up again.
struct ScratchAddr {
  CUcontext ctx;
  void* addr;
};
ScratchAddr g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (CtxGetCurrentFn)p;
  }
  return fn;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The device address of the scratch array on the current device, looked up
// (cudaGetSymbolAddress, with that device current) on the first call in each
// context.
bsa_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return BSA_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (ctx == nullptr || g_scratch[dev].addr == nullptr || g_scratch[dev].ctx != ctx) {
    // (the lookup also makes the device's primary context current when this
    // thread has none yet)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return BSA_ERR_CUDA;
    g_scratch[dev].ctx = ctx;
    g_scratch[dev].addr = p;
  }
  *out = g_scratch[dev].addr;
  return BSA_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

bsa_status bsa_attn_fwd_noalloc(const bsa_shape* s, const void* q, const void* k, const void* v,
                                const int32_t* kv_count, const int32_t* kv_idx, float scale, void* o,
                                float* lse_or_null, uint32_t* error_word_or_null, bsa_stream_t stream) {
  bsa_status st = bsa_validate_shape(s);
  if (st != BSA_OK) return st;
  Dims g;
  g.B = s->B;
  g.T = s->T;
  g.H = s->H;
  g.W = s->W;
  g.heads = s->heads;
  g.d = s->d;
  g.bs = s->block;
  g.P = s->patch;
  g.N = (int)bsa_seq_len(s);
  g.Npad = (int)bsa_padded_len(s);
  g.nb = (int)bsa_num_blocks(s);
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || kv_count == nullptr || kv_idx == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(kv_count) ||
      !aligned16(kv_idx) || (lse_or_null != nullptr && !aligned16(lse_or_null)) ||
      (error_word_or_null != nullptr && ((uintptr_t)error_word_or_null & 3u) != 0))
    return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.0f) return BSA_ERR_INVALID_ARG;
  if (scale == 0.0f) scale = (float)(1.0 / std::sqrt((double)g.d));
  // Scratch this shape needs: control block + work plan.  Larger shapes are
  // refused before anything is launched.
  const size_t need = sizeof(Ctrl) + align256(bsa::plan_region_bytes(g));
  if (need > (size_t)BSA_NOALLOC_SCRATCH_BYTES) return BSA_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != BSA_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  Ctrl* ctrl = (Ctrl*)scratch;
  int2* items = (int2*)((char*)scratch + sizeof(Ctrl));
  // The control block keeps the last call's contents: clear it first.
  if (cudaMemsetAsync(ctrl, 0, sizeof(Ctrl), cs) != cudaSuccess) return BSA_ERR_CUDA;
  if (bsa::launch_plan(g, kv_count, kv_idx, items, cs) != cudaSuccess) return BSA_ERR_CUDA;
  if (bsa::launch_attn(g, q, k, v, kv_count, kv_idx, items, bsa::plan_work_counter(g, items), scale, o, lse_or_null,
                       nullptr, ctrl, bsa::next_launch_seq(), cs) != cudaSuccess)
    return BSA_ERR_CUDA;
  if (error_word_or_null != nullptr &&
      cudaMemcpyAsync(error_word_or_null, &ctrl->error, sizeof(uint32_t), cudaMemcpyDeviceToDevice, cs) !=
          cudaSuccess)
    return BSA_ERR_CUDA;
  return BSA_OK;
}

}  // extern "C"
