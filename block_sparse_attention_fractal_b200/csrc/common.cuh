// Shared device-side definitions of libbsa: shape arithmetic, the fractal
// token order, the workspace control block and error bits.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bsa.h"

namespace bsa {

// Device error word bits (control block of the workspace).
enum : uint32_t {
  kErrIndex = 1u,    // a KV index outside [0, nb)
  kErrCount = 2u,    // a KV count outside [1, nb]
  kErrTimeout = 4u,  // a bounded wait expired
  kErrLayout = 8u,   // shared memory not aligned as the kernel's layout needs
  kErrWeight = 16u,  // an inclusion weight that is not positive and finite
};

// Control block at the start of every workspace.
struct Ctrl {
  uint32_t error;       // OR of kErr* bits
  uint32_t detail[3];   // first offending (row, value, site) for diagnostics
  // Sequence number of the launch whose CTAs are giving up after a bounded
  // wait expired.  Every launch gets its own nonzero number, and a CTA gives
  // up early only on its own launch's number, so a timeout left behind by an
  // earlier call never cuts a later call short.
  uint32_t abort_seq;
  uint32_t pad[59];
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

struct Dims {
  int B, T, H, W, heads, d, bs, P;
  int N, Npad, nb;
};

__device__ __forceinline__ void report_error(Ctrl* c, uint32_t bits, uint32_t row, uint32_t value, uint32_t site) {
  uint32_t old = atomicOr(&c->error, bits);
  if (old == 0u) {
    c->detail[0] = row;
    c->detail[1] = value;
    c->detail[2] = site;
  }
}

// Original token index n = t*H*W + h*W + w of fractal position p < N.
// Frames in order; inside a frame the P x P patches row-major (edge patches
// clipped), inside a patch the tokens row-major.
__host__ __device__ __forceinline__ int fractal_token(int p, int H, int W, int P) {
  const int HW = H * W;
  const int t = p / HW;
  const int r = p - t * HW;
  const int band = P * W;                 // tokens of one full band of patch rows
  const int pr = r / band;
  const int r2 = r - pr * band;
  const int ph = min(P, H - pr * P);      // rows of this band (last band may be short)
  const int pc = r2 / (ph * P);
  const int r3 = r2 - pc * ph * P;
  const int pw = min(P, W - pc * P);      // columns of this patch (last patch may be narrow)
  const int hh = r3 / pw;
  const int ww = r3 - hh * pw;
  return t * HW + (pr * P + hh) * W + (pc * P + ww);
}

}  // namespace bsa
