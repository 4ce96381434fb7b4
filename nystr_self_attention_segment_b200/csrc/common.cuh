// Shared device helpers: dtype conversion, warp reductions, workspace layout.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/nys_attn.h"

namespace nys {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxIters = 64;
constexpr int kMaxConvK = 63;
constexpr int kNumSms = 148;       // streaming multiprocessors of a B200

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Records the first failure a kernel sees in the workspace error word.
__device__ __forceinline__ void set_error(uint32_t *err, uint32_t code) {
  if (err) atomicCAS(err, 0u, code);
}

// Workspace layout, a pure function of the shape so that it can be sized on
// a machine without a GPU.  All regions are 256-byte aligned.
// Per-head words of the bf16 path's hand-off, zeroed by every call:
// [0, BH) key-split blocks done, [BH, 2 BH) W inputs (merged Y, Z) in global
// memory, [2 BH, 3 BH) W of the head stored (the output kernel's flag).
constexpr int kCountsPerHead = 3;

struct Layout {
  size_t q_land, k_land, z, y, w, err;     // parity-visible fp32 intermediates
  size_t count;                            // kCountsPerHead words per head (bf16 path)
  size_t pmax, psum, py;                   // split-n partials of B~ V
  size_t scratch;                          // per-head pinv scratch (m > 64)
  size_t w_bf;                             // W as the bf16 operand of P W
  size_t total;
  int splits;                              // B~ V partials per head
  int keys_per_split;                      // SIMT path: keys per split
  int bv_ctas_per_head;                    // tensor-core path: CTAs per head
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace nys
