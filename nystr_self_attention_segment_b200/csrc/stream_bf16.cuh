// Segment means of the bf16 path (head_dim = 64): Q~ and K~ in one pass over
// Q and K ("Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, Eq. 16 with the page's 1/l correction).
// Segment j holds tokens j*l .. min(j*l + l, L) - 1, l = ceil(L / m), L the
// sequence length of the element (n, or its own length for ragged batches):
// the sequence read as padded to m*l tokens, each landmark the mean over the
// real tokens of its segment.
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace segm {

using namespace sm100;

// Tokens per element: lens (device, one per batch element) or n.
struct Shape {
  int n, m, heads;
  const int *lens;   // [batch] or null
};

// 16-byte load that leaves its L2 lines normal (0) or first to evict (1).
template <int EVICT_FIRST>
__device__ __forceinline__ uint4 load16(const uint4 *p, uint64_t policy) {
  if constexpr (EVICT_FIRST) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(policy));
    return v;
  } else {
    (void)policy;
    return __ldg(p);
  }
}

#ifndef NYS_SEG_EVICT_FIRST
#define NYS_SEG_EVICT_FIRST 0
#endif

// One block per (segment, batch*head, tensor): 8 threads cover the 64
// features of a row (8 bf16 each) and `groups` groups of threads stride over
// the segment's rows, four rows in flight per thread; a fixed-order tree
// over the groups gives the sum, divided by the segment's real tokens.  An
// element whose length is invalid (outside [m, n], or with an empty segment)
// records NYS_ERR_INVALID_ARG and leaves its landmarks unwritten.
__global__ void __launch_bounds__(256)
seg_means_bf16(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
               float *__restrict__ Qt, float *__restrict__ Kt, Shape sh, uint32_t *err) {
  __shared__ float part[32][64];
  NYS_MARK(kTrSeg, 0);
  griddep_launch_dependents();   // the next kernel waits for this grid anyway
  const int j = blockIdx.x, bh = blockIdx.y, m = sh.m, n = sh.n;
  const __nv_bfloat16 *X = blockIdx.z == 0 ? Q : K;
  float *Xt = blockIdx.z == 0 ? Qt : Kt;
  int L = n;
  if (sh.lens) {
    L = sh.lens[bh / sh.heads];
    if (L < m || L > n || (long)(m - 1) * ((L + m - 1) / m) >= L) {
      if (threadIdx.x == 0 && j == 0 && blockIdx.z == 0) set_error(err, NYS_ERR_INVALID_ARG);
      return;
    }
  }
  const int len = (L + m - 1) / m;                 // l
  const int seg = min(len, L - j * len);           // real tokens of segment j (>= 1)
  const int groups = blockDim.x >> 3;              // row groups (<= 32)
  const int g = threadIdx.x >> 3, ch = threadIdx.x & 7;
  const uint4 *src = (const uint4 *)(X + ((size_t)bh * n + (size_t)j * len) * 64) + ch;
  const uint64_t policy = NYS_SEG_EVICT_FIRST ? policy_evict_first() : 0;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto add = [&](const uint4 &v) {
    const __nv_bfloat162 *hh = (const __nv_bfloat162 *)&v;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(hh[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  };
  int r = g;
  for (; r + 3 * groups < seg; r += 4 * groups) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = load16<NYS_SEG_EVICT_FIRST>(src + (size_t)(r + u * groups) * 8, policy);
#pragma unroll
    for (int u = 0; u < 4; ++u) add(v[u]);
  }
  for (; r < seg; r += groups) add(load16<NYS_SEG_EVICT_FIRST>(src + (size_t)r * 8, policy));
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][ch * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < 64; c += blockDim.x) {   // blocks of 8..256 threads
    float s = 0.f;
    for (int q = 0; q < groups; ++q) s += part[q][c];
    Xt[((size_t)bh * m + j) * 64 + c] = s / (float)seg;
  }
  NYS_MARK(kTrSeg, 1);
}

// Threads per block: 8 per row group, min(l, 32) groups (l of the longest
// element, ceil(n / m)).
inline int threads_for(int n, int m) {
  const int l = (n + m - 1) / m;
  return 8 * (l < 32 ? l : 32);
}

}  // namespace segm
}  // namespace nys
