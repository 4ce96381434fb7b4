// Memory-bound helpers of the bf16 path (head_dim = 64):
//  * seg_means_bf16: Q~, K~ segment means ("Nystromformer: A Nystrom-Based
//    Algorithm for Approximating Self-Attention", section 3.4, Eq. 16 with the
//    page's 1/l correction), one pass over Q and K with 16-byte loads.
//    Segment j holds tokens j*l .. min(j*l + l, n) - 1, l = ceil(n / m) (the
//    sequence read as padded to m*l tokens), averaged over its real tokens;
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {

// One block per (segment, head, tensor): 8 threads cover the 64 features of a
// row (8 bf16 each) and `rows` groups of threads stride over the segment's l
// rows; a fixed-order tree over the groups gives the sum, divided by l.
__global__ void __launch_bounds__(256)
seg_means_bf16(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
               float *__restrict__ Qt, float *__restrict__ Kt, int n, int m) {
  __shared__ float part[32][64];
  NYS_MARK(kTrSeg, 0);
  sm100::griddep_launch_dependents();   // the next kernel waits for this grid anyway
  const int j = blockIdx.x, bh = blockIdx.y;
  const __nv_bfloat16 *X = blockIdx.z == 0 ? Q : K;
  float *Xt = blockIdx.z == 0 ? Qt : Kt;
  const int len = (n + m - 1) / m;                 // l
  const int seg = min(len, n - j * len);           // real tokens of segment j (>= 1)
  const int groups = blockDim.x >> 3;          // row groups (<= 32)
  const int g = threadIdx.x >> 3, ch = threadIdx.x & 7;
  const uint4 *src = (const uint4 *)(X + ((size_t)bh * n + (size_t)j * len) * 64) + ch;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int r = g;
  // four rows in flight per thread
  for (; r + 3 * groups < seg; r += 4 * groups) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(src + (size_t)(r + u * groups) * 8);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162 *h = (const __nv_bfloat162 *)&v[u];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  for (; r < seg; r += groups) {
    const uint4 v = __ldg(src + (size_t)r * 8);
    const __nv_bfloat162 *h = (const __nv_bfloat162 *)&v;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
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

}  // namespace nys
