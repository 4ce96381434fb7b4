// Memory-bound helpers of the bf16 path (head_dim = 64):
//  * seg_means_bf16: Q~, K~ segment means ("Nystromformer: A Nystrom-Based
//    Algorithm for Approximating Self-Attention", section 3.4, Eq. 16 with the
//    page's 1/l correction), one pass over Q and K with 16-byte loads;
//  * merge_w: the B~ V partials of all CTAs / row copies of a head combined in
//    a fixed order (Y = B~ V), then W = Z Y (Eq. 17 product chain).
#pragma once

#include "common.cuh"

namespace nys {

// One block per (segment, head, tensor): 8 threads cover the 64 features of a
// row (8 bf16 each) and `rows` groups of threads stride over the segment's l
// rows; a fixed-order tree over the groups gives the sum, divided by l.
__global__ void __launch_bounds__(256)
seg_means_bf16(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
               float *__restrict__ Qt, float *__restrict__ Kt, int n, int m) {
  __shared__ float part[32][64];
  const int j = blockIdx.x, bh = blockIdx.y;
  const __nv_bfloat16 *X = blockIdx.z == 0 ? Q : K;
  float *Xt = blockIdx.z == 0 ? Qt : Kt;
  const int seg = n / m;
  const int groups = blockDim.x >> 3;          // row groups (<= 32)
  const int g = threadIdx.x >> 3, ch = threadIdx.x & 7;
  const uint4 *src = (const uint4 *)(X + ((size_t)bh * n + (size_t)j * seg) * 64) + ch;
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
}

// One block per head, 256 threads.  pmax / psum / py hold `parts` partial
// softmax states per landmark row: running max (log2 units), running sum and
// the unnormalised sum of p_i v_i.
template <int M>
__global__ void __launch_bounds__(256)
merge_w(const float *__restrict__ pmax, const float *__restrict__ psum,
        const float *__restrict__ py, const float *__restrict__ Zg, float *__restrict__ Yg,
        float *__restrict__ Wg, int parts) {
  extern __shared__ float sm[];
  float *zs = sm;                         // [M][M]
  float *ys = zs + M * M;                 // [M][64]
  float *wgt = ys + M * 64;               // [parts][M]
  const int bh = blockIdx.x, t = threadIdx.x;
  {
    const float4 *z4 = (const float4 *)(Zg + (size_t)bh * M * M);
    constexpr int kPer = M * M / 4 / 256;
    float4 v[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) v[i] = z4[t + 256 * i];
#pragma unroll
    for (int i = 0; i < kPer; ++i) ((float4 *)zs)[t + 256 * i] = v[i];
  }
  const size_t pb = (size_t)bh * parts * M;
  if (t < M) {
    float mx = -INFINITY;
    for (int p = 0; p < parts; ++p) mx = fmaxf(mx, pmax[pb + (size_t)p * M + t]);
    float den = 0.f;
    for (int p = 0; p < parts; ++p) {
      const float f = exp2f(pmax[pb + (size_t)p * M + t] - mx);
      wgt[p * M + t] = f;
      den = fmaf(psum[pb + (size_t)p * M + t], f, den);
    }
    const float inv = 1.f / den;
    for (int p = 0; p < parts; ++p) wgt[p * M + t] *= inv;
  }
  __syncthreads();
  // Y rows: thread -> (row, 4 features), partials in a fixed order
  for (int idx = t; idx < M * 16; idx += 256) {
    const int j = idx >> 4, c4 = idx & 15;
    const float4 *src = (const float4 *)(py + (pb + j) * 64) + c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int p = 0;
    for (; p + 4 <= parts; p += 4) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = src[(size_t)(p + u) * M * 16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = wgt[(p + u) * M + j];
        acc.x = fmaf(w, v[u].x, acc.x);
        acc.y = fmaf(w, v[u].y, acc.y);
        acc.z = fmaf(w, v[u].z, acc.z);
        acc.w = fmaf(w, v[u].w, acc.w);
      }
    }
    for (; p < parts; ++p) {
      const float4 v = src[(size_t)p * M * 16];
      const float w = wgt[p * M + j];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    ((float4 *)ys)[idx] = acc;
    ((float4 *)(Yg + (size_t)bh * M * 64))[idx] = acc;
  }
  __syncthreads();
  // W = Z Y: thread -> R rows x 4 features
  constexpr int R = M * 16 / 256;    // rows per thread (M = 32: 2, 64: 4, 128: 8)
  const int c4 = t & 15, j0 = (t >> 4) * R;
  float4 acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < M; ++k) {
    const float4 y = ((const float4 *)ys)[k * 16 + c4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float z = zs[(j0 + r) * M + k];
      acc[r].x = fmaf(z, y.x, acc[r].x);
      acc[r].y = fmaf(z, y.y, acc[r].y);
      acc[r].z = fmaf(z, y.z, acc[r].z);
      acc[r].w = fmaf(z, y.w, acc[r].w);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) ((float4 *)(Wg + (size_t)bh * M * 64))[(j0 + r) * 16 + c4] = acc[r];
}

}  // namespace nys
