// Merge of the B~ V partial states and W = Z (B~ V) for the bf16 path
// ("Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, Eq. 17 / Algorithm 1: the m x d product that
// the output F~ W needs; the spec order F~ (Z (B~ V))).
//
// The S key splits of a head left, per landmark j, a running maximum m_s
// (log2 units), a sum l_s and an unnormalised Y_s over their keys.  With
// f_s = 2^(m_s - max_s m_s):
//   Y_j = sum_s f_s Y_s,j / sum_s f_s l_s,j     (splits in order s = 0..S-1)
// then W = Z Y in fp32 (k in order), stored as fp32 rows and as the bf16 B
// operand of the output kernel's P W (row = landmark, 16-byte chunk c of the
// 128-byte row at c ^ (row & 7): the 128-byte swizzle of a 1 KB-aligned tile).
//
// Grid: batch*heads x R blocks, R = m / 16; block r forms W rows
// [16 r, 16 r + 16) and merges the whole Y (every block merges the same Y in
// the same order, so they agree bit for bit); block 0 also stores Y for the
// parity checks.  Every sum runs in a fixed order.
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace wmerge {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kRows = 16;          // W rows per block
constexpr int kMaxSplits = 16;
constexpr int kYs = 68;            // Y row stride (floats): float4 rows, no conflicts

struct Params {
  const float *pmax, *psum, *py;   // [BH][S][m], [BH][S][m], [BH][S][m][64]
  const float *z;                  // [BH][m][m]
  float *y, *w;                    // [BH][m][64]
  uint8_t *w_op;                   // [BH][m][128 B]
  int splits;
};

template <int M>
struct Smem {
  static constexpr uint32_t ys = 0;                              // Y [M][kYs]
  static constexpr uint32_t zs = ys + M * kYs * 4u;              // Z rows [kRows][M + 4]
  static constexpr uint32_t wgt = zs + kRows * (M + 4) * 4u;     // f [S][M]
  static constexpr uint32_t psm = wgt + kMaxSplits * M * 4u;     // l [S][M]
  static constexpr uint32_t den = psm + kMaxSplits * M * 4u;     // 1 / sum f l [M]
  static constexpr uint32_t total = den + M * 4u;
};

template <int M>
__global__ void __launch_bounds__(kThreads)
wmerge_kernel(const Params prm) {
  using C = Smem<M>;
  extern __shared__ __align__(16) uint8_t smem[];
  NYS_MARK(kTrW, 0);
  // the output kernel may launch now: it waits for this whole grid before it
  // reads W
  griddep_launch_dependents();
  constexpr int R = M / kRows;
  const int bh = blockIdx.x / R, r0 = (blockIdx.x % R) * kRows;
  const int t = threadIdx.x, S = prm.splits;
  float *ys = (float *)(smem + C::ys), *zs = (float *)(smem + C::zs);
  float *wgt = (float *)(smem + C::wgt), *psm = (float *)(smem + C::psm);
  float *den = (float *)(smem + C::den);
  griddep_wait();   // partials and Z of the previous kernel
  NYS_MARK(kTrW, 1);
  const size_t pb = (size_t)bh * S * M;
  {   // maxima and sums of the splits, and this block's Z rows (loads first)
    constexpr int kPer = (kMaxSplits * M + kThreads - 1) / kThreads;
    constexpr int kZ4 = kRows * M / 4, kZPer = (kZ4 + kThreads - 1) / kThreads;
    float a[kPer], b[kPer];
    float4 zv[kZPer];
    const float4 *zg = (const float4 *)(prm.z + ((size_t)bh * M + r0) * M);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = t + u * kThreads;
      if (i < S * M) {
        a[u] = __ldcg(prm.pmax + pb + i);
        b[u] = __ldcg(prm.psum + pb + i);
      }
    }
#pragma unroll
    for (int u = 0; u < kZPer; ++u) {
      const int i = t + u * kThreads;
      if (i < kZ4) zv[u] = __ldcg(zg + i);
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = t + u * kThreads;
      if (i < S * M) {
        wgt[i] = a[u];
        psm[i] = b[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kZPer; ++u) {
      const int i = t + u * kThreads;
      if (i < kZ4) *(float4 *)(zs + (i * 4 / M) * (M + 4) + (i * 4) % M) = zv[u];
    }
  }
  __syncthreads();
  if (t < M) {   // weights f_s and 1 / sum_s f_s l_s of landmark t
    float mx = -INFINITY;
    for (int s = 0; s < S; ++s) mx = fmaxf(mx, wgt[s * M + t]);
    float d = 0.f;
    for (int s = 0; s < S; ++s) {
      const float f = mx == -INFINITY ? 0.f : fast_exp2(wgt[s * M + t] - mx);
      wgt[s * M + t] = f;
      d = fmaf(psm[s * M + t], f, d);
    }
    den[t] = 1.f / d;
  }
  __syncthreads();
  {   // Y = sum_s f_s Y_s / den, a batch of splits loaded at once
    constexpr int kItems = M * 16;                 // float4 items of Y
    constexpr int kIpt = kItems / kThreads;        // 2, 4 or 8 items per thread
    constexpr int kBatch = 16 / kIpt;              // splits per load batch
    float4 acc[kIpt];
#pragma unroll
    for (int q = 0; q < kIpt; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < S; s0 += kBatch) {
      float4 v[kIpt][kBatch];
#pragma unroll
      for (int q = 0; q < kIpt; ++q) {
        const int idx = q * kThreads + t;
        const float4 *src = (const float4 *)(prm.py + (pb + (idx >> 4)) * 64) + (idx & 15);
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (s0 + u < S) v[q][u] = __ldcg(src + (size_t)(s0 + u) * M * 16);
      }
#pragma unroll
      for (int q = 0; q < kIpt; ++q) {
        const int j = (q * kThreads + t) >> 4;
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (s0 + u < S) {
            const float f = wgt[(s0 + u) * M + j];
            acc[q].x = fmaf(f, v[q][u].x, acc[q].x);
            acc[q].y = fmaf(f, v[q][u].y, acc[q].y);
            acc[q].z = fmaf(f, v[q][u].z, acc[q].z);
            acc[q].w = fmaf(f, v[q][u].w, acc[q].w);
          }
      }
    }
#pragma unroll
    for (int q = 0; q < kIpt; ++q) {
      const int idx = q * kThreads + t;
      const float inv = den[idx >> 4];
      const float4 y = make_float4(acc[q].x * inv, acc[q].y * inv, acc[q].z * inv, acc[q].w * inv);
      *(float4 *)(ys + (idx >> 4) * kYs + (idx & 15) * 4) = y;
      if (r0 == 0) ((float4 *)(prm.y + (size_t)bh * M * 64))[idx] = y;
    }
  }
  __syncthreads();
  {   // W rows r0 + i: thread (i, c4) forms 4 columns, k in order
    const int i = t >> 4, c4 = t & 15;
    const float *zr = zs + i * (M + 4);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int k = 0; k < M; ++k) {
      const float zk = zr[k];
      const float4 y = *(const float4 *)(ys + k * kYs + 4 * c4);
      a.x = fmaf(zk, y.x, a.x);
      a.y = fmaf(zk, y.y, a.y);
      a.z = fmaf(zk, y.z, a.z);
      a.w = fmaf(zk, y.w, a.w);
    }
    const int row = r0 + i;
    *(float4 *)(prm.w + ((size_t)bh * M + row) * 64 + 4 * c4) = a;
    uint8_t *op = prm.w_op + ((size_t)bh * M + row) * 128;
    *(uint2 *)(op + (((c4 >> 1) ^ (row & 7)) << 4) + (c4 & 1) * 8) =
        make_uint2(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w));
  }
  NYS_MARK(kTrW, 2);
}

}  // namespace wmerge
}  // namespace nys
