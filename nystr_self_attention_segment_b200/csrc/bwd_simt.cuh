// Backward pass of the Nystrom attention: gradients of the loss with respect
// to Q, K, V and the DConv kernel, given dO ("Nystromformer: A Nystrom-Based
// Algorithm for Approximating Self-Attention", section 3.4: "Moore-Penrose
// Pseudoinverse Computation" -- the gradient flows through the iteration's
// matrix products like through any other layer; Eq. 17 / Algorithm 1 and
// Figure 4 for the forward it differentiates).
//
// The chain rule of every forward step, in reverse (s = 1/sqrt(d)):
//   DConv:  dV += conv^T(dO),  dw[t] = sum_i dO_i . V_{i+t-half}
//   O = F W:  dF = dO W^T,  dW = F^T dO
//   W = Z Y:  dZ = dW Y^T,  dY = Z^T dW
//   Y = B V:  dB = dY V^T,  dV += B^T dY
//   softmax rows (F, B, A):  dS = P * (dP - rowsum(dP * P))
//   B = softmax(s Q~ K^T):  dQ~ += s dS_B K,  dK += s dS_B^T Q~
//   F = softmax(s Q K~^T):  dQ += s dS_F K~,  dK~ += s dS_F^T Q
//   Z = Lemma 1 steps from Z0:  each step back through its four products
//   Z0 = A^T / (||A||_1 ||A||_inf):  the norms' maximising column / row
//   A = softmax(s Q~ K~^T):  dQ~ += s dS_A K~,  dK~ += s dS_A^T Q~
//   Q~, K~ = segment means:  each token of segment j gets dX~_j / count_j
// with rowsum(dB * B)_j = dY_j . Y_j (Y = B V), so B is never stored.
//
// Kernels (fp32 arithmetic on the CUDA cores; inputs and gradients in the
// forward's dtype, the conv gradient fp32), after the forward's own segment
// means, pseudoinverse (all iterates kept), B~ V partials and merge:
//   bwd_rows   per 64-row tile: F, dF, dS_F; dQ (the F part); block partials
//              of dW, dK~ and dw
//   bwd_head   per head: dW, dY, dZ, the Lemma 1 steps backwards, dA, dQ~_A,
//              dK~ (total), D = rowsum(dY * Y)
//   bwd_keys   per 64-key tile: B, dB, dS_B; dK (without its dK~ part), dV
//              (with the conv part); block partials of dQ~.  It starts
//              while bwd_head runs (programmatic launch) and waits only for
//              the head's dY and D flag
//   bwd_dqt_total  dQ~ = dQ~_A + the key blocks' partials, in order
//   bwd_dqk    dQ += dQ~_{seg(i)} / count, dK += dK~_{seg(i)} / count
//   bwd_dconv  dw summed over the batch and the row blocks, in order
// Every sum runs in a fixed order: results are bitwise reproducible.
#pragma once

#include "common.cuh"
#include "simt.cuh"
#include "sm100.cuh"

namespace nys {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kHeadThreads = 512;   // bwd_head: one block per head, twice the warps
constexpr int kTile = 64;   // rows / keys per tile

// mm_acc (simt.cuh): the register-tiled block product every kernel here uses.

template <int RM, int RN>
__device__ __forceinline__ void zero(float (&acc)[RM][RN]) {
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int c = 0; c < RN; ++c) acc[r][c] = 0.f;
}

// C(i, j) = alpha * acc for the owned outputs (C row stride ldc).
template <int RM, int RN>
__device__ __forceinline__ void store(const float (&acc)[RM][RN], float *C, int ldc, int M, int N,
                                      float alpha = 1.f) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int c = 0; c < RN; ++c) {
      const int i = ty + 16 * r, j = tx + 16 * c;
      if (i < M && j < N) C[i * ldc + j] = alpha * acc[r][c];
    }
}

// segment of token i, and its token count, for l = ceil(L / m)
__device__ __forceinline__ int seg_of(int i, int l) { return i / l; }
__device__ __forceinline__ int seg_count(int j, int l, int L) { return min(l, L - j * l); }

// ---------------------------------------------------------------------------
struct RowsParams {
  const void *Q, *V, *G;        // [BH][n][d] (T)
  const float *kt, *w;          // [BH][m][d] K~, W
  const float *conv_w;          // [H][k] or null
  void *dQ;                     // [BH][n][d] (T): the F part of dQ
  float *dw_part, *dkt_part;    // [BH][R][m][d] partials of dW, dK~ (F part)
  float *dconv_part;            // [BH][R][k]
  int n, d, m, heads, conv_k, R;
  float scale;
};

// Row stride of the 64-column tiles: 16-byte aligned rows, 4 mod 32 words.
constexpr int kLd = 68;

template <int M>
struct RowsSmem {
  // padded fp32 tiles (rows of 16-byte multiples, zero beyond the data); the V halo is only read by the conv gradient, which
  // runs before F and dS_F are formed, so they share their bytes (two
  // blocks per SM at m <= 64)
  static constexpr int LD = kLd, LM = M + 4;
  static constexpr uint32_t kHalo = (kTile + 62) * LD * 4, kFD = 2 * kTile * LM * 4;
  static constexpr uint32_t kt = 0;                            // [M][LD]
  static constexpr uint32_t w = kt + M * LD * 4;               // [M][LD]
  static constexpr uint32_t q = w + M * LD * 4;                // [64][LD]
  static constexpr uint32_t g = q + kTile * LD * 4;            // [64][LD]
  static constexpr uint32_t vh = g + kTile * LD * 4;           // [64 + 62][LD] V halo, or
  static constexpr uint32_t f = vh;                            // [64][LM]
  static constexpr uint32_t ds = f + kTile * LM * 4;           // [64][LM]
  static constexpr uint32_t cw = vh + (kHalo > kFD ? kHalo : kFD);   // [64]
  static constexpr uint32_t dwc = cw + 64 * 4;                 // [64] conv partial
  static constexpr uint32_t cpart = dwc + 64 * 4;              // [64][2] the tile's tap halves
  static constexpr uint32_t total = cpart + 128 * 4;
};

// Taps per thread of the conv gradient: 64 columns x ceil(k / kTapGroup)
// groups fill the block once for k <= 36.
constexpr int kTapGroup = 9;

template <typename T, int M>
__global__ void __launch_bounds__(kThreads, M <= 64 ? 2 : 1) bwd_rows(const RowsParams p) {
  using S = RowsSmem<M>;
  constexpr int LD = S::LD, LM = S::LM;
  constexpr int RM = M / 16;   // landmarks per thread (dW, dK~ rows; F, dF columns)
  extern __shared__ __align__(16) uint8_t smem[];
  float *kt = (float *)(smem + S::kt), *w = (float *)(smem + S::w);
  float *qs = (float *)(smem + S::q), *gs = (float *)(smem + S::g);
  float *fs = (float *)(smem + S::f), *ds = (float *)(smem + S::ds);
  float *vh = (float *)(smem + S::vh), *cw = (float *)(smem + S::cw);
  float *dwc = (float *)(smem + S::dwc), *cpart = (float *)(smem + S::cpart);
  const int blk = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int n = p.n, d = p.d, m = p.m, head = bh % p.heads;
  const int d4 = round4(d), m4 = round4(m);
  const int k = p.conv_w ? p.conv_k : 0, half = (k - 1) / 2;
  const T *Q = (const T *)p.Q + (size_t)bh * n * d;
  const T *V = (const T *)p.V + (size_t)bh * n * d;
  const T *G = (const T *)p.G + (size_t)bh * n * d;
  T *dQ = (T *)p.dQ + (size_t)bh * n * d;
  for (int i = t; i < M * LD; i += kThreads) {
    const int j = i / LD, c = i % LD;
    const bool in = j < m && c < d;
    kt[i] = in ? p.kt[((size_t)bh * m + j) * d + c] : 0.f;
    w[i] = in ? p.w[((size_t)bh * m + j) * d + c] : 0.f;
  }
  if (t < 64) {
    cw[t] = t < k ? p.conv_w[head * k + t] : 0.f;
    dwc[t] = 0.f;
  }
  const int tiles = (n + kTile - 1) / kTile;
  const int tb = (int)((long)blk * tiles / p.R), te = (int)((long)(blk + 1) * tiles / p.R);
  float dW[RM][4], dK[RM][4];
  zero(dW);
  zero(dK);
  for (int tile = tb; tile < te; ++tile) {
    const int r0 = tile * kTile;
    __syncthreads();
    if (sizeof(T) == 2 && (d & 7) == 0) {
      load_tile<LD>(qs, Q, r0, kTile, n, d);
      load_tile<LD>(gs, G, r0, kTile, n, d);
      if (k > 0) load_tile<LD>(vh, V, r0 - half, kTile + k - 1, n, d);
    } else {
      for (int i = t; i < kTile * LD; i += kThreads) {
        const int r = i / LD, c = i % LD, row = r0 + r;
        const bool in = row < n && c < d;
        qs[i] = in ? to_f(Q[(size_t)row * d + c]) : 0.f;
        gs[i] = in ? to_f(G[(size_t)row * d + c]) : 0.f;
      }
      if (k > 0)
        for (int i = t; i < (kTile + k - 1) * LD; i += kThreads) {
          const int r = i / LD, c = i % LD, row = r0 - half + r;
          vh[i] = (row >= 0 && row < n && c < d) ? to_f(V[(size_t)row * d + c]) : 0.f;
        }
    }
    __syncthreads();
    // conv kernel gradient: tap j gets sum_i sum_c dO_i,c V_{i+j-half},c
    // (halo row i + j).  A thread takes one column c and kTapGroup taps
    // j0 ..: down the rows it keeps the halo rows i + j0 .. in a sliding
    // window of registers, so each row costs two loads; a warp's 32 columns
    // are then summed by shuffles, and the two halves of 64 in order.
    if (k > 0) {
      const int hr = kTile + k - 1;   // halo rows loaded
      const int items = ((k + kTapGroup - 1) / kTapGroup) * 64;
      for (int u = t; u < items; u += kThreads) {
        const int j0 = (u >> 6) * kTapGroup, c = u & 63;
        float acc[kTapGroup], win[kTapGroup];
#pragma unroll
        for (int q = 0; q < kTapGroup; ++q) {
          acc[q] = 0.f;
          win[q] = j0 + q < hr ? vh[(j0 + q) * LD + c] : 0.f;
        }
        for (int r = 0; r < kTile; ++r) {
          const float g = gs[r * LD + c];
#pragma unroll
          for (int q = 0; q < kTapGroup; ++q) acc[q] = fmaf(g, win[q], acc[q]);
#pragma unroll
          for (int q = 0; q + 1 < kTapGroup; ++q) win[q] = win[q + 1];
          const int nr = r + j0 + kTapGroup;   // the row entering the window
          win[kTapGroup - 1] = nr < hr ? vh[nr * LD + c] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kTapGroup; ++q) {
          const float v = warp_sum(acc[q]);
          if ((t & 31) == 0 && j0 + q < k) cpart[(j0 + q) * 2 + ((u >> 5) & 1)] = v;
        }
      }
      __syncthreads();   // fs and ds overwrite the halo; cpart complete
      if (t < k) dwc[t] += cpart[2 * t] + cpart[2 * t + 1];
    }
    {   // logits S = Q K~^T (64 x m) into fs, dF = dO W^T into ds
      float a[4][RM];
      zero(a);
      mm_vec<4, RM, false, false>(a, qs, LD, kt, LD, d4);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < RM; ++c) {
          const int col = vec_col<RM, false>(c);
          if (col < m) fs[vec_row<4>(r) * LM + col] = p.scale * a[r][c];
        }
      zero(a);
      mm_vec<4, RM, false, false>(a, gs, LD, w, LD, d4);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < RM; ++c) {
          const int col = vec_col<RM, false>(c);
          if (col < m) ds[vec_row<4>(r) * LM + col] = a[r][c];
        }
    }
    __syncthreads();
    // row softmax of F and dS_F = F (dF - rowsum(dF F)): a warp per row;
    // columns m .. m4 - 1 are zeroed for the products over the landmarks
    {
      const int warp = t >> 5, lane = t & 31;
      for (int r = warp; r < kTile; r += 8) {
        const bool in = r0 + r < n;
        float mx = -INFINITY;
        for (int j = lane; j < m; j += 32) mx = fmaxf(mx, fs[r * LM + j]);
        mx = warp_max(mx);
        float sum = 0.f;
        for (int j = lane; j < m; j += 32) {
          const float e = expf(fs[r * LM + j] - mx);
          fs[r * LM + j] = e;
          sum += e;
        }
        const float inv = 1.f / warp_sum(sum);
        float dot = 0.f;
        for (int j = lane; j < m; j += 32) {
          const float f = fs[r * LM + j] * inv;
          fs[r * LM + j] = in ? f : 0.f;
          dot = fmaf(f, ds[r * LM + j], dot);
        }
        dot = warp_sum(dot);
        for (int j = lane; j < m; j += 32) {
          const float f = fs[r * LM + j];
          ds[r * LM + j] = in ? f * (ds[r * LM + j] - dot) : 0.f;
        }
        for (int j = m + lane; j < m4; j += 32) {
          fs[r * LM + j] = 0.f;
          ds[r * LM + j] = 0.f;
        }
      }
    }
    __syncthreads();
    {   // dQ (F part) = s dS_F K~ (64 x d)
      float a[4][4];
      zero(a);
      mm_vec<4, 4, false, true>(a, ds, LM, kt, LD, m4);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = r0 + vec_row<4>(r), col = vec_col<4, true>(c);
          if (row < n && col < d) dQ[(size_t)row * d + col] = from_f<T>(p.scale * a[r][c]);
        }
    }
    // dW += F^T dO, dK~ += dS_F^T Q (m x d, over the tile's rows)
    mm_vec<RM, 4, true, true>(dW, fs, LM, gs, LD, kTile);
    mm_vec<RM, 4, true, true>(dK, ds, LM, qs, LD, kTile);
  }
  // block partials
  const size_t pb = ((size_t)bh * p.R + blk) * m * d;
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = vec_row<RM>(r), col = vec_col<4, true>(c);
      if (j < m && col < d) {
        p.dw_part[pb + (size_t)j * d + col] = dW[r][c];
        p.dkt_part[pb + (size_t)j * d + col] = p.scale * dK[r][c];
      }
    }
  __syncthreads();
  if (t < k) p.dconv_part[((size_t)bh * p.R + blk) * k + t] = dwc[t];
}

// ---------------------------------------------------------------------------
struct HeadParams {
  const float *dw_part, *dkt_part;   // [BH][R][m][d]
  const float *qt, *kt, *y;          // [BH][m][d]
  const float *a, *zs;               // [BH][m][m], [BH][iters + 1][m][m]
  float *dy, *dqt_a, *dkt;           // [BH][m][d]
  float *dd;                         // [BH][m]: rowsum(dY * Y)
  float *scratch;                    // [BH][head_bytes] when the matrices do not fit smem
  uint32_t *ready;                   // [BH]: set once dY and D of the head are stored
  int publish;                       // 1: set `ready` (0 only in a test of the wait)
  int d, m, iters, R, use_smem;
  float scale;
};

// C = alpha A B (+ beta C) over m x m (or m x d) matrices with row stride
// ld, all in one block; the product runs with every thread (mm_vec: A, B
// stored k-major when AK, BK, else transposed; K4 = the inner size rounded
// up to 4, over zero padding).
template <int RM, int RN, bool AK, bool BK>
__device__ __forceinline__ void mm_block(float *C, int ldc, const float *A, int lda,
                                         const float *B, int ldb, int K4, int M, int N,
                                         float alpha, float beta) {
  float acc[RM][RN];
  zero(acc);
  mm_vec<RM, RN, AK, BK>(acc, A, lda, B, ldb, K4);
  __syncthreads();   // C may alias an operand's previous contents
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int c = 0; c < RN; ++c) {
      const int i = vec_row<RM>(r), j = vec_col<RN, BK>(c);
      if (i < M && j < N) {
        float *o = C + i * ldc + j;
        *o = alpha * acc[r][c] + (beta != 0.f ? beta * *o : 0.f);
      }
    }
  __syncthreads();
}

// sum_{r < R} x[r * stride], added in order of r; four loads in flight.
__device__ __forceinline__ float sum_parts(const float *x, size_t stride, int R) {
  float s = 0.f;
  int r = 0;
  for (; r + 4 <= R; r += 4) {
    const float v0 = x[r * stride], v1 = x[(r + 1) * stride], v2 = x[(r + 2) * stride],
                v3 = x[(r + 3) * stride];
    s += v0;
    s += v1;
    s += v2;
    s += v3;
  }
  for (; r < R; ++r) s += x[r * stride];
  return s;
}

// out[e] = sum_{r < R} x[r * md + e] (+ add[e]) for the elements
// e = t, t + kHeadThreads, ... < md of a bwd_head thread, each added in order
// of r; 16 loads in flight per step.
template <typename Store>
__device__ __forceinline__ void head_sum_parts(const float *x, int md, int R, Store store) {
  constexpr int kE = 8;
  for (int e0 = threadIdx.x; e0 < md; e0 += kE * kHeadThreads) {
    float acc[kE];
#pragma unroll
    for (int i = 0; i < kE; ++i) acc[i] = 0.f;
    int r = 0;
    for (; r + 2 <= R; r += 2) {
      float v0[kE], v1[kE];
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const int e = e0 + i * kHeadThreads;
        v0[i] = e < md ? x[(size_t)r * md + e] : 0.f;
        v1[i] = e < md ? x[(size_t)(r + 1) * md + e] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        acc[i] += v0[i];
        acc[i] += v1[i];
      }
    }
    for (; r < R; ++r)
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const int e = e0 + i * kHeadThreads;
        acc[i] += e < md ? x[(size_t)r * md + e] : 0.f;
      }
#pragma unroll
    for (int i = 0; i < kE; ++i) {
      const int e = e0 + i * kHeadThreads;
      if (e < md) store(e, acc[i]);
    }
  }
}

// dst[(e / cols) * ld + e % cols] = src[e] for e < rows * cols (a row-major
// matrix into the padded layout), by a bwd_head thread; eight loads in
// flight.
__device__ __forceinline__ void head_copy(float *dst, int ld, const float *src, int rows,
                                          int cols) {
  constexpr int kU = 8;
  const int total = rows * cols;
  for (int e0 = threadIdx.x; e0 < total; e0 += kU * kHeadThreads) {
    float v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int e = e0 + u * kHeadThreads;
      v[u] = e < total ? src[e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int e = e0 + u * kHeadThreads;
      if (e < total) dst[(e / cols) * ld + e % cols] = v[u];
    }
  }
}

// Row stride of bwd_head<M>'s matrices: m columns or the d <= 64 columns of
// the m x d ones, plus four (16-byte rows, 4 mod 32 words).
template <int M>
__host__ __device__ constexpr int head_ld() {
  return (M > 64 ? M : 64) + 4;
}

// Bytes of the twelve matrices of bwd_head<M>.
template <int M>
__host__ __device__ constexpr size_t head_bytes() {
  return (size_t)12 * M * head_ld<M>() * 4;
}

template <int M>
__global__ void __launch_bounds__(kHeadThreads) bwd_head(const HeadParams p) {
  // 512 threads: products own rows ty * RR + r (ty < 32) and 16 column
  // threads; m x m outputs take RM columns per thread
  constexpr int RR = M / 32, RM = M / 16;
  extern __shared__ __align__(16) float smem_f[];
  const int bh = blockIdx.x, t = threadIdx.x;
  // twelve M x ld matrices (m <= M rows)
  constexpr int ld = head_ld<M>(), kMat = M * ld;
  const int m = p.m, d = p.d, m4 = round4(m), d4 = round4(d);
  float *base = p.use_smem ? smem_f : p.scratch + (size_t)bh * (head_bytes<M>() / 4);
  float *A = base, *Zj = A + kMat, *P = Zj + kMat, *T1 = P + kMat, *T2 = T1 + kMat,
        *T3 = T2 + kMat, *dZ = T3 + kMat, *dP = dZ + kMat, *dT = dP + kMat,
        *dA = dT + kMat, *X = dA + kMat, *Y2 = X + kMat;
  // every matrix starts zero: rows m .. M - 1 and the columns past its own
  // stay zero, which the products over m4 or d4 terms read
  for (int e = t; e < 12 * kMat; e += kHeadThreads) base[e] = 0.f;
  __syncthreads();
  // X: dW (m x d) then scratch; Y2: Y (m x d)
  const size_t hd = (size_t)bh * m * d;
  head_sum_parts(p.dw_part + (size_t)bh * p.R * m * d, m * d, p.R,
                 [&](int e, float v) { X[(e / d) * ld + e % d] = v; });
  head_copy(Y2, ld, p.y + hd, m, d);
  head_copy(A, ld, p.a + (size_t)bh * m * m, m, m);
  head_copy(Zj, ld, p.zs + ((size_t)bh * (p.iters + 1) + p.iters) * m * m, m, m);
  __syncthreads();
  // dZ = dW Y^T (m x m), dY = Z^T dW (m x d)
  mm_block<RR, RM, false, false>(dZ, ld, X, ld, Y2, ld, d4, m, m, 1.f, 0.f);
  mm_block<RR, 4, true, true>(T1, ld, Zj, ld, X, ld, m4, m, d, 1.f, 0.f);
  for (int e = t; e < m * d; e += kHeadThreads) {
    const int i = e / d, c = e % d;
    p.dy[hd + e] = T1[i * ld + c];
  }
  if (t < m) {   // D_j = dY_j . Y_j
    float s = 0.f;
    for (int c = 0; c < d; ++c) s = fmaf(T1[t * ld + c], Y2[t * ld + c], s);
    p.dd[(size_t)bh * m + t] = s;
  }
  __syncthreads();
  // dY and D are all bwd_keys reads of this kernel's results: publish them,
  // and let bwd_keys start on the SMs this kernel leaves free
  if (t == 0 && p.publish) sm100::flag_release(p.ready + bh, 1u);
  sm100::griddep_launch_dependents();
  // Lemma 1 steps backwards: Z' = 1/4 Z T3, T3 = 13I - P T2, T2 = 15I - P T1,
  // T1 = 7I - P, P = A Z
  for (int j = p.iters - 1; j >= 0; --j) {
    head_copy(Zj, ld, p.zs + ((size_t)bh * (p.iters + 1) + j) * m * m, m, m);
    __syncthreads();
    mm_block<RR, RM, false, true>(P, ld, A, ld, Zj, ld, m4, m, m, 1.f, 0.f);            // P = A Z
    for (int e = t; e < m * m; e += kHeadThreads) {
      const int i = e / m, c = e % m;
      T1[i * ld + c] = (i == c ? 7.f : 0.f) - P[i * ld + c];
    }
    __syncthreads();
    mm_block<RR, RM, false, true>(T2, ld, P, ld, T1, ld, m4, m, m, -1.f, 0.f);          // -P T1
    for (int e = t; e < m * m; e += kHeadThreads) {
      const int i = e / m, c = e % m;
      T2[i * ld + c] += (i == c ? 15.f : 0.f);
    }
    __syncthreads();
    mm_block<RR, RM, false, true>(T3, ld, P, ld, T2, ld, m4, m, m, -1.f, 0.f);          // -P T2
    for (int e = t; e < m * m; e += kHeadThreads) {
      const int i = e / m, c = e % m;
      T3[i * ld + c] += (i == c ? 13.f : 0.f);
    }
    __syncthreads();
    mm_block<RR, RM, true, true>(dT, ld, Zj, ld, dZ, ld, m4, m, m, 0.25f, 0.f);       // dT3 = 1/4 Z^T dZ
    mm_block<RR, RM, false, false>(X, ld, dZ, ld, T3, ld, m4, m, m, 0.25f, 0.f);        // dZ_prev = 1/4 dZ T3^T
    mm_block<RR, RM, false, false>(dP, ld, dT, ld, T2, ld, m4, m, m, -1.f, 0.f);        // dP = -dT3 T2^T
    mm_block<RR, RM, true, true>(T3, ld, P, ld, dT, ld, m4, m, m, -1.f, 0.f);         // dT2 = -P^T dT3
    mm_block<RR, RM, false, false>(dP, ld, T3, ld, T1, ld, m4, m, m, -1.f, 1.f);        // dP -= dT2 T1^T
    mm_block<RR, RM, true, true>(dT, ld, P, ld, T3, ld, m4, m, m, -1.f, 0.f);         // dT1 = -P^T dT2
    for (int e = t; e < m * m; e += kHeadThreads) {
      const int i = e / m, c = e % m;
      dP[i * ld + c] -= dT[i * ld + c];                                          // dP -= dT1
    }
    __syncthreads();
    mm_block<RR, RM, false, false>(dA, ld, dP, ld, Zj, ld, m4, m, m, 1.f, 1.f);         // dA += dP Z^T
    mm_block<RR, RM, true, true>(X, ld, A, ld, dP, ld, m4, m, m, 1.f, 1.f);           // dZ_prev += A^T dP
    for (int e = t; e < m * m; e += kHeadThreads) dZ[(e / m) * ld + e % m] = X[(e / m) * ld + e % m];
    __syncthreads();
  }
  // Z0 = A^T c, c = 1 / (||A||_1 ||A||_inf): gradients through c and the
  // maximising column / row (first index at ties).  Column sums, row sums
  // and the rows of dc = sum_ij dZ_ij A_ji run one per thread, each in index
  // order; one thread then takes the maxima and adds the rows in order.
  __shared__ float red[4];
  __shared__ int arg[2];
  __shared__ float cs[M], rs[M], dcr[M];
  for (int u = t; u < 3 * m; u += kHeadThreads) {
    const int i = u % m;
    float s = 0.f;
    if (u < m) {
      for (int r = 0; r < m; ++r) s += fabsf(A[r * ld + i]);
      cs[i] = s;
    } else if (u < 2 * m) {
      for (int j = 0; j < m; ++j) s += fabsf(A[i * ld + j]);
      rs[i] = s;
    } else {
      for (int j = 0; j < m; ++j) s = fmaf(dZ[i * ld + j], A[j * ld + i], s);
      dcr[i] = s;
    }
  }
  __syncthreads();
  if (t == 0) {
    float n1 = -1.f, ninf = -1.f, dc = 0.f;
    int jc = 0, ir = 0;
    for (int j = 0; j < m; ++j)
      if (cs[j] > n1) { n1 = cs[j]; jc = j; }
    for (int i = 0; i < m; ++i)
      if (rs[i] > ninf) { ninf = rs[i]; ir = i; }
    for (int i = 0; i < m; ++i) dc += dcr[i];
    red[0] = 1.f / (n1 * ninf);
    red[1] = dc;
    red[2] = n1;
    red[3] = ninf;
    arg[0] = jc;
    arg[1] = ir;
  }
  __syncthreads();
  {
    const float c = red[0], dc = red[1], n1 = red[2], ninf = red[3];
    for (int e = t; e < m * m; e += kHeadThreads) {
      const int i = e / m, j = e % m;
      float g = dA[i * ld + j] + c * dZ[j * ld + i];
      if (j == arg[0]) g += -dc * c / n1 * (A[i * ld + j] > 0.f ? 1.f : (A[i * ld + j] < 0.f ? -1.f : 0.f));
      if (i == arg[1]) g += -dc * c / ninf * (A[i * ld + j] > 0.f ? 1.f : (A[i * ld + j] < 0.f ? -1.f : 0.f));
      dA[i * ld + j] = g;
    }
  }
  __syncthreads();
  // softmax backward of A: dS_A = A (dA - rowsum(dA A)), into dP
  if (t < m) {
    float dot = 0.f;
    for (int j = 0; j < m; ++j) dot = fmaf(dA[t * ld + j], A[t * ld + j], dot);
    for (int j = 0; j < m; ++j) dP[t * ld + j] = A[t * ld + j] * (dA[t * ld + j] - dot);
  }
  // Q~, K~ into T1, T2 (m x d)
  head_copy(T1, ld, p.qt + hd, m, d);
  head_copy(T2, ld, p.kt + hd, m, d);
  __syncthreads();
  // dQ~_A = s dS_A K~ ; dK~ = (F part) + s dS_A^T Q~
  mm_block<RR, 4, false, true>(T3, ld, dP, ld, T2, ld, m4, m, d, p.scale, 0.f);
  for (int e = t; e < m * d; e += kHeadThreads) p.dqt_a[hd + e] = T3[(e / d) * ld + e % d];
  mm_block<RR, 4, true, true>(X, ld, dP, ld, T1, ld, m4, m, d, p.scale, 0.f);
  head_sum_parts(p.dkt_part + (size_t)bh * p.R * m * d, m * d, p.R,
                 [&](int e, float v) { p.dkt[hd + e] = v + X[(e / d) * ld + e % d]; });
}

// ---------------------------------------------------------------------------
struct KeysParams {
  const void *K, *V, *G;        // [BH][n][d] (T)
  const float *qt, *dy;         // [BH][m][d]
  const float *lse2, *dd;       // [BH][m]: log2-sum-exp of B~'s scaled logits, rowsum(dY Y)
  const float *conv_w;          // [H][k] or null
  const uint32_t *ready;        // [BH]: bwd_head's flag for dY and D
  uint32_t *err;                // workspace error word
  void *dK, *dV;                // [BH][n][d] (T)
  float *dqt_part;              // [BH][S2][m][d]
  int n, d, m, heads, conv_k, S2;
  float scale, scale_log2;
};

template <int M>
struct KeysSmem {
  // the dO halo is only read by conv^T, which runs (into registers) before
  // B and dS_B are formed, so they share their bytes (two blocks per SM at
  // m <= 64)
  static constexpr int LD = kLd, LK = kLd;
  static constexpr uint32_t kHalo = (kTile + 62) * LD * 4, kBD = 2 * M * LK * 4;
  static constexpr uint32_t qt = 0;                              // [M][LD]
  static constexpr uint32_t dy = qt + M * LD * 4;                // [M][LD]
  static constexpr uint32_t ks = dy + M * LD * 4;                // [64][LD]
  static constexpr uint32_t vs = ks + kTile * LD * 4;            // [64][LD]
  static constexpr uint32_t gh = vs + kTile * LD * 4;            // [64 + 62][LD] dO halo, or
  static constexpr uint32_t b = gh;                              // [M][LK]
  static constexpr uint32_t db = b + M * LK * 4;                 // [M][LK]
  static constexpr uint32_t cw = gh + (kHalo > kBD ? kHalo : kBD);   // [64]
  static constexpr uint32_t lse = cw + 64 * 4;                   // [M]
  static constexpr uint32_t dd = lse + M * 4;                    // [M]
  static constexpr uint32_t total = dd + M * 4;
};

template <typename T, int M>
__global__ void __launch_bounds__(kThreads, M <= 64 ? 2 : 1) bwd_keys(const KeysParams p) {
  using S = KeysSmem<M>;
  constexpr int LD = S::LD, LK = S::LK, RM = M / 16;
  extern __shared__ __align__(16) uint8_t smem[];
  float *qt = (float *)(smem + S::qt), *dy = (float *)(smem + S::dy);
  float *ks = (float *)(smem + S::ks), *vs = (float *)(smem + S::vs);
  float *bs = (float *)(smem + S::b), *dbs = (float *)(smem + S::db);
  float *gh = (float *)(smem + S::gh);
  float *cw = (float *)(smem + S::cw), *lse = (float *)(smem + S::lse);
  float *ddv = (float *)(smem + S::dd);
  const int blk = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int n = p.n, d = p.d, m = p.m, head = bh % p.heads;
  const int d4 = round4(d), m4 = round4(m);
  const int k = p.conv_w ? p.conv_k : 0, half = (k - 1) / 2;
  const T *K = (const T *)p.K + (size_t)bh * n * d;
  const T *V = (const T *)p.V + (size_t)bh * n * d;
  const T *G = (const T *)p.G + (size_t)bh * n * d;
  T *dK = (T *)p.dK + (size_t)bh * n * d;
  T *dV = (T *)p.dV + (size_t)bh * n * d;
  const size_t hd = (size_t)bh * m * d;
  // this kernel may start while bwd_head runs: wait (bounded) for the head's
  // dY and D; on a timeout (recorded in the error word) the block leaves
  __shared__ uint32_t abort_flag;
  if (t == 0) {
    abort_flag = 0u;
    const sm100::Abort ab{&abort_flag, p.err};
    sm100::flag_wait(p.ready + bh, ab, sm100::kWaitLimitCycles);
  }
  __syncthreads();
  if (abort_flag) {
    if (t == 0) sm100::griddep_wait();
    return;
  }
  for (int i = t; i < M * LD; i += kThreads) {
    const int j = i / LD, c = i % LD;
    const bool in = j < m && c < d;
    qt[i] = in ? p.qt[hd + j * d + c] : 0.f;
    dy[i] = in ? p.dy[hd + j * d + c] : 0.f;
  }
  if (t < 64) cw[t] = t < k ? p.conv_w[head * k + t] : 0.f;
  for (int j = t; j < M; j += kThreads) {
    lse[j] = j < m ? p.lse2[(size_t)bh * m + j] : 0.f;
    ddv[j] = j < m ? p.dd[(size_t)bh * m + j] : 0.f;
  }
  const int tiles = (n + kTile - 1) / kTile;
  const int tb = (int)((long)blk * tiles / p.S2), te = (int)((long)(blk + 1) * tiles / p.S2);
  float dq[RM][4];
  zero(dq);
  for (int tile = tb; tile < te; ++tile) {
    const int k0 = tile * kTile;
    __syncthreads();
    load_tile<LD>(ks, K, k0, kTile, n, d);
    load_tile<LD>(vs, V, k0, kTile, n, d);
    if (k > 0)   // dO rows k0 + half - (k - 1) .. k0 + 63 + half: conv^T
      load_tile<LD>(gh, G, k0 + half - (k - 1), kTile + k - 1, n, d);
    __syncthreads();
    // conv^T(dO) for the tile's dV outputs (key vec_row<4>(r), column
    // vec_col<4, true>(c)): dV_row += w[tp] dO[row - tp + half]
    float cv[4][4];
    zero(cv);
    if (k > 0) {
      for (int tp = 0; tp < k; ++tp) {
        const float wt = cw[tp];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          float g[4];
          ld_vec<4>(g, gh + (vec_row<4>(r) + (k - 1) - tp) * LD + vec_col<4, true>(0));
#pragma unroll
          for (int c = 0; c < 4; ++c) cv[r][c] = fmaf(wt, g[c], cv[r][c]);
        }
      }
      __syncthreads();   // bs and dbs overwrite the halo
    }
    {   // B = 2^(s log2e Q~ K^T - lse) (m x 64), dB = dY V^T; rows m .. M - 1
        // zeroed for the products over the landmarks
      float a[RM][4], b[RM][4];
      zero(a);
      zero(b);
      mm_vec<RM, 4, false, false>(a, qt, LD, ks, LD, d4);
      mm_vec<RM, 4, false, false>(b, dy, LD, vs, LD, d4);
#pragma unroll
      for (int r = 0; r < RM; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = vec_row<RM>(r), key = vec_col<4, false>(c);
          float bv = 0.f, dbv = 0.f;
          if (j < m) {
            bv = (k0 + key < n) ? exp2f(a[r][c] * p.scale_log2 - lse[j]) : 0.f;
            dbv = bv * (b[r][c] - ddv[j]);   // dS_B
          }
          bs[j * LK + key] = bv;
          dbs[j * LK + key] = dbv;
        }
    }
    __syncthreads();
    {   // dK = s dS_B^T Q~ (bwd_dqk adds dK~_seg / count) ; dV = B^T dY + conv^T(dO)
      float a[4][4], b[4][4];
      zero(a);
      zero(b);
      mm_vec<4, 4, true, true>(a, dbs, LK, qt, LD, m4);
      mm_vec<4, 4, true, true>(b, bs, LK, dy, LD, m4);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = vec_col<4, true>(c), row = k0 + vec_row<4>(r);
          if (row < n && col < d) {
            dK[(size_t)row * d + col] = from_f<T>(p.scale * a[r][c]);
            dV[(size_t)row * d + col] = from_f<T>(b[r][c] + cv[r][c]);
          }
        }
    }
    // dQ~ += s dS_B K (m x d, over the tile's keys)
    mm_vec<RM, 4, false, true>(dq, dbs, LK, ks, LD, kTile);
  }
  const size_t pb = ((size_t)bh * p.S2 + blk) * m * d;
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = vec_row<RM>(r), col = vec_col<4, true>(c);
      if (j < m && col < d) p.dqt_part[pb + (size_t)j * d + col] = p.scale * dq[r][c];
    }
  // complete only after bwd_head, whose other results the next kernels read
  if (t == 0) sm100::griddep_wait();
}

// ---------------------------------------------------------------------------
// dQ~ = dQ~_A + the key blocks' partials in order, in place of dQ~_A: one
// thread per element of the head's m x d matrix.
__global__ void __launch_bounds__(kThreads)
bwd_dqt_total(float *dqt, const float *dqt_part, int md, int S2) {
  const int bh = blockIdx.y, e = blockIdx.x * kThreads + threadIdx.x;
  if (e >= md) return;
  const float s = sum_parts(dqt_part + (size_t)bh * S2 * md + e, (size_t)md, S2);
  dqt[(size_t)bh * md + e] += s;
}

// dQ += dQ~_{seg(i)} / count and dK += dK~_{seg(i)} / count over the block's
// rows: the m x d quotients once into shared memory, then thread t takes
// column t % 64 of every fourth row (d <= 64).
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_dqk(void *dQv, void *dKv, const float *dqt, const float *dkt, int n, int d, int m,
        int rows_per_block) {
  extern __shared__ float quot[];   // [2][m][d]
  float *dq = quot, *dk = quot + m * d;
  const int bh = blockIdx.y, t = threadIdx.x;
  const size_t hd = (size_t)bh * m * d;
  const int l = (n + m - 1) / m;
  for (int e0 = t; e0 < m * d; e0 += 4 * kThreads) {   // four elements' loads in flight
    float vq[4], vk[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * kThreads;
      vq[u] = e < m * d ? dqt[hd + e] : 0.f;
      vk[u] = e < m * d ? dkt[hd + e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * kThreads;
      if (e < m * d) {
        const float cnt = (float)seg_count(e / d, l, n);
        dq[e] = vq[u] / cnt;
        dk[e] = vk[u] / cnt;
      }
    }
  }
  __syncthreads();
  T *dQ = (T *)dQv + (size_t)bh * n * d;
  T *dK = (T *)dKv + (size_t)bh * n * d;
  const int r0 = blockIdx.x * rows_per_block, r1 = min(n, r0 + rows_per_block);
  if constexpr (sizeof(T) == 2) {
    if ((d & 7) == 0) {   // bf16 rows of 16-byte chunks: eight values per load
      const int cpr = d >> 3;
      constexpr int kU = 4;
      for (int u0 = t; u0 < (r1 - r0) * cpr; u0 += kU * kThreads) {
        uint4 vq[kU], vk[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i = u0 + u * kThreads, row = r0 + i / cpr, c8 = (i % cpr) * 8;
          vq[u] = vk[u] = make_uint4(0u, 0u, 0u, 0u);
          if (row < r1) {
            vq[u] = *reinterpret_cast<const uint4 *>(dQ + (size_t)row * d + c8);
            vk[u] = *reinterpret_cast<const uint4 *>(dK + (size_t)row * d + c8);
          }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i = u0 + u * kThreads, row = r0 + i / cpr, c8 = (i % cpr) * 8;
          if (row >= r1) continue;
          const int q = seg_of(row, l) * d + c8;
          __nv_bfloat162 *hq = reinterpret_cast<__nv_bfloat162 *>(&vq[u]);
          __nv_bfloat162 *hk = reinterpret_cast<__nv_bfloat162 *>(&vk[u]);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 a = __bfloat1622float2(hq[h]), b = __bfloat1622float2(hk[h]);
            hq[h] = __floats2bfloat162_rn(a.x + dq[q + 2 * h], a.y + dq[q + 2 * h + 1]);
            hk[h] = __floats2bfloat162_rn(b.x + dk[q + 2 * h], b.y + dk[q + 2 * h + 1]);
          }
          *reinterpret_cast<uint4 *>(dQ + (size_t)row * d + c8) = vq[u];
          *reinterpret_cast<uint4 *>(dK + (size_t)row * d + c8) = vk[u];
        }
      }
      return;
    }
  }
  const int c = t & 63;
  if (c >= d) return;
  constexpr int kStep = kThreads / 64, kU = 8;   // rows per pass; passes in flight
  for (int row0 = r0 + (t >> 6); row0 < r1; row0 += kStep * kU) {
    float gq[kU], gk[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int row = row0 + u * kStep;
      const size_t o = (size_t)row * d + c;
      gq[u] = row < r1 ? to_f(dQ[o]) : 0.f;
      gk[u] = row < r1 ? to_f(dK[o]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int row = row0 + u * kStep;
      if (row < r1) {
        const size_t o = (size_t)row * d + c;
        const int q = seg_of(row, l) * d + c;
        dQ[o] = from_f<T>(gq[u] + dq[q]);
        dK[o] = from_f<T>(gk[u] + dk[q]);
      }
    }
  }
}

// dconv[h][t] = sum over batch elements b (in order) of the row blocks'
// partials (in order).
__global__ void bwd_dconv(float *dconv, const float *part, int batch, int heads, int R, int k) {
  const int h = blockIdx.x, t = threadIdx.x;
  if (t >= k) return;
  float s = 0.f;
  for (int b = 0; b < batch; ++b)
    for (int r = 0; r < R; ++r) s += part[(((size_t)b * heads + h) * R + r) * k + t];
  dconv[h * k + t] = s;
}

}  // namespace bwd
}  // namespace nys
