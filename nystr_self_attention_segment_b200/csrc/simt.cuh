// SIMT kernels of the Nystrom forward: the fp32 path (any head_dim <= 64,
// m <= 64) and the generic building blocks shared with the bf16 path
// (segment means, the split merge and W = Z Y).
//
// Method: "Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4 -- Eq. 16 (segment means), Lemma 1 and its
// initialisation (pseudoinverse), Eq. 17 / Algorithm 1 (the three softmax
// kernels and the product chain), Figure 4 (DConv skip on V).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace nys {

// Tokens of element bh / heads: its own length for ragged batches (lens, one
// per batch element, on the device), else n.  A length outside [m, n] or with
// an empty segment reads as 0 (the element's output is all zero) and records
// NYS_ERR_INVALID_ARG.
__device__ __forceinline__ int seq_len_of(const int *lens, int bh, int heads, int n, int m,
                                          uint32_t *err) {
  if (!lens) return n;
  const int L = lens[bh / heads];
  if (L < m || L > n || (long)(m - 1) * ((L + m - 1) / m) >= L) {
    set_error(err, NYS_ERR_INVALID_ARG);
    return 0;
  }
  return L;
}

// ---------------------------------------------------------------------------
// Segment means (Eq. 16, mean over l = ceil(L/m) contiguous tokens, L the
// element's length).  One thread per (head, landmark, feature); blockIdx.y
// selects Q (0) or K (1).  Sums in fp32 in token order, then divides by the
// segment's real tokens.
template <typename T>
__global__ void seg_means_scalar(const T *__restrict__ Q, const T *__restrict__ K,
                                 float *__restrict__ Qt, float *__restrict__ Kt, int BH, int n,
                                 int d, int m, const int *lens, int heads, uint32_t *err) {
  const T *X = blockIdx.y == 0 ? Q : K;
  float *Xt = blockIdx.y == 0 ? Qt : Kt;
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  long total = (long)BH * m * d;
  if (idx >= total) return;
  int c = (int)(idx % d);
  long jb = idx / d;            // bh * m + j
  int j = (int)(jb % m);
  long bh = jb / m;
  const int L = seq_len_of(lens, (int)bh, heads, n, m, err);
  if (L == 0) return;
  const int len = (L + m - 1) / m;            // l = ceil(L / m)
  const int seg = min(len, L - j * len);      // real tokens of segment j (>= 1)
  const T *src = X + ((size_t)bh * n + (size_t)j * len) * d + c;
  float acc = 0.f;
  for (int t = 0; t < seg; ++t) acc += to_f(src[(size_t)t * d]);
  Xt[idx] = acc / (float)seg;
}

// ---------------------------------------------------------------------------
// dst[r * LD + c] = X[row0 + r][c] as fp32 for r < rows, c < LD: zero for
// rows outside [0, n) and columns past d.  bf16 rows of a multiple of 8
// features (16-byte aligned: the inputs are) move as 16-byte loads of eight
// values; otherwise eight scalar loads in flight per thread.
template <int LD, int kThreads = 256, typename T>
__device__ __forceinline__ void load_tile(float *dst, const T *X, int row0, int rows, int n,
                                          int d) {
  if constexpr (sizeof(T) == 2) {
    if ((d & 7) == 0) {
      const int cpr = d >> 3, total = rows * cpr;   // 16-byte chunks per row, in all
      for (int u = threadIdx.x; u < total; u += kThreads) {
        const int r = u / cpr, c8 = (u - r * cpr) * 8, row = row0 + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row >= 0 && row < n) v = *reinterpret_cast<const uint4 *>(X + (size_t)row * d + c8);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
        float4 lo, hi;
        float2 f;
        f = __bfloat1622float2(h[0]); lo.x = f.x; lo.y = f.y;
        f = __bfloat1622float2(h[1]); lo.z = f.x; lo.w = f.y;
        f = __bfloat1622float2(h[2]); hi.x = f.x; hi.y = f.y;
        f = __bfloat1622float2(h[3]); hi.z = f.x; hi.w = f.y;
        *reinterpret_cast<float4 *>(dst + r * LD + c8) = lo;
        *reinterpret_cast<float4 *>(dst + r * LD + c8 + 4) = hi;
      }
      for (int u = threadIdx.x; u < rows * (LD - d); u += kThreads) {   // the padding
        const int r = u / (LD - d);
        dst[r * LD + d + (u - r * (LD - d))] = 0.f;
      }
      return;
    }
  }
  constexpr int kU = 8;
  const int total = rows * LD;
  for (int i0 = threadIdx.x; i0 < total; i0 += kU * kThreads) {
    float v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kThreads, r = i / LD, c = i % LD, row = row0 + r;
      v[u] = (i < total && row >= 0 && row < n && c < d) ? to_f(X[(size_t)row * d + c]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kThreads;
      if (i < total) dst[i] = v[u];
    }
  }
}

// ---------------------------------------------------------------------------
// Register-tiled block product on 256 threads: acc[r][c] += sum_k A(i, k)
// B(k, j) for the outputs this thread owns, i = ty + 16 r, j = tx + 16 c
// (ty = t / 16, tx = t % 16), i < M, j < N, terms added in order of k.
// A(i, k) = A[i * sai + k * sak], B(k, j) = B[k * sbk + j * sbj].
template <int RM, int RN>
__device__ __forceinline__ void mm_acc(float (&acc)[RM][RN], const float *A, int sai, int sak,
                                       const float *B, int sbk, int sbj, int K, int M, int N) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    float a[RM], b[RN];
#pragma unroll
    for (int r = 0; r < RM; ++r) {
      const int i = ty + 16 * r;
      a[r] = i < M ? A[i * sai + k * sak] : 0.f;
    }
#pragma unroll
    for (int c = 0; c < RN; ++c) {
      const int j = tx + 16 * c;
      b[c] = j < N ? B[k * sbk + j * sbj] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < RN; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
  }
}

// ---------------------------------------------------------------------------
// The same product from 16-byte shared-memory loads, for operands whose rows
// are 16-byte aligned (row strides a multiple of 4 floats) and zero-padded
// to K4, a multiple of 4.  Thread (ty, tx) owns rows ty * RM + r and
// columns tx * RN + c when B is stored k-major (B(k, j) = B[k * ldb + j]),
// else tx + 16 c (B(k, j) = B[j * ldb + k]); A(i, k) = A[k * lda + i] when
// A is stored k-major, else A[i * lda + k].  Each k-step then costs one
// load of A's rows and one of B's columns; a row stride of 4 mod 32 words
// keeps the strided forms to the minimum number of bank wavefronts.
template <int N>
__device__ __forceinline__ void ld_vec(float (&v)[N], const float *p) {
  if constexpr (N == 1) {
    v[0] = p[0];
  } else if constexpr (N == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(p);
    v[0] = x.x, v[1] = x.y;
  } else {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 x = *reinterpret_cast<const float4 *>(p + 4 * q);
      v[4 * q] = x.x, v[4 * q + 1] = x.y, v[4 * q + 2] = x.z, v[4 * q + 3] = x.w;
    }
  }
}

template <int RM, int RN, bool AK, bool BK>
__device__ __forceinline__ void mm_vec(float (&acc)[RM][RN], const float *A, int lda,
                                       const float *B, int ldb, int K4) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const float *a0 = AK ? A + ty * RM : A + ty * RM * lda;
  const float *b0 = BK ? B + tx * RN : B + tx * ldb;
  for (int k = 0; k < K4; k += 4) {
    float a[4][RM], b[4][RN];
    if constexpr (AK) {
#pragma unroll
      for (int q = 0; q < 4; ++q) ld_vec<RM>(a[q], a0 + (k + q) * lda);
    } else {
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        const float4 x = *reinterpret_cast<const float4 *>(a0 + r * lda + k);
        a[0][r] = x.x, a[1][r] = x.y, a[2][r] = x.z, a[3][r] = x.w;
      }
    }
    if constexpr (BK) {
#pragma unroll
      for (int q = 0; q < 4; ++q) ld_vec<RN>(b[q], b0 + (k + q) * ldb);
    } else {
#pragma unroll
      for (int c = 0; c < RN; ++c) {
        const float4 x = *reinterpret_cast<const float4 *>(b0 + 16 * c * ldb + k);
        b[0][c] = x.x, b[1][c] = x.y, b[2][c] = x.z, b[3][c] = x.w;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int r = 0; r < RM; ++r)
#pragma unroll
        for (int c = 0; c < RN; ++c) acc[r][c] = fmaf(a[q][r], b[q][c], acc[r][c]);
  }
}

// The output row and column that mm_vec<RM, RN, *, BK> accumulates in
// acc[r][c].
template <int RM>
__device__ __forceinline__ int vec_row(int r) {
  return (threadIdx.x >> 4) * RM + r;
}
template <int RN, bool BK>
__device__ __forceinline__ int vec_col(int c) {
  return BK ? (threadIdx.x & 15) * RN + c : (threadIdx.x & 15) + 16 * c;
}

// k rounded up to a multiple of 4
__host__ __device__ constexpr int round4(int k) { return (k + 3) & ~3; }

// ---------------------------------------------------------------------------
// Landmark kernel A = softmax(Q~ K~^T / sqrt(d)) and its pseudoinverse by
// Lemma 1 as printed: Z <- 1/4 Z (13I - AZ (15I - AZ (7I - AZ))), from
// Z0 = A^T / (||A||_1 ||A||_inf).  One block of 256 threads per head; all
// five m x m fp32 matrices live in `mats` (shared memory when it fits, else
// the per-head workspace scratch), each 16 RM rows (m <= 16 RM) of stride
// 16 RM + 4, zero past row and column m: the products read whole rows and
// columns of their 16 RM x 16 RM tiles.
template <int RM>
__host__ __device__ constexpr int pinv_ld() {
  return 16 * RM + 4;
}

// bytes of pinv_simt<RM>'s five matrices
template <int RM>
__host__ __device__ constexpr size_t pinv_mats_bytes() {
  return (size_t)5 * 16 * RM * pinv_ld<RM>() * 4;
}

// C = X Y (m x m, row stride ld), register-tiled on mm_vec: each output adds
// its terms in index order with fmaf.
template <int RM>
__device__ __forceinline__ void block_gemm(float *C, const float *X, const float *Y, int m) {
  constexpr int ld = pinv_ld<RM>(), RR = RM;
  float acc[RR][RM];
#pragma unroll
  for (int r = 0; r < RR; ++r)
#pragma unroll
    for (int c = 0; c < RM; ++c) acc[r][c] = 0.f;
  mm_vec<RR, RM, false, true>(acc, X, ld, Y, ld, round4(m));
#pragma unroll
  for (int r = 0; r < RR; ++r)
#pragma unroll
    for (int c = 0; c < RM; ++c) {
      const int i = vec_row<RR>(r), j = vec_col<RM, true>(c);
      if (i < m && j < m) C[i * ld + j] = acc[r][c];
    }
  __syncthreads();
}

// dst = c I - src (m x m, row stride ld)
__device__ __forceinline__ void block_diag_minus(float *dst, const float *src, float c, int m,
                                                 int ld) {
  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
    const int i = idx / m, j = idx % m;
    dst[i * ld + j] = (i == j ? c : 0.f) - src[i * ld + j];
  }
  __syncthreads();
}

// a_out, z_all (optional, for the backward pass): A [BH][m][m] and every
// iterate Z0 .. Z_iters [BH][iters + 1][m][m].
template <int RM>   // m <= 16 RM
__global__ void __launch_bounds__(256)
pinv_simt(const float *__restrict__ Qt, const float *__restrict__ Kt, float *__restrict__ Zout,
          float *__restrict__ scratch, int m, int d, float scale, int iters, int use_smem,
          float *__restrict__ a_out = nullptr, float *__restrict__ z_all = nullptr) {
  extern __shared__ __align__(16) float smem[];
  constexpr int ld = pinv_ld<RM>();
  const int bh = blockIdx.x, t = threadIdx.x;
  constexpr int mm = 16 * RM * ld;
  // all five in shared memory, or (m > 64) A and Z in the scratch and the
  // three the products write in shared memory
  float *mats = use_smem ? smem : scratch + (size_t)bh * (pinv_mats_bytes<RM>() / 4);
  float *A = mats, *Z = A + mm;
  float *P = use_smem ? Z + mm : smem, *T1 = P + mm, *T2 = T1 + mm;
  __shared__ float red[2];
  __shared__ float nsum[2 * 16 * RM];   // column sums, then row sums
  const float *qt = Qt + (size_t)bh * m * d;
  const float *kt = Kt + (size_t)bh * m * d;
  // the B~ V partials that follow read nothing of this kernel: they may run
  // beside it (programmatic launch)
  sm100::griddep_launch_dependents();
  for (int e = t; e < 2 * mm; e += blockDim.x) A[e] = 0.f;   // A, Z
  for (int e = t; e < 3 * mm; e += blockDim.x) P[e] = 0.f;   // P, T1, T2
  __syncthreads();
  {   // logits, each a dot product over the features in order: thread
      // (ty, tx) = (t / 16, t % 16) takes rows ty + 16 r, columns tx + 16 c
    constexpr int RR = RM;
    const int ty = t >> 4, tx = t & 15;
    float acc[RR][RM];
#pragma unroll
    for (int r = 0; r < RR; ++r)
#pragma unroll
      for (int c = 0; c < RM; ++c) acc[r][c] = 0.f;
    for (int k = 0; k < d; ++k) {
      float a[RR], b[RM];
#pragma unroll
      for (int r = 0; r < RR; ++r) a[r] = ty + 16 * r < m ? qt[(ty + 16 * r) * d + k] : 0.f;
#pragma unroll
      for (int c = 0; c < RM; ++c) b[c] = tx + 16 * c < m ? kt[(tx + 16 * c) * d + k] : 0.f;
#pragma unroll
      for (int r = 0; r < RR; ++r)
#pragma unroll
        for (int c = 0; c < RM; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
#pragma unroll
    for (int r = 0; r < RR; ++r)
#pragma unroll
      for (int c = 0; c < RM; ++c) {
        const int i = ty + 16 * r, j = tx + 16 * c;
        if (i < m && j < m) A[i * ld + j] = acc[r][c] * scale;
      }
  }
  __syncthreads();
  {   // row softmax, a warp per row
    const int warp = t >> 5, lane = t & 31, warps = blockDim.x >> 5;
    for (int i = warp; i < m; i += warps) {
      float mx = -INFINITY;
      for (int j = lane; j < m; j += 32) mx = fmaxf(mx, A[i * ld + j]);
      mx = warp_max(mx);
      float s = 0.f;
      for (int j = lane; j < m; j += 32) {
        const float e = __expf(A[i * ld + j] - mx);
        A[i * ld + j] = e;
        s += e;
      }
      const float inv = 1.f / warp_sum(s);
      for (int j = lane; j < m; j += 32) A[i * ld + j] *= inv;
    }
  }
  __syncthreads();
  // ||A||_1 (max column sum) and ||A||_inf (max row sum): each sum in index
  // order by its own thread, the maxima in order by one thread, so the
  // result is deterministic.
  for (int u = t; u < 2 * m; u += blockDim.x) {
    float s = 0.f;
    if (u < m) {
      for (int i = 0; i < m; ++i) s += fabsf(A[i * ld + u]);
    } else {
      for (int j = 0; j < m; ++j) s += fabsf(A[(u - m) * ld + j]);
    }
    nsum[u] = s;
  }
  __syncthreads();
  if (t == 0) {
    float n1 = 0.f, ninf = 0.f;
    for (int j = 0; j < m; ++j) n1 = fmaxf(n1, nsum[j]);
    for (int i = 0; i < m; ++i) ninf = fmaxf(ninf, nsum[m + i]);
    red[0] = 1.f / (n1 * ninf);
  }
  __syncthreads();
  const float c0 = red[0];
  for (int idx = t; idx < m * m; idx += blockDim.x) {
    const int i = idx / m, j = idx % m;
    Z[i * ld + j] = A[j * ld + i] * c0;
    if (a_out) a_out[(size_t)bh * m * m + idx] = A[i * ld + j];
    if (z_all) z_all[(size_t)bh * (iters + 1) * m * m + idx] = A[j * ld + i] * c0;
  }
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    block_gemm<RM>(P, A, Z, m);               // AZ
    block_diag_minus(T1, P, 7.f, m, ld);      // 7I - AZ
    block_gemm<RM>(T2, P, T1, m);             // AZ (7I - AZ)
    block_diag_minus(T1, T2, 15.f, m, ld);    // 15I - ...
    block_gemm<RM>(T2, P, T1, m);             // AZ (15I - ...)
    block_diag_minus(T1, T2, 13.f, m, ld);    // 13I - ...
    block_gemm<RM>(T2, Z, T1, m);             // Z (13I - ...)
    for (int idx = t; idx < m * m; idx += blockDim.x) {
      const int i = idx / m, j = idx % m;
      Z[i * ld + j] = 0.25f * T2[i * ld + j];
      if (z_all)
        z_all[((size_t)bh * (iters + 1) + it + 1) * m * m + idx] = 0.25f * T2[i * ld + j];
    }
    __syncthreads();
  }
  float *zo = Zout + (size_t)bh * m * m;
  for (int idx = t; idx < m * m; idx += blockDim.x) zo[idx] = Z[(idx / m) * ld + idx % m];
}

// pinv_simt for m landmarks (m <= 128), and the bytes of its matrices
inline auto pinv_simt_for(int m) {
  return m <= 32 ? pinv_simt<2> : (m <= 64 ? pinv_simt<4> : pinv_simt<8>);
}
// dynamic shared memory of pinv_simt for m landmarks: all five matrices for
// m <= 64, else the three the products write
inline size_t pinv_simt_smem(int m) {
  return m <= 32 ? pinv_mats_bytes<2>() : (m <= 64 ? pinv_mats_bytes<4>() : pinv_mats_bytes<8>() / 5 * 3);
}
inline size_t pinv_simt_mats_bytes(int m) {
  return m <= 32 ? pinv_mats_bytes<2>() : (m <= 64 ? pinv_mats_bytes<4>() : pinv_mats_bytes<8>());
}

// ---------------------------------------------------------------------------
// B~ V over one split of the keys (Eq. 17): for every landmark row j, an
// online softmax over the split's keys of s * q~_j . k_i, keeping the running
// maximum (log2 units), the running sum and the unnormalised sum of p_i v_i.
// Grid (splits, heads), 256 threads; per 64-key tile the logits and the
// P V product run register-tiled on mm_vec (thread (ty, tx) owns rows
// ty * RM + r, keys tx + 16 c and features tx * 4 + c), and the 16 threads
// of a row reduce its tile maximum and sum by shuffles.
constexpr int kSimtKeyTile = 64;
constexpr int kSimtLd = 68;   // row stride of the tiles (d <= 64 or 64 keys): 16-byte rows

template <int RM>   // m <= 16 RM
__host__ __device__ constexpr size_t bv_partial_smem() {
  return (size_t)(2 * 16 * RM + 2 * kSimtKeyTile) * kSimtLd * 4;
}

template <typename T, int RM>   // m <= 16 RM
__global__ void __launch_bounds__(256)
bv_partial_simt(const float *__restrict__ Qt, const T *__restrict__ K, const T *__restrict__ V,
                float *__restrict__ pmax, float *__restrict__ psum, float *__restrict__ py,
                int n, int d, int m, int splits, int keys_per_split, float scale_log2,
                const int *lens, int heads) {
  constexpr int LD = kSimtLd, kT = kSimtKeyTile;
  extern __shared__ __align__(16) float smem[];
  const int split = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int tx = t & 15, d4 = round4(d);
  float *qs = smem;                 // [16 RM][LD] Q~ rows
  float *ks = qs + 16 * RM * LD;    // [64][LD]
  float *vs = ks + kT * LD;         // [64][LD]
  float *ps = vs + kT * LD;         // [16 RM][LD] the tile's p (row j, key)
  for (int i = t; i < 16 * RM * LD; i += 256) {
    const int j = i / LD, c = i % LD;
    qs[i] = (j < m && c < d) ? Qt[((size_t)bh * m + j) * d + c] : 0.f;
  }
  float Mx[RM], Sm[RM], y[RM][4];
#pragma unroll
  for (int r = 0; r < RM; ++r) {
    Mx[r] = -INFINITY;
    Sm[r] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) y[r][c] = 0.f;
  }
  // keys of the element: [0, L) (an invalid length reads as 0: no keys)
  const int L = seq_len_of(lens, bh, heads, n, m, nullptr);
  const int k0 = split * keys_per_split;
  const int k1 = min(L, k0 + keys_per_split);
  const T *Kh = K + (size_t)bh * n * d;
  const T *Vh = V + (size_t)bh * n * d;
  for (int t0 = k0; t0 < k1; t0 += kT) {
    __syncthreads();
    load_tile<LD>(ks, Kh, t0, kT, k1, d);   // keys t0 .. t0 + 63, zero from k1 on
    load_tile<LD>(vs, Vh, t0, kT, k1, d);
    __syncthreads();
    float sc[RM][4];
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) sc[r][c] = 0.f;
    mm_vec<RM, 4, false, false>(sc, qs, LD, ks, LD, d4);
#pragma unroll
    for (int r = 0; r < RM; ++r) {
      float l2[4], mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        l2[c] = t0 + tx + 16 * c < k1 ? sc[r][c] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, l2[c]);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mnew = fmaxf(Mx[r], mx);     // finite: the tile's first key is in range
      const float alpha = exp2f(Mx[r] - mnew);  // 0 when Mx was -inf
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = exp2f(l2[c] - mnew);
        ps[vec_row<RM>(r) * LD + vec_col<4, false>(c)] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      Sm[r] = Sm[r] * alpha + sum;
      Mx[r] = mnew;
#pragma unroll
      for (int c = 0; c < 4; ++c) y[r][c] *= alpha;
    }
    __syncthreads();
    mm_vec<RM, 4, false, true>(y, ps, LD, vs, LD, kT);
  }
  const size_t base = ((size_t)bh * splits + split) * m;
#pragma unroll
  for (int r = 0; r < RM; ++r) {
    const int j = vec_row<RM>(r);
    if (j >= m) continue;
    if (tx == 0) {
      pmax[base + j] = Mx[r];
      psum[base + j] = Sm[r];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = vec_col<4, true>(c);
      if (col < d) py[(base + j) * d + col] = y[r][c];
    }
  }
  // launched beside pinv_simt: complete only after it, whose Z the merge
  // reads
  if (t == 0) sm100::griddep_wait();
}

// bv_partial_simt for m landmarks (m <= 128)
template <typename T>
inline auto bv_partial_simt_for(int m) {
  return m <= 32 ? bv_partial_simt<T, 2> : (m <= 64 ? bv_partial_simt<T, 4> : bv_partial_simt<T, 8>);
}
inline size_t bv_partial_simt_smem(int m) {
  return m <= 32 ? bv_partial_smem<2>() : (m <= 64 ? bv_partial_smem<4>() : bv_partial_smem<8>());
}

// ---------------------------------------------------------------------------
// Merge of the key splits in split order (Y = B~ V), then W = Z Y.  Grid
// (heads, column blocks of kMergeCols): a thread per landmark row takes the
// row's maximum and split weights, every output of the block's columns then
// adds its splits in order, and W's columns follow from Z and those of Y.
constexpr int kMergeCols = 16;

inline size_t merge_w_smem(int m, int d, int splits) {
  (void)d;
  return ((size_t)m * kMergeCols + (size_t)m * m + 2 * (size_t)splits * m + m) * 4;
}

__global__ void __launch_bounds__(256)
merge_w_simt(const float *__restrict__ pmax, const float *__restrict__ psum,
             const float *__restrict__ py, const float *__restrict__ Zg, float *__restrict__ Yg,
             float *__restrict__ Wg, int m, int d, int splits, float *__restrict__ lse2 = nullptr) {
  extern __shared__ float smem[];
  const int bh = blockIdx.x, c0 = blockIdx.y * kMergeCols, t = threadIdx.x;
  const int nc = min(kMergeCols, d - c0);
  float *ys = smem;                    // [m][kMergeCols]
  float *zs = ys + m * kMergeCols;     // [m][m]
  float *fac = zs + m * m;             // [splits][m]: the split maxima, then 2^(max_s - max)
  float *sms = fac + splits * m;       // [splits][m]: the split sums
  float *tot = sms + splits * m;       // [m]: the row's merged sum
  const size_t pb = (size_t)bh * splits * m;
  for (int e = t; e < splits * m; e += 256) {
    fac[e] = pmax[pb + e];
    sms[e] = psum[pb + e];
  }
  __syncthreads();
  for (int j = t; j < m; j += 256) {
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, fac[s * m + j]);
    float sum = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float f = exp2f(fac[s * m + j] - mx);
      fac[s * m + j] = f;
      sum = fmaf(sms[s * m + j], f, sum);
    }
    tot[j] = sum;
    if (lse2 && blockIdx.y == 0) lse2[(size_t)bh * m + j] = mx + log2f(sum);   // backward pass
  }
  for (int e = t; e < m * m; e += 256) zs[e] = Zg[(size_t)bh * m * m + e];
  __syncthreads();
  for (int idx = t; idx < m * kMergeCols; idx += 256) {
    const int j = idx / kMergeCols, c = idx % kMergeCols;
    if (c >= nc) continue;
    const float *src = py + (pb + j) * d + c0 + c;
    const size_t stride = (size_t)m * d;
    float acc = 0.f;
    int s = 0;
    for (; s + 4 <= splits; s += 4) {   // four loads in flight, added in order
      const float v0 = src[s * stride], v1 = src[(s + 1) * stride], v2 = src[(s + 2) * stride],
                  v3 = src[(s + 3) * stride];
      acc = fmaf(v0, fac[s * m + j], acc);
      acc = fmaf(v1, fac[(s + 1) * m + j], acc);
      acc = fmaf(v2, fac[(s + 2) * m + j], acc);
      acc = fmaf(v3, fac[(s + 3) * m + j], acc);
    }
    for (; s < splits; ++s) acc = fmaf(src[s * stride], fac[s * m + j], acc);
    const float y = acc / tot[j];
    ys[idx] = y;
    Yg[((size_t)bh * m + j) * d + c0 + c] = y;
  }
  __syncthreads();
  for (int idx = t; idx < m * kMergeCols; idx += 256) {
    const int j = idx / kMergeCols, c = idx % kMergeCols;
    if (c >= nc) continue;
    float acc = 0.f;
    for (int k = 0; k < m; ++k) acc = fmaf(zs[j * m + k], ys[k * kMergeCols + c], acc);
    Wg[((size_t)bh * m + j) * d + c0 + c] = acc;
  }
}

// ---------------------------------------------------------------------------
// Output rows: out_i = softmax_m(s q_i . K~^T) W + sum_t w[t] V[i + t - (k-1)/2]
// (Eq. 17 with the Figure 4 DConv skip).  One warp per row; lane owns
// features lane and lane+32 and landmarks lane and lane+32.
constexpr int kSimtOutRowsPerBlock = 32;

template <typename T, int LPL>   // landmarks per lane: m <= 32 * LPL
__global__ void __launch_bounds__(256)
out_simt(const T *__restrict__ Q, const T *__restrict__ V, const float *__restrict__ Kt,
         const float *__restrict__ Wg, const float *__restrict__ convw, T *__restrict__ out,
         int n, int d, int m, int heads, int convk, float scale_log2, const int *lens) {
  extern __shared__ float smem[];
  const int bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = bh % heads;
  float *kts = smem;                   // [m][d+1]
  float *ws = kts + m * (d + 1);       // [m][d]
  float *qrow = ws + m * d;            // [8][d]
  float *wc = qrow + 8 * d;            // [convk]
  for (int i = threadIdx.x; i < m * d; i += blockDim.x) {
    int j = i / d, c = i % d;
    kts[j * (d + 1) + c] = Kt[(size_t)bh * m * d + i];
    ws[i] = Wg[(size_t)bh * m * d + i];
  }
  if (convw)
    for (int t = threadIdx.x; t < convk; t += blockDim.x) wc[t] = convw[head * convk + t];
  __syncthreads();
  const T *Qh = Q + (size_t)bh * n * d;
  const T *Vh = V + (size_t)bh * n * d;
  T *Oh = out + (size_t)bh * n * d;
  const int half = (convk - 1) / 2;
  // rows of the element: [0, L); padding rows (and every row of an element
  // with an invalid length) are zero, and the conv pads with zeros from L on
  const int L = seq_len_of(lens, bh, heads, n, m, nullptr);
  for (int rr = warp; rr < kSimtOutRowsPerBlock; rr += 8) {
    const int i = blockIdx.x * kSimtOutRowsPerBlock + rr;
    if (i >= n) break;
    if (i >= L) {
      if (lane < d) Oh[(size_t)i * d + lane] = from_f<T>(0.f);
      if (lane + 32 < d) Oh[(size_t)i * d + lane + 32] = from_f<T>(0.f);
      continue;
    }
    if (lane < d) qrow[warp * d + lane] = to_f(Qh[(size_t)i * d + lane]);
    if (lane + 32 < d) qrow[warp * d + lane + 32] = to_f(Qh[(size_t)i * d + lane + 32]);
    __syncwarp();
    float l[LPL];
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < LPL; ++t) {
      int j = lane + 32 * t;
      float acc = 0.f;
      if (j < m)
        for (int c = 0; c < d; ++c) acc = fmaf(qrow[warp * d + c], kts[j * (d + 1) + c], acc);
      l[t] = j < m ? acc * scale_log2 : -INFINITY;
      mx = fmaxf(mx, l[t]);
    }
    mx = warp_max(mx);
    float ps = 0.f;
#pragma unroll
    for (int t = 0; t < LPL; ++t) {
      l[t] = exp2f(l[t] - mx);
      ps += l[t];
    }
    const float inv = 1.f / warp_sum(ps);
#pragma unroll
    for (int t = 0; t < LPL; ++t) l[t] *= inv;
    float o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int t = 0; t < LPL; ++t)
    for (int jj = 0; jj < 32; ++jj) {
      const int j = 32 * t + jj;
      if (j >= m) break;
      float f = __shfl_sync(0xffffffffu, l[t], jj);
      if (lane < d) o0 = fmaf(f, ws[j * d + lane], o0);
      if (lane + 32 < d) o1 = fmaf(f, ws[j * d + lane + 32], o1);
    }
    if (convw) {
      float c0 = 0.f, c1 = 0.f;
      for (int t = 0; t < convk; ++t) {
        int src = i + t - half;
        if (src < 0 || src >= L) continue;
        if (lane < d) c0 = fmaf(wc[t], to_f(Vh[(size_t)src * d + lane]), c0);
        if (lane + 32 < d) c1 = fmaf(wc[t], to_f(Vh[(size_t)src * d + lane + 32]), c1);
      }
      o0 += c0;
      o1 += c1;
    }
    if (lane < d) Oh[(size_t)i * d + lane] = from_f<T>(o0);
    if (lane + 32 < d) Oh[(size_t)i * d + lane + 32] = from_f<T>(o1);
    __syncwarp();
  }
}

}  // namespace nys
