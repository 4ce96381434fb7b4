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
// Landmark kernel A = softmax(Q~ K~^T / sqrt(d)) and its pseudoinverse by
// Lemma 1 as printed: Z <- 1/4 Z (13I - AZ (15I - AZ (7I - AZ))), from
// Z0 = A^T / (||A||_1 ||A||_inf).  One block per head; all five m x m fp32
// matrices live in `mats` (shared memory when it fits, else the per-head
// workspace scratch).
__device__ __forceinline__ void block_gemm(float *C, const float *X, const float *Y, int m) {
  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
    int i = idx / m, j = idx % m;
    float acc = 0.f;
    for (int k = 0; k < m; ++k) acc = fmaf(X[i * m + k], Y[k * m + j], acc);
    C[idx] = acc;
  }
  __syncthreads();
}

__device__ __forceinline__ void block_diag_minus(float *dst, const float *src, float c, int m) {
  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
    int i = idx / m, j = idx % m;
    dst[idx] = (i == j ? c : 0.f) - src[idx];
  }
  __syncthreads();
}

// a_out, z_all (optional, for the backward pass): A [BH][m][m] and every
// iterate Z0 .. Z_iters [BH][iters + 1][m][m].
__global__ void pinv_simt(const float *__restrict__ Qt, const float *__restrict__ Kt,
                          float *__restrict__ Zout, float *__restrict__ scratch, int m, int d,
                          float scale, int iters, int use_smem, float *__restrict__ a_out = nullptr,
                          float *__restrict__ z_all = nullptr) {
  extern __shared__ float smem[];
  const int bh = blockIdx.x;
  float *mats = use_smem ? smem : scratch + (size_t)bh * 5 * m * m;
  float *A = mats, *Z = A + m * m, *P = Z + m * m, *T1 = P + m * m, *T2 = T1 + m * m;
  __shared__ float red[2];
  const float *qt = Qt + (size_t)bh * m * d;
  const float *kt = Kt + (size_t)bh * m * d;

  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
    int i = idx / m, j = idx % m;
    float acc = 0.f;
    for (int c = 0; c < d; ++c) acc = fmaf(qt[i * d + c], kt[j * d + c], acc);
    A[idx] = acc * scale;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {        // row softmax
    float mx = -INFINITY;
    for (int j = 0; j < m; ++j) mx = fmaxf(mx, A[i * m + j]);
    float s = 0.f;
    for (int j = 0; j < m; ++j) {
      float e = __expf(A[i * m + j] - mx);
      A[i * m + j] = e;
      s += e;
    }
    float inv = 1.f / s;
    for (int j = 0; j < m; ++j) A[i * m + j] *= inv;
  }
  __syncthreads();
  // ||A||_1 (max column sum) and ||A||_inf (max row sum), sequential in a
  // fixed order by one thread so the result is deterministic.
  if (threadIdx.x == 0) {
    float n1 = 0.f, ninf = 0.f;
    for (int j = 0; j < m; ++j) {
      float cs = 0.f;
      for (int i = 0; i < m; ++i) cs += fabsf(A[i * m + j]);
      n1 = fmaxf(n1, cs);
    }
    for (int i = 0; i < m; ++i) {
      float rs = 0.f;
      for (int j = 0; j < m; ++j) rs += fabsf(A[i * m + j]);
      ninf = fmaxf(ninf, rs);
    }
    red[0] = 1.f / (n1 * ninf);
  }
  __syncthreads();
  const float c0 = red[0];
  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
    int i = idx / m, j = idx % m;
    Z[idx] = A[j * m + i] * c0;
    if (a_out) a_out[(size_t)bh * m * m + idx] = A[idx];
    if (z_all) z_all[(size_t)bh * (iters + 1) * m * m + idx] = A[j * m + i] * c0;
  }
  __syncthreads();
  for (int it = 0; it < iters; ++it) {
    block_gemm(P, A, Z, m);               // AZ
    block_diag_minus(T1, P, 7.f, m);      // 7I - AZ
    block_gemm(T2, P, T1, m);             // AZ (7I - AZ)
    block_diag_minus(T1, T2, 15.f, m);    // 15I - ...
    block_gemm(T2, P, T1, m);             // AZ (15I - ...)
    block_diag_minus(T1, T2, 13.f, m);    // 13I - ...
    block_gemm(T2, Z, T1, m);             // Z (13I - ...)
    for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
      Z[idx] = 0.25f * T2[idx];
      if (z_all) z_all[((size_t)bh * (iters + 1) + it + 1) * m * m + idx] = 0.25f * T2[idx];
    }
    __syncthreads();
  }
  float *zo = Zout + (size_t)bh * m * m;
  for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) zo[idx] = Z[idx];
}

// ---------------------------------------------------------------------------
// B~ V over one split of the keys (Eq. 17): for every landmark row j, an
// online softmax over the split's keys of s * q~_j . k_i, keeping the running
// maximum (log2 units), the running sum and the unnormalised sum of p_i v_i.
// Grid (splits, heads), 8 warps; warp w owns rows j = w, w+8, ...; lane owns
// features lane and lane+32.
constexpr int kSimtKeyTile = 32;

template <typename T, int kSimtMaxRowsPerWarp>   // m <= 8 * kSimtMaxRowsPerWarp
__global__ void __launch_bounds__(256)
bv_partial_simt(const float *__restrict__ Qt, const T *__restrict__ K, const T *__restrict__ V,
                float *__restrict__ pmax, float *__restrict__ psum, float *__restrict__ py,
                int n, int d, int m, int splits, int keys_per_split, float scale_log2,
                const int *lens, int heads) {
  extern __shared__ float smem[];
  const int split = blockIdx.x, bh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *qs = smem;                            // [m][d]
  float *ks = qs + m * d;                      // [32][d+1]
  float *vs = ks + kSimtKeyTile * (d + 1);     // [32][d]
  for (int i = threadIdx.x; i < m * d; i += blockDim.x) qs[i] = Qt[(size_t)bh * m * d + i];

  float M[kSimtMaxRowsPerWarp], S[kSimtMaxRowsPerWarp], y0[kSimtMaxRowsPerWarp],
      y1[kSimtMaxRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kSimtMaxRowsPerWarp; ++r) {
    M[r] = -INFINITY;
    S[r] = 0.f;
    y0[r] = 0.f;
    y1[r] = 0.f;
  }
  // keys of the element: [0, L) (an invalid length reads as 0: no keys)
  const int L = seq_len_of(lens, bh, heads, n, m, nullptr);
  const int k0 = split * keys_per_split;
  const int k1 = min(L, k0 + keys_per_split);
  const T *Kh = K + (size_t)bh * n * d;
  const T *Vh = V + (size_t)bh * n * d;
  for (int t0 = k0; t0 < k1; t0 += kSimtKeyTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kSimtKeyTile * d; i += blockDim.x) {
      int r = i / d, c = i % d;
      int key = t0 + r;
      float kv = 0.f, vv = 0.f;
      if (key < k1) {
        kv = to_f(Kh[(size_t)key * d + c]);
        vv = to_f(Vh[(size_t)key * d + c]);
      }
      ks[r * (d + 1) + c] = kv;
      vs[r * d + c] = vv;
    }
    __syncthreads();
    const bool valid = (t0 + lane) < k1;
#pragma unroll
    for (int r = 0; r < kSimtMaxRowsPerWarp; ++r) {
      const int j = warp + 8 * r;
      if (j >= m) break;
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(qs[j * d + c], ks[lane * (d + 1) + c], acc);
      float l2 = valid ? acc * scale_log2 : -INFINITY;
      float mnew = fmaxf(M[r], warp_max(l2));
      float alpha = exp2f(M[r] - mnew);        // 0 when M was -inf
      float p = exp2f(l2 - mnew);
      S[r] = S[r] * alpha + warp_sum(p);
      float a0 = y0[r] * alpha, a1 = y1[r] * alpha;
      for (int i = 0; i < kSimtKeyTile; ++i) {
        float pi = __shfl_sync(0xffffffffu, p, i);
        if (lane < d) a0 = fmaf(pi, vs[i * d + lane], a0);
        if (lane + 32 < d) a1 = fmaf(pi, vs[i * d + lane + 32], a1);
      }
      y0[r] = a0;
      y1[r] = a1;
      M[r] = mnew;
    }
  }
  const size_t base = ((size_t)bh * splits + split) * m;
#pragma unroll
  for (int r = 0; r < kSimtMaxRowsPerWarp; ++r) {
    const int j = warp + 8 * r;
    if (j >= m) break;
    if (lane == 0) {
      pmax[base + j] = M[r];
      psum[base + j] = S[r];
    }
    if (lane < d) py[(base + j) * d + lane] = y0[r];
    if (lane + 32 < d) py[(base + j) * d + lane + 32] = y1[r];
  }
}

// ---------------------------------------------------------------------------
// Merge of the key splits in split order (Y = B~ V), then W = Z Y.  One block
// per head.
__global__ void merge_w_simt(const float *__restrict__ pmax, const float *__restrict__ psum,
                             const float *__restrict__ py, const float *__restrict__ Zg,
                             float *__restrict__ Yg, float *__restrict__ Wg, int m, int d,
                             int splits, float *__restrict__ lse2 = nullptr) {
  extern __shared__ float ys[];   // [m][d]
  const int bh = blockIdx.x;
  const size_t pb = (size_t)bh * splits * m;
  for (int idx = threadIdx.x; idx < m * d; idx += blockDim.x) {
    int j = idx / d, c = idx % d;
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, pmax[pb + (size_t)s * m + j]);
    float sum = 0.f, acc = 0.f;
    for (int s = 0; s < splits; ++s) {
      float f = exp2f(pmax[pb + (size_t)s * m + j] - mx);
      sum = fmaf(psum[pb + (size_t)s * m + j], f, sum);
      acc = fmaf(py[(pb + (size_t)s * m + j) * d + c], f, acc);
    }
    float y = acc / sum;
    if (lse2 && c == 0) lse2[(size_t)bh * m + j] = mx + log2f(sum);   // backward pass
    ys[idx] = y;
    Yg[(size_t)bh * m * d + idx] = y;
  }
  __syncthreads();
  const float *z = Zg + (size_t)bh * m * m;
  for (int idx = threadIdx.x; idx < m * d; idx += blockDim.x) {
    int j = idx / d, c = idx % d;
    float acc = 0.f;
    for (int k = 0; k < m; ++k) acc = fmaf(z[j * m + k], ys[k * d + c], acc);
    Wg[(size_t)bh * m * d + idx] = acc;
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
