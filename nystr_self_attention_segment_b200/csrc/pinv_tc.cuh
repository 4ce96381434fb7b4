// Landmark kernel and iterative pseudoinverse on 5th-generation tensor cores
// (tf32 inputs, fp32 accumulation in TMEM), one CTA per (batch, head).
//
// "Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, "Moore-Penrose Pseudoinverse Computation":
//   A  = softmax(Q~ K~^T / sqrt(d))
//   Z0 = A^T / (||A||_1 ||A||_inf)
//   Z_{j+1} = 1/4 Z_j (13I - A Z_j (15I - A Z_j (7I - A Z_j)))   (Lemma 1)
//
// Q~ K~^T is formed with the 3xTF32 split (hi*hi + hi*lo + lo*hi, hi = tf32
// rounding, lo = tf32 of the remainder), accurate to about fp32, because the
// logits can be large (peaky attention) and A feeds an ill-conditioned
// inverse.  The softmax runs in registers on the TMEM rows.
//
// Evaluation order of the iteration.  With P_j = A Z_j the step is
// Z_{j+1} = 1/4 Z_j X5 where X1 = 7I - P_j, X3 = 15I - P_j X1,
// X5 = 13I - P_j X3.  Since A Z_{j+1} = 1/4 (A Z_j) X5, the next P is
// 1/4 P_j X5: the same product that gives Z_{j+1}.  So every step is three
// dependent MMA stages,
//   T2 = P X1,   T4 = P X3,   [P'; Z'] = 1/4 [P; Z] X5,
// the last one with P and Z stacked into one 128-row A operand (m <= 64), and
// P_0 = A A^T / (||A||_1 ||A||_inf).  Equal to the printed recurrence in exact
// arithmetic; only rounding differs (tf32 operands, fp32 accumulation).
//
// 128 threads; thread r owns accumulator row r (TMEM lane r) and writes that
// row of the next operands.  Both operands are K-major with the 128-byte
// swizzle (32 fp32 per swizzle row); B operands are written transposed
// because an MN-major tf32 B operand reads as zero on this hardware.
#pragma once

#include "sm100.cuh"

namespace nys {
namespace pinvtc {

using namespace sm100;

constexpr int kThreads = 128;

template <int M>
struct Cfg {
  static constexpr uint32_t kAop = (M / 32) * 16384u;   // 128 rows x M (K-major)
  static constexpr uint32_t kBop = (M / 32) * M * 128u; // M rows x M (K-major)
  static constexpr uint32_t kQop = 2 * 16384u;          // 128 rows x 64 features
  static constexpr uint32_t kKop = 2 * M * 128u;        // M rows x 64 features
  // iteration operands
  static constexpr uint32_t aop = 0;
  static constexpr uint32_t zop = aop + kAop;                      // M = 128 only
  static constexpr uint32_t bop = zop + (M == 128 ? kAop : 0u);
  // landmark operands, dead once the logits are in TMEM; for M = 128 they
  // overlay the Z and B operands, which are written only after that point
  static constexpr uint32_t qh = M == 128 ? zop : bop + kBop;
  static constexpr uint32_t ql = qh + kQop;
  static constexpr uint32_t kh = ql + kQop;
  static constexpr uint32_t kl = kh + kKop;
  static constexpr uint32_t end0 = kl + kKop;
  static constexpr uint32_t end1 = bop + kBop;
  static constexpr uint32_t bars = ((end0 > end1 ? end0 : end1) + 1023u) & ~1023u;
  static constexpr uint32_t total = bars + 2048u + 1024u;
  static constexpr uint32_t kTmemCols = M == 128 ? 256 : (M == 64 ? 64 : 32);
};

struct Params {
  const float *q_land, *k_land;   // [BH][m][64]
  float *z_out;                   // [BH][m][m]
  uint32_t *err;
  int iters;
  float scale_log2;               // log2(e) / sqrt(d)
};

__device__ __forceinline__ float to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// byte offset of element (row, k) of a K-major operand with `slab`-byte slabs
__device__ __forceinline__ uint32_t kmaj_off(uint32_t slab, int row, int k) {
  return (uint32_t)(k >> 5) * slab + sw128_offset(row, (k & 31) >> 2) + (k & 3) * 4u;
}

// Row `row`, columns c0..c0+31 (c0 a multiple of 32) of a K-major operand.
__device__ __forceinline__ void put_kmaj32(uint32_t base, uint32_t slab, int row, int c0,
                                           const float *v) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    st_shared_v4(base + (uint32_t)(c0 >> 5) * slab + sw128_offset(row, q),
                 __float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                 __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
}
// Row `k` of a matrix X, columns n0..n0+31, into the K-major B operand of X
// (M rows of 128-byte swizzled slabs): element (k, n) goes to row n, column
// k.  The 32 threads of a warp hold 32 consecutive k, so every store
// instruction fills one 128-byte row without bank conflicts.
template <int M>
__device__ __forceinline__ void put_bT32(uint32_t base, int k, int n0, const float *v) {
  const uint32_t col = (uint32_t)(k >> 5) * (M * 128u) + (k & 3) * 4u;
#pragma unroll
  for (int e = 0; e < 32; ++e)
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(base + col + sw128_offset(n0 + e, (k & 31) >> 2)),
                 "r"(__float_as_uint(v[e]))
                 : "memory");
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return __uint_as_float(v);
}

// Runs on threads 0..127 of a block (4 warps, one per TMEM lane quarter);
// synchronises them with named barrier 1 only, so other warps of the block
// may do something else meanwhile.  smem: Cfg<M>::total bytes, 1 KB aligned.
__device__ __forceinline__ void sync128() { named_barrier(1, 128); }

template <int M>
__device__ __forceinline__ void pinv_body(const Params &prm, uint8_t *smem, int bh) {
  using C = Cfg<M>;
  const int t = threadIdx.x, warp = t >> 5;
  uint64_t *bar = (uint64_t *)(smem + C::bars);
  uint32_t *tmem_slot = (uint32_t *)(bar + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  float *red = (float *)(smem + C::bars + 1024);   // [2 * M] column / row sums
  const Abort ab{abort_flag, prm.err};
  if (t == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::kTmemCols);
  sync128();

  const uint32_t aop = smem_u32(smem + C::aop), zop = smem_u32(smem + C::zop);
  const uint32_t bop = smem_u32(smem + C::bop);
  const uint32_t qh = smem_u32(smem + C::qh), ql = smem_u32(smem + C::ql);
  const uint32_t kh = smem_u32(smem + C::kh), kl = smem_u32(smem + C::kl);

  // ---- landmarks -> hi/lo tf32 operands (all loads issued before the stores)
  {
    const float4 *qg = (const float4 *)(prm.q_land + (size_t)bh * M * 64);
    const float4 *kg = (const float4 *)(prm.k_land + (size_t)bh * M * 64);
    constexpr int kPer = M * 16 / kThreads;   // float4 per thread per tensor
    float4 qv[kPer], kv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      qv[i] = qg[t + i * kThreads];
      kv[i] = kg[t + i * kThreads];
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int idx = t + i * kThreads, row = idx >> 4, k = (idx & 15) * 4;
      const float q[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
      const float kk[4] = {kv[i].x, kv[i].y, kv[i].z, kv[i].w};
      uint32_t hq[4], lq[4], hk[4], lk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = to_tf32(q[e]), b = to_tf32(kk[e]);
        hq[e] = __float_as_uint(a);
        lq[e] = __float_as_uint(to_tf32(q[e] - a));
        hk[e] = __float_as_uint(b);
        lk[e] = __float_as_uint(to_tf32(kk[e] - b));
      }
      const uint32_t oq = kmaj_off(16384u, row, k), ok = kmaj_off(M * 128u, row, k);
      st_shared_v4(qh + oq, hq[0], hq[1], hq[2], hq[3]);
      st_shared_v4(ql + oq, lq[0], lq[1], lq[2], lq[3]);
      st_shared_v4(kh + ok, hk[0], hk[1], hk[2], hk[3]);
      st_shared_v4(kl + ok, lk[0], lk[1], lk[2], lk[3]);
    }
    if (M < 128)   // A-operand rows M..127 are zero
      for (int idx = t; idx < (128 - M) * 16; idx += kThreads) {
        const int row = M + (idx >> 4), k = (idx & 15) * 4;
        st_shared_v4(qh + kmaj_off(16384u, row, k), 0, 0, 0, 0);
        st_shared_v4(ql + kmaj_off(16384u, row, k), 0, 0, 0, 0);
      }
  }
  fence_async_smem();
  tc_fence_before();
  sync128();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t idesc = make_idesc(kFmtTF32, 128, M, 0, 0);   // both operands K-major
  uint32_t phase = 0;

  // D (+)= A B^T over K = kk, A slabs of 16 KB (128 rows), B slabs of b_slab
  auto issue = [&](uint32_t a_base, uint32_t d_col, uint32_t b_base, uint32_t b_slab, int kk,
                   bool acc0) {
    for (int k = 0; k < kk / 8; ++k) {
      const uint64_t ad = make_sdesc(a_base + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
      const uint64_t bd = make_sdesc(b_base + (k >> 2) * b_slab + (k & 3) * 32u, 16, 1024);
      mma_tf32(tmem + d_col, ad, bd, idesc, (acc0 || k > 0) ? 1u : 0u);
    }
  };
  auto wait_mma = [&]() -> bool {
    const bool done = mbar_wait(bar, phase, ab);
    phase ^= 1u;
    tc_fence_after();
    return done;
  };
  auto sync_operands = [&]() {
    fence_async_smem();
    tc_fence_before();
    sync128();
    tc_fence_after();
  };
  auto ld32 = [&](uint32_t col, float *v) {
    tmem_ld32(tmem + lane_base + col, v);
    tmem_ld_wait();
  };
  auto diag_minus = [&](float *v, int cb, int row, float a) {
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = (cb + e == row ? a : 0.f) - v[e];
  };

  // ---- logits Q~ K~^T (3xTF32) -> TMEM
  if (t == 0) {
    issue(qh, 0, kh, M * 128u, 64, false);
    issue(qh, 0, kl, M * 128u, 64, true);
    issue(ql, 0, kh, M * 128u, 64, true);
    mma_commit(bar);
  }
  bool ok = wait_mma();
  float *zg = prm.z_out + (size_t)bh * M * M;
  // ---- row softmax in registers; A rows into the K-major operand
  if (ok && t < M) {
    float v[M];
#pragma unroll
    for (int c = 0; c < M; c += 32) tmem_ld32(tmem + lane_base + c, v + c);
    tmem_ld_wait();
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < M; ++j) mx = fmaxf(mx, v[j]);
    const float moff = mx * prm.scale_log2;
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[j] = exp2f(fmaf(v[j], prm.scale_log2, -moff));
      s += v[j];
    }
    const float inv = 1.f / s;
    float rs = 0.f;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[j] *= inv;
      rs += fabsf(v[j]);
    }
    red[M + t] = rs;
#pragma unroll
    for (int c = 0; c < M; c += 32) put_kmaj32(aop, 16384u, t, c, v + c);
  }
  if (M < 128)   // A-operand rows M..127 are zero (they also pad P)
    for (int idx = t; idx < (128 - M) * (M / 4); idx += kThreads) {
      const int row = M + idx / (M / 4), k = (idx % (M / 4)) * 4;
      st_shared_v4(aop + kmaj_off(16384u, row, k), 0, 0, 0, 0);
    }
  sync128();
  if (t < M) {   // column sums: a warp reads 32 consecutive columns of one row
    float cs = 0.f;
    for (int i = 0; i < M; ++i) cs += fabsf(ld_shared_f32(aop + kmaj_off(16384u, i, t)));
    red[t] = cs;
  }
  sync128();
  float n1 = 0.f, ninf = 0.f;
  for (int i = 0; i < M; ++i) {
    n1 = fmaxf(n1, red[i]);
    ninf = fmaxf(ninf, red[M + i]);
  }
  const float c0 = 1.f / (n1 * ninf);

  if (prm.iters == 0) {   // Z = Z0 = c0 A^T
    if (t < M)
      for (int j = 0; j < M; ++j) zg[(size_t)t * M + j] = c0 * ld_shared_f32(aop + kmaj_off(16384u, j, t));
  } else if (ok) {
    const uint32_t z_a = M == 128 ? zop : aop;   // Z rows: own buffer, or rows M.. of aop
    const int z_row0 = M == 128 ? 0 : M;
    // ---- P0 = c0 A A^T (B = A read K-major)
    sync_operands();
    if (t == 0) {
      issue(aop, 0, aop, 16384u, M, false);
      mma_commit(bar);
    }
    ok = wait_mma();
    // Z0 rows (c0 times the columns of A); A stays in rows 0..M-1 until P0
    // replaces it below, after this barrier
    if (ok && t < M)
      for (int cb = 0; cb < M; cb += 32) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = c0 * ld_shared_f32(aop + kmaj_off(16384u, cb + e, t));
        put_kmaj32(z_a, 16384u, z_row0 + t, cb, v);
      }
    sync128();
    if (ok && t < M)   // P0 rows and X1 = 7I - P0
      for (int cb = 0; cb < M; cb += 32) {
        float v[32];
        ld32(cb, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= c0;
        put_kmaj32(aop, 16384u, t, cb, v);
        diag_minus(v, cb, t, 7.f);
        put_bT32<M>(bop, t, cb, v);
      }
    for (int it = 0; it < prm.iters && ok; ++it) {
      const bool last = it + 1 == prm.iters;
      // T2 = P X1  ->  X3 = 15I - T2
      sync_operands();
      if (t == 0) {
        issue(aop, 0, bop, M * 128u, M, false);
        mma_commit(bar);
      }
      if (!(ok = wait_mma())) break;
      if (t < M)
        for (int cb = 0; cb < M; cb += 32) {
          float v[32];
          ld32(cb, v);
          diag_minus(v, cb, t, 15.f);
          put_bT32<M>(bop, t, cb, v);
        }
      // T4 = P X3  ->  X5 = 13I - T4
      sync_operands();
      if (t == 0) {
        issue(aop, 0, bop, M * 128u, M, false);
        mma_commit(bar);
      }
      if (!(ok = wait_mma())) break;
      if (t < M)
        for (int cb = 0; cb < M; cb += 32) {
          float v[32];
          ld32(cb, v);
          diag_minus(v, cb, t, 13.f);
          put_bT32<M>(bop, t, cb, v);
        }
      // [P'; Z'] = 1/4 [P; Z] X5
      sync_operands();
      if (t == 0) {
        issue(aop, 0, bop, M * 128u, M, false);
        if (M == 128) issue(zop, 128, bop, M * 128u, M, false);
        mma_commit(bar);
      }
      if (!(ok = wait_mma())) break;
      if (M <= 64) {
        if (t < 2 * M)
          for (int cb = 0; cb < M; cb += 32) {
            float v[32];
            ld32(cb, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
            if (t >= M && last) {
              float4 *dst = (float4 *)(zg + (size_t)(t - M) * M + cb);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            put_kmaj32(aop, 16384u, t, cb, v);
            if (t < M) {
              diag_minus(v, cb, t, 7.f);
              put_bT32<M>(bop, t, cb, v);
            }
          }
      } else {
        for (int cb = 0; cb < M; cb += 32) {
          float v[32];
          ld32(cb, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
          put_kmaj32(aop, 16384u, t, cb, v);
          diag_minus(v, cb, t, 7.f);
          put_bT32<M>(bop, t, cb, v);
          ld32(128 + cb, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
          put_kmaj32(zop, 16384u, t, cb, v);
          if (last) {
            float4 *dst = (float4 *)(zg + (size_t)t * M + cb);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  sync128();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int M>
__global__ void __launch_bounds__(kThreads, 1) pinv_tc_kernel(const Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  pinv_body<M>(prm, smem, blockIdx.x);
}

}  // namespace pinvtc
}  // namespace nys
