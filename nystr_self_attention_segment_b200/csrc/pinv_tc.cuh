// Landmark kernel and iterative pseudoinverse on 5th-generation tensor cores
// (tf32 inputs, fp32 accumulation in TMEM), one block per (batch, head).
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
// Each stage is one full-width MMA batch (at N = 64 an MMA instruction costs
// about as much as at N = 32, so products are not split); after it, two
// threads per accumulator row (one column half each) turn the product into
// the next operands.
//
// Operands are K-major with the 128-byte swizzle (32 fp32 per swizzle row);
// B operands are written transposed (element (k, n) at row n) because an
// MN-major tf32 B operand reads as zero on this hardware.  (X is symmetric
// in exact arithmetic, but substituting its rows for its columns lets the
// tf32 rounding asymmetry of P feed back through the iteration; the peaky
// headline workload then misses 2e-2, so the transpose is exact.)
//
// Threads: 0..255; thread t owns accumulator row t % 128 (TMEM lane t % 128)
// and column half t / 128 (m = 32 uses one half); thread 0 issues the MMAs.
#pragma once

#include "sm100.cuh"

namespace nys {
namespace pinvtc {

using namespace sm100;

constexpr int kThreads = 256;

template <int M>
struct Cfg {
  static constexpr int kHalves = M >= 64 ? 2 : 1;      // column halves
  static constexpr int kCols = M / kHalves;            // columns per half
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
__host__ __device__ __forceinline__ uint32_t kmaj_off(uint32_t slab, int row, int k) {
  return (uint32_t)(k >> 5) * slab + (uint32_t)row * 128u +
         ((((uint32_t)(k & 31) >> 2) ^ ((uint32_t)row & 7u)) << 4) + (k & 3) * 4u;
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

// Runs on threads 0..255 of a block and synchronises them with named barrier
// 1 only, so other warps of the block may do something else meanwhile.
// smem: Cfg<M>::total bytes, 1 KB aligned.
__device__ __forceinline__ void sync_pinv() { named_barrier(1, kThreads); }

// tmem_in: a TMEM allocation of at least Cfg<M>::kTmemCols columns owned by
// the caller, or ~0u to allocate (and free) one here.
template <int M>
__device__ __forceinline__ void pinv_body(const Params &prm, uint8_t *smem, int bh,
                                          uint32_t tmem_in = ~0u) {
  using C = Cfg<M>;
  constexpr int NC = C::kCols;
  const int t = threadIdx.x, warp = t >> 5;
  const int r = t & 127, h = t >> 7;                // accumulator row, column half
  const bool active = h < C::kHalves;
  const int c_lo = h * NC;                          // first column of this thread's half
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
  if (tmem_in != ~0u) {
    if (t == 0) *tmem_slot = tmem_in;
  } else if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
  }

  const uint32_t aop = smem_u32(smem + C::aop), zop = smem_u32(smem + C::zop);
  const uint32_t bop = smem_u32(smem + C::bop);
  const uint32_t qh = smem_u32(smem + C::qh), ql = smem_u32(smem + C::ql);
  const uint32_t kh = smem_u32(smem + C::kh), kl = smem_u32(smem + C::kl);
  const float *aop_f = (const float *)(smem + C::aop);

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
  sync_pinv();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  uint32_t phase = 0;

  // D (+)= A B^T over K = kk; A slabs of 16 KB (128 rows), B slabs of
  // b_slab bytes; N = M columns
  auto issue = [&](uint32_t a_base, uint32_t d_col, uint32_t b_base, uint32_t b_slab, int kk,
                   bool acc0) {
    const uint32_t idesc = make_idesc(kFmtTF32, 128, M, 0, 0);
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
  // makes prior shared-memory operand writes visible to the tensor cores and
  // synchronises the operand threads
  auto sync_operands = [&]() {
    fence_async_smem();
    tc_fence_before();
    sync_pinv();
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
  // ---- row softmax in registers (one thread per row); A into the A operand
  if (ok && h == 0 && r < M) {
    float v[M];
#pragma unroll
    for (int c = 0; c < M; c += 32) tmem_ld32(tmem + lane_base + c, v + c);
    tmem_ld_wait();
    float mx[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
    for (int j = 4; j < M; ++j) mx[j & 3] = fmaxf(mx[j & 3], v[j]);
    const float moff = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * prm.scale_log2;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[j] = fast_exp2(fmaf(v[j], prm.scale_log2, -moff));
      s[j & 3] += v[j];
    }
    const float inv = 1.f / ((s[0] + s[1]) + (s[2] + s[3]));
    float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < M; ++j) {
      v[j] *= inv;
      rs[j & 3] += fabsf(v[j]);
    }
    red[M + r] = (rs[0] + rs[1]) + (rs[2] + rs[3]);
#pragma unroll
    for (int c = 0; c < M; c += 32) put_kmaj32(aop, 16384u, r, c, v + c);
  }
  if (M < 128)   // A-operand rows M..127 are zero (they also pad P)
    for (int idx = t; idx < (128 - M) * (M / 4); idx += kThreads) {
      const int row = M + idx / (M / 4), k = (idx % (M / 4)) * 4;
      st_shared_v4(aop + kmaj_off(16384u, row, k), 0, 0, 0, 0);
    }
  sync_pinv();
  if (t < M) {   // column sums: a warp reads 32 consecutive columns of one row
    float cs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int i = 0; i < M; ++i) cs[i & 3] += fabsf(aop_f[kmaj_off(16384u, i, t) >> 2]);
    red[t] = (cs[0] + cs[1]) + (cs[2] + cs[3]);
  }
  sync_pinv();
  float n1 = 0.f, ninf = 0.f;
  for (int i = 0; i < M; ++i) {
    n1 = fmaxf(n1, red[i]);
    ninf = fmaxf(ninf, red[M + i]);
  }
  const float c0 = 1.f / (n1 * ninf);

  if (prm.iters == 0) {   // Z = Z0 = c0 A^T
    for (int idx = t; idx < M * M; idx += kThreads) {
      const int i = idx / M, j = idx % M;
      zg[idx] = c0 * aop_f[kmaj_off(16384u, j, i) >> 2];
    }
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
    if (ok && active && r < M)
      for (int cb = c_lo; cb < c_lo + NC; cb += 32) {
        float v[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = c0 * aop_f[kmaj_off(16384u, cb + e, r) >> 2];
        put_kmaj32(z_a, 16384u, z_row0 + r, cb, v);
      }
    sync_pinv();
    if (ok && active && r < M)   // P0 rows and X1 = 7I - P0
      for (int cb = c_lo; cb < c_lo + NC; cb += 32) {
        float v[32];
        ld32(cb, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= c0;
        put_kmaj32(aop, 16384u, r, cb, v);
        diag_minus(v, cb, r, 7.f);
        put_bT32<M>(bop, r, cb, v);
      }
    for (int it = 0; it < prm.iters && ok; ++it) {
      const bool last = it + 1 == prm.iters;
      // T2 = P X1  ->  X3 = 15I - T2 ;  T4 = P X3  ->  X5 = 13I - T4
      for (int stage = 0; stage < 2 && ok; ++stage) {
        sync_operands();
        if (t == 0) {
          issue(aop, 0, bop, M * 128u, M, false);
          mma_commit(bar);
        }
        if (!(ok = wait_mma())) break;
        if (active && r < M)
          for (int cb = c_lo; cb < c_lo + NC; cb += 32) {
            float v[32];
            ld32(cb, v);
            diag_minus(v, cb, r, stage == 0 ? 15.f : 13.f);
            put_bT32<M>(bop, r, cb, v);
          }
      }
      if (!ok) break;
      // [P'; Z'] = 1/4 [P; Z] X5
      sync_operands();
      if (t == 0) {
        issue(aop, 0, bop, M * 128u, M, false);
        if (M == 128) issue(zop, 128, bop, M * 128u, M, false);
        mma_commit(bar);
      }
      if (!(ok = wait_mma())) break;
      if (M <= 64) {
        if (active && r < 2 * M)
          for (int cb = c_lo; cb < c_lo + NC; cb += 32) {
            float v[32];
            ld32(cb, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
            if (r >= M && last) {
              float4 *dst = (float4 *)(zg + (size_t)(r - M) * M + cb);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
            put_kmaj32(aop, 16384u, r, cb, v);
            if (r < M) {
              diag_minus(v, cb, r, 7.f);
              put_bT32<M>(bop, r, cb, v);
            }
          }
      } else {
        for (int cb = c_lo; cb < c_lo + NC; cb += 32) {
          float v[32];
          ld32(cb, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
          put_kmaj32(aop, 16384u, r, cb, v);
          diag_minus(v, cb, r, 7.f);
          put_bT32<M>(bop, r, cb, v);
          ld32(128 + cb, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= 0.25f;
          put_kmaj32(zop, 16384u, r, cb, v);
          if (last) {
            float4 *dst = (float4 *)(zg + (size_t)r * M + cb);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  sync_pinv();
  if (t == 0 && !*abort_flag) mbar_inval(bar);
  if (warp == 0 && tmem_in == ~0u) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pinvtc
}  // namespace nys
