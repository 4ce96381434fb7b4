// Landmark kernel and iterative pseudoinverse for m = 128 on 5th-generation
// tensor cores, one block per (batch, head): the power form of the m <= 64
// kernel (pinv_pow.cuh) at full width.
//
// "Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, "Moore-Penrose Pseudoinverse Computation":
//   A  = softmax(Q~ K~^T / sqrt(d))
//   Z0 = A^T / (||A||_1 ||A||_inf)
//   Z_{j+1} = 1/4 Z_j (13I - A Z_j (15I - A Z_j (7I - A Z_j)))   (Lemma 1)
//
// Evaluation order (as for m <= 64).  With P_j = A Z_j the step is
// Z_{j+1} = Z_j r_j, r_j = 1/4 (13I - 15 P_j + 7 P_j^2 - P_j^3), and
// P_{j+1} = P_j r_j = 1/4 (13 P - 15 P^2 + 7 P^3 - P^4).  Every P_j is a
// polynomial in P_0 = A A^T / (||A||_1 ||A||_inf), so the P_j are symmetric
// and a matrix's rows serve as its columns.  One step is two dependent
// stages of MMAs:
//   stage 1:  P2 = P P                     (U = 7P - P2 formed from it)
//   stage 2:  U P2 = 7P^3 - P^4,  U P = 7P^2 - P^3
// after which P_{j+1} and r_j are elementwise; Z_j = Z_{j-1} r_{j-1} is a
// third product off the chain, issued beside stage 1.  Equal to the printed
// recurrence in exact arithmetic; only rounding differs.
//
// Precision.  The landmark logits use split bf16 (hi*hi + hi*lo + lo*hi,
// about 16 bits) and A A^T split fp16 (about 21 bits); the iteration runs on
// fp16 operands (10-bit significands, as tf32) with fp32 accumulation in
// TMEM.  At m = 128 the operands of the split products would not fit in
// shared memory beside the Z update's.
//
// Threads 0..255: thread t owns TMEM lane (matrix row) t % 128 and column
// half t / 128 (64 columns).  Thread 256 (warp 8) issues the MMAs.
// TMEM (512 columns): stage 1 / logits / A A^T at 0, U P2 at 128, U P at 256,
// the Z update at 384.
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace pinvpow128 {

using namespace sm100;

constexpr int M = 128;
constexpr int kThreads = 256;      // matrix-row threads
constexpr int kBarThreads = 288;   // plus the issuer warp
constexpr int NC = 64;             // columns per thread

struct Cfg {
  // fp16 operands, K-major, 128 rows x 128 columns: two 16 KB atoms of 64
  // columns (element (row, k) in atom k / 64, 128-byte swizzle row `row`)
  static constexpr uint32_t kOp = 32768u;
  static constexpr uint32_t op_p = 0;              // P_j (A of stage 1, B of stages 1, 2)
  static constexpr uint32_t op_p2 = op_p + kOp;    // P_j^2 (B of stage 2)
  static constexpr uint32_t op_u = op_p2 + kOp;    // U (A of stage 2)
  static constexpr uint32_t op_z = op_u + kOp;     // Z_j (A of the update)
  static constexpr uint32_t op_r = op_z + kOp;     // r_j (B of the update)
  // setup overlays: the landmark operands (bf16 hi / lo, 128 rows x 64
  // features) over Z and r; A in fp32 over P2 and U; A's lo half over r
  static constexpr uint32_t qh = op_z, ql = qh + 16384u;
  static constexpr uint32_t kh = ql + 16384u, kl = kh + 16384u;
  static constexpr uint32_t af = op_p2;            // [128][128] fp32, 16-byte chunks swizzled
  static constexpr uint32_t red = op_r + kOp;      // [4][2][128] fp32 row / column partials
  static constexpr uint32_t bars = red + 4096u;
  static constexpr uint32_t total = bars + 1024u;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t t_d1 = 0, t_x = 128, t_y = 256, t_z = 384;
};

// Byte offset of element (row, k) of a K-major fp16 operand of Cfg::kOp.
__device__ __forceinline__ uint32_t op_off(int row, int k) {
  return (uint32_t)(k >> 6) * 16384u + sw128_offset(row, (k & 63) >> 3) + (uint32_t)(k & 7) * 2u;
}

// 16 values of row `row`, columns c0.. (c0 a multiple of 16) into a K-major
// fp16 operand (rounded to nearest).
__device__ __forceinline__ void put16_f16(uint32_t base, int row, int c0, const float *v) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int c = c0 + 8 * q;
    st_shared_v4(base + (uint32_t)(c >> 6) * 16384u + sw128_offset(row, (c & 63) >> 3),
                 pack_f16(v[8 * q], v[8 * q + 1]), pack_f16(v[8 * q + 2], v[8 * q + 3]),
                 pack_f16(v[8 * q + 4], v[8 * q + 5]), pack_f16(v[8 * q + 6], v[8 * q + 7]));
  }
}
// The same, as the lo half of a split: rounding of v - fp16(v).
__device__ __forceinline__ void put16_f16_lo(uint32_t base, int row, int c0, const float *v) {
  float lo[16];
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const float2 hf = __half22float2(__floats2half2_rn(v[e], v[e + 1]));
    lo[e] = v[e] - hf.x;
    lo[e + 1] = v[e + 1] - hf.y;
  }
  put16_f16(base, row, c0, lo);
}

// fp32 [128][128] scratch, 16-byte chunks XOR-swizzled by row so that row
// and column accesses avoid bank conflicts: element (r, c)
__device__ __forceinline__ int af_idx(int r, int c) {
  return r * 128 + ((((c >> 2) ^ (r & 31)) << 2) | (c & 3));
}

// Runs on threads 0..287 of a block and synchronises them with named barrier
// 1 only.  smem: Cfg::total bytes, 1 KB aligned.  Prm carries q_land, k_land
// ([BH][128][64] fp32), z_out ([BH][128][128] fp32), err, iters and
// scale_log2 = log2(e) / sqrt(d).  tmem: a 512-column TMEM allocation owned
// by the caller.  zs_hi, zs_lo (shared-memory addresses, or 0): the final Z
// is also written there as a split bf16 operand pair, K-major (two 16 KB
// atoms of 64 columns each), for a product with Z that follows in the same
// block; they may lie over this function's operands (written after its
// last MMA has completed).
template <class Prm>
__device__ __forceinline__ void pinv_body(const Prm &prm, uint8_t *smem, int bh, uint32_t tmem,
                                          uint32_t zs_hi = 0, uint32_t zs_lo = 0) {
  using C = Cfg;
  const int t = threadIdx.x, warp = t >> 5;
  const int r = t & 127, h = t >> 7;
  const bool rows = t < kThreads;
  const bool issuer = t == kThreads;
  const int c_lo = h * NC;
  uint64_t *bar_main = (uint64_t *)(smem + C::bars);
  uint64_t *bar_z = bar_main + 1;
  volatile uint32_t *abort_flag = (volatile uint32_t *)(bar_main + 2);
  float *red = (float *)(smem + C::red);   // [4][2][128]: maxima, sums, |A| row / column sums
  float *af = (float *)(smem + C::af);
  const Abort ab{abort_flag, prm.err};
  if (t == 0) {
    mbar_init(bar_main, 1);
    mbar_init(bar_z, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t s0 = smem_u32(smem);
  const uint32_t op_p = s0 + C::op_p, op_p2 = s0 + C::op_p2, op_u = s0 + C::op_u;
  const uint32_t op_z = s0 + C::op_z, op_r = s0 + C::op_r;
  const uint32_t qh = s0 + C::qh, ql = s0 + C::ql, kh = s0 + C::kh, kl = s0 + C::kl;
  float *zg = prm.z_out + (size_t)bh * M * M;

  // 8 values as a split bf16 pair (hi = rounding of x, lo = rounding of
  // x - hi) at byte offset `off` of two operands
  auto put8_bf16_split = [](uint32_t hi_base, uint32_t lo_base, uint32_t off, const float *x) {
    uint32_t hh[4], ll[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
      const float2 bf = __bfloat1622float2(b);
      hh[e] = *reinterpret_cast<const uint32_t *>(&b);
      ll[e] = pack_bf16(x[2 * e] - bf.x, x[2 * e + 1] - bf.y);
    }
    st_shared_v4(hi_base + off, hh[0], hh[1], hh[2], hh[3]);
    st_shared_v4(lo_base + off, ll[0], ll[1], ll[2], ll[3]);
  };

  // ---- landmarks -> split bf16 operands (all loads issued first)
  if (rows) {
    const float4 *qg = (const float4 *)(prm.q_land + (size_t)bh * M * 64);
    const float4 *kg = (const float4 *)(prm.k_land + (size_t)bh * M * 64);
    float4 qv[4][2], kv[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = t + i * kThreads;
      qv[i][0] = __ldcg(qg + 2 * idx);
      qv[i][1] = __ldcg(qg + 2 * idx + 1);
      kv[i][0] = __ldcg(kg + 2 * idx);
      kv[i][1] = __ldcg(kg + 2 * idx + 1);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = t + i * kThreads, rr = idx >> 3, ch = idx & 7;
      const float q[8] = {qv[i][0].x, qv[i][0].y, qv[i][0].z, qv[i][0].w,
                          qv[i][1].x, qv[i][1].y, qv[i][1].z, qv[i][1].w};
      const float k[8] = {kv[i][0].x, kv[i][0].y, kv[i][0].z, kv[i][0].w,
                          kv[i][1].x, kv[i][1].y, kv[i][1].z, kv[i][1].w};
      put8_bf16_split(qh, ql, sw128_offset(rr, ch), q);
      put8_bf16_split(kh, kl, sw128_offset(rr, ch), k);
    }
  }
  fence_async_smem();
  tc_fence_before();
  named_barrier(1, kBarThreads);
  tc_fence_after();
  const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  uint32_t pm = 0, pz = 0;   // mbarrier phases
  bool ok = true;
  auto wait_main = [&](bool mine) {
    if (mine && ok) ok = mbar_wait(bar_main, pm, ab);
    pm ^= 1u;
    tc_fence_after();
  };
  auto wait_z = [&](bool mine) {
    if (mine && ok) ok = mbar_wait(bar_z, pz, ab);
    pz ^= 1u;
    tc_fence_after();
  };
  // operand writes -> tensor cores, and a block-uniform abort decision
  auto sync_ops = [&]() -> bool {
    fence_async_smem();
    tc_fence_before();
    const bool failed = named_barrier_or(1, kBarThreads, !ok);
    tc_fence_after();
    return !failed;
  };
  // K step k of a K-major operand: atom k / 4, 32 bytes per step inside it
  auto dk = [](uint32_t base, int k) -> uint64_t {
    return make_sdesc(base + (uint32_t)(k >> 2) * 16384u + 32u * (uint32_t)(k & 3), 16, 1024);
  };
  // D (+)= A B^T over K = 16 ks
  auto mma_k = [&](uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, int ks, bool acc) {
    for (int k = 0; k < ks; ++k) mma_bf16(d, dk(a, k), dk(b, k), idesc, (acc || k > 0) ? 1u : 0u);
  };
  const uint32_t id_bf = make_idesc(kFmtBF16, 128, 128, 0, 0);
  const uint32_t id_h = make_idesc(kFmtF16, 128, 128, 0, 0);

  // ---- logits Q~ K~^T (split bf16, K = 64)
  if (issuer) {
    mma_k(tmem + C::t_d1, qh, kh, id_bf, 4, false);
    mma_k(tmem + C::t_d1, qh, kl, id_bf, 4, true);
    mma_k(tmem + C::t_d1, ql, kh, id_bf, 4, true);
    mma_commit(bar_main);
  }
  wait_main(rows);
  // ---- row softmax, two threads per row (a column half each, combined in
  //      order through shared memory): A as a split fp16 pair (hi over P,
  //      lo over r) and in fp32 (over P2 and U); the halves' |A| row sums
  float av[NC];
  if (ok && rows) {
    tmem_ld32(t_row + C::t_d1 + c_lo, av);
    tmem_ld32(t_row + C::t_d1 + c_lo + 32, av + 32);
    tmem_ld_wait();
    float mx = av[0];
#pragma unroll
    for (int k = 1; k < NC; ++k) mx = fmaxf(mx, av[k]);
    red[h * 128 + r] = mx;
  }
  named_barrier(1, kBarThreads);
  if (ok && rows) {
    const float moff = fmaxf(red[r], red[128 + r]) * prm.scale_log2;
    float sm = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      av[k] = fast_exp2(fmaf(av[k], prm.scale_log2, -moff));
      sm += av[k];
    }
    red[256 + h * 128 + r] = sm;
  }
  named_barrier(1, kBarThreads);
  if (ok && rows) {
    const float inv = 1.f / (red[256 + r] + red[384 + r]);
    float rs = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      av[k] *= inv;
      rs += fabsf(av[k]);
    }
    red[512 + h * 128 + r] = rs;
#pragma unroll
    for (int c = 0; c < NC; c += 16) {
      put16_f16(op_p, r, c_lo + c, av + c);
      put16_f16_lo(op_r, r, c_lo + c, av + c);
    }
#pragma unroll
    for (int c = 0; c < NC; c += 4)
      *(float4 *)(af + af_idx(r, c_lo + c)) = make_float4(av[c], av[c + 1], av[c + 2], av[c + 3]);
  }
  if (!sync_ops()) ok = false;
  NYS_MARK(kTrMid, 8);
  // ---- A A^T (split fp16, K = 128); meanwhile Z0's rows are A's columns
  if (ok && issuer) {
    mma_k(tmem + C::t_d1, op_p, op_p, id_h, 8, false);
    mma_k(tmem + C::t_d1, op_p, op_r, id_h, 8, true);
    mma_k(tmem + C::t_d1, op_r, op_p, id_h, 8, true);
    mma_commit(bar_main);
  }
  float zc[NC];   // row r of A^T, columns c_lo..: A[c_lo + k][r]
  if (ok && rows) {
    float cs = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      zc[k] = af[af_idx(c_lo + k, r)];
      cs += fabsf(zc[k]);
    }
    red[768 + h * 128 + r] = cs;
  }
  named_barrier(1, kBarThreads);
  // ||A||_1 (largest column sum) and ||A||_inf (largest row sum): every warp
  // reduces the 128 rows' partials, lane l taking rows l, l + 32, ...
  float n1 = 0.f, ninf = 0.f;
  {
    const int l = t & 31;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = l + 32 * q;
      n1 = fmaxf(n1, red[768 + i] + red[896 + i]);
      ninf = fmaxf(ninf, red[512 + i] + red[640 + i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n1 = fmaxf(n1, __shfl_xor_sync(0xffffffffu, n1, o));
      ninf = fmaxf(ninf, __shfl_xor_sync(0xffffffffu, ninf, o));
    }
  }
  const float c0 = 1.f / (n1 * ninf);
  if (ok && rows) {   // Z0 = c0 A^T into the Z operand (over the dead landmark operands)
#pragma unroll
    for (int k = 0; k < NC; ++k) zc[k] *= c0;
#pragma unroll
    for (int c = 0; c < NC; c += 16) put16_f16(op_z, r, c_lo + c, zc + c);
    if (prm.iters == 0) {
#pragma unroll
      for (int q = 0; q < NC / 4; ++q)
        *(float4 *)(zg + (size_t)r * M + c_lo + 4 * q) =
            make_float4(zc[4 * q], zc[4 * q + 1], zc[4 * q + 2], zc[4 * q + 3]);
    }
  }
  wait_main(rows);
  // P_j of this thread's row half stays in registers through the steps
  float preg[NC];
  if (ok && rows) {   // P0 = c0 A A^T
    tmem_ld32(t_row + C::t_d1 + c_lo, preg);
    tmem_ld32(t_row + C::t_d1 + c_lo + 32, preg + 32);
    tmem_ld_wait();
#pragma unroll
    for (int k = 0; k < NC; ++k) preg[k] *= c0;
#pragma unroll
    for (int c = 0; c < NC; c += 16) put16_f16(op_p, r, c_lo + c, preg + c);
  }
  if (!sync_ops()) ok = false;
  NYS_MARK(kTrMid, 9);

  // ---- Lemma 1 steps.  The update Z_j = Z_{j-1} r_{j-1} goes out with
  //      stage 1 of step j and is read back into the Z operand while stage 2
  //      runs, before r_j is written over r_{j-1}.
  const int iters = ok ? prm.iters : 0;
  bool good = ok;   // block-uniform: no stage failed
  for (int j = 0; j < iters; ++j) {
    // stage 1: P2 = P P
    if (issuer) {
      mma_k(tmem + C::t_d1, op_p, op_p, id_h, 8, false);
      mma_commit(bar_main);
      if (j > 0) {
        mma_k(tmem + C::t_z, op_z, op_r, id_h, 8, false);
        mma_commit(bar_z);
      }
    }
    wait_main(rows);
    if (j < 8) NYS_MARK(kTrMid, 40 + j);
    if (ok && rows) {
#pragma unroll
      for (int c = 0; c < NC; c += 16) {
        float p2[16], uu[16];
        tmem_ld16(t_row + C::t_d1 + c_lo + c, p2);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) uu[e] = fmaf(7.f, preg[c + e], -p2[e]);
        put16_f16(op_p2, r, c_lo + c, p2);
        put16_f16(op_u, r, c_lo + c, uu);
      }
    }
    if (!sync_ops()) {
      good = false;
      break;
    }
    // stage 2: U P2 and U P
    if (issuer) {
      mma_k(tmem + C::t_x, op_u, op_p2, id_h, 8, false);
      mma_k(tmem + C::t_y, op_u, op_p, id_h, 8, false);
      mma_commit(bar_main);
    }
    if (j > 0) {   // Z_j into the Z operand
      wait_z(rows);
      if (ok && rows) {
#pragma unroll
        for (int c = 0; c < NC; c += 16) {
          float z[16];
          tmem_ld16(t_row + C::t_z + c_lo + c, z);
          tmem_ld_wait();
          put16_f16(op_z, r, c_lo + c, z);
        }
      }
    }
    wait_main(rows);
    if (j < 8) NYS_MARK(kTrMid, 48 + j);
    if (ok && rows) {
      // P_{j+1} = 1/4 (13 P - 15 P2 + 7 P^3 - P^4), r_j = 1/4 (13I - 15 P + 7 P^2 - P^3)
#pragma unroll
      for (int c = 0; c < NC; c += 16) {
        float x[16], y[16], p2[16];
        tmem_ld16(t_row + C::t_x + c_lo + c, x);
        tmem_ld16(t_row + C::t_y + c_lo + c, y);
        tmem_ld16(t_row + C::t_d1 + c_lo + c, p2);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float pj = preg[c + e];
          preg[c + e] = 0.25f * fmaf(13.f, pj, fmaf(-15.f, p2[e], x[e]));
          y[e] = 0.25f * ((c_lo + c + e == r ? 13.f : 0.f) + fmaf(-15.f, pj, y[e]));
        }
        put16_f16(op_p, r, c_lo + c, preg + c);
        put16_f16(op_r, r, c_lo + c, y);
      }
    }
    if (j < 8) NYS_MARK(kTrMid, 16 + j);
    if (!sync_ops()) {
      good = false;
      break;
    }
  }
  // ---- Z = Z_{iters-1} r_{iters-1}: to global memory and the caller's operand
  if (iters > 0 && good) {
    if (issuer) {
      mma_k(tmem + C::t_z, op_z, op_r, id_h, 8, false);
      mma_commit(bar_z);
    }
    wait_z(rows);
    if (ok && rows) {
#pragma unroll
      for (int c = 0; c < NC; c += 16) {
        float z[16];
        tmem_ld16(t_row + C::t_z + c_lo + c, z);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *(float4 *)(zg + (size_t)r * M + c_lo + c + 4 * q) =
              make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
        if (zs_hi) {
          put8_bf16_split(zs_hi, zs_lo, op_off(r, c_lo + c), z);
          put8_bf16_split(zs_hi, zs_lo, op_off(r, c_lo + c + 8), z + 8);
        }
      }
    }
  } else if (ok && rows && prm.iters == 0 && zs_hi) {
    // Z = Z0, stored above by this thread
#pragma unroll
    for (int c = 0; c < NC; c += 8) {
      const float4 a = *(const float4 *)(zg + (size_t)r * M + c_lo + c);
      const float4 b = *(const float4 *)(zg + (size_t)r * M + c_lo + c + 4);
      const float z[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      put8_bf16_split(zs_hi, zs_lo, op_off(r, c_lo + c), z);
    }
  }
  tc_fence_before();
  named_barrier(1, kBarThreads);
  if (t == 0 && !*abort_flag) {
    mbar_inval(bar_main);
    mbar_inval(bar_z);
  }
}

}  // namespace pinvpow128
}  // namespace nys
