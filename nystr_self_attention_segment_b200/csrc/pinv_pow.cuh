// Landmark kernel and iterative pseudoinverse for m <= 64 on 5th-generation
// tensor cores, one block per (batch, head), with a short dependent chain.
//
// "Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, "Moore-Penrose Pseudoinverse Computation":
//   A  = softmax(Q~ K~^T / sqrt(d))
//   Z0 = A^T / (||A||_1 ||A||_inf)
//   Z_{j+1} = 1/4 Z_j (13I - A Z_j (15I - A Z_j (7I - A Z_j)))   (Lemma 1)
//
// Evaluation order.  With P_j = A Z_j the step is Z_{j+1} = Z_j r_j where
//   r_j = 1/4 (13I - 15 P_j + 7 P_j^2 - P_j^3),
// and then P_{j+1} = A Z_{j+1} = P_j r_j = 1/4 (13 P - 15 P^2 + 7 P^3 - P^4):
// every P_j is a polynomial in P_0 = A Z_0 = A A^T / (||A||_1 ||A||_inf), so
// the P_j are symmetric and commute.  One step is two dependent products,
//   stage 1:  P2 = P P                       (U = 7P - P2 formed from it)
//   stage 2:  U [P2 | P] = [7P^3 - P^4 | 7P^2 - P^3]   (one N = 128 MMA)
// after which P_{j+1} and r_j are elementwise in the thread that holds the
// row (P_j and P_j^2 stay in its registers).  Z_{j+1} = Z_j r_j is a third
// product off the dependent chain (issued beside the chain's MMAs).  Equal
// to the printed recurrence in exact arithmetic; only rounding differs.
// Because the P_j are symmetric, a matrix's rows serve as its columns: every
// operand is written once, K-major, and used as A and B.
//
// Precision.  Every product is formed from split operands, x = hi + lo with
// hi the rounding of x and lo the rounding of x - hi, as hi*hi + hi*lo +
// lo*hi with fp32 accumulation in TMEM (about 21 bits for fp16, 16 for
// bf16).  The P-chain operands are fp16 (K = 16 per MMA); P0 and the first
// kSplitIters steps use the split, later steps hi*hi alone (the iteration
// corrects its own errors in P once P is near a projector).  The Z update
// uses split bf16 (fp32 range: Z can grow with the iteration count).  The
// landmark logits Q~ K~^T use split bf16.  A single 10-bit product in the
// early steps or in Z leaves Z about 3e-3 off, which ill-conditioned heads
// amplify to several 1e-2 in the output.
//
// Threads 0..255: thread t owns TMEM lane r = t % 128 and column half
// h = t / 128.  Lanes 0..m-1 carry the P chain and r_j, lanes 64..64+m-1
// the Z update (its MMA rows are stacked at row 64), so the two run on
// different warps.  Thread 256 (warp 8) issues the MMAs: an MMA issue
// blocks the issuing thread until the tensor pipe takes it, which must not
// hold up a row thread.
#pragma once

#include <type_traits>

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace pinvpow {

using namespace sm100;

// Arguments of the pseudoinverse bodies (this file's and pinv_pow128.cuh's).
struct Params {
  const float *q_land, *k_land;   // [BH][m][64]
  float *z_out;                   // [BH][m][m]
  uint32_t *err;
  int iters;
  float scale_log2;               // log2(e) / sqrt(d)
};

constexpr int kThreads = 256;       // matrix-row threads
constexpr int kBarThreads = 288;    // plus one issuer warp (warp 8, lane 0 issues)

constexpr int kSplitIters = 3;   // Lemma 1 steps with split fp16 products

template <int M>
struct Cfg {
  static_assert(M == 32 || M == 64, "m <= 64 only");
  static constexpr int NC = M / 2;                  // columns per thread
  // 16-bit operands, K-major, one 128-byte swizzle row per matrix row (K = M
  // <= 64), each as a hi and a lo copy:
  //   a2  [P2 ; P ; P] fp16: rows 0..M-1 = P2, rows 64..64+M-1 = P and rows
  //       128..128+M-1 = P again (stage 1 reads 128 rows from row 64, so that
  //       lanes 64.. of its result repeat lanes 0..)
  //   u   U = 7P - P2 fp16: rows 0..M-1 and again 64..64+M-1
  //   az  Z bf16 at rows 64..64+M-1 (128 rows)
  //   br  r bf16: M rows, two buffers (by step parity: the Z update of a step
  //       reads r of the step before while the new r is written)
  //   q, k  landmark logits operands (bf16, 64 features)
  static constexpr uint32_t kA2 = 192u * 128u, kU = 128u * 128u;
  static constexpr uint32_t a2h = 0, a2l = a2h + kA2;
  static constexpr uint32_t uh = a2l + kA2, ul = uh + kU;
  static constexpr uint32_t azh = ul + kU, azl = azh + 128u * 128u;
  static constexpr uint32_t brh = azl + 128u * 128u, brl = brh + 2u * 64u * 128u;
  static constexpr uint32_t qh = brl + 2u * 64u * 128u;   // br hi / lo: 2 x 8 KB each
  static constexpr uint32_t ql = qh + 128u * 128u;
  static constexpr uint32_t kh = ql + 128u * 128u;
  static constexpr uint32_t kl = kh + 64u * 128u;
  // fp32 scratch over the logits operands (dead once A is formed): P by step
  // parity (A during setup) and P2, [M][64] each with 16-byte chunks
  // XOR-swizzled by row so that row and column accesses avoid bank conflicts
  static constexpr uint32_t pf = qh;                     // [2][64][64] fp32
  static constexpr uint32_t p2f = pf + 2u * 64u * 64u * 4u;
  static constexpr uint32_t red = kl + 64u * 128u;      // [3][M]
  static constexpr uint32_t bars = (red + 3u * M * 4u + 1023u) & ~1023u;
  static constexpr uint32_t total = bars + 1024u;
  static constexpr uint32_t kTmemCols = 256;        // D at column 0 (128 wide), Z update at 128
};

// N (a multiple of 8) values of row `row`, columns c0.. (c0 a multiple of 8),
// into a K-major 16-bit operand pair: hi = rounding of x, lo = rounding of
// x - hi (fp16 when F16, else bf16)
template <int N, bool F16>
__device__ __forceinline__ void put_split(uint32_t hi_base, uint32_t lo_base, int row, int c0,
                                          const float *v, bool with_lo = true) {
  // with_lo is uniform over the block: the lo halves are formed only when
  // they are stored
#pragma unroll
  for (int q = 0; q < N / 8; ++q) {
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = v[8 * q + 2 * e], x1 = v[8 * q + 2 * e + 1];
      h[e] = F16 ? pack_f16(x0, x1) : pack_bf16(x0, x1);
    }
    const uint32_t off = sw128_offset(row, (c0 >> 3) + q);
    st_shared_v4(hi_base + off, h[0], h[1], h[2], h[3]);
  }
  if (!with_lo) return;
#pragma unroll
  for (int q = 0; q < N / 8; ++q) {
    uint32_t l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = v[8 * q + 2 * e], x1 = v[8 * q + 2 * e + 1];
      if constexpr (F16) {
        const float2 hf = __half22float2(__floats2half2_rn(x0, x1));
        l[e] = pack_f16(x0 - hf.x, x1 - hf.y);
      } else {
        const float2 hf = __bfloat1622float2(__floats2bfloat162_rn(x0, x1));
        l[e] = pack_bf16(x0 - hf.x, x1 - hf.y);
      }
    }
    st_shared_v4(lo_base + sw128_offset(row, (c0 >> 3) + q), l[0], l[1], l[2], l[3]);
  }
}

// fp32 [64][64] scratch, 16-byte chunks XOR-swizzled by row: element (r, c)
__device__ __forceinline__ int sw_idx(int r, int c) {
  return r * 64 + ((((c >> 2) ^ (r & 7)) << 2) | (c & 3));
}
template <int N>
__device__ __forceinline__ void put_row(float *buf, int r, int c0, const float *v) {
#pragma unroll
  for (int q = 0; q < N / 4; ++q)
    *(float4 *)(buf + sw_idx(r, c0 + 4 * q)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
template <int N>
__device__ __forceinline__ void get_row(const float *buf, int r, int c0, float *v) {
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    const float4 x = *(const float4 *)(buf + sw_idx(r, c0 + 4 * q));
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
}

template <int N>
__device__ __forceinline__ void ld_cols(uint32_t taddr, float *v) {
  if constexpr (N == 32) {
    tmem_ld32(taddr, v);
  } else if constexpr (N == 16) {
    tmem_ld16(taddr, v);
  } else {
    tmem_ld8(taddr, v);
  }
  tmem_ld_wait();
}

// Runs on threads 0..287 of a block and synchronises them with named barrier
// 1 only.  smem: Cfg<M>::total bytes, 1 KB aligned.  Prm carries q_land,
// k_land ([BH][m][64] fp32), z_out ([BH][m][m] fp32), err, iters and
// scale_log2 = log2(e) / sqrt(d).
// tmem_in: a TMEM allocation of at least Cfg<M>::kTmemCols columns owned by
// the caller, or ~0u to allocate (and free) one here.
// zs_hi, zs_lo (shared-memory addresses, or 0): the final Z is also written
// there as a split bf16 operand pair, K-major, one 128-byte swizzle row per
// matrix row (hi = rounding of z, lo = rounding of z - hi), for a product
// with Z that follows in the same block.  They may lie over this function's
// own operands: they are written after its last MMA has completed.
template <int M, class Prm>
__device__ __forceinline__ void pinv_body(const Prm &prm, uint8_t *smem, int bh,
                                          uint32_t tmem_in = ~0u, uint32_t zs_hi = 0,
                                          uint32_t zs_lo = 0) {
  using C = Cfg<M>;
  constexpr int NC = C::NC;
  const int t = threadIdx.x, warp = t >> 5;
  const int r = t & 127, h = t >> 7;
  const bool rows = t < kThreads;
  const bool issuer = t == kThreads;
  const bool crit = rows && r < M;               // P chain rows
  const bool aux = rows && r >= 64 && r < 64 + M;   // Z update rows
  const int row = crit ? r : r - 64;             // matrix row of this thread
  const int c_lo = h * NC;
  // the P chain's elementwise work: the results of stages 1 and 2 repeat in
  // lanes 64.. (their A operands hold every row twice), so four threads share
  // each row, a quarter of its columns each
  constexpr int NQ = M / 4;
  const bool pc = rows && (r & 63) < M;
  const int prow = r & 63;
  const int cq = ((r >> 6) * 2 + h) * NQ;
  uint64_t *bar_main = (uint64_t *)(smem + C::bars);
  uint64_t *bar_z = bar_main + 1;
  uint32_t *tmem_slot = (uint32_t *)(bar_main + 2);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  float *red = (float *)(smem + C::red);         // row sums [M], column halves [2][M]
  float *pf0 = (float *)(smem + C::pf);          // fp32 P by step parity (A during setup)
  float *p2f = (float *)(smem + C::p2f);         // fp32 P2 of the current step
  const Abort ab{abort_flag, prm.err};
  if (t == 0) {
    mbar_init(bar_main, 1);
    mbar_init(bar_z, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tmem_in != ~0u) {
    if (t == 0) *tmem_slot = tmem_in;
  } else if (warp == 0) {
    tmem_alloc(tmem_slot, C::kTmemCols);
  }

  const uint32_t a2h = smem_u32(smem + C::a2h), a2l = smem_u32(smem + C::a2l);
  const uint32_t uh = smem_u32(smem + C::uh), ul = smem_u32(smem + C::ul);
  const uint32_t azh = smem_u32(smem + C::azh), azl = smem_u32(smem + C::azl);
  const uint32_t brh = smem_u32(smem + C::brh), brl = smem_u32(smem + C::brl);
  const uint32_t qh = smem_u32(smem + C::qh), ql = smem_u32(smem + C::ql);
  const uint32_t kh = smem_u32(smem + C::kh), kl = smem_u32(smem + C::kl);
  const uint32_t ph = a2h + 64u * 128u, pl = a2l + 64u * 128u;   // P at row 64 of a2

  // ---- landmarks -> split bf16 operands (all loads issued first)
  if (rows) {
    constexpr int kPer = M * 8 / kThreads;      // 16-byte chunks per thread per tensor
    const float4 *qg = (const float4 *)(prm.q_land + (size_t)bh * M * 64);
    const float4 *kg = (const float4 *)(prm.k_land + (size_t)bh * M * 64);
    float4 qv[kPer][2], kv[kPer][2];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int idx = t + i * kThreads;
      qv[i][0] = __ldcg(qg + 2 * idx);
      qv[i][1] = __ldcg(qg + 2 * idx + 1);
      kv[i][0] = __ldcg(kg + 2 * idx);
      kv[i][1] = __ldcg(kg + 2 * idx + 1);
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int idx = t + i * kThreads, rr = idx >> 3, ch = idx & 7;
      const float q[8] = {qv[i][0].x, qv[i][0].y, qv[i][0].z, qv[i][0].w,
                          qv[i][1].x, qv[i][1].y, qv[i][1].z, qv[i][1].w};
      const float k[8] = {kv[i][0].x, kv[i][0].y, kv[i][0].z, kv[i][0].w,
                          kv[i][1].x, kv[i][1].y, kv[i][1].z, kv[i][1].w};
      put_split<8, false>(qh, ql, rr, ch * 8, q);
      put_split<8, false>(qh, ql, 64 + rr, ch * 8, q);   // logits repeat in lanes 64..
      put_split<8, false>(kh, kl, rr, ch * 8, k);
    }
  }
  fence_async_smem();
  tc_fence_before();
  named_barrier(1, kBarThreads);
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t t_d = tmem + lane_base, t_z = tmem + lane_base + 128;
  const uint32_t id_bf = make_idesc(kFmtBF16, 128, M, 0, 0);
  const uint32_t id_f16 = make_idesc(kFmtF16, 128, M, 0, 0);
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
  // D (+)= A B^T over K = KK (steps of 16), K-major 16-bit operands given by
  // their descriptors (a K step adds 32 bytes, i.e. 2 to the address field)
  auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, auto kk, bool acc) {
    constexpr int KK = decltype(kk)::value;
#pragma unroll
    for (int k = 0; k < KK / 16; ++k)
      mma_bf16(d, a + 2u * k, b + 2u * k, idesc, (acc || k > 0) ? 1u : 0u);
  };
  using KM = std::integral_constant<int, M>;
  using K64 = std::integral_constant<int, 64>;
  // split product: hi*hi + hi*lo + lo*hi (or hi*hi alone)
  auto mma3 = [&](uint32_t d, uint64_t a_h, uint64_t a_l, uint64_t b_h, uint64_t b_l,
                  uint32_t idesc, auto kk, bool split) {
    mma(d, a_h, b_h, idesc, kk, false);
    if (split) {
      mma(d, a_h, b_l, idesc, kk, true);
      mma(d, a_l, b_h, idesc, kk, true);
    }
  };
  // operand descriptors (built where an MMA is issued)
  auto sd = [](uint32_t a) { return make_sdesc(a, 16, 1024); };
  float *zg = prm.z_out + (size_t)bh * M * M;

  // ---- logits (split bf16) -> TMEM columns 0..M-1
  if (issuer) {
    mma3(tmem, sd(qh), sd(ql), sd(kh), sd(kl), id_bf, K64{}, true);
    mma_commit(bar_main);
  }
  wait_main(pc);
  // ---- row softmax, four threads per row (a quarter of the columns each;
  //      the row's maximum and sum combine the quarters in order through
  //      shared memory): A into the split fp16 operand at rows 64.. and
  //      128.. of a2 (the P position, twice, for A A^T) and an fp32 copy;
  //      quarter row sums of |A|
  float* red4 = p2f;   // [3][4][64]: maxima, sums, |A| sums (logits operands are dead)
  const int qi = cq / NQ;
  float av[NQ];
  if (ok && pc) {
    ld_cols<NQ>(t_d + cq, av);
    float mx = av[0];
#pragma unroll
    for (int k = 1; k < NQ; ++k) mx = fmaxf(mx, av[k]);
    red4[qi * 64 + prow] = mx;
  }
  named_barrier(1, kBarThreads);
  if (ok && pc) {
    const float moff = fmaxf(fmaxf(red4[prow], red4[64 + prow]),
                             fmaxf(red4[128 + prow], red4[192 + prow])) * prm.scale_log2;
    float sm = 0.f;
#pragma unroll
    for (int k = 0; k < NQ; ++k) {
      av[k] = fast_exp2(fmaf(av[k], prm.scale_log2, -moff));
      sm += av[k];
    }
    red4[256 + qi * 64 + prow] = sm;
  }
  named_barrier(1, kBarThreads);
  if (ok && pc) {
    const float inv = 1.f / (((red4[256 + prow] + red4[320 + prow]) + red4[384 + prow]) +
                             red4[448 + prow]);
    float rs = 0.f;
#pragma unroll
    for (int k = 0; k < NQ; ++k) {
      av[k] *= inv;
      rs += fabsf(av[k]);
    }
    red4[512 + qi * 64 + prow] = rs;
    put_split<NQ, true>(ph, pl, prow, cq, av);
    put_split<NQ, true>(ph, pl, 64 + prow, cq, av);
    put_row<NQ>(pf0, prow, cq, av);
  }
  if (!sync_ops()) ok = false;
  NYS_MARK(kTrMid, 8);
  // ---- A A^T on the tensor cores; meanwhile the Z rows take the columns of
  //      A (their Z0 rows up to c0) and their partial column sums
  if (ok && issuer) {
    mma3(tmem, sd(ph), sd(pl), sd(ph), sd(pl), id_f16, KM{}, true);
    mma_commit(bar_main);
  }
  float acol[NC];
  if (ok && aux) {
    float cs = 0.f;
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      acol[k] = pf0[sw_idx(c_lo + k, row)];
      cs += fabsf(acol[k]);
    }
    red[M + h * M + row] = cs;
  }
  named_barrier(1, kBarThreads);
  // ||A||_1 (largest column sum) and ||A||_inf (largest row sum): every warp
  // reduces the m rows' partials, lane l taking rows l and l + 32
  float n1 = 0.f, ninf = 0.f;
  {
    const int l = t & 31;
#pragma unroll
    for (int i = l; i < M; i += 32) {
      n1 = fmaxf(n1, red[M + i] + red[2 * M + i]);
      ninf = fmaxf(ninf, ((red4[512 + i] + red4[576 + i]) + red4[640 + i]) + red4[704 + i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n1 = fmaxf(n1, __shfl_xor_sync(0xffffffffu, n1, o));
      ninf = fmaxf(ninf, __shfl_xor_sync(0xffffffffu, ninf, o));
    }
  }
  const float c0 = 1.f / (n1 * ninf);
  if (ok && aux) {   // Z0 = c0 A^T, rows 64.. of the Z operand
#pragma unroll
    for (int k = 0; k < NC; ++k) acol[k] *= c0;
    if (prm.iters == 0) {
#pragma unroll
      for (int q = 0; q < NC / 4; ++q)
        *(float4 *)(zg + (size_t)row * M + c_lo + 4 * q) =
            make_float4(acol[4 * q], acol[4 * q + 1], acol[4 * q + 2], acol[4 * q + 3]);
      if (zs_hi) put_split<NC, false>(zs_hi, zs_lo, row, c_lo, acol);
    } else {
      put_split<NC, false>(azh, azl, 64 + row, c_lo, acol);
    }
  }
  wait_main(pc);
  // P_j of this thread's row quarter stays in registers through the steps
  float preg[NQ];
  if (ok && pc) {   // P0 = c0 A A^T
    ld_cols<NQ>(t_d + cq, preg);
#pragma unroll
    for (int k = 0; k < NQ; ++k) preg[k] *= c0;
    put_split<NQ, true>(ph, pl, prow, cq, preg);
    put_split<NQ, true>(ph, pl, 64 + prow, cq, preg);
  }
  if (!sync_ops()) ok = false;
  NYS_MARK(kTrMid, 9);

  // ---- Lemma 1 steps.  Z pipeline: the update Z_j = Z_{j-1} r_{j-1} is
  //      issued in stage 2 of step j (behind the chain's MMA) and read back
  //      by the Z rows in stage 1 of step j + 1; r_j alternates between two
  //      buffers by step parity.
  const int iters = ok ? prm.iters : 0;
  bool good = ok;   // block-uniform: no stage failed
  const uint32_t id_z = make_idesc(kFmtBF16, 128, M, 0, 0);
  constexpr uint32_t kBr = 64u * 128u;            // one r buffer
  // stage 2 multiplies U (A, 128 rows of which the first m are U) by the
  // 128 rows of [P2; P] (B, N = 128): columns 0.. give U P2 = 7P^3 - P^4 and
  // columns 64.. give U P = 7P^2 - P^3, in the same TMEM lane (the P_j
  // commute), so the thread that holds P_j and P_j^2 of a row forms both
  // P_{j+1} and r_j of it
  const uint32_t id_s2 = make_idesc(kFmtF16, 128, 128, 0, 0);
  for (int j = 0; j < iters; ++j) {
    const bool split = j < kSplitIters, split_next = j + 1 < kSplitIters;
    // stage 1: P2 = P P
    if (issuer) {
      mma3(tmem, sd(ph), sd(pl), sd(ph), sd(pl), id_f16, KM{}, split);
      mma_commit(bar_main);
    }
    if (j >= 2) {   // Z_{j-1} back into the Z operand
      wait_z(aux);
      if (ok && aux) {
        float z[NC];
        ld_cols<NC>(t_z + c_lo, z);
        put_split<NC, false>(azh, azl, 64 + row, c_lo, z);
      }
    }
    wait_main(pc);
    if (j < 8) NYS_MARK(kTrMid, 40 + j);
    float p2[NQ];
    if (ok && pc) {
      float uu[NQ];
      ld_cols<NQ>(t_d + cq, p2);
#pragma unroll
      for (int k = 0; k < NQ; ++k) uu[k] = fmaf(7.f, preg[k], -p2[k]);
      put_split<NQ, true>(a2h, a2l, prow, cq, p2, split);
      put_split<NQ, true>(uh, ul, prow, cq, uu, split);
      put_split<NQ, true>(uh, ul, 64 + prow, cq, uu, split);
    }
    if (!sync_ops()) {
      good = false;
      break;
    }
    // stage 2: U [P2; P], then Z_j = Z_{j-1} r_{j-1}
    if (issuer) {
      mma3(tmem, sd(uh), sd(ul), sd(a2h), sd(a2l), id_s2, KM{}, split);
      mma_commit(bar_main);
      if (j > 0) {
        const uint32_t rb = ((j - 1) & 1) * (kBr >> 4);
        mma3(tmem + 128, sd(azh), sd(azl), sd(brh) + rb, sd(brl) + rb, id_z, KM{}, true);
        mma_commit(bar_z);
      }
    }
    wait_main(pc);
    if (j < 8) NYS_MARK(kTrMid, 48 + j);
    if (ok && pc) {
      // P_{j+1} = 1/4 (13 P - 15 P2 + 7 P^3 - P^4), r_j = 1/4 (13I - 15 P + 7 P^2 - P^3)
      float x[NQ], y[NQ];
      ld_cols<NQ>(t_d + cq, x);
      ld_cols<NQ>(t_d + 64 + cq, y);
#pragma unroll
      for (int k = 0; k < NQ; ++k) {
        const float pj = preg[k];
        preg[k] = 0.25f * fmaf(13.f, pj, fmaf(-15.f, p2[k], x[k]));
        y[k] = 0.25f * ((cq + k == prow ? 13.f : 0.f) + fmaf(-15.f, pj, y[k]));
      }
      put_split<NQ, true>(ph, pl, prow, cq, preg, split_next);
      put_split<NQ, true>(ph, pl, 64 + prow, cq, preg, split_next);
      const uint32_t rb = (j & 1) * kBr;
      put_split<NQ, false>(brh + rb, brl + rb, prow, cq, y);
    }
    if (j < 8) NYS_MARK(kTrMid, 16 + j);
    if (!sync_ops()) {
      good = false;
      break;
    }
  }
  // ---- Z = Z_{iters-1} r_{iters-1}
  if (iters > 0 && good) {
    if (iters >= 2) {   // Z_{iters-1} from the last update into the Z operand
      wait_z(aux);
      if (ok && aux) {
        float z[NC];
        ld_cols<NC>(t_z + c_lo, z);
        put_split<NC, false>(azh, azl, 64 + row, c_lo, z);
      }
      good = sync_ops();
    }
    if (good) {
      if (issuer) {
        const uint32_t rb = ((iters - 1) & 1) * (kBr >> 4);
        mma3(tmem + 128, sd(azh), sd(azl), sd(brh) + rb, sd(brl) + rb, id_z, KM{}, true);
        mma_commit(bar_z);
      }
      wait_z(aux);
      float z[NC];
      if (ok && aux) {
        ld_cols<NC>(t_z + c_lo, z);
#pragma unroll
        for (int q = 0; q < NC / 4; ++q)
          *(float4 *)(zg + (size_t)row * M + c_lo + 4 * q) =
              make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
        if (zs_hi) put_split<NC, false>(zs_hi, zs_lo, row, c_lo, z);
      }
    }
  }
  tc_fence_before();
  named_barrier(1, kBarThreads);
  if (t == 0 && !*abort_flag) {
    mbar_inval(bar_main);
    mbar_inval(bar_z);
  }
  if (warp == 0 && tmem_in == ~0u) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pinvpow
}  // namespace nys
