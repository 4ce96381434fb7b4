// The projections of the attention layer on 5th-generation tensor cores:
//   Q, K, V = X W_Q^T, X W_K^T, X W_V^T   ("Nystromformer: A Nystrom-Based
//   Algorithm for Approximating Self-Attention", "Standard Self-Attention:
//   The Mathematical Baseline"; Figure 4 takes the layer input X), and
//   Y = concat_h(O_h) W_O^T
// as C[rows, N] = A[rows, K] B[N, K]^T with bf16 operands and fp32
// accumulation in TMEM.
//
// A block computes one 128 x 128 tile of C.  Its 128 rows are tokens of one
// batch element (tile i0 .. i0 + 127 of n; rows past n read as zero and are
// not stored), so the A tiles come straight from the [B][n][D] input (QKV
// projection: K block kb = features kb*64 ..) or from the [B][H][n][64]
// attention output (output projection: K block kb = head kb), both through
// one 3-D tensor map with a 64 x 128 box.  B is the [N][K] weight
// (nn.Linear layout).  Warp 0 streams A and B tiles through a kStages ring
// (TMA, no multicast), warp 1 issues the MMAs (M = 128, N = 128, K = 16
// each) into a 128-column TMEM accumulator, and warps 4-7 (TMEM lanes 0-127,
// one row each) convert the accumulator to bf16 and store it:
//   kQkv  columns c of [Q | K | V] go to tensor c / D, head (c % D) / 64 of
//         the [B][H][n][64] outputs;
//   kOut  the [B][n][N] output.
#pragma once

#include "sm100.cuh"

namespace nys {
namespace gemm {

using namespace sm100;

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = 6;
constexpr int kThreads = 256;
constexpr uint32_t kStageBytes = 2u * kBM * kBK * 2u;   // A + B tiles, 32 KB
constexpr uint32_t kSmem = kStages * kStageBytes + 1024u + 1024u;

enum Mode { kQkv = 0, kOut = 1 };

struct Params {
  int n, batch, heads, N, K;     // rows per element, elements, heads, C columns, K
  int mtiles, ntiles;            // tiles per element along n, along N
  __nv_bfloat16 *q, *k, *v;      // kQkv: [B][H][n][64]
  __nv_bfloat16 *y;              // kOut: [B][n][N]
  uint32_t *err;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
            const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = (uint64_t *)(smem + kStages * kStageBytes);
  uint64_t *full = bars, *empty = bars + kStages, *acc_full = bars + 2 * kStages;
  uint32_t *tmem_slot = (uint32_t *)(acc_full + 1);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  const Abort ab{abort_flag, p.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tile: N fastest, so that neighbouring blocks share their A tile in L2
  const int tile = blockIdx.x;
  const int nt = tile % p.ntiles;
  const int mt = (tile / p.ntiles) % p.mtiles;
  const int b = tile / (p.ntiles * p.mtiles);
  const int i0 = mt * kBM, n0 = nt * kBN;
  const int kblocks = p.K / kBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages && !mbar_wait(&empty[s], ((kb / kStages) & 1) ^ 1, ab)) break;
      uint8_t *sa = smem + s * kStageBytes, *sb = sa + kBM * kBK * 2;
      mbar_expect_tx(&full[s], kStageBytes);
      if (MODE == kQkv)
        tma_load_3d(sa, &map_a, &full[s], kb * kBK, i0, b);   // X [B][n][K]
      else
        tma_load_3d(sa, &map_a, &full[s], 0, i0, b * p.heads + kb);   // O [B*H][n][64]
      tma_load_3d(sb, &map_b, &full[s], kb * kBK, n0, 0);     // W [N][K]
    }
    for (int kb = kblocks > kStages ? kblocks - kStages : 0; kb < kblocks; ++kb)
      if (!mbar_wait(&empty[kb % kStages], (kb / kStages) & 1, ab)) break;
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = make_idesc(kFmtBF16, kBM, kBN, 0, 0);
    bool ok = true;
    for (int kb = 0; kb < kblocks && ok; ++kb) {
      const int s = kb % kStages;
      if (!(ok = mbar_wait(&full[s], (kb / kStages) & 1, ab))) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * kStageBytes), sb = sa + kBM * kBK * 2;
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)
        mma_bf16(tmem, make_sdesc(sa + 32 * k, 16, 1024), make_sdesc(sb + 32 * k, 16, 1024), idesc,
                 (kb > 0 || k > 0) ? 1u : 0u);
      mma_commit(&empty[s]);
    }
    mma_commit(acc_full);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int r = threadIdx.x - 128;   // tile row == TMEM lane
    const int i = i0 + r;
    const uint32_t t_acc = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    if (mbar_wait(acc_full, 0, ab)) {
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kBN; c0 += 64) {
        float v[64];
        tmem_ld32(t_acc + c0, v);
        tmem_ld32(t_acc + c0 + 32, v + 32);
        tmem_ld_wait();
        if (i < p.n && n0 + c0 < p.N) {
          uint4 o[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            o[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                              pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                              pack_bf16(v[8 * q + 6], v[8 * q + 7]));
          __nv_bfloat16 *dst;
          if (MODE == kQkv) {
            const int c = n0 + c0, D = p.heads * 64;
            const int which = c / D, h = (c % D) / 64;
            __nv_bfloat16 *base = which == 0 ? p.q : (which == 1 ? p.k : p.v);
            dst = base + (((size_t)b * p.heads + h) * p.n + i) * 64;
          } else {
            dst = p.y + ((size_t)b * p.n + i) * p.N + n0 + c0;
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) ((uint4 *)dst)[q] = o[q];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag)
    for (int s = 0; s < 2 * kStages + 1; ++s) mbar_inval(bars + s);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace gemm
}  // namespace nys
