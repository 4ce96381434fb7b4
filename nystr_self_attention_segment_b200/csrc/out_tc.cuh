// Output kernel of the bf16 path on 5th-generation tensor cores:
//
//   out[i] = softmax_m(s q_i . K~^T) W + sum_t w_h[t] V[i + t - (k-1)/2]
//
// ("Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4: Eq. 17 / Algorithm 1 for F~ W, Figure 4 for
// the DConv skip).  W = Z (B~ V) comes from the workspace.
//
// A block owns a run of 128-row tiles of one (batch, head).  Per tile:
//   TMA  Q tile (128 x 64 bf16) and the V tile with its conv halo
//        (kconv = 128 + k - 1 rounded up to 16 rows; zero outside [0, n)),
//   MMA  S = Q K~^T                 (M=128, N=m, K=64; operands in smem),
//   MMA  O = T_h V_halo             (M=128, N=64, K=kconv; T_h in TMEM),
//        T_h is the banded Toeplitz matrix of the head's conv kernel
//        (T_h[r][j] = w_h[j - r]), so the depthwise conv runs on the tensor
//        cores,
//   softmax warpgroup: row softmax of S (one TMEM lane = one row); P (the F~
//        tile, bf16) written into TMEM over S,
//   MMA  O += P W                   (M=128, N=64, K=m; P read from TMEM),
//   softmax warpgroup: O -> bf16 -> shared memory -> TMA store (clipped at n).
// Two softmax warpgroups take alternate tiles.
// Warps: 0 TMA producer, 1 and 2 MMA issuers (one per softmax warpgroup;
// warp 1 owns TMEM), 4-7 and 8-11 softmax + epilogue.  TMEM: warpgroup w has
// S at w*(m+64) and O right after it; T_h follows at 2*(m+64).
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace outtc {

using namespace sm100;

constexpr int kStages = 4;

// Softmax warpgroups per block (tiles in flight): three for m <= 64, two for
// m = 128 (TMEM holds S and O of each, plus the Toeplitz operand).  Warps: 0
// TMA producer, 1..NW MMA issuers (one per softmax warpgroup; warp 1 owns
// TMEM), 4.. the softmax warpgroups, kLoader the W operand copy and the
// ragged-batch masking.
template <int M>
struct Warps {
  static constexpr int NW = M <= 64 ? 3 : 2;
  static constexpr int kLoader = NW == 3 ? 4 + 4 * NW : 3;
  static constexpr int kThreads = NW == 3 ? 32 * (kLoader + 1) : 384;
};
constexpr int kTileRows = 128;
constexpr int kMaxKconv = 192;

struct SmemLayout {
  uint32_t kt, w, q[kStages], v[kStages], o[3], cw, bars, total;
};

__host__ __device__ inline SmemLayout smem_layout(int m, int kconv) {
  SmemLayout L;
  uint32_t off = 0;
  auto take = [&](uint32_t b) {
    uint32_t at = off;
    off += (b + 1023u) & ~1023u;
    return at;
  };
  L.kt = take(m * 128u);
  L.w = take(m * 128u);
  for (int s = 0; s < kStages; ++s) {
    L.q[s] = take(16384u);
    L.v[s] = take(kconv * 128u);
  }
  // an output staging tile per softmax warpgroup (three for m <= 64)
  for (int w = 0; w < 3; ++w) L.o[w] = w < (m <= 64 ? 3 : 2) ? take(16384u) : 0u;
  L.cw = take(256u);
  L.bars = take(256u);
  L.total = off + 1024u;   // slack for aligning the dynamic smem base to 1 KB
  return L;
}

struct Params {
  const float *k_land;     // [BH][m][64] fp32
  const uint8_t *w_op;     // [BH][m][128 B]: W as the bf16 B operand of P W
                           // (row j = landmark, 64 features, 128-byte swizzle)
  const float *conv_w;     // [H][k] or null
  uint32_t *err;
  int n, heads, conv_k, kconv;
  int tiles_per_head, ctas_per_head;
  float scale_log2;
  const int *lens;         // [batch] tokens per element (ragged batches) or null
  int m;
  const uint32_t *w_flag;  // [BH]: nonzero once the previous kernel has stored W of the head
};

// One run of 128-row tiles [t_begin, t_end) of (batch, head) bh.  tmem_in: a
// 512-column TMEM allocation owned by the caller, or ~0u to allocate (and
// free) one here.  smem: smem_layout(M, kconv).total bytes, 1 KB aligned.
template <int M>
// wait_prev: launched with programmatic dependent launch while the previous
// kernel still runs.  Everything that reads only the inputs and K~ (barriers,
// TMEM, the Toeplitz operand, the first kStages tiles' S and conv) runs at
// once; the W operand is loaded once the head's flag (prm.w_flag) says the
// previous kernel has stored it, so a head's P W starts as soon as its own W
// exists, not when the whole previous grid has completed.  The block waits
// for the previous grid before it exits, so that this grid completes after
// it.
__device__ __forceinline__ void out_body(const CUtensorMap *map_q, const CUtensorMap *map_v,
                                         const CUtensorMap *map_o, const Params &prm,
                                         uint8_t *smem, int bh, int t_begin, int t_end,
                                         uint32_t tmem_in, bool wait_prev = false) {
  const SmemLayout L = smem_layout(M, prm.kconv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = bh % prm.heads;
  const int ntiles = t_end - t_begin;
  const bool conv = prm.conv_w != nullptr;
  const int half = (prm.conv_k - 1) / 2;
  // rows [0, L) of the element are real (L = n, or its own length for ragged
  // batches; an invalid length reads as 0).  Output rows from L on are zero,
  // and V rows from L on read as zero in the conv: a warp (3) clears them in
  // the staged V tile before the conv MMA may read it.
  int seq = prm.n;
  if (prm.lens) {
    seq = prm.lens[bh / prm.heads];
    if (seq < prm.m || seq > prm.n || (long)(prm.m - 1) * ((seq + prm.m - 1) / prm.m) >= seq)
      seq = 0;
  }
  const bool mask_v = conv && prm.lens != nullptr;
  // Q and V are read here for the last time in the pass and out is not read
  // again: their lines leave L2 first
  const uint64_t last_use = policy_evict_first();
  // TMEM per softmax warpgroup: S (M columns, P written over it as bf16
  // pairs) and O (64 columns); the Toeplitz operand after them.
  constexpr int NW = Warps<M>::NW, kThreads = Warps<M>::kThreads;
  constexpr uint32_t kOcol = M;
  constexpr uint32_t kStride = kOcol + 64;    // TMEM columns per softmax warpgroup
  constexpr uint32_t kT = NW * kStride;       // Toeplitz operand columns
  static_assert(kT + kMaxKconv / 2 <= 512, "TMEM");

  uint64_t *bars = (uint64_t *)(smem + L.bars);
  uint64_t *full = bars;                   // [kStages]
  uint64_t *empty = bars + kStages;        // [kStages]
  uint64_t *s_full = bars + 2 * kStages;   // [NW] per softmax warpgroup
  uint64_t *p_ready = s_full + NW;
  uint64_t *o_full = p_ready + NW;
  uint64_t *tm_free = o_full + NW;
  uint64_t *w_ready = tm_free + NW;        // W operand in shared memory
  uint64_t *v_ready = w_ready + 1;         // [kStages] V tile masked past L
  uint32_t *tmem_slot = (uint32_t *)(v_ready + kStages);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  const Abort ab{abort_flag, prm.err};
  float *cw = (float *)(smem + L.cw);
  NYS_MARK(kTrOut, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NW; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_ready[b], 128);
      mbar_init(&o_full[b], 1);
      mbar_init(&tm_free[b], 128);
    }
    mbar_init(w_ready, 1);
    for (int s = 0; s < kStages; ++s) mbar_init(&v_ready[s], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(map_q);
    tma_prefetch_desc(map_o);
    if (conv) tma_prefetch_desc(map_v);
  }
  if (tmem_in != ~0u) {
    if (threadIdx.x == 0) *tmem_slot = tmem_in;
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
  }

  if (conv && threadIdx.x < prm.conv_k)
    cw[threadIdx.x] = prm.conv_w[(size_t)head * prm.conv_k + threadIdx.x];
  tc_fence_before();
  __syncthreads();   // barriers, TMEM address, conv weights
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t bytes = 16384u + (conv ? (uint32_t)prm.kconv * 128u : 0u);
  const int pre = ntiles < kStages ? ntiles : kStages;   // tile loads issued up front
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      const int r0 = (t_begin + i) * kTileRows;
      mbar_expect_tx(&full[i], bytes);
      tma_load_3d_hint(smem + L.q[i], map_q, &full[i], 0, r0, bh, last_use);
      if (conv) tma_load_3d_hint(smem + L.v[i], map_v, &full[i], 0, r0 - half, bh, last_use);
    }
  }
  // Toeplitz operand into TMEM: row r (lane r), columns j = halo rows
  if (conv && warp >= 4 && warp < 8) {
    const int r = threadIdx.x - 128;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    for (int c0 = 0; c0 < prm.kconv / 2; c0 += 16) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j0 = 2 * (c0 + e) - r, j1 = j0 + 1;
        const float lo = (j0 >= 0 && j0 < prm.conv_k) ? cw[j0] : 0.f;
        const float hi = (j1 >= 0 && j1 < prm.conv_k) ? cw[j1] : 0.f;
        pk[e] = pack_bf16(lo, hi);
      }
      tmem_st16(tmem + lane_base + kT + c0, pk);
    }
    tmem_st_wait();
  }
  // ---- per-head operands, bf16 with the 128-byte swizzle: K~ (B of S,
  // K-major; written by the segment-mean kernel, which has completed before
  // this grid launches: every block of the previous kernel lets it launch
  // only after its own wait for that kernel) now; W (B of P W, MN-major; written by
  // the previous kernel) by warp 3 after the wait, so that the first tiles'
  // S, conv and softmax overlap the previous kernel's tail.  W arrives as
  // the ready bf16 operand in one bulk copy.
  auto put_op = [&](uint32_t base, const float4 *src, int idx) {
    const float4 a0 = __ldcg(src + 2 * idx), a1 = __ldcg(src + 2 * idx + 1);
    st_shared_v4(base + sw128_offset(idx >> 3, idx & 7), pack_bf16(a0.x, a0.y),
                 pack_bf16(a0.z, a0.w), pack_bf16(a1.x, a1.y), pack_bf16(a1.z, a1.w));
  };
  {
    const float4 *kt = (const float4 *)(prm.k_land + (size_t)bh * M * 64);
    for (int idx = threadIdx.x; idx < M * 8; idx += kThreads) put_op(smem_u32(smem + L.kt), kt, idx);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  NYS_MARK(kTrOut, 1);
  if (warp == Warps<M>::kLoader && lane == 0) {
    // the flag's acquire orders the previous kernel's W stores before this
    // thread's generic accesses; the proxy fence then orders them before the
    // bulk copy
    const bool have_w = !wait_prev || flag_wait(prm.w_flag + bh, ab, kWaitLimitCycles);
    NYS_MARK_T(kTrOut, 2);
    if (have_w) {
      fence_async_global();
      mbar_expect_tx(w_ready, M * 128u);
      bulk_load(smem + L.w, prm.w_op + (size_t)bh * M * 128, M * 128u, w_ready);
    }
  }
  if (warp == Warps<M>::kLoader && mask_v) {
    // ragged batches: halo rows at or past L of every staged V tile become
    // zero before its conv MMA (v_ready); tiles are taken in order, each
    // after its load, so the barrier phases cannot run ahead
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % kStages;
      if (!mbar_wait(&full[s], (i / kStages) & 1, ab)) break;
      const int first = seq - ((t_begin + i) * kTileRows - half);   // first halo row past L
      if (first < prm.kconv) {
        const uint32_t base = smem_u32(smem + L.v[s]);
        for (int q = (first > 0 ? first : 0) * 8 + lane; q < prm.kconv * 8; q += 32)
          st_shared_v4(base + (uint32_t)q * 16u, 0u, 0u, 0u, 0u);
        fence_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_ready[s]);
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int i = pre; i < ntiles; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, ab)) break;
        const int r0 = (t_begin + i) * kTileRows;
        mbar_expect_tx(&full[s], bytes);
        tma_load_3d_hint(smem + L.q[s], map_q, &full[s], 0, r0, bh, last_use);
        if (conv) tma_load_3d_hint(smem + L.v[s], map_v, &full[s], 0, r0 - half, bh, last_use);
      }
      // consume the stage releases nobody else waits for (no tensor-core
      // arrival may be pending when the barriers are invalidated)
      for (int i = ntiles > kStages ? ntiles - kStages : 0; i < ntiles; ++i)
        if (!mbar_wait(&empty[i % kStages], (i / kStages) & 1, ab)) break;
    }
  } else if (warp >= 1 && warp <= NW) {
    // ------------------------------------------------------------ MMA issuers
    // one per softmax warpgroup, so that neither waits behind the other
    if (lane == 0) {
      const int w = warp - 1;
      const uint32_t id_s = make_idesc(kFmtBF16, 128, M, 0, 0);
      const uint32_t id_o = make_idesc(kFmtBF16, 128, 64, 0, 1);
      const uint32_t kt_a = smem_u32(smem + L.kt), w_a = smem_u32(smem + L.w);
      // S of the next tile goes out right after P W of the current one (the
      // tensor pipe runs one issuer's MMAs in order, so it cannot overwrite
      // P before P W has read it); only the conv into O waits for the
      // epilogue to release O.
      auto issue_s = [&](int i) -> bool {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1, ab)) return false;
        tc_fence_after();
        const uint32_t q_a = smem_u32(smem + L.q[s]);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem + w * kStride, make_sdesc(q_a + 32 * k, 16, 1024),
                   make_sdesc(kt_a + 32 * k, 16, 1024), id_s, k > 0);
        mma_commit(&s_full[w]);
        return true;
      };
      bool ok = w < ntiles ? issue_s(w) : true;
      for (int i = w; i < ntiles && ok; i += NW) {
        const int s = i % kStages, u = i / NW;
        if (!mbar_wait(&tm_free[w], (u & 1) ^ 1, ab)) break;
        tc_fence_after();
        if (conv) {
          if (mask_v && !mbar_wait(&v_ready[s], (i / kStages) & 1, ab)) break;
          tc_fence_after();
          const uint32_t v_a = smem_u32(smem + L.v[s]);
          for (int k = 0; k < prm.kconv / 16; ++k)
            mma_bf16_ts(tmem + w * kStride + kOcol, tmem + kT + 8 * k,
                        make_sdesc(v_a + k * 2048u, 16, 1024), id_o, k > 0);
        }
        mma_commit(&empty[s]);
        if (!mbar_wait(&p_ready[w], u & 1, ab)) break;
        if (u == 0 && !mbar_wait(w_ready, 0, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < M / 16; ++k)
          mma_bf16_ts(tmem + w * kStride + kOcol, tmem + w * kStride + 8 * k,
                      make_sdesc(w_a + k * 2048u, 16, 1024), id_o, (conv || k > 0) ? 1u : 0u);
        mma_commit(&o_full[w]);
        if (i + NW < ntiles) ok = issue_s(i + NW);
      }
    }
  } else if (warp >= 4 && warp < 4 + 4 * NW) {
    // ------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) >> 2;
    const int r = threadIdx.x & 127;                 // tile row == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + wg * kStride;
    for (int i = wg; i < ntiles; i += NW) {
      const int u = i / NW;
      if (!mbar_wait(&s_full[wg], u & 1, ab)) break;
      if (threadIdx.x == 128 && blockIdx.x == 0 && u < 8) NYS_MARK_T(kTrOut, 16 + u);
      tc_fence_after();
      float v[M];
#pragma unroll
      for (int c = 0; c < M; c += 32) tmem_ld32(t_s + c, v + c);
      tmem_ld_wait();
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = v[q];
#pragma unroll
      for (int c = 8; c < M; ++c) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
      const float moff = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         prm.scale_log2;
      float ps[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) ps[q] = 0.f;
#pragma unroll
      for (int c = 0; c < M; ++c) {
        v[c] = fast_exp2(fmaf(v[c], prm.scale_log2, -moff));
        ps[c & 7] += v[c];
      }
      const float inv =
          1.f / (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7])));
      uint32_t pk[M / 2];
#pragma unroll
      for (int c = 0; c < M; c += 2) pk[c >> 1] = pack_bf16(v[c] * inv, v[c + 1] * inv);
#pragma unroll
      for (int c = 0; c < M / 2; c += 16) tmem_st16(t_s + c, pk + c);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[wg]);
      if (threadIdx.x == 128 && blockIdx.x == 0 && u < 8) NYS_MARK_T(kTrOut, 24 + u);
      if (!mbar_wait(&o_full[wg], u & 1, ab)) break;
      if (threadIdx.x == 128 && blockIdx.x == 0 && u < 8) NYS_MARK_T(kTrOut, 32 + u);
      tc_fence_after();
      float o[64];
      tmem_ld32(t_s + kOcol, o);
      tmem_ld32(t_s + kOcol + 32, o + 32);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&tm_free[wg]);
      if (threadIdx.x == 128 && u < 4) NYS_MARK_T(kTrOut, 8 + u);
      // this warpgroup's staging buffer was last used NW tiles ago
      if (r == 0) bulk_wait_read0();
      named_barrier(2 + wg, 128);
      if ((t_begin + i) * kTileRows + r >= seq) {   // padding rows of a ragged element
#pragma unroll
        for (int c = 0; c < 64; ++c) o[c] = 0.f;
      }
      const uint32_t o_row = smem_u32(smem + L.o[wg]);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(o_row + sw128_offset(r, c), pack_bf16(o[8 * c], o[8 * c + 1]),
                     pack_bf16(o[8 * c + 2], o[8 * c + 3]), pack_bf16(o[8 * c + 4], o[8 * c + 5]),
                     pack_bf16(o[8 * c + 6], o[8 * c + 7]));
      fence_async_smem();
      named_barrier(2 + wg, 128);
      if (r == 0) {
        tma_store_3d_hint(map_o, smem + L.o[wg], 0, (t_begin + i) * kTileRows, bh, last_use);
        bulk_commit();
      }
      if (threadIdx.x == 128 && blockIdx.x == 0 && u < 8) NYS_MARK_T(kTrOut, 40 + u);
    }
    if (r == 0) bulk_wait0();

  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag)
    for (int b = 0; b < 3 * kStages + 4 * NW + 1; ++b) mbar_inval(bars + b);
  if (warp == 1 && tmem_in == ~0u) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (wait_prev && threadIdx.x == 0) griddep_wait();
  NYS_MARK(kTrOut, 4);
}

template <int M>
__global__ void __launch_bounds__(Warps<M>::kThreads, 1)
out_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_v,
              const __grid_constant__ CUtensorMap map_o, const Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int bh = blockIdx.x / prm.ctas_per_head;
  const int part = blockIdx.x % prm.ctas_per_head;
  const int t_begin = (int)((long)part * prm.tiles_per_head / prm.ctas_per_head);
  const int t_end = (int)((long)(part + 1) * prm.tiles_per_head / prm.ctas_per_head);
  // launched early (programmatic dependent launch): out_body reads K~ at
  // once (its kernel completed before the previous one could let this grid
  // launch) and W after the head's flag
  out_body<M>(&map_q, &map_v, &map_o, prm, smem, bh, t_begin, t_end, ~0u, true);
}

}  // namespace outtc
}  // namespace nys
