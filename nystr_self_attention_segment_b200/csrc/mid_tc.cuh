// Middle stage of the bf16 path, one launch:
//   blocks [0, BH)            the landmark kernel A and its pseudoinverse Z
//                             (one head each: pinv_pow.cuh for m <= 64,
//                             pinv_pow128.cuh for m = 128),
//   blocks [BH, BH*(1+S))     Y = B~ V streamed over the keys, S blocks per head
//                             ("Nystromformer: A Nystrom-Based Algorithm for
//                             Approximating Self-Attention", section 3.4,
//                             Eq. 17 / Algorithm 1; B~ = softmax(Q~ K^T/sqrt(d))
//                             over the n keys is never stored).
// Each B~ V block leaves one partial softmax state per landmark (running
// maximum, sum, unnormalised Y); the last B~ V block of a head merges them
// into Y, and the second of {that block, the pseudoinverse block} to finish
// forms W = Z Y on the tensor cores (merge_y, form_w below).
//
// B~ V block.  The 128 accumulator rows (TMEM lanes) hold G = 128 / m copies
// of the m landmark rows; copy g handles keys g*m .. g*m + m - 1 of every
// 128-key chunk, so every TMEM lane has work.  Per chunk:
//   TMA  K and V chunks (128 x 64 bf16, zero past n),
//   MMA  S = [Q~; ..; Q~] K_c^T       (M=128, N=128, K=64, operands in smem),
//   softmax: P = 2^(s - m_ref) as bf16 straight into TMEM (zero outside the
//        row's key group), row sums in fp32,
//   MMA  Y += P V_c                    (M=128, N=64, K=128, P read from TMEM,
//        Y accumulated in TMEM).
// m <= 64 (bv_body): two softmax warpgroups take alternate chunks, each with
// its own TMEM buffers, reference maxima and sums; warps 0 TMA producer, 1
// and 2 MMA issuers (one per softmax warpgroup), 4-7 and 8-11 softmax.
// m = 128 (bv_body_split): both warpgroups work on every chunk, warpgroup h
// on half h of each row's keys, with S and P double-buffered; warps 0 TMA
// producer, 1 MMA issuer, 4-11 softmax.  Either way the states of a landmark
// are merged in the block at the end, giving one partial per (block,
// landmark); warp 1 owns TMEM.
#pragma once

#include "pinv_pow.cuh"
#include "pinv_pow128.cuh"
#include "trace.cuh"

namespace nys {
namespace midtc {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kStages = 6;   // ~1.5 us of loads in flight per SM
constexpr int kChunk = 128;
constexpr int kMaxSplits = 16;   // B~ V partials per head (bounds the merge scratch)

struct BvSmem {
  uint32_t q, k[kStages], v[kStages], bars, total;
};
__host__ __device__ inline BvSmem bv_smem() {
  BvSmem L;
  uint32_t off = 0;
  auto take = [&](uint32_t b) {
    uint32_t at = off;
    off += (b + 1023u) & ~1023u;
    return at;
  };
  L.q = take(16384u);
  for (int s = 0; s < kStages; ++s) {
    L.k[s] = take(16384u);
    L.v[s] = take(16384u);
  }
  L.bars = take(1024u);
  L.total = off;
  return L;
}

template <int M>
__host__ __device__ constexpr uint32_t pinv_smem() {
  if constexpr (M <= 64) {
    return pinvpow::Cfg<M>::total;
  } else {
    return pinvpow128::Cfg::total;
  }
}


struct Params {
  pinvpow::Params pinv;
  const float *q_land;        // [BH][m][64]
  float *pmax, *psum, *py;    // [BH][S][m], [BH][S][m], [BH][S][m][64]
  const float *z;             // [BH][m][m] (the pseudoinverse blocks' result)
  float *y, *w;               // [BH][m][64]
  uint8_t *w_op;              // [BH][m][128 B]: W as the bf16 B operand of P W
  uint32_t *count;            // [kCountsPerHead BH], zeroed per call
  uint32_t *err;
  const int *lens;            // [batch] tokens per element (ragged batches) or null
  int heads;
  int BH, n, chunks_per_head, splits;
  float scale_log2;
};

// ------------------------------------------------------------------ B~ V body
// Softmax over the keys with a lazily updated reference maximum: P =
// 2^(s - m_ref) with m_ref raised only when a chunk's maximum exceeds it by
// more than kTau (log2 units), so P <= 2^kTau and the Y accumulator (in TMEM,
// summed by the P V MMAs) is rescaled only then.  In bv_body (m <= 64) the
// two softmax warpgroups take alternate chunks and turns through their
// exponential sections (named barriers 2 and 3); in bv_body_split (m = 128)
// they split every chunk's keys between them (named barrier 2: the halves'
// maxima), so a chunk's softmax is half as long a chain.
constexpr float kTau = 8.f;
// Turn-taking of the two softmax warpgroups of bv_body through their
// exponential sections (1), or both at once (0).
#ifndef NYS_BV_TURNS
#define NYS_BV_TURNS 1
#endif
// V's loads with the evict-first policy (1) or not (0: the output kernel
// reads V again).
#ifndef NYS_V_EVICT_FIRST
#define NYS_V_EVICT_FIRST 0
#endif

// tmem_in: a 512-column TMEM allocation owned by the caller, or ~0u to
// allocate (and free) one here.
// wait_prev: launched with programmatic dependent launch; the first K / V
// chunk loads are issued before the wait for the previous kernel, the Q~
// operand (its result) is read after it, and the next kernel may launch once
// the wait has returned.
template <int M>
__device__ __forceinline__ void bv_body(const CUtensorMap *map_k, const CUtensorMap *map_v,
                                        const Params &prm, uint8_t *smem, int bh, int split,
                                        uint32_t tmem_in, bool wait_prev = false) {
  constexpr int G = 128 / M;
  const BvSmem L = bv_smem();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // keys [0, L): L = n, or the element's own length (an invalid one reads as
  // 0 and leaves the split empty; the segment-mean kernel reports it)
  int seq = prm.n;
  if (prm.lens) {
    seq = prm.lens[bh / prm.heads];
    if (seq < M || seq > prm.n || (long)(M - 1) * ((seq + M - 1) / M) >= seq) seq = 0;
  }
  const int c_begin = (int)((long)split * prm.chunks_per_head / prm.splits);
  const int c_end = min((int)((long)(split + 1) * prm.chunks_per_head / prm.splits),
                        (seq + kChunk - 1) / kChunk);
  const int nch = c_end > c_begin ? c_end - c_begin : 0;

  uint64_t *bars = (uint64_t *)(smem + L.bars);
  uint64_t *full = bars;                  // [kStages]
  uint64_t *empty = bars + kStages;       // [kStages]
  uint64_t *s_full = bars + 2 * kStages;  // [2] per softmax warpgroup
  uint64_t *s_free = s_full + 2;
  uint64_t *p_ready = s_free + 2;
  uint64_t *y_full = p_ready + 2;
  constexpr int kBars = 2 * kStages + 8;
  uint32_t *tmem_slot = (uint32_t *)(bars + kBars);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  const Abort ab{abort_flag, prm.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
      mbar_init(&p_ready[b], 128);
      mbar_init(&y_full[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(map_k);
    tma_prefetch_desc(map_v);
  }
  if (tmem_in != ~0u) {
    if (threadIdx.x == 0) *tmem_slot = tmem_in;
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
  }
  __syncthreads();   // barriers initialised
  const int pre = nch < kStages ? nch : kStages;   // chunk loads issued up front
  // K is read here for the last time in the pass (V again by the output
  // kernel): its lines leave L2 first
  const uint64_t last_use = policy_evict_first();
  auto load_v = [&](int s, int k0) {
    if (NYS_V_EVICT_FIRST)
      tma_load_3d_hint(smem + L.v[s], map_v, &full[s], 0, k0, bh, last_use);
    else
      tma_load_3d(smem + L.v[s], map_v, &full[s], 0, k0, bh);
  };
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      const int k0 = (c_begin + i) * kChunk;
      mbar_expect_tx(&full[i], 32768u);
      tma_load_3d_hint(smem + L.k[i], map_k, &full[i], 0, k0, bh, last_use);
      load_v(i, k0);
    }
  }
  if (wait_prev) {
    griddep_wait();
    griddep_launch_dependents();
    NYS_MARK(kTrMid, 1);
  }
  // A operand rows: row r holds landmark r % M (bf16, 128-byte swizzle)
  if (threadIdx.x < 256) {
    const float4 *qt = (const float4 *)(prm.q_land + (size_t)bh * M * 64);
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;   // 4 chunks each
    float4 a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = __ldcg(qt + (row % M) * 16 + half * 8 + u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      st_shared_v4(smem_u32(smem + L.q) + sw128_offset(row, half * 4 + u),
                   pack_bf16(a[2 * u].x, a[2 * u].y), pack_bf16(a[2 * u].z, a[2 * u].w),
                   pack_bf16(a[2 * u + 1].x, a[2 * u + 1].y),
                   pack_bf16(a[2 * u + 1].z, a[2 * u + 1].w));
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM per softmax warpgroup w: S at 256w (128 cols), P at 256w + 128
  // (64 cols of bf16 pairs), Y at 256w + 192 (64 cols)

  if (warp == 0) {
    if (lane == 0) {
      for (int i = pre; i < nch; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, ab)) break;
        const int k0 = (c_begin + i) * kChunk;
        mbar_expect_tx(&full[s], 32768u);
        tma_load_3d_hint(smem + L.k[s], map_k, &full[s], 0, k0, bh, last_use);
        load_v(s, k0);
      }
      // consume the stage releases nobody else waits for, so that no
      // tensor-core arrival is pending when the barriers are invalidated
      for (int i = nch > kStages ? nch - kStages : 0; i < nch; ++i)
        if (!mbar_wait(&empty[i % kStages], (i / kStages) & 1, ab)) break;
    }
  } else if (warp == 1 || warp == 2) {
    // one MMA issuer per softmax warpgroup
    if (lane == 0) {
      const int w = warp - 1;
      const uint32_t id_s = make_idesc(kFmtBF16, 128, 128, 0, 0);
      const uint32_t id_y = make_idesc(kFmtBF16, 128, 64, 0, 1);
      const uint64_t dq = make_sdesc(smem_u32(smem + L.q), 16, 1024);
      auto issue_s = [&](int i) -> bool {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1, ab)) return false;
        tc_fence_after();
        const uint64_t dk = make_sdesc(smem_u32(smem + L.k[s]), 16, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem + 256 * w, dq + 2u * k, dk + 2u * k, id_s, k > 0);
        mma_commit(&s_full[w]);
        return true;
      };
      bool ok = w < nch ? issue_s(w) : true;
      for (int i = w; i < nch && ok; i += 2) {
        const int s = i % kStages, u = i >> 1;
        // the next S as soon as this warpgroup has read the current one
        if (i + 2 < nch) {
          if (!mbar_wait(&s_free[w], u & 1, ab)) break;
          if (!(ok = issue_s(i + 2))) break;
        }
        if (!mbar_wait(&p_ready[w], u & 1, ab)) break;
        tc_fence_after();
        const uint64_t dv = make_sdesc(smem_u32(smem + L.v[s]), 16, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ts(tmem + 256 * w + 192, tmem + 256 * w + 128 + 8 * k, dv + 128u * k, id_y,
                      (u > 0 || k > 0) ? 1u : 0u);
        mma_commit(&y_full[w]);
        mma_commit(&empty[s]);
      }
    }
  }
  // softmax warpgroups; their running states are kept for the merge below
  float run_max = -INFINITY, run_sum = 0.f;
  float acc[64];
  const int wg = (warp >= 8) ? 1 : 0;
  const int r = threadIdx.x & 127;          // accumulator row == TMEM lane
  const int j = r % M, g = r / M;           // landmark, key group
  if (warp >= 4) {
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_base + 256 * wg;
    {   // P starts at zero: each row only ever writes its own key group
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tmem_st32(t_s + 128, z);
      tmem_st32(t_s + 160, z);
      tmem_st_wait();
    }
    if (NYS_BV_TURNS && wg == 1 && nch > 0) named_barrier_arrive(2, 256);   // warpgroup 0 first
    bool ok = true;
    int u = 0;
    for (int i = wg; i < nch; i += 2, ++u) {
      if (!(ok = mbar_wait(&s_full[wg], u & 1, ab))) break;
      if (threadIdx.x == 128 && blockIdx.x == (unsigned)prm.BH && u < 32) NYS_MARK_T(kTrMid, 32 + u);
      tc_fence_after();
      float v[M];
#pragma unroll
      for (int c = 0; c < M; c += 32) tmem_ld32(t_s + g * M + c, v + c);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s_free[wg]);
      const int key0 = (c_begin + i) * kChunk + g * M;
      const int valid = min(M, seq - key0);       // keys of this group inside [0, L)
      if (NYS_BV_TURNS) named_barrier(2 + wg, 256);   // this warpgroup's turn
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
      if (valid == M) {
#pragma unroll
        for (int c = 0; c < M; ++c) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
      } else {
#pragma unroll
        for (int c = 0; c < M; ++c)
          if (c < valid) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
      }
      const float cmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         prm.scale_log2;
      const bool up = cmax > run_max + kTau;
      bool y_done = false;
      if (__any_sync(0xffffffffu, up)) {
        // raise the reference of the rows that need it and rescale their Y
        // (warp-uniform: the TMEM accesses are warp-wide)
        const float m_new = up ? cmax : run_max;
        const float alpha = (run_max == -INFINITY) ? 0.f : fast_exp2(run_max - m_new);
        if (u > 0) {
          if (!(ok = mbar_wait(&y_full[wg], (u - 1) & 1, ab))) break;
          tc_fence_after();
          y_done = true;
          float y[64];
          tmem_ld32(t_s + 192, y);
          tmem_ld32(t_s + 224, y + 32);
          tmem_ld_wait();
          uint32_t ys[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) ys[c] = __float_as_uint(y[c] * alpha);
          tmem_st32(t_s + 192, ys);
          tmem_st32(t_s + 224, ys + 32);
          tmem_st_wait();
        }
        run_sum *= alpha;
        run_max = m_new;
      }
      const float mref = run_max;
      const bool none = (mref == -INFINITY);
      float ps[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) ps[q] = 0.f;
      uint32_t pk[M / 2];
      if (valid == M && !none) {
#pragma unroll
        for (int c = 0; c < M; c += 2) {
          const float p0 = fast_exp2(fmaf(v[c], prm.scale_log2, -mref));
          const float p1 = fast_exp2(fmaf(v[c + 1], prm.scale_log2, -mref));
          ps[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < M; c += 2) {
          const float p0 = (c < valid && !none) ? fast_exp2(fmaf(v[c], prm.scale_log2, -mref)) : 0.f;
          const float p1 =
              (c + 1 < valid && !none) ? fast_exp2(fmaf(v[c + 1], prm.scale_log2, -mref)) : 0.f;
          ps[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16(p0, p1);
        }
      }
      run_sum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      if (NYS_BV_TURNS && i + 1 < nch) named_barrier_arrive(2 + (wg ^ 1), 256);   // the other's turn
      // P is read by the previous P V of this warpgroup: wait for it
      if (u > 0 && !y_done) {
        if (!(ok = mbar_wait(&y_full[wg], (u - 1) & 1, ab))) break;
        tc_fence_after();
      }
#pragma unroll
      for (int c = 0; c < M / 2; c += 16) tmem_st16(t_s + 128 + g * (M / 2) + c, pk + c);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[wg]);
      if (threadIdx.x == 128 && blockIdx.x == (unsigned)prm.BH && u < 32) NYS_MARK_T(kTrMid, 96 + u);
    }
    if (NYS_BV_TURNS && !ok) {
      // let the other warpgroup leave a turn it may be waiting for
      named_barrier_arrive(2 + (wg ^ 1), 256);
    }
    // the state: Y of this row after the last P V of this warpgroup
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = 0.f;
    if (ok && u > 0 && mbar_wait(&y_full[wg], (u - 1) & 1, ab)) {
      tc_fence_after();
      tmem_ld32(t_s + 192, acc);
      tmem_ld32(t_s + 224, acc + 32);
      tmem_ld_wait();
    }
  }
  tc_fence_before();
  __syncthreads();   // pipeline drained: stage buffers are free for the merge
  if (threadIdx.x == 0 && !*abort_flag)
    for (int b = 0; b < kBars; ++b) mbar_inval(bars + b);
  if (warp == 1 && tmem_in == ~0u) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // In-block merge of the 2G states of every landmark, in a fixed order.
  float *st = (float *)(smem + L.k[0]);   // [2][128][66]: max, sum, acc[64]
  if (warp >= 4) {
    float *o = st + (wg * 128 + r) * 66;
    o[0] = run_max;
    o[1] = run_sum;
#pragma unroll
    for (int c = 0; c < 64; ++c) o[2 + c] = acc[c];
  }
  __syncthreads();
  if (warp >= 4 && wg == 0 && g == 0) {
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < 2 * G; ++q) mx = fmaxf(mx, st[((q / G) * 128 + (q % G) * M + j) * 66]);
    float f[2 * G], den = 0.f;
#pragma unroll
    for (int q = 0; q < 2 * G; ++q) {
      const float *o = st + ((q / G) * 128 + (q % G) * M + j) * 66;
      f[q] = (mx == -INFINITY) ? 0.f : fast_exp2(o[0] - mx);
      den = fmaf(o[1], f[q], den);
    }
    const size_t base = ((size_t)bh * prm.splits + split) * M + j;
    prm.pmax[base] = mx;
    prm.psum[base] = den;
    float4 *dst = (float4 *)(prm.py + base * 64);
#pragma unroll 4
    for (int c4 = 0; c4 < 16; ++c4) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 2 * G; ++q) {
        const float *o = st + ((q / G) * 128 + (q % G) * M + j) * 66 + 2 + 4 * c4;
        a.x = fmaf(f[q], o[0], a.x);
        a.y = fmaf(f[q], o[1], a.y);
        a.z = fmaf(f[q], o[2], a.z);
        a.w = fmaf(f[q], o[3], a.w);
      }
      dst[c4] = a;
    }
  }
}

// The same with the softmax warpgroups splitting every chunk's keys (used
// for m = 128, whose rows hold 128 keys of a chunk: one thread per row would
// keep 128 scores in registers).
template <int M>
__device__ __forceinline__ void bv_body_split(const CUtensorMap *map_k, const CUtensorMap *map_v,
                                        const Params &prm, uint8_t *smem, int bh, int split,
                                        uint32_t tmem_in, bool wait_prev = false) {
  constexpr int G = 128 / M;
  const BvSmem L = bv_smem();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // keys [0, L): L = n, or the element's own length (an invalid one reads as
  // 0 and leaves the split empty; the segment-mean kernel reports it)
  int seq = prm.n;
  if (prm.lens) {
    seq = prm.lens[bh / prm.heads];
    if (seq < M || seq > prm.n || (long)(M - 1) * ((seq + M - 1) / M) >= seq) seq = 0;
  }
  const int c_begin = (int)((long)split * prm.chunks_per_head / prm.splits);
  const int c_end = min((int)((long)(split + 1) * prm.chunks_per_head / prm.splits),
                        (seq + kChunk - 1) / kChunk);
  const int nch = c_end > c_begin ? c_end - c_begin : 0;

  uint64_t *bars = (uint64_t *)(smem + L.bars);
  uint64_t *full = bars;                  // [kStages]
  uint64_t *empty = bars + kStages;       // [kStages]
  uint64_t *s_full = bars + 2 * kStages;  // [2] per softmax warpgroup
  uint64_t *s_free = s_full + 2;
  uint64_t *p_ready = s_free + 2;
  uint64_t *y_full = p_ready + 2;
  constexpr int kBars = 2 * kStages + 8;
  uint32_t *tmem_slot = (uint32_t *)(bars + kBars);
  volatile uint32_t *abort_flag = tmem_slot + 1;
  const Abort ab{abort_flag, prm.err};

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 256);
      mbar_init(&p_ready[b], 256);
      mbar_init(&y_full[b], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(map_k);
    tma_prefetch_desc(map_v);
  }
  if (tmem_in != ~0u) {
    if (threadIdx.x == 0) *tmem_slot = tmem_in;
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
  }
  __syncthreads();   // barriers initialised
  const int pre = nch < kStages ? nch : kStages;   // chunk loads issued up front
  // K is read here for the last time in the pass (V again by the output
  // kernel): its lines leave L2 first
  const uint64_t last_use = policy_evict_first();
  auto load_v = [&](int s, int k0) {
    if (NYS_V_EVICT_FIRST)
      tma_load_3d_hint(smem + L.v[s], map_v, &full[s], 0, k0, bh, last_use);
    else
      tma_load_3d(smem + L.v[s], map_v, &full[s], 0, k0, bh);
  };
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < pre; ++i) {
      const int k0 = (c_begin + i) * kChunk;
      mbar_expect_tx(&full[i], 32768u);
      tma_load_3d_hint(smem + L.k[i], map_k, &full[i], 0, k0, bh, last_use);
      load_v(i, k0);
    }
  }
  if (wait_prev) {
    griddep_wait();
    griddep_launch_dependents();
    NYS_MARK(kTrMid, 1);
  }
  // A operand rows: row r holds landmark r % M (bf16, 128-byte swizzle)
  if (threadIdx.x < 256) {
    const float4 *qt = (const float4 *)(prm.q_land + (size_t)bh * M * 64);
    const int row = threadIdx.x >> 1, half = threadIdx.x & 1;   // 4 chunks each
    float4 a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = __ldcg(qt + (row % M) * 16 + half * 8 + u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      st_shared_v4(smem_u32(smem + L.q) + sw128_offset(row, half * 4 + u),
                   pack_bf16(a[2 * u].x, a[2 * u].y), pack_bf16(a[2 * u].z, a[2 * u].w),
                   pack_bf16(a[2 * u + 1].x, a[2 * u + 1].y),
                   pack_bf16(a[2 * u + 1].z, a[2 * u + 1].w));
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM: S of chunk i in buffer i & 1 (columns 128 (i & 1), 128 wide), P of
  // chunk i at 256 + 64 (i & 1) (bf16 pairs, 64 wide), Y at 384 (64 wide).
  // Both softmax warpgroups work on every chunk: warpgroup h takes half h of
  // each row's keys, the two halves of a row agree on the row's reference
  // maximum through shared memory, and P V runs once both halves of P are in.
  constexpr uint32_t kP = 256, kY = 384;
  __shared__ float xmax[2][2][128];   // chunk parity, half, row: the halves' maxima

  if (warp == 0) {
    if (lane == 0) {
      for (int i = pre; i < nch; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, ab)) break;
        const int k0 = (c_begin + i) * kChunk;
        mbar_expect_tx(&full[s], 32768u);
        tma_load_3d_hint(smem + L.k[s], map_k, &full[s], 0, k0, bh, last_use);
        load_v(s, k0);
      }
      // consume the stage releases nobody else waits for, so that no
      // tensor-core arrival is pending when the barriers are invalidated
      for (int i = nch > kStages ? nch - kStages : 0; i < nch; ++i)
        if (!mbar_wait(&empty[i % kStages], (i / kStages) & 1, ab)) break;
    }
  } else if (warp == 1) {
    // MMA issuer: S of the next chunks as soon as their buffer has been read,
    // P V of a chunk once both halves of its P are in TMEM
    if (lane == 0) {
      const uint32_t id_s = make_idesc(kFmtBF16, 128, 128, 0, 0);
      const uint32_t id_y = make_idesc(kFmtBF16, 128, 64, 0, 1);
      const uint64_t dq = make_sdesc(smem_u32(smem + L.q), 16, 1024);
      auto issue_s = [&](int i) -> bool {
        const int s = i % kStages;
        if (!mbar_wait(&full[s], (i / kStages) & 1, ab)) return false;
        tc_fence_after();
        const uint64_t dk = make_sdesc(smem_u32(smem + L.k[s]), 16, 1024);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem + 128 * (i & 1), dq + 2u * k, dk + 2u * k, id_s, k > 0);
        mma_commit(&s_full[i & 1]);
        return true;
      };
      bool ok = nch > 0 ? issue_s(0) : true;
      if (ok && nch > 1) ok = issue_s(1);
      for (int i = 0; i < nch && ok; ++i) {
        const int s = i % kStages, b = i & 1, u = i >> 1;
        if (!mbar_wait(&p_ready[b], u & 1, ab)) break;
        tc_fence_after();
        const uint64_t dv = make_sdesc(smem_u32(smem + L.v[s]), 16, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16_ts(tmem + kY, tmem + kP + 64 * b + 8 * k, dv + 128u * k, id_y,
                      (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(&y_full[b]);
        mma_commit(&empty[s]);
        if (i + 2 < nch) {
          if (!mbar_wait(&s_free[b], u & 1, ab)) break;
          ok = issue_s(i + 2);
        }
      }
    }
  }
  // softmax warpgroups; their running states are kept for the merge below
  constexpr int H = M / 2;                 // keys of a row per chunk and half
  float run_max = -INFINITY, run_sum = 0.f;
  float acc[32];                           // this half of the row's Y
  const int h = (warp >= 8) ? 1 : 0;
  const int r = threadIdx.x & 127;          // accumulator row == TMEM lane
  const int j = r % M, g = r / M;           // landmark, key group
  if (warp >= 4) {
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    {   // P starts at zero: each row only ever writes its own keys
      uint32_t z[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) z[e] = 0u;
      tmem_st32(t_row + kP + 32 * h, z);
      tmem_st32(t_row + kP + 64 + 32 * h, z);
      tmem_st_wait();
    }
    // ok stays uniform over the 256 softmax threads: a failed wait is
    // reported at the next exchange barrier, where every thread leaves the
    // loop (a thread that left before it would leave the others waiting)
    bool ok = true;
    for (int i = 0; i < nch; ++i) {
      const int b = i & 1, u = i >> 1;
      const bool got = ok && mbar_wait(&s_full[b], u & 1, ab);
      if (threadIdx.x == 128 && blockIdx.x == (unsigned)prm.BH && i < 32) NYS_MARK_T(kTrMid, 32 + i);
      tc_fence_after();
      float v[H];
      const int key0 = (c_begin + i) * kChunk + g * M + h * H;
      const int valid = max(0, min(H, seq - key0));   // keys of this half inside [0, L)
      float hmax = -INFINITY;
      if (got) {
        const uint32_t t_s = t_row + 128 * b + g * M + h * H;
        if constexpr (H >= 32) {
#pragma unroll
          for (int c = 0; c < H; c += 32) tmem_ld32(t_s + c, v + c);
        } else {
          tmem_ld16(t_s, v);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[b]);
        float mx[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
        if (valid == H) {
#pragma unroll
          for (int c = 0; c < H; ++c) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
        } else {
#pragma unroll
          for (int c = 0; c < H; ++c)
            if (c < valid) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
        }
        hmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                     fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      }
      // the row's maximum over both halves (the same value in both threads)
      xmax[b][h][r] = hmax;
      if (named_barrier_or(2, 256, !got)) {
        ok = false;
        break;
      }
      const float cmax = fmaxf(hmax, xmax[b][h ^ 1][r]) * prm.scale_log2;
      const bool up = cmax > run_max + kTau;
      bool y_done = false;   // P V of chunk i - 1 (and so of i - 2) has completed
      // warp-uniform, and the same in the two warps that share these rows
      if (__any_sync(0xffffffffu, up)) {
        // raise the reference of the rows that need it and rescale this half
        // of their Y
        const float m_new = up ? cmax : run_max;
        const float alpha = (run_max == -INFINITY) ? 0.f : fast_exp2(run_max - m_new);
        if (i > 0) {
          if (!(ok = mbar_wait(&y_full[(i - 1) & 1], ((i - 1) >> 1) & 1, ab))) continue;
          tc_fence_after();
          y_done = true;
          float y[32];
          tmem_ld32(t_row + kY + 32 * h, y);
          tmem_ld_wait();
          uint32_t ys[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) ys[c] = __float_as_uint(y[c] * alpha);
          tmem_st32(t_row + kY + 32 * h, ys);
          tmem_st_wait();
        }
        run_sum *= alpha;
        run_max = m_new;
      }
      const float mref = run_max;
      const bool none = (mref == -INFINITY);
      float ps[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) ps[q] = 0.f;
      uint32_t pk[H / 2];
      if (valid == H && !none) {
#pragma unroll
        for (int c = 0; c < H; c += 2) {
          const float p0 = fast_exp2(fmaf(v[c], prm.scale_log2, -mref));
          const float p1 = fast_exp2(fmaf(v[c + 1], prm.scale_log2, -mref));
          ps[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < H; c += 2) {
          const float p0 = (c < valid && !none) ? fast_exp2(fmaf(v[c], prm.scale_log2, -mref)) : 0.f;
          const float p1 =
              (c + 1 < valid && !none) ? fast_exp2(fmaf(v[c + 1], prm.scale_log2, -mref)) : 0.f;
          ps[(c >> 1) & 7] += p0 + p1;
          pk[c >> 1] = pack_bf16(p0, p1);
        }
      }
      run_sum += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      // P buffer b was read by P V of chunk i - 2
      if (i >= 2 && !y_done) {
        if (!(ok = mbar_wait(&y_full[b], ((i - 2) >> 1) & 1, ab))) continue;
        tc_fence_after();
      }
      const uint32_t t_p = t_row + kP + 64 * b + g * (M / 2) + h * (H / 2);
      if constexpr (H / 2 >= 16) {
#pragma unroll
        for (int c = 0; c < H / 2; c += 16) tmem_st16(t_p + c, pk + c);
      } else {
        tmem_st8(t_p, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_ready[b]);
      if (threadIdx.x == 128 && blockIdx.x == (unsigned)prm.BH && i < 32) NYS_MARK_T(kTrMid, 96 + i);
    }
    // the state: this half of the row's Y after the last P V
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;
    if (ok && nch > 0 &&
        mbar_wait(&y_full[(nch - 1) & 1], ((nch - 1) >> 1) & 1, ab)) {
      tc_fence_after();
      tmem_ld32(t_row + kY + 32 * h, acc);
      tmem_ld_wait();
    }
  }
  tc_fence_before();
  __syncthreads();   // pipeline drained: stage buffers are free for the merge
  if (threadIdx.x == 0 && !*abort_flag)
    for (int bb = 0; bb < kBars; ++bb) mbar_inval(bars + bb);
  if (warp == 1 && tmem_in == ~0u) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // In-block merge of the G key groups of every landmark (two halves each),
  // in a fixed order.
  float *st = (float *)(smem + L.k[0]);   // [2][128][66]: max, half sum, Y (this half's columns)
  if (warp >= 4) {
    float *o = st + (h * 128 + r) * 66;
    o[0] = run_max;
    o[1] = run_sum;
#pragma unroll
    for (int c = 0; c < 32; ++c) o[2 + 32 * h + c] = acc[c];
  }
  __syncthreads();
  if (warp >= 4 && h == 0 && g == 0) {
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < G; ++q) mx = fmaxf(mx, st[(q * M + j) * 66]);
    float f[G], den = 0.f;
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float m_q = st[(q * M + j) * 66];
      f[q] = (mx == -INFINITY || m_q == -INFINITY) ? 0.f : fast_exp2(m_q - mx);
      den = fmaf(st[(q * M + j) * 66 + 1] + st[(128 + q * M + j) * 66 + 1], f[q], den);
    }
    const size_t base = ((size_t)bh * prm.splits + split) * M + j;
    prm.pmax[base] = mx;
    prm.psum[base] = den;
    float4 *dst = (float4 *)(prm.py + base * 64);
#pragma unroll 4
    for (int c4 = 0; c4 < 16; ++c4) {
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < G; ++q) {
        // columns 4 c4 .. 4 c4 + 3 come from half (4 c4) / 32
        const float *o = st + (((c4 >= 8) ? 128 : 0) + q * M + j) * 66 + 2 + 4 * c4;
        a.x = fmaf(f[q], o[0], a.x);
        a.y = fmaf(f[q], o[1], a.y);
        a.z = fmaf(f[q], o[2], a.z);
        a.w = fmaf(f[q], o[3], a.w);
      }
      dst[c4] = a;
    }
  }
}

// ------------------------------------------------------------------ merge + W
// The last B~ V block of a head (counted with an atomic) merges the head's S
// partial states (m_s, l_s, Y_s) of every landmark into Y, in split order
// with a running maximum:
//   M <- max(M, m_s),  a = 2^(M_old - M),  b = 2^(m_s - M),
//   L <- a L + b l_s,  Y~ <- a Y~ + b Y_s,   and finally Y = Y~ / L.
// The second of {that block, the head's pseudoinverse block} to finish forms
// W = Z Y (form_w).  Each of the two can leave its own result in the W
// operands in shared memory (the same split of the same values that form_w
// would load), so form_w loads only the other one; either way W is the same.

// W operand scratch: Z (A, K-major, m rows) and Y (B, MN-major, m landmark
// rows of 64 features), each as a split bf16 pair; the MMA barrier.
template <int M>
struct WSmem {
  static constexpr int kAtoms = M > 64 ? M / 64 : 1;     // 128-byte K atoms of Z
  static constexpr uint32_t ah = 0, al = ah + kAtoms * 16384u;
  static constexpr uint32_t bh = al + kAtoms * 16384u, bl = bh + M * 128u;
  static constexpr uint32_t bar = bl + M * 128u;
  static constexpr uint32_t total = bar + 64u;
};

__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[e] = *reinterpret_cast<const uint32_t *>(&hh);
    l[e] = pack_bf16(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Merge scratch, after the W operands: per split of a batch its partial Y
// rows [M][64] fp32, then the batch's maxima and sums [kMergeBatch][M]; an
// mbarrier for the bulk copies.
template <int M>
struct MergeSmem {
  static constexpr uint32_t base = (WSmem<M>::total + 1023u) & ~1023u;
  static constexpr uint32_t kPy = M * 256u;
  static constexpr int kBatch = M <= 64 ? 8 : 3;   // splits per batch of copies
  static constexpr uint32_t py = base;
  static constexpr uint32_t pm = py + kBatch * kPy;
  static constexpr uint32_t pl = pm + kBatch * M * 4u;
  static constexpr uint32_t bar = pl + kBatch * M * 4u;
  // Z in fp32 for W, copied with the first batch (m <= 64; at m = 128 it
  // does not fit and form_w loads it)
  static constexpr bool kZ = M <= 64;
  static constexpr uint32_t zf = (bar + 64u + 1023u) & ~1023u;
  static constexpr uint32_t total = kZ ? zf + M * M * 4u : bar + 64u;
};

// All kThreads threads.  Thread 0 brings a batch of splits' partials (rows,
// maxima, sums) into shared memory with bulk copies, all in flight at once
// (the partials were stored by other blocks' generic stores, ordered before
// this block's count by their fences and ours; the proxy fence orders them
// before the copies); then threads 0..255, 256 / M per landmark row and
// 64 M / 256 features each, fold the batch into their running state.  Y goes
// to global memory in fp32 and, when stage_y, into the W operand's Y pair in
// shared memory.
template <int M>
__device__ __forceinline__ void merge_y(const Params &prm, uint8_t *smem, int bh, bool stage_y,
                                        const Abort &ab, bool load_z) {
  using C = MergeSmem<M>;
  constexpr int kTpr = 256 / M, kF = 64 / kTpr;   // threads per row, features per thread
  const int t = threadIdx.x, S = prm.splits;
  const int j = (t & 255) / kTpr, f0 = (t % kTpr) * kF;
  uint64_t *bar = (uint64_t *)(smem + C::bar);
  const float *sp = (const float *)(smem + C::py);
  const float *sm = (const float *)(smem + C::pm);
  const float *sl = (const float *)(smem + C::pl);
  const size_t pb = (size_t)bh * S * M;
  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  float mx = -INFINITY, den = 0.f, acc[kF];
#pragma unroll
  for (int f = 0; f < kF; ++f) acc[f] = 0.f;
  bool ok = true;
  uint32_t phase = 0;
  for (int s0 = 0; s0 < S; s0 += C::kBatch) {
    const int nb = min(C::kBatch, S - s0);
    if (t == 0) {
      const bool z = C::kZ && load_z && s0 == 0;   // Z of the head with the first batch
      fence_async_global();
      mbar_expect_tx(bar, (uint32_t)nb * (C::kPy + 2u * M * 4u) + (z ? M * M * 4u : 0u));
      if (z) bulk_load(smem + C::zf, prm.z + (size_t)bh * M * M, M * M * 4u, bar);
      for (int u = 0; u < nb; ++u) {
        const size_t i = pb + (size_t)(s0 + u) * M;
        bulk_load(smem + C::py + u * C::kPy, prm.py + i * 64, C::kPy, bar);
        bulk_load(smem + C::pm + u * M * 4u, prm.pmax + i, M * 4u, bar);
        bulk_load(smem + C::pl + u * M * 4u, prm.psum + i, M * 4u, bar);
      }
    }
    ok = ok && mbar_wait(bar, phase, ab);
    phase ^= 1u;
    if (t < 256 && ok) {
      for (int u = 0; u < nb; ++u) {
        const float pm = sm[u * M + j], pl = sl[u * M + j];
        const float nm = fmaxf(mx, pm);
        const float a = mx == -INFINITY ? 0.f : fast_exp2(mx - nm);
        const float b = pm == -INFINITY ? 0.f : fast_exp2(pm - nm);
        den = fmaf(den, a, pl * b);
        const float4 *row = (const float4 *)(sp + u * (M * 64) + j * 64 + f0);
#pragma unroll
        for (int q = 0; q < kF / 4; ++q) {
          const float4 y = row[q];
          acc[4 * q] = fmaf(acc[4 * q], a, y.x * b);
          acc[4 * q + 1] = fmaf(acc[4 * q + 1], a, y.y * b);
          acc[4 * q + 2] = fmaf(acc[4 * q + 2], a, y.z * b);
          acc[4 * q + 3] = fmaf(acc[4 * q + 3], a, y.w * b);
        }
        mx = nm;
      }
    }
    // the buffers are refilled by the next batch; a failed wait ends the merge
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
  }
  if (t == 0 && ok) mbar_inval(bar);
  if (t >= 256) return;
  const float inv = 1.f / den;
#pragma unroll
  for (int f = 0; f < kF; ++f) acc[f] *= inv;
  float4 *dst = (float4 *)(prm.y + ((size_t)bh * M + j) * 64 + f0);
#pragma unroll
  for (int q = 0; q < kF / 4; ++q)
    dst[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
  if (stage_y) {
    const uint32_t s_bh = smem_u32(smem + WSmem<M>::bh), s_bl = smem_u32(smem + WSmem<M>::bl);
#pragma unroll
    for (int c = 0; c < kF / 8; ++c) {
      uint4 hi, lo;
      split8(acc + 8 * c, hi, lo);
      const uint32_t off = sw128_offset(j, f0 / 8 + c);
      st_shared_v4(s_bh + off, hi.x, hi.y, hi.z, hi.w);
      st_shared_v4(s_bl + off, lo.x, lo.y, lo.z, lo.w);
    }
  }
}

// W = Z Y on the tensor cores from split bf16 operands (hi = rounding of x,
// lo = rounding of x - hi; Z_h Y_h + Z_h Y_l + Z_l Y_h, fp32 accumulation,
// about 16 bits), Z K-major (A, m rows), Y MN-major (B, row k = landmark, 64
// features); W stored in fp32 and as the bf16 operand of P W (128 bytes per
// landmark row, 16-byte chunk c at c ^ (row & 7)).  All kThreads threads;
// TMEM columns 0..63 of the block's allocation.  z_staged / y_staged: that
// operand pair is already in place (written by this block from the values it
// stored to global memory, split the same way), so it is not loaded.  z_smem:
// Z in fp32 in this block's shared memory (copied there by merge_y), or null
// to read it from global memory.
template <int M>
__device__ __forceinline__ void form_w(const Params &prm, uint8_t *smem, int bh, uint32_t tmem,
                                       const Abort &ab, bool z_staged, bool y_staged,
                                       const float *z_smem) {
  using C = WSmem<M>;
  const int t = threadIdx.x, warp = t >> 5;
  uint64_t *bar = (uint64_t *)(smem + C::bar);
  if (t == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  const uint32_t s_ah = smem_u32(smem + C::ah), s_al = smem_u32(smem + C::al);
  const uint32_t s_bh = smem_u32(smem + C::bh), s_bl = smem_u32(smem + C::bl);
  {   // operands: 16-byte chunks of 8 values, every load issued before the
      // first is used, split on the way in
    constexpr int kZc = M * M / 8, kYc = M * 64 / 8;
    constexpr int kPer = (kZc + kYc + kThreads - 1) / kThreads;
    const float4 *zg = (const float4 *)(z_smem ? z_smem : prm.z + (size_t)bh * M * M);
    const float4 *yg = (const float4 *)(prm.y + (size_t)bh * M * 64);
    const int c0 = z_staged ? kZc : 0, c1 = y_staged ? kZc : kZc + kYc;
    float4 va[kPer], vb[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int c = c0 + t + u * kThreads;
      if (c < c1) {
        if (c < kZc && z_smem) {
          va[u] = zg[2 * c];
          vb[u] = zg[2 * c + 1];
        } else {
          const float4 *src = c < kZc ? zg + 2 * c : yg + 2 * (c - kZc);
          va[u] = __ldcg(src);
          vb[u] = __ldcg(src + 1);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int c = c0 + t + u * kThreads;
      if (c >= c1) break;
      const float x[8] = {va[u].x, va[u].y, va[u].z, va[u].w, vb[u].x, vb[u].y, vb[u].z, vb[u].w};
      uint4 hi, lo;
      split8(x, hi, lo);
      if (c < kZc) {   // Z row i, K chunk kc (8 columns): atom kc / 8
        const int i = c / (M / 8), kc = c % (M / 8);
        const uint32_t off = (uint32_t)(kc >> 3) * 16384u + sw128_offset(i, kc & 7);
        st_shared_v4(s_ah + off, hi.x, hi.y, hi.z, hi.w);
        st_shared_v4(s_al + off, lo.x, lo.y, lo.z, lo.w);
      } else {         // Y row k (landmark), feature chunk fc
        const int k = (c - kZc) >> 3, fc = (c - kZc) & 7;
        const uint32_t off = sw128_offset(k, fc);
        st_shared_v4(s_bh + off, hi.x, hi.y, hi.z, hi.w);
        st_shared_v4(s_bl + off, lo.x, lo.y, lo.z, lo.w);
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (t == 0) {
    const uint32_t idesc = make_idesc(kFmtBF16, 128, 64, 0, 1);
    auto da = [&](uint32_t base, int k) {
      return make_sdesc(base + (uint32_t)(k >> 2) * 16384u + 32u * (k & 3), 16, 1024);
    };
    auto db = [&](uint32_t base, int k) { return make_sdesc(base + 2048u * k, 16, 1024); };
#pragma unroll
    for (int k = 0; k < M / 16; ++k) mma_bf16(tmem, da(s_ah, k), db(s_bh, k), idesc, k > 0);
#pragma unroll
    for (int k = 0; k < M / 16; ++k) mma_bf16(tmem, da(s_ah, k), db(s_bl, k), idesc, 1u);
#pragma unroll
    for (int k = 0; k < M / 16; ++k) mma_bf16(tmem, da(s_al, k), db(s_bh, k), idesc, 1u);
    mma_commit(bar);
  }
  if (warp < 4) {
    const int r = t;   // W row == TMEM lane
    const bool done = mbar_wait(bar, 0, ab);
    tc_fence_after();
    float v[64];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v);
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32, v + 32);
    tmem_ld_wait();
    if (done && r < M) {
      float4 *wr = (float4 *)(prm.w + ((size_t)bh * M + r) * 64);
#pragma unroll
      for (int q = 0; q < 16; ++q) wr[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      uint4 *op = (uint4 *)(prm.w_op + ((size_t)bh * M + r) * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        op[c ^ (r & 7)] = make_uint4(pack_bf16(v[8 * c], v[8 * c + 1]),
                                     pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                                     pack_bf16(v[8 * c + 4], v[8 * c + 5]),
                                     pack_bf16(v[8 * c + 6], v[8 * c + 7]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (t == 0 && !*ab.flag) mbar_inval(bar);
}

template <int M>
__host__ __device__ constexpr uint32_t smem_bytes() {
  // pinv operands or B~ V buffers, then the W operands
  constexpr uint32_t bv = 16384u + kStages * 32768u + 1024u;
  constexpr uint32_t body = pinv_smem<M>() > bv ? pinv_smem<M>() : bv;
  constexpr uint32_t tail = MergeSmem<M>::total;
  return 1024u + (body > tail ? body : tail);
}

#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
// Test builds only: a busy delay (bounded by the SM clock, waiting on
// nothing) before a block reports its W input, so that the tests can make
// either block the second to finish: 1 delays the pseudoinverse blocks, 2 the
// Y-merging blocks.
__device__ int g_test_w_order;
__device__ __forceinline__ void test_delay(int side) {
  if (g_test_w_order != side) return;
  const long long t0 = clock64();
  while (clock64() - t0 < 200000ll) {
  }
}
#else
__device__ __forceinline__ void test_delay(int) {}
#endif

template <int M>
__global__ void __launch_bounds__(kThreads, 1)
mid_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
           const Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint32_t tmem_base;
  const int t = threadIdx.x;
  NYS_MARK(kTrMid, 0);
  // one TMEM allocation for every body this block runs (an allocation
  // relinquishes the block's permit to allocate again)
  if ((t >> 5) == 1) tmem_alloc(&tmem_base, 512);
  // launched early (programmatic dependent launch): the bodies wait for the
  // previous kernel before they read the landmarks, and only then let the
  // next kernel launch.  So the next kernel starts after the segment-mean
  // kernel has completed and may read K~ at once; it reads a head's W after
  // that head's W flag (count[2 BH + bh]) and waits for this whole grid only
  // before it exits.
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const bool is_pinv = (int)blockIdx.x < prm.BH;
  if (is_pinv) {
    const int bh = blockIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    NYS_MARK(kTrMid, 1);
    if constexpr (M <= 64) {
      if (t < pinvpow::kBarThreads)
        pinvpow::pinv_body<M>(prm.pinv, smem, bh, tmem, smem_u32(smem + WSmem<M>::ah),
                              smem_u32(smem + WSmem<M>::al));
    } else {
      if (t < pinvpow128::kBarThreads)
        pinvpow128::pinv_body(prm.pinv, smem, bh, tmem, smem_u32(smem + WSmem<M>::ah),
                              smem_u32(smem + WSmem<M>::al));
    }
  } else {
    const int b = blockIdx.x - prm.BH;
    const int bh = b / prm.splits, split = b % prm.splits;
    if constexpr (M == 128)
      bv_body_split<M>(&map_k, &map_v, prm, smem, bh, split, tmem, true);
    else
      bv_body<M>(&map_k, &map_v, prm, smem, bh, split, tmem, true);
  }
  NYS_MARK(kTrMid, 2);
  // hand-off.  Counts per head: count[bh] key-split blocks done,
  // count[BH + bh] W inputs (merged Y, Z) in global memory, count[2 BH + bh]
  // W stored (the output kernel's flag).  The last split block merges the
  // partials at once; W is formed by whichever of {that block, the
  // pseudoinverse block} comes second: if the pseudoinverse block has
  // already counted in, the split block merges and forms W in one go (with
  // Z copied in beside the partials, m <= 64); otherwise it stores Y and
  // counts in, and the second to count forms W.  Each count is taken by
  // thread 0 between block barriers, with a fence on each side of the
  // atomic: the barrier orders the block's stores before the first fence,
  // the second fence orders the other blocks' stores (seen through the
  // count) before the block's loads after the next barrier.
  __shared__ uint32_t last;
  __shared__ volatile uint32_t w_abort;
  const int bh = is_pinv ? (int)blockIdx.x : (int)(blockIdx.x - prm.BH) / prm.splits;
  uint32_t *cnt_w = prm.count + prm.BH + bh;
  auto count_in = [&](uint32_t *c, uint32_t target) {
    tc_fence_before();
    __syncthreads();
    if (t == 0) {
      __threadfence();
      last = atomicAdd(c, 1u) == target;
      __threadfence();
    }
    __syncthreads();
    tc_fence_after();
  };
  if (t == 0) {
    w_abort = 0;
    test_delay(is_pinv ? 1 : 2);
  }
  const Abort wab{&w_abort, prm.err};
  bool form = false, z_staged = is_pinv, y_staged = false, z_copy = false;
  if (is_pinv) {
    count_in(cnt_w, 1u);
    form = last;
  } else {
    count_in(prm.count + bh, (uint32_t)prm.splits - 1u);
    if (last) {   // block-uniform
      __shared__ uint32_t z_ready;
      if (t == 0) z_ready = flag_acquire(cnt_w);
      __syncthreads();
      const bool direct = z_ready != 0;   // Z stored: this block forms W
      z_copy = direct && MergeSmem<M>::kZ;
      NYS_MARK(kTrMid, 3);
      merge_y<M>(prm, smem, bh, true, wab, z_copy);
      NYS_MARK(kTrMid, 4);
      y_staged = true;
      if (direct) {
        form = true;
      } else {
        count_in(cnt_w, 1u);
        form = last;
      }
    }
  }
  if (form) {   // block-uniform
    NYS_MARK(kTrMid, 5);
    form_w<M>(prm, smem, bh, tmem, wab, z_staged, y_staged,
              z_copy ? (const float *)(smem + MergeSmem<M>::zf) : nullptr);
    // form_w ends with a block barrier after every thread's stores
    if (t == 0) {
      fence_async_global();   // the output kernel reads W with a bulk copy
      flag_release(prm.count + 2 * prm.BH + bh, 1u);
    }
    NYS_MARK(kTrMid, 6);
  }
  tc_fence_before();
  __syncthreads();
  if ((t >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  NYS_MARK(kTrMid, 7);
}

}  // namespace midtc
}  // namespace nys
