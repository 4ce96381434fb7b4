// The whole bf16 forward (m <= 64) as one persistent launch: one block per
// SM pulls tasks from a global queue in a fixed order and runs them to
// completion ("Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, Eq. 16-17 / Algorithm 1, Figure 4).  Per
// (batch, head) h the tasks are
//   SEG(h, c)   segment sums of a run of Q or K rows -> Q~, K~ (Eq. 16),
//   PINV(h)     landmark kernel A and its pseudoinverse Z (Lemma 1),
//   BV(h, s)    B~ V over a range of keys (one partial softmax state per
//               landmark),
//   OUT(h, t)   a run of 128-row output tiles: F~ W + DConv(V),
// and the last of PINV(h) / BV(h, *) to finish merges the B~ V partials and
// forms W = Z Y.  The queue is a sequence of steps k = 0, 1, ...; step k
// holds SEG(k, *), PINV(k - lag_p), BV(k - lag_b, *) and OUT(k - lag_o, *)
// (those that exist), so a head's pseudoinverse starts as soon as its
// landmarks are summed while later heads still stream, and its output tiles
// come late enough that W is usually ready.  A task waits only for tasks
// earlier in the queue, which running blocks already hold, so the schedule
// cannot deadlock whatever the number of resident blocks.  Every wait is
// bounded; a timeout records NYS_ERR_TIMEOUT and the blocks stop taking
// tasks.
#pragma once

#include "mid_tc.cuh"
#include "out_tc.cuh"

namespace nys {
namespace fused {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kSegStages = 6;

enum TaskType : int { kNone = 0, kSeg = 1, kPinv = 2, kBv = 3, kOut = 4 };

struct Params {
  midtc::Params mid;      // pseudoinverse, B~ V, merge
  outtc::Params out;      // output tiles
  float *q_land, *k_land;
  uint32_t *err;          // error word
  uint32_t *queue;        // next task
  uint32_t *seg_cnt;      // [BH] SEG tasks done
  uint32_t *head_cnt;     // [BH] PINV + BV tasks done
  uint32_t *w_ready;      // [BH] W formed
  int BH, seg_len;        // l = n / m
  int seg_per_task, seg_tasks;   // segments per SEG task; SEG tasks per tensor per head
  int splits;             // BV tasks per head
  int tiles_per_task, out_tasks;   // output tiles per OUT task; OUT tasks per head
  int lag_p, lag_b, lag_o;
  int steps, total;       // queue steps, tasks
  float inv_len;          // 1 / l
};

struct Task {
  int type, h, idx;
};

// Sequential decoder of the queue order; task ids given to one block grow,
// so the decoder only moves forward.
struct Decoder {
  int k = 0, base = 0;
  __device__ int size(const Params &p, int k) const {
    int s = 0;
    if (k < p.BH) s += 2 * p.seg_tasks;
    if (k - p.lag_p >= 0 && k - p.lag_p < p.BH) s += 1;
    if (k - p.lag_b >= 0 && k - p.lag_b < p.BH) s += p.splits;
    if (k - p.lag_o >= 0 && k - p.lag_o < p.BH) s += p.out_tasks;
    return s;
  }
  __device__ Task decode(const Params &p, int id) {
    Task t{kNone, 0, 0};
    if (id >= p.total) return t;
    while (k < p.steps && id >= base + size(p, k)) {
      base += size(p, k);
      ++k;
    }
    int o = id - base;
    if (k < p.BH) {
      if (o < 2 * p.seg_tasks) return Task{kSeg, k, o};
      o -= 2 * p.seg_tasks;
    }
    if (k - p.lag_p >= 0 && k - p.lag_p < p.BH) {
      if (o == 0) return Task{kPinv, k - p.lag_p, 0};
      o -= 1;
    }
    if (k - p.lag_b >= 0 && k - p.lag_b < p.BH) {
      if (o < p.splits) return Task{kBv, k - p.lag_b, o};
      o -= p.splits;
    }
    return Task{kOut, k - p.lag_o, o};
  }
};

// Bounded wait for a global counter to reach `target` (acquire).  Gives up
// when another block has recorded an error, or after kWaitLimitCycles.
__device__ __forceinline__ bool wait_counter(const uint32_t *c, uint32_t target, uint32_t *err) {
  const long long t0 = clock64();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    if (v >= target) return true;
    if (*(volatile uint32_t *)err != 0) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      set_error(err, NYS_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(128);
  }
}

// ------------------------------------------------------------------ SEG
// Sums of the rows of segments [s0, s1) of one tensor of head bh, on the
// tensor cores: each 128-row TMA tile X is multiplied by an indicator matrix
// A (slot s, row k) = 1 if row k of the tile belongs to segment s0 + s, and
// D (128 slots x 64 features, fp32 in TMEM) accumulates over the tiles.  Any
// segment length works (segments may straddle tiles).  Warps: 0 TMA, 1 MMA
// issue, 4..11 build A (double-buffered) and read D.
struct SegSmem {
  static constexpr uint32_t x = 0;                              // [kSegStages] 16 KB tiles
  static constexpr uint32_t a = x + kSegStages * 16384u;        // [2] 32 KB indicators
  static constexpr uint32_t bars = a + 2 * 32768u;
  static constexpr uint32_t total = bars + 1024u;
};

template <int M>
__device__ __forceinline__ void seg_body(const CUtensorMap *map, const Params &prm, uint8_t *smem,
                                         int bh, int chunk, float *dst, uint32_t tmem) {
  using L = SegSmem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int len = prm.seg_len;
  const int s0 = chunk * prm.seg_per_task;
  const int s1 = min(M, s0 + prm.seg_per_task);
  const int nseg = s1 - s0;
  const int r0 = s0 * len, r1 = s1 * len;
  const int nst = (r1 - r0 + 127) / 128;
  uint64_t *bars = (uint64_t *)(smem + L::bars);
  uint64_t *full = bars, *empty = bars + kSegStages;
  uint64_t *a_ready = bars + 2 * kSegStages, *a_free = a_ready + 2, *d_full = a_free + 2;
  constexpr int kBars = 2 * kSegStages + 5;
  volatile uint32_t *abort_flag = (volatile uint32_t *)(bars + kBars);
  const Abort ab{abort_flag, prm.err};
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSegStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_ready[b], 256);
      mbar_init(&a_free[b], 1);
    }
    mbar_init(d_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const uint32_t xs = smem_u32(smem + L::x), as = smem_u32(smem + L::a);

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nst; ++i) {
        const int s = i % kSegStages;
        if (!mbar_wait(&empty[s], ((i / kSegStages) & 1) ^ 1, ab)) break;
        mbar_expect_tx(&full[s], 16384u);
        tma_load_3d(smem + L::x + s * 16384u, map, &full[s], 0, r0 + 128 * i, bh);
      }
      for (int i = nst > kSegStages ? nst - kSegStages : 0; i < nst; ++i)
        if (!mbar_wait(&empty[i % kSegStages], (i / kSegStages) & 1, ab)) break;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kFmtBF16, 128, 64, 0, 1);
      bool ok = true;
      for (int i = 0; i < nst && ok; ++i) {
        const int s = i % kSegStages, b = i & 1;
        if (!(ok = mbar_wait(&full[s], (i / kSegStages) & 1, ab))) break;
        if (!(ok = mbar_wait(&a_ready[b], (i >> 1) & 1, ab))) break;
        tc_fence_after();
        const uint64_t da = make_sdesc(as + b * 32768u, 16, 1024);
        const uint64_t dx = make_sdesc(xs + s * 16384u, 16, 1024);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_bf16(tmem, da + (k >> 2) * 1024u + (k & 3) * 2u, dx + 128u * k, idesc,
                   (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&a_free[b]);
      }
      if (ok) mma_commit(d_full);
    }
  } else if (warp >= 4) {
    const int u = threadIdx.x - 128;             // 0..255
    const int slot = u >> 1, kh = u & 1;         // A row, K half
    const int lo_row = (s0 + slot) * len;
    const int hi_row = min(lo_row + len, r1);
    const bool live = slot < nseg;
    bool ok = true;
    for (int i = 0; i < nst && ok; ++i) {
      const int b = i & 1;
      if (i >= 2 && !(ok = mbar_wait(&a_free[b], ((i - 2) >> 1) & 1, ab))) break;
      const int rbase = r0 + 128 * i + kh * 64;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ra = rbase + q * 8 + 2 * e, rb = ra + 1;
          const uint32_t lo = (live && ra >= lo_row && ra < hi_row) ? 0x3F80u : 0u;
          const uint32_t hi = (live && rb >= lo_row && rb < hi_row) ? 0x3F80u : 0u;
          w[e] = lo | (hi << 16);
        }
        st_shared_v4(as + b * 32768u + kh * 16384u + sw128_offset(slot, q), w[0], w[1], w[2],
                     w[3]);
      }
      fence_async_smem();
      mbar_arrive(&a_ready[b]);
    }
    // the last indicator releases are not waited for by anyone else
    for (int i = nst > 2 ? nst - 2 : 0; i < nst && ok; ++i)
      ok = mbar_wait(&a_free[i & 1], (i >> 1) & 1, ab);
    if (warp < 8 && ok && mbar_wait(d_full, 0, ab)) {
      tc_fence_after();
      float v[64];
      const uint32_t t_d = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      tmem_ld32(t_d, v);
      tmem_ld32(t_d + 32, v + 32);
      tmem_ld_wait();
      if (u < nseg) {
        float4 *o = (float4 *)(dst + ((size_t)bh * M + s0 + u) * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          o[q] = make_float4(v[4 * q] * prm.inv_len, v[4 * q + 1] * prm.inv_len,
                             v[4 * q + 2] * prm.inv_len, v[4 * q + 3] * prm.inv_len);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag)
    for (int b = 0; b < kBars; ++b) mbar_inval(bars + b);
}

template <int M>
__host__ __device__ constexpr uint32_t smem_bytes(int kconv) {
  const uint32_t a = midtc::smem_bytes<M>();   // includes the 1 KB alignment slack
  const uint32_t b = outtc::smem_layout(M, kconv).total;
  const uint32_t c = SegSmem::total + 1024u;
  const uint32_t ab = a > b ? a : b;
  return ab > c ? ab : c;
}

// Each task body is a separate function so that it gets its own register
// allocation (inlined together they spill).
template <int M>
__device__ __forceinline__ void run_seg(const CUtensorMap *map, const Params &prm, uint8_t *smem,
                                     int bh, int chunk, float *dst, uint32_t tmem) {
  seg_body<M>(map, prm, smem, bh, chunk, dst, tmem);
}
template <int M>
__device__ __forceinline__ void run_out(const CUtensorMap *mq, const CUtensorMap *mvh,
                                     const CUtensorMap *mo, const Params &prm, uint8_t *smem,
                                     int bh, int tb, int te, uint32_t tmem) {
  outtc::out_body<M>(mq, mvh, mo, prm.out, smem, bh, tb, te, tmem);
}
template <int M>
__device__ __forceinline__ void run_pinv(const Params &prm, uint8_t *smem, int bh, uint32_t tmem) {
  pinvpow::pinv_body<M>(prm.mid.pinv, smem, bh, tmem);
}
template <int M>
__device__ __forceinline__ void run_bv(const CUtensorMap *mk, const CUtensorMap *mv,
                                    const Params &prm, uint8_t *smem, int bh, int split,
                                    uint32_t tmem) {
  midtc::bv_body<M>(mk, mv, prm.mid, smem, bh, split, tmem);
}
template <int M>
__device__ __forceinline__ void run_merge(const Params &prm, uint8_t *smem, int bh, uint32_t tmem) {
  midtc::merge_body<M>(prm.mid, smem, bh);
}

template <int M>
__global__ void __launch_bounds__(kThreads, 1)
fused_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
             const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_vh,
             const __grid_constant__ CUtensorMap map_o, const __grid_constant__ Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint32_t tmem_base, last;
  __shared__ Task task;
  const int warp = threadIdx.x >> 5;
  if (warp == 1) tmem_alloc(&tmem_base, 512);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&map_q);
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
    tma_prefetch_desc(&map_vh);
    tma_prefetch_desc(&map_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  Decoder dec;
  while (true) {
    if (threadIdx.x == 0) {
      Task t{kNone, 0, 0};
      if (*(volatile uint32_t *)prm.err == 0) t = dec.decode(prm, (int)atomicAdd(prm.queue, 1u));
      bool ok = true;
      if (t.type == kPinv || t.type == kBv)
        ok = wait_counter(prm.seg_cnt + t.h, 2u * prm.seg_tasks, prm.err);
      else if (t.type == kOut)
        ok = wait_counter(prm.w_ready + t.h, 1u, prm.err);
      if (!ok) t.type = kNone;
      task = t;
    }
    __syncthreads();
    const Task t = task;
    if (t.type == kNone) break;
    if (t.type == kSeg) {
      const bool is_k = t.idx >= prm.seg_tasks;
      run_seg<M>(is_k ? &map_k : &map_q, prm, smem, t.h, is_k ? t.idx - prm.seg_tasks : t.idx,
                 is_k ? prm.k_land : prm.q_land, tmem);
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) atomicAdd(prm.seg_cnt + t.h, 1u);
    } else if (t.type == kOut) {
      const int tb = t.idx * prm.tiles_per_task;
      const int te = min(prm.out.tiles_per_head, tb + prm.tiles_per_task);
      run_out<M>(&map_q, &map_vh, &map_o, prm, smem, t.h, tb, te, tmem);
    } else {
      if (t.type == kPinv) {
        if (threadIdx.x < pinvpow::kBarThreads) run_pinv<M>(prm, smem, t.h, tmem);
      } else {
        run_bv<M>(&map_k, &map_v, prm, smem, t.h, t.idx, tmem);
      }
      // publish, count; the last of the head's splits + 1 tasks merges
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) last = atomicAdd(prm.head_cnt + t.h, 1u) == (uint32_t)prm.splits;
      __syncthreads();
      if (last) {
        __threadfence();
        run_merge<M>(prm, smem, t.h, tmem);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0)
          asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(prm.w_ready + t.h), "r"(1u)
                       : "memory");
      }
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fused
}  // namespace nys
