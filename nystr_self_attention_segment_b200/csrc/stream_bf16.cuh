// Segment means of the bf16 path (head_dim = 64): Q~ and K~ in one pass over
// Q and K ("Nystromformer: A Nystrom-Based Algorithm for Approximating
// Self-Attention", section 3.4, Eq. 16 with the page's 1/l correction).
// Segment j holds tokens j*l .. min(j*l + l, L) - 1, l = ceil(L / m), L the
// sequence length of the element (n, or its own length for ragged batches):
// the sequence read as padded to m*l tokens, each landmark the mean over the
// real tokens of its segment.
//
// A block owns a run of consecutive segments of one (batch*head, tensor).
// Its rows stream through shared memory in pieces of at most 128 rows (16 KB)
// by bulk copies (cp.async.bulk, no multicast) into a ring of kStages
// buffers, so that up to 64 KB per block are in flight; thread 256 issues the
// copies.  A piece holds k = floor(128 / l) whole segments (l <= 128) or 128
// rows of one segment (l > 128).  The 8 consumer warps split a piece:
//   k >= 8  warp w sums whole segments w, w + 8, ... (lane = 2 features);
//   k <  8  floor(8 / k) warps per segment sum disjoint row ranges, and the
//           partial sums of a segment (carried across its pieces) are added
//           in warp order at the segment's end.
// Every sum runs in a fixed order, so the result is bitwise reproducible.
#pragma once

#include "sm100.cuh"
#include "trace.cuh"

namespace nys {
namespace segm {

using namespace sm100;

constexpr int kStages = 4;
constexpr int kPieceRows = 128;
constexpr int kConsumers = 256;
constexpr int kThreads = kConsumers + 32;
constexpr uint32_t kSmem = kStages * kPieceRows * 128u + 1024u;   // + slack for alignment

// Tokens of element b: lens (device, per batch element) or n.
struct Shape {
  int n, m, heads;
  const int *lens;   // [batch] or null
};

__device__ __forceinline__ int elem_len(const Shape &sh, int bh) {
  return sh.lens ? sh.lens[bh / sh.heads] : sh.n;
}

// Pieces of segments [j0, j1) of a sequence of L tokens, segment length l:
// piece p covers rows [row0, row0 + rows) and segments [s0, s0 + ns) (ns >= 1;
// for l > 128 the piece is part `part` of segment s0).
struct Piece {
  int row0, rows, s0, ns, last;   // last: the piece ends segment s0 + ns - 1
};

__device__ __forceinline__ int seg_rows(int j, int l, int L) {
  return min(l, L - j * l);
}

__device__ __forceinline__ int n_pieces(int j0, int j1, int l, int L) {
  if (j1 <= j0) return 0;
  if (l <= kPieceRows) {
    const int k = kPieceRows / l;
    return (j1 - j0 + k - 1) / k;
  }
  // whole segments of l rows, except possibly the last segment of the sequence
  const int per = (l + kPieceRows - 1) / kPieceRows;
  int total = (j1 - j0 - 1) * per;
  total += (seg_rows(j1 - 1, l, L) + kPieceRows - 1) / kPieceRows;
  return total;
}

__device__ __forceinline__ Piece piece_at(int p, int j0, int j1, int l, int L) {
  Piece r;
  if (l <= kPieceRows) {
    const int k = kPieceRows / l;
    r.s0 = j0 + p * k;
    r.ns = min(k, j1 - r.s0);
    r.row0 = r.s0 * l;
    r.rows = min((r.s0 + r.ns) * l, L) - r.row0;
    r.last = 1;
  } else {
    const int per = (l + kPieceRows - 1) / kPieceRows;
    const int j = j0 + p / per, part = p % per;
    const int cnt = seg_rows(j, l, L);
    r.s0 = j;
    r.ns = 1;
    r.row0 = j * l + part * kPieceRows;
    r.rows = min(kPieceRows, cnt - part * kPieceRows);
    r.last = (part + 1) * kPieceRows >= cnt;
  }
  return r;
}

// Grid (groups, batch*heads, 2): block x sums segments
// [x*m/groups, (x+1)*m/groups) of tensor z (0: Q, 1: K) of element y.
// lens elements must hold m <= L <= n with no empty segment (checked on the
// host for lens == null; for device lengths, an invalid length records
// NYS_ERR_INVALID_ARG and its landmarks are left unwritten).
__global__ void __launch_bounds__(kThreads)
seg_means_bf16(const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
               float *__restrict__ Qt, float *__restrict__ Kt, Shape sh, uint32_t *err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *ring = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ float red[8][64];
  __shared__ uint32_t abort_flag;
  NYS_MARK(kTrSeg, 0);
  griddep_launch_dependents();   // the next kernel waits for this grid anyway
  const int bh = blockIdx.y;
  const __nv_bfloat16 *X = blockIdx.z == 0 ? Q : K;
  float *Xt = blockIdx.z == 0 ? Qt : Kt;
  const int L = elem_len(sh, bh);
  const int m = sh.m;
  if (L < m || L > sh.n || (long)(m - 1) * ((L + m - 1) / m) >= L) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) set_error(err, NYS_ERR_INVALID_ARG);
    return;
  }
  const int l = (L + m - 1) / m;
  const int j0 = (int)((long)blockIdx.x * m / gridDim.x);
  const int j1 = (int)((long)(blockIdx.x + 1) * m / gridDim.x);
  const int np = n_pieces(j0, j1, l, L);
  const uint8_t *src = (const uint8_t *)(X + (size_t)bh * sh.n * 64);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);   // one arrival per consumer warp
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Abort ab{&abort_flag, err};
  if (t == kConsumers) {
    // ---------------------------------------------------------- producer
    for (int p = 0; p < np; ++p) {
      const int s = p % kStages;
      if (p >= kStages && !mbar_wait(&empty[s], ((p / kStages) & 1) ^ 1, ab)) break;
      const Piece pc = piece_at(p, j0, j1, l, L);
      const uint32_t bytes = (uint32_t)pc.rows * 128u;
      mbar_expect_tx(&full[s], bytes);
      bulk_load(ring + s * (kPieceRows * 128), src + (size_t)pc.row0 * 128, bytes, &full[s]);
    }
    // wait for the last releases, so that no arrival is pending at exit
    for (int p = np > kStages ? np - kStages : 0; p < np; ++p)
      if (!mbar_wait(&empty[p % kStages], (p / kStages) & 1, ab)) break;
  } else if (t < kConsumers) {
    // ---------------------------------------------------------- consumers
    float a0 = 0.f, a1 = 0.f;   // features 2*lane, 2*lane + 1
    for (int p = 0; p < np; ++p) {
      const int s = p % kStages;
      if (!mbar_wait(&full[s], (p / kStages) & 1, ab)) break;
      const Piece pc = piece_at(p, j0, j1, l, L);
      const uint8_t *buf = ring + s * (kPieceRows * 128);
      if (pc.ns >= 8) {
        // whole segments per warp (l <= 16): the mean straight out
        for (int q = warp; q < pc.ns; q += 8) {
          const int j = pc.s0 + q;
          const int r0 = j * l - pc.row0, cnt = seg_rows(j, l, L);
          float b0 = 0.f, b1 = 0.f;
          for (int r = 0; r < cnt; ++r) {
            const float2 f = __bfloat1622float2(
                *(const __nv_bfloat162 *)(buf + (r0 + r) * 128 + lane * 4));
            b0 += f.x;
            b1 += f.y;
          }
          const float inv = 1.f / (float)cnt;
          *(float2 *)(Xt + ((size_t)bh * m + j) * 64 + 2 * lane) = make_float2(b0 * inv, b1 * inv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      } else {
        // wps warps per segment, each a contiguous row range of the piece
        const int wps = 8 / pc.ns;
        const int q = warp / wps, part = warp % wps;
        if (q < pc.ns) {
          const int j = pc.s0 + q;
          const int seg_lo = max(j * l, pc.row0) - pc.row0;
          const int seg_hi = min(j * l + seg_rows(j, l, L), pc.row0 + pc.rows) - pc.row0;
          const int per = (seg_hi - seg_lo + wps - 1) / wps;
          const int r_lo = seg_lo + part * per, r_hi = min(seg_hi, r_lo + per);
          for (int r = r_lo; r < r_hi; ++r) {
            const float2 f =
                __bfloat1622float2(*(const __nv_bfloat162 *)(buf + r * 128 + lane * 4));
            a0 += f.x;
            a1 += f.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (pc.last) {
          // the piece ends its segments: partials of each segment in warp order
          if (q < pc.ns) {
            red[warp][2 * lane] = a0;
            red[warp][2 * lane + 1] = a1;
          }
          named_barrier(1, kConsumers);
          for (int i = t; i < pc.ns * 64; i += kConsumers) {
            const int qq = i >> 6, c = i & 63, j = pc.s0 + qq;
            float sum = 0.f;
            for (int w = qq * wps; w < (qq + 1) * wps; ++w) sum += red[w][c];
            Xt[((size_t)bh * m + j) * 64 + c] = sum / (float)seg_rows(j, l, L);
          }
          named_barrier(1, kConsumers);
          a0 = a1 = 0.f;
        }
      }
    }
  }
  __syncthreads();
  if (t == 0 && !abort_flag)
    for (int s = 0; s < kStages; ++s) {
      mbar_inval(&full[s]);
      mbar_inval(&empty[s]);
    }
  NYS_MARK(kTrSeg, 1);
}

// Blocks per (batch*head, tensor): about one wave of kResident blocks per SM
// over the whole grid, at most one block per segment.
constexpr int kResident = 3;
inline int groups_for(int BH, int m) {
  int g = (kNumSms * kResident) / (2 * BH);
  if (g < 1) g = 1;
  if (g > m) g = m;
  return g;
}

}  // namespace segm
}  // namespace nys
