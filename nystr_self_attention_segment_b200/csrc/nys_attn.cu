// C ABI of the Nystrom attention forward: argument validation, workspace
// layout and the stream-ordered launch sequence.  See include/nys_attn.h for
// the contract of every entry point.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>
#include <utility>

#include "common.cuh"
#include "simt.cuh"
#include "sm100.cuh"
#include "mid_tc.cuh"
#include "out_tc.cuh"
#include "bwd_simt.cuh"
#include "gemm_tc.cuh"
#include "stream_bf16.cuh"

using namespace nys;

namespace {

size_t elem_size(int dtype) { return dtype == NYS_BF16 ? 2 : 4; }

nys_status validate_shape(const nys_desc *desc, int m) {
  if (!desc) return NYS_ERR_INVALID_ARG;
  if (desc->dtype != NYS_F32 && desc->dtype != NYS_BF16) return NYS_ERR_INVALID_ARG;
  if (desc->batch < 0 || desc->heads < 0 || desc->seq_len < 0 || desc->head_dim < 1)
    return NYS_ERR_INVALID_ARG;
  if (m < 1) return NYS_ERR_INVALID_ARG;
  if ((long)desc->batch * desc->heads * desc->seq_len == 0) return NYS_OK;   // empty
  if (m > desc->seq_len) return NYS_ERR_INVALID_ARG;
  {   // segments of ceil(n / m) tokens, the last one possibly shorter: none empty
    const long seg = ((long)desc->seq_len + m - 1) / m;
    if ((long)(m - 1) * seg >= desc->seq_len) return NYS_ERR_NOT_DIVISIBLE;
  }
  if (desc->dtype == NYS_F32) {
    if (desc->head_dim > 64 || m > 64) return NYS_ERR_UNSUPPORTED;
  } else {
    if (desc->head_dim != 64) return NYS_ERR_UNSUPPORTED;
    if (m != 32 && m != 64 && m != 128) return NYS_ERR_UNSUPPORTED;
  }
  // batch * heads indexes gridDim.y of the segment-mean and SIMT launches
  // (at most 65535); seq_len indexes TMA coordinates and int offsets
  if ((long)desc->batch * desc->heads > 65535L || desc->seq_len > (1 << 24))
    return NYS_ERR_UNSUPPORTED;
  return NYS_OK;
}

bool is_empty(const nys_desc *desc) {
  return (long)desc->batch * desc->heads * desc->seq_len == 0;
}


// Key splits per head of the SIMT B~ V pass (whole 64-key tiles each): one
// wave of three blocks per SM, at most 64 (the merge keeps a weight per split
// and row in shared memory); *keys_per_split gets the split length.
int simt_key_splits(size_t BH, size_t n, int *keys_per_split) {
  const int tile = kSimtKeyTile;
  const int ntiles = (int)((n + tile - 1) / tile);
  int splits = BH ? (int)((3 * kNumSms) / BH) : 1;
  if (splits > 64) splits = 64;
  if (splits > ntiles) splits = ntiles;
  if (splits < 1) splits = 1;
  const int tiles_per_split = (ntiles + splits - 1) / splits;
  *keys_per_split = tiles_per_split * tile;
  return (ntiles + tiles_per_split - 1) / tiles_per_split;
}

Layout make_layout(const nys_desc *desc, int m) {
  Layout L;
  memset(&L, 0, sizeof(L));
  const size_t BH = (size_t)desc->batch * desc->heads;
  const size_t n = desc->seq_len, d = desc->head_dim;
  int splits;
  if (desc->dtype == NYS_BF16) {
    // one B~ V CTA per SM: chunk-aligned key splits per head, times the
    // 128 / m row copies inside a CTA
    // one pseudoinverse block per head plus `splits` B~ V blocks per head in
    // one wave of 148 blocks; each B~ V block leaves one merged partial
    const int chunks = (int)((n + midtc::kChunk - 1) / midtc::kChunk);
    int per_head = BH ? (int)((kNumSms - (int)BH) / (int)BH) : 1;
    if (per_head < 1) per_head = 1;
    if (per_head > chunks) per_head = chunks;
    if (per_head > midtc::kMaxSplits) per_head = midtc::kMaxSplits;
    L.bv_ctas_per_head = per_head;
    splits = per_head;
    L.keys_per_split = 0;
  } else {
    splits = simt_key_splits(BH, n, &L.keys_per_split);
    L.bv_ctas_per_head = 0;
  }
  L.splits = splits;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.q_land = take(BH * m * d * 4);
  L.k_land = take(BH * m * d * 4);
  L.z = take(BH * m * m * 4);
  L.y = take(BH * m * d * 4);
  L.w = take(BH * m * d * 4);
  // the error word, then the hand-off words of every head; all zeroed by
  // every call
  L.err = take(256 + BH * 4 * kCountsPerHead);
  L.count = L.err + 256;
  L.pmax = take(BH * splits * m * 4);
  L.psum = take(BH * splits * m * 4);
  L.py = take(BH * splits * m * d * 4);
  L.scratch = take(desc->dtype == NYS_F32 && m > 64 ? BH * pinv_simt_mats_bytes(m) : 0);
  L.w_bf = take(desc->dtype == NYS_BF16 ? BH * m * 128 : 0);   // W as the bf16 P W operand
  L.total = off;
  return L;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  uintptr_t x0 = (uintptr_t)a, x1 = x0 + na, y0 = (uintptr_t)b, y1 = y0 + nb;
  return x0 < y1 && y0 < x1;
}

// Records events[i + 1] after the i-th kernel when the caller asked for
// per-kernel timing.
// Inside a stream capture the records become external event nodes of the
// graph, so that a replayed graph still times every kernel.
struct Marks {
  cudaEvent_t const *ev = nullptr;
  int n = 0, next = 1;
  int launched = 0;   // kernels enqueued so far by this call
  static void record(cudaEvent_t e, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else
      cudaEventRecord(e, s);
  }
  void first(cudaStream_t s) {
    if (ev) record(ev[0], s);
  }
  void after(cudaStream_t s) {
    ++launched;
    if (ev && next < n) record(ev[next++], s);
  }
};

#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
// Test builds only (a separate library the tests load): the launch with this
// index in the next forward call asks for more dynamic shared memory than a
// block may have, so that the launch is refused and nothing of it runs.
int g_fail_launch = -1;
// Test builds only: while set, bwd_head never publishes its dY / D flag, so
// that bwd_keys' bounded wait runs out.
bool g_hold_head_flag = false;
#endif

// Whether bwd_head publishes its per-head flag (always, outside the test
// build).
int head_publishes() {
#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
  return g_hold_head_flag ? 0 : 1;
#else
  return 1;
#endif
}

// Dynamic shared memory of launch `idx` of a call (a test build may make one
// launch impossible, see above).
size_t launch_smem(int idx, size_t smem) {
#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
  if (idx == g_fail_launch) {
    g_fail_launch = -1;
    return (size_t)1 << 20;
  }
#endif
  (void)idx;
  return smem;
}

// Launches one kernel and reports the launch's own status (the return value
// of cudaLaunchKernelEx, so an unrelated earlier error cannot be mistaken
// for it).  pdl: programmatic stream serialisation, i.e. the kernel may start
// while the previous kernel of the stream drains and must wait
// (griddepcontrol.wait) before it reads that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, bool pdl, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
// Test build only: a bounded wait that runs out (see nys_test_timeout_probe).
__global__ void timeout_probe(uint32_t *err, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ uint32_t flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const sm100::Abort ab{&flag, err};
    if (!sm100::mbar_wait_for(&bar, 0, ab, limit_cycles)) sm100::mbar_inval(&bar);
  }
}
#endif

// Opts a kernel in to `smem` bytes of dynamic shared memory when it needs
// more than the default 48 KB.
template <typename... KArgs>
bool allow_smem(void (*kern)(KArgs...), size_t smem) {
  return smem <= 48 * 1024 ||
         cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
             cudaSuccess;
}

constexpr int kSimtLaunches = 5;
const char *kSimtNames = "seg_means,pinv,bv_partial,merge_w,out";

template <typename T>
nys_status launch_simt(const T *Q, const T *K, const T *V, const nys_desc *desc, int m,
                       int iters, const float *conv_w, int conv_k, const int *lens, T *out,
                       char *ws, const Layout &L, cudaStream_t stream, Marks &mk) {
  const int BH = desc->batch * desc->heads;
  const int n = desc->seq_len, d = desc->head_dim;
  float *qt = (float *)(ws + L.q_land), *kt = (float *)(ws + L.k_land);
  float *z = (float *)(ws + L.z), *y = (float *)(ws + L.y), *w = (float *)(ws + L.w);
  float *pmax = (float *)(ws + L.pmax), *psum = (float *)(ws + L.psum);
  float *py = (float *)(ws + L.py), *scratch = (float *)(ws + L.scratch);
  uint32_t *err = (uint32_t *)(ws + L.err);
  const int heads = desc->heads;
  const float scale = 1.0f / sqrtf((float)d);
  const float scale_log2 = scale * kLog2e;

  // every launch is checked at once: a refused launch returns before the
  // next one is enqueued
  {
    long total = (long)BH * m * d;
    dim3 grid((unsigned)((total + 255) / 256), 2);
    if (launch(seg_means_scalar<T>, grid, dim3(256), launch_smem(mk.launched, 0), stream, false,
               Q, K, qt, kt, BH, n, d, m, lens, heads, err) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {
    const int use_smem = m <= 64;
    size_t sm = pinv_simt_smem(m);
    auto kern = pinv_simt_for(m);
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH), dim3(256), launch_smem(mk.launched, sm), stream, false, qt,
               kt, z, scratch, m, d, scale, iters, use_smem, (float *)nullptr,
               (float *)nullptr) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {
    const size_t sm = bv_partial_simt_smem(m);
    dim3 grid(L.splits, BH);
    auto kern = bv_partial_simt_for<T>(m);
    if (!allow_smem(kern, sm) ||
        launch(kern, grid, dim3(256), launch_smem(mk.launched, sm), stream, true, qt, K, V,
               pmax, psum, py, n, d, m, L.splits, L.keys_per_split, scale_log2, lens,
               heads) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {
    const size_t sm = merge_w_smem(m, d, L.splits);
    auto kern = merge_w_simt;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH, (d + kMergeCols - 1) / kMergeCols), dim3(256),
               launch_smem(mk.launched, sm), stream, false, pmax, psum, py, z, y, w, m, d,
               L.splits, (float *)nullptr) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {
    size_t sm = ((size_t)m * (d + 1) + (size_t)m * d + 8 * d + (conv_w ? conv_k : 0)) * 4;
    dim3 grid((n + kSimtOutRowsPerBlock - 1) / kSimtOutRowsPerBlock, BH);
    const int ck = conv_w ? conv_k : 0;
    auto kern = m <= 64 ? out_simt<T, 2> : out_simt<T, 4>;
    if (!allow_smem(kern, sm) ||
        launch(kern, grid, dim3(256), launch_smem(mk.launched, sm), stream, false, Q, V, kt, w,
               conv_w, out, n, d, m, desc->heads, ck, scale_log2, lens) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  return NYS_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, resolved through the runtime so that the
// library does not link libcuda (it loads on machines without a GPU).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;   // resolved once; never changes afterwards
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// [BH][n][64] bf16 viewed as a 3-D tensor (64, n, BH); box of `rows` rows;
// 128-byte swizzle; out-of-range rows read as zero and are not written.
bool make_map(CUtensorMap *map, const void *base, int BH, int n, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)n, (cuuint64_t)BH};
  cuuint64_t strides[2] = {128, (cuuint64_t)n * 128};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// A bf16 tensor [d2][d1][d0] (d0 contiguous) as a 3-D map with a box of
// 64 x rows x 1 and the 128-byte swizzle; reads outside the tensor are zero.
bool make_map3(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
               int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// launches of the bf16 path
constexpr int kTcLaunches = 3;
const char *kTcNames = "seg_means,mid_tc,out_tc";

template <int M>
nys_status launch_tc_m(const __nv_bfloat16 *Q, const __nv_bfloat16 *K, const __nv_bfloat16 *V,
                       const nys_desc *desc, int iters, const float *conv_w, int conv_k,
                       const int *lens, __nv_bfloat16 *out, char *ws, const Layout &L,
                       cudaStream_t stream, Marks &mk) {
  const int BH = desc->batch * desc->heads;
  const int n = desc->seq_len;
  float *qt = (float *)(ws + L.q_land), *kt = (float *)(ws + L.k_land);
  float *z = (float *)(ws + L.z), *y = (float *)(ws + L.y), *w = (float *)(ws + L.w);
  float *pmax = (float *)(ws + L.pmax), *psum = (float *)(ws + L.psum);
  float *py = (float *)(ws + L.py);
  uint32_t *err = (uint32_t *)(ws + L.err);
  const float scale_log2 = 0.125f * kLog2e;   // log2(e) / sqrt(64)
  const bool conv = conv_w != nullptr;
  const int kconv = conv ? ((128 + conv_k - 1 + 15) / 16) * 16 : 0;

  CUtensorMap mq, mkk, mv, mvh, mo;
  if (!make_map(&mq, Q, BH, n, 128) || !make_map(&mkk, K, BH, n, 128) ||
      !make_map(&mv, V, BH, n, 128) || !make_map(&mvh, V, BH, n, conv ? kconv : 128) ||
      !make_map(&mo, out, BH, n, 128))
    return NYS_ERR_CUDA;

  {   // segment means of Q and K (Eq. 16)
    const segm::Shape sh{n, M, desc->heads, lens};
    if (launch(segm::seg_means_bf16, dim3(M, BH, 2), dim3(segm::threads_for(n, M)),
               launch_smem(mk.launched, 0), stream, false, Q, K, qt, kt, sh, err) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {   // pseudoinverse || B~ V, then the merge of Y and W = Z Y
    midtc::Params p;
    p.pinv = pinvpow::Params{qt, kt, z, err, iters, scale_log2};
    p.q_land = qt;
    p.pmax = pmax;
    p.psum = psum;
    p.py = py;
    p.z = z;
    p.y = y;
    p.w = w;
    p.w_op = (uint8_t *)(ws + L.w_bf);
    p.count = (uint32_t *)(ws + L.count);
    p.err = err;
    p.lens = lens;
    p.heads = desc->heads;
    p.BH = BH;
    p.n = n;
    p.chunks_per_head = (n + midtc::kChunk - 1) / midtc::kChunk;
    p.splits = L.splits;
    p.scale_log2 = scale_log2;
    auto kern = midtc::mid_kernel<M>;
    const uint32_t sm = midtc::smem_bytes<M>();
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH * (1 + L.splits)), dim3(midtc::kThreads),
               launch_smem(mk.launched, sm), stream, true, mkk, mv, p) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  {   // F~ W + DConv(V)
    const int tph = (n + outtc::kTileRows - 1) / outtc::kTileRows;
    // blocks per head: the SMs that the pseudoinverse blocks (one per head,
    // busy until about W) leave free, so that no block starts late
    int cpb = (kNumSms - BH) / BH;
    if (cpb < 1) cpb = 1;
    if (cpb > tph) cpb = tph;
    const uint32_t *w_flag = (const uint32_t *)(ws + L.count) + 2 * (size_t)BH;
    outtc::Params p{kt,  (const uint8_t *)(ws + L.w_bf), conv_w, err, n, desc->heads,
                    conv ? conv_k : 1, kconv, tph, cpb, scale_log2, lens, M, w_flag};
    auto kern = outtc::out_tc_kernel<M>;
    const uint32_t sm = outtc::smem_layout(M, conv ? kconv : 0).total;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH * cpb), dim3(outtc::Warps<M>::kThreads), launch_smem(mk.launched, sm),
               stream,
               true, mq, mvh, mo, p) != cudaSuccess)
      return NYS_ERR_CUDA;
    mk.after(stream);
  }
  return NYS_OK;
}

nys_status launch_tc(const __nv_bfloat16 *Q, const __nv_bfloat16 *K, const __nv_bfloat16 *V,
                     const nys_desc *desc, int m, int iters, const float *conv_w, int conv_k,
                     const int *lens, __nv_bfloat16 *out, char *ws, const Layout &L,
                     cudaStream_t stream, Marks &mk) {
  switch (m) {
    case 32: return launch_tc_m<32>(Q, K, V, desc, iters, conv_w, conv_k, lens, out, ws, L, stream, mk);
    case 64: return launch_tc_m<64>(Q, K, V, desc, iters, conv_w, conv_k, lens, out, ws, L, stream, mk);
    case 128:
      return launch_tc_m<128>(Q, K, V, desc, iters, conv_w, conv_k, lens, out, ws, L, stream, mk);
  }
  return NYS_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// The attention layer: QKV projection, the forward, output projection.
struct LayerLayout {
  size_t q, k, v, o, ws, total;
};

LayerLayout make_layer_layout(const nys_desc *desc, int m) {
  LayerLayout L;
  const size_t t = (size_t)desc->batch * desc->heads * desc->seq_len * 64 * 2;
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t at = off;
    off = align256(off + b);
    return at;
  };
  L.q = take(t);
  L.k = take(t);
  L.v = take(t);
  L.o = take(t);
  L.ws = take(make_layout(desc, m).total);
  L.total = off;
  return L;
}

template <int MODE>
nys_status launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, const gemm::Params &p,
                       cudaStream_t stream) {
  auto kern = gemm::gemm_kernel<MODE>;
  const int grid = p.batch * p.mtiles * p.ntiles;
  if (!allow_smem(kern, gemm::kSmem) ||
      launch(kern, dim3(grid), dim3(gemm::kThreads), gemm::kSmem, stream, false, ma, mb, p) !=
          cudaSuccess)
    return NYS_ERR_CUDA;
  return NYS_OK;
}

// ---------------------------------------------------------------------------
// Backward pass: workspace layout and launch sequence (bwd_simt.cuh).
struct BwdLayout {
  size_t qt, kt, z, a, zall, pscr, pmax, psum, py, y, w, lse, dwp, dktp, dcp, dy, dqta, dkt,
      dd, hscr, dqtp, err, ready, total;
  int S, keys_per_split, R, S2, mb;
};

int bwd_mbucket(int m) { return m <= 32 ? 32 : (m <= 64 ? 64 : 128); }

BwdLayout make_bwd_layout(const nys_desc *desc, int m, int iters, int conv_k) {
  BwdLayout L;
  memset(&L, 0, sizeof(L));
  const size_t BH = (size_t)desc->batch * desc->heads;
  const size_t n = desc->seq_len, d = desc->head_dim;
  L.S = simt_key_splits(BH, n, &L.keys_per_split);
  // row / key blocks per head: one wave of the resident blocks (two per SM
  // for m <= 64, one for m = 128), so that no SM runs a tail of its own
  L.mb = bwd_mbucket(m);
  const int t64 = (int)((n + bwd::kTile - 1) / bwd::kTile);
  const int per_sm = L.mb <= 64 ? 2 : 1;
  int r = BH ? (int)(kNumSms * per_sm / BH) : 1;
  if (r > t64) r = t64;
  if (r < 1) r = 1;
  L.R = r;
  // key blocks run beside bwd_head, one block per head on its own SM: one
  // wave on the SMs it leaves
  const int free_sms = BH < (size_t)kNumSms ? kNumSms - (int)BH : kNumSms;
  int s2 = BH ? (int)(free_sms * per_sm / BH) : 1;
  if (s2 > t64) s2 = t64;
  if (s2 < 1) s2 = 1;
  L.S2 = s2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t md = BH * m * d * 4, mm = BH * m * m * 4;
  // the error word first (offset 0), then bwd_head's per-head flags; one
  // memset per call clears both
  L.err = take(256);
  L.ready = take(BH * 4);
  L.qt = take(md);
  L.kt = take(md);
  L.z = take(mm);
  L.a = take(mm);
  L.zall = take(mm * (iters + 1));
  L.pscr = take(m > 64 ? BH * pinv_simt_mats_bytes(m) : 0);
  L.pmax = take(BH * L.S * m * 4);
  L.psum = take(BH * L.S * m * 4);
  L.py = take(BH * L.S * m * d * 4);
  L.y = take(md);
  L.w = take(md);
  L.lse = take(BH * m * 4);
  L.dwp = take(md * L.R);
  L.dktp = take(md * L.R);
  L.dcp = take(BH * L.R * (conv_k > 0 ? conv_k : 0) * 4);
  L.dy = take(md);
  L.dqta = take(md);
  L.dkt = take(md);
  L.dd = take(BH * m * 4);
  L.hscr = take(L.mb > 64 ? BH * bwd::head_bytes<128>() : 0);
  L.dqtp = take(md * L.S2);
  L.total = off;
  return L;
}

template <typename T, int MB>
nys_status launch_bwd(const T *Q, const T *K, const T *V, const nys_desc *desc, int m, int iters,
                      const float *conv_w, int conv_k, const T *dO, T *dQ, T *dK, T *dV,
                      float *dconv, char *ws, const BwdLayout &L, cudaStream_t stream) {
  const int BH = desc->batch * desc->heads, H = desc->heads;
  const int n = desc->seq_len, d = desc->head_dim;
  const float scale = 1.0f / sqrtf((float)d), scale_log2 = scale * kLog2e;
  float *qt = (float *)(ws + L.qt), *kt = (float *)(ws + L.kt), *z = (float *)(ws + L.z);
  float *a = (float *)(ws + L.a), *zall = (float *)(ws + L.zall);
  float *pmax = (float *)(ws + L.pmax), *psum = (float *)(ws + L.psum);
  float *py = (float *)(ws + L.py), *y = (float *)(ws + L.y), *w = (float *)(ws + L.w);
  float *lse = (float *)(ws + L.lse);
  uint32_t *err = (uint32_t *)(ws + L.err);
  const int ck = conv_w ? conv_k : 0;
  // the forward's landmark steps, keeping A, every Z iterate and B~'s
  // log-sum-exp
  if constexpr (sizeof(T) == 2) {
    if (d == 64) {   // the bf16 path's streaming segment means
      const segm::Shape sh{n, m, H, nullptr};
      if (launch(segm::seg_means_bf16, dim3(m, BH, 2), dim3(segm::threads_for(n, m)), 0, stream,
                 false, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K, qt, kt, sh,
                 err) != cudaSuccess)
        return NYS_ERR_CUDA;
    }
  }
  if (sizeof(T) != 2 || d != 64) {
    long total = (long)BH * m * d;
    if (launch(seg_means_scalar<T>, dim3((unsigned)((total + 255) / 256), 2), dim3(256), 0,
               stream, false, Q, K, qt, kt, BH, n, d, m, (const int *)nullptr, H,
               err) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  {
    const int use_smem = m <= 64;
    const size_t sm = pinv_simt_smem(m);
    auto kern = pinv_simt_for(m);
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH), dim3(256), sm, stream, false, (const float *)qt,
               (const float *)kt, z, (float *)(ws + L.pscr), m, d, scale, iters, use_smem, a,
               zall) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  {
    const size_t sm = bv_partial_simt_smem(m);
    auto kern = bv_partial_simt_for<T>(m);
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(L.S, BH), dim3(256), sm, stream, true, (const float *)qt, K, V, pmax,
               psum, py, n, d, m, L.S, L.keys_per_split, scale_log2, (const int *)nullptr,
               H) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  {
    const size_t sm = merge_w_smem(m, d, L.S);
    auto kern = merge_w_simt;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH, (d + kMergeCols - 1) / kMergeCols), dim3(256), sm, stream, false,
               (const float *)pmax,
               (const float *)psum, (const float *)py, (const float *)z, y, w, m, d, L.S,
               lse) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  // the backward proper
  {
    const bwd::RowsParams p{Q,  V,  dO, kt,  w,    conv_w, dQ,     (float *)(ws + L.dwp),
                            (float *)(ws + L.dktp), (float *)(ws + L.dcp), n, d, m, H, ck,
                            L.R, scale};
    auto kern = bwd::bwd_rows<T, MB>;
    const size_t sm = bwd::RowsSmem<MB>::total;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(L.R, BH), dim3(bwd::kThreads), sm, stream, false, p) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  {
    const bwd::HeadParams p{(const float *)(ws + L.dwp), (const float *)(ws + L.dktp), qt, kt, y,
                            a, zall, (float *)(ws + L.dy), (float *)(ws + L.dqta),
                            (float *)(ws + L.dkt), (float *)(ws + L.dd),
                            (float *)(ws + L.hscr), (uint32_t *)(ws + L.ready),
                            head_publishes(), d, m, iters, L.R, MB <= 64 ? 1 : 0, scale};
    auto kern = bwd::bwd_head<MB>;
    const size_t sm = MB <= 64 ? bwd::head_bytes<MB>() : 0;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(BH), dim3(bwd::kHeadThreads), sm, stream, false, p) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  {
    // programmatic launch: the key tiles run beside bwd_head once every
    // head has published dY and D
    const bwd::KeysParams p{K, V, dO, qt, (const float *)(ws + L.dy), lse,
                            (const float *)(ws + L.dd), conv_w,
                            (const uint32_t *)(ws + L.ready), err, dK, dV,
                            (float *)(ws + L.dqtp), n, d, m, H, ck, L.S2, scale, scale_log2};
    auto kern = bwd::bwd_keys<T, MB>;
    const size_t sm = bwd::KeysSmem<MB>::total;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3(L.S2, BH), dim3(bwd::kThreads), sm, stream, true, p) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  if (launch(bwd::bwd_dqt_total, dim3((m * d + bwd::kThreads - 1) / bwd::kThreads, BH),
             dim3(bwd::kThreads), 0, stream, false, (float *)(ws + L.dqta),
             (const float *)(ws + L.dqtp), m * d, L.S2) != cudaSuccess)
    return NYS_ERR_CUDA;
  {
    const int rpb = 256;
    const size_t sm = (size_t)2 * m * d * 4;
    auto kern = bwd::bwd_dqk<T>;
    if (!allow_smem(kern, sm) ||
        launch(kern, dim3((n + rpb - 1) / rpb, BH), dim3(bwd::kThreads), sm, stream, false,
               (void *)dQ, (void *)dK, (const float *)(ws + L.dqta),
               (const float *)(ws + L.dkt), n, d, m, rpb) != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  if (ck > 0 &&
      launch(bwd::bwd_dconv, dim3(H), dim3(64), 0, stream, false, dconv,
             (const float *)(ws + L.dcp), desc->batch, H, L.R, ck) != cudaSuccess)
    return NYS_ERR_CUDA;
  return NYS_OK;
}

}  // namespace

extern "C" {

NYS_ATTN_API const char *nys_status_string(nys_status s) {
  switch (s) {
    case NYS_OK: return "NYS_OK";
    case NYS_ERR_INVALID_ARG: return "NYS_ERR_INVALID_ARG: null pointer, negative size or bad enum";
    case NYS_ERR_UNSUPPORTED: return "NYS_ERR_UNSUPPORTED: no kernel for this head_dim / landmarks / dtype / conv_k";
    case NYS_ERR_NOT_DIVISIBLE: return "NYS_ERR_NOT_DIVISIBLE: a segment of ceil(seq_len / num_landmarks) tokens would be empty";
    case NYS_ERR_ALIAS: return "NYS_ERR_ALIAS: output overlaps an input or the workspace";
    case NYS_ERR_WORKSPACE: return "NYS_ERR_WORKSPACE: workspace too small";
    case NYS_ERR_CUDA: return "NYS_ERR_CUDA: CUDA runtime or launch failure";
    case NYS_ERR_TIMEOUT: return "NYS_ERR_TIMEOUT: a bounded device wait gave up";
  }
  return "unknown nys_status";
}

NYS_ATTN_API int nys_version(void) { return 100; }

NYS_ATTN_API nys_status nys_attn_workspace_size(const nys_desc *desc, int m, size_t *bytes) {
  if (!bytes) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  *bytes = is_empty(desc) ? 0 : make_layout(desc, m).total;
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_intermediates(const nys_desc *desc, int m,
                                               nys_intermediates *out) {
  if (!out) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) {
    memset(out, 0, sizeof(*out));
    return NYS_OK;
  }
  Layout L = make_layout(desc, m);
  out->q_landmarks = L.q_land;
  out->k_landmarks = L.k_land;
  out->z = L.z;
  out->y = L.y;
  out->w = L.w;
  out->error_word = L.err;
  out->total = L.total;
  return NYS_OK;
}

static nys_status validate_call(const void *Q, const void *K, const void *V,
                                const nys_desc *desc, int m, int iters, const float *conv_w,
                                int conv_k, const void *out) {
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (iters < 0) return NYS_ERR_INVALID_ARG;
  if (iters > kMaxIters) return NYS_ERR_UNSUPPORTED;
  if (conv_w) {
    if (conv_k < 1) return NYS_ERR_INVALID_ARG;
    if (conv_k % 2 == 0) return NYS_ERR_INVALID_ARG;
    if (conv_k > kMaxConvK) return NYS_ERR_UNSUPPORTED;
  }
  if (is_empty(desc)) return NYS_OK;
  if (!Q || !K || !V || !out) return NYS_ERR_INVALID_ARG;
  // tensor-memory-access maps and 16-byte loads (bf16), 4-byte loads (fp32)
  const uintptr_t align = desc->dtype == NYS_BF16 ? 15 : 3;
  if ((((uintptr_t)Q | (uintptr_t)K | (uintptr_t)V | (uintptr_t)out) & align) != 0)
    return NYS_ERR_INVALID_ARG;
  if (conv_w && ((uintptr_t)conv_w & 3) != 0) return NYS_ERR_INVALID_ARG;
  return NYS_OK;
}

static nys_status forward_impl(const void *Q, const void *K, const void *V,
                               const nys_desc *desc, int m, int iters, const float *conv_w,
                               int conv_k, void *out, void *workspace, size_t workspace_bytes,
                               nys_stream_t stream_, void *const *events, int n_events,
                               const int *lens = nullptr, bool clear_err = true) {
  nys_status st = validate_call(Q, K, V, desc, m, iters, conv_w, conv_k, out);
  if (st != NYS_OK) return st;
  if (events && n_events < (desc->dtype == NYS_BF16 ? kTcLaunches : kSimtLaunches) + 1)
    return NYS_ERR_INVALID_ARG;
  if (is_empty(desc)) return NYS_OK;
  Marks mk;
  mk.ev = (cudaEvent_t const *)events;
  mk.n = events ? n_events : 0;
  cudaStream_t stream = (cudaStream_t)stream_;
  const size_t tbytes = (size_t)desc->batch * desc->heads * desc->seq_len * desc->head_dim *
                        elem_size(desc->dtype);
  Layout L = make_layout(desc, m);
  if (overlaps(out, tbytes, Q, tbytes) || overlaps(out, tbytes, K, tbytes) ||
      overlaps(out, tbytes, V, tbytes))
    return NYS_ERR_ALIAS;
  if (workspace) {
    if (workspace_bytes < L.total) return NYS_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255) != 0) return NYS_ERR_INVALID_ARG;
    if (overlaps(out, tbytes, workspace, L.total)) return NYS_ERR_ALIAS;
  }
  char *ws = (char *)workspace;
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync((void **)&ws, L.total, stream) != cudaSuccess) return NYS_ERR_CUDA;
    owned = true;
  }
  const size_t ncount = (size_t)desc->batch * desc->heads * 4 * kCountsPerHead;
  const size_t nclear = clear_err ? 256 + ncount : 0;
  if (nclear && cudaMemsetAsync(ws + L.err, 0, nclear, stream) != cudaSuccess) st = NYS_ERR_CUDA;
  // the layer clears the error word itself; the counters still start at zero
  if (!clear_err &&
      cudaMemsetAsync(ws + L.count, 0, ncount, stream) !=
          cudaSuccess)
    st = NYS_ERR_CUDA;
  mk.first(stream);
  if (st == NYS_OK) {
    if (desc->dtype == NYS_F32)
      st = launch_simt<float>((const float *)Q, (const float *)K, (const float *)V, desc, m,
                              iters, conv_w, conv_k, lens, (float *)out, ws, L, stream, mk);
    else
      st = launch_tc((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                     (const __nv_bfloat16 *)V, desc, m, iters, conv_w, conv_k, lens,
                     (__nv_bfloat16 *)out, ws, L, stream, mk);
  }
  if (owned && cudaFreeAsync(ws, stream) != cudaSuccess && st == NYS_OK) st = NYS_ERR_CUDA;
  return st;
}

NYS_ATTN_API nys_status nys_attn_forward(const void *Q, const void *K, const void *V,
                                         const nys_desc *desc, int m, int iters,
                                         const float *conv_w, int conv_k, void *out,
                                         void *workspace, size_t workspace_bytes,
                                         nys_stream_t stream) {
  return forward_impl(Q, K, V, desc, m, iters, conv_w, conv_k, out, workspace, workspace_bytes,
                      stream, nullptr, 0);
}

NYS_ATTN_API nys_status nys_attn_forward_lens(const void *Q, const void *K, const void *V,
                                              const nys_desc *desc, int m, int iters,
                                              const float *conv_w, int conv_k,
                                              const int *lens_dev, void *out, void *workspace,
                                              size_t workspace_bytes, nys_stream_t stream) {
  const nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if ((!lens_dev && !is_empty(desc)) || ((uintptr_t)lens_dev & 3) != 0) return NYS_ERR_INVALID_ARG;
  return forward_impl(Q, K, V, desc, m, iters, conv_w, conv_k, out, workspace, workspace_bytes,
                      stream, nullptr, 0, lens_dev);
}

NYS_ATTN_API nys_status nys_attn_layer_workspace_size(const nys_desc *desc, int m,
                                                      size_t *bytes) {
  if (!bytes) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (desc->dtype != NYS_BF16) return NYS_ERR_UNSUPPORTED;
  *bytes = is_empty(desc) ? 0 : make_layer_layout(desc, m).total;
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_layer_forward(const void *X, const void *Wqkv, const void *Wo,
                                               const nys_desc *desc, int m, int iters,
                                               const float *conv_w, int conv_k, void *Y,
                                               void *workspace, size_t workspace_bytes,
                                               nys_stream_t stream_) {
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (desc->dtype != NYS_BF16) return NYS_ERR_UNSUPPORTED;
  if (iters < 0) return NYS_ERR_INVALID_ARG;
  if (iters > kMaxIters) return NYS_ERR_UNSUPPORTED;
  if (conv_w && (conv_k < 1 || conv_k % 2 == 0 || ((uintptr_t)conv_w & 3) != 0))
    return NYS_ERR_INVALID_ARG;
  if (conv_w && conv_k > kMaxConvK) return NYS_ERR_UNSUPPORTED;
  if (is_empty(desc)) return NYS_OK;
  if (!X || !Wqkv || !Wo || !Y || !workspace) return NYS_ERR_INVALID_ARG;
  if ((((uintptr_t)X | (uintptr_t)Wqkv | (uintptr_t)Wo | (uintptr_t)Y) & 15) != 0 ||
      ((uintptr_t)workspace & 255) != 0)
    return NYS_ERR_INVALID_ARG;
  const LayerLayout LL = make_layer_layout(desc, m);
  if (workspace_bytes < LL.total) return NYS_ERR_WORKSPACE;
  const int B = desc->batch, H = desc->heads, n = desc->seq_len, D = H * 64;
  const size_t xbytes = (size_t)B * n * D * 2;
  if (overlaps(Y, xbytes, X, xbytes) || overlaps(Y, xbytes, workspace, LL.total) ||
      overlaps(Y, xbytes, Wqkv, (size_t)3 * D * D * 2) || overlaps(Y, xbytes, Wo, (size_t)D * D * 2))
    return NYS_ERR_ALIAS;
  cudaStream_t stream = (cudaStream_t)stream_;
  char *ws = (char *)workspace;
  __nv_bfloat16 *q = (__nv_bfloat16 *)(ws + LL.q), *k = (__nv_bfloat16 *)(ws + LL.k),
                *v = (__nv_bfloat16 *)(ws + LL.v), *o = (__nv_bfloat16 *)(ws + LL.o);
  CUtensorMap mx, mwq, mo, mwo;
  if (!make_map3(&mx, X, D, n, B, gemm::kBM) || !make_map3(&mwq, Wqkv, D, 3 * D, 1, gemm::kBN) ||
      !make_map3(&mo, o, 64, n, (uint64_t)B * H, gemm::kBM) ||
      !make_map3(&mwo, Wo, D, D, 1, gemm::kBN))
    return NYS_ERR_CUDA;
  if (cudaMemsetAsync(ws + LL.ws + make_layout(desc, m).err, 0, 256, stream) != cudaSuccess)
    return NYS_ERR_CUDA;
  gemm::Params gp{};
  gp.n = n;
  gp.batch = B;
  gp.heads = H;
  gp.mtiles = (n + gemm::kBM - 1) / gemm::kBM;
  gp.err = (uint32_t *)(ws + LL.ws + make_layout(desc, m).err);
  // Q, K, V = X W^T, written per head
  gp.N = 3 * D;
  gp.K = D;
  gp.ntiles = (3 * D + gemm::kBN - 1) / gemm::kBN;
  gp.q = q;
  gp.k = k;
  gp.v = v;
  st = launch_gemm<gemm::kQkv>(mx, mwq, gp, stream);
  if (st != NYS_OK) return st;
  // the attention proper, with its workspace after Q, K, V, O
  st = forward_impl(q, k, v, desc, m, iters, conv_w, conv_k, o, ws + LL.ws, LL.total - LL.ws,
                    stream_, nullptr, 0, nullptr, false);
  if (st != NYS_OK) return st;
  // Y = concat_h(O_h) Wo^T
  gp.N = D;
  gp.K = D;
  gp.ntiles = (D + gemm::kBN - 1) / gemm::kBN;
  gp.y = (__nv_bfloat16 *)Y;
  return launch_gemm<gemm::kOut>(mo, mwo, gp, stream);
}

NYS_ATTN_API nys_status nys_attn_layer_check_error(void *workspace, const nys_desc *desc, int m,
                                                   nys_stream_t stream) {
  if (!workspace) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (desc->dtype != NYS_BF16) return NYS_ERR_UNSUPPORTED;
  if (is_empty(desc)) return NYS_OK;
  return nys_attn_check_error((char *)workspace + make_layer_layout(desc, m).ws, desc, m, stream);
}

NYS_ATTN_API nys_status nys_attn_backward_workspace_size(const nys_desc *desc, int m,
                                                         int pinv_iters, int conv_k,
                                                         size_t *bytes) {
  if (!bytes) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (pinv_iters < 0 || conv_k < 0) return NYS_ERR_INVALID_ARG;
  if (pinv_iters > kMaxIters || conv_k > kMaxConvK) return NYS_ERR_UNSUPPORTED;
  *bytes = is_empty(desc) ? 0 : make_bwd_layout(desc, m, pinv_iters, conv_k).total;
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_backward(const void *Q, const void *K, const void *V,
                                          const nys_desc *desc, int m, int iters,
                                          const float *conv_w, int conv_k, const void *dO,
                                          void *dQ, void *dK, void *dV, float *dconv_w,
                                          void *workspace, size_t workspace_bytes,
                                          nys_stream_t stream_) {
  nys_status st = validate_call(Q, K, V, desc, m, iters, conv_w, conv_k, dQ);
  if (st != NYS_OK) return st;
  if ((conv_w == nullptr) != (dconv_w == nullptr)) return NYS_ERR_INVALID_ARG;
  if (conv_w && ((uintptr_t)dconv_w & 3) != 0) return NYS_ERR_INVALID_ARG;
  if (is_empty(desc)) {
    if (conv_w && desc->heads > 0)   // no tokens: the conv gradient is zero
      return cudaMemsetAsync(dconv_w, 0, (size_t)desc->heads * conv_k * 4,
                             (cudaStream_t)stream_) == cudaSuccess
                 ? NYS_OK
                 : NYS_ERR_CUDA;
    return NYS_OK;
  }
  if (!dO || !dK || !dV) return NYS_ERR_INVALID_ARG;
  const uintptr_t align = desc->dtype == NYS_BF16 ? 15 : 3;
  if ((((uintptr_t)dO | (uintptr_t)dK | (uintptr_t)dV) & align) != 0) return NYS_ERR_INVALID_ARG;
  const size_t tbytes = (size_t)desc->batch * desc->heads * desc->seq_len * desc->head_dim *
                        elem_size(desc->dtype);
  // gradients overlap neither each other nor any input
  const void *ins[4] = {Q, K, V, dO};
  void *outs[3] = {dQ, dK, dV};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 4; ++j)
      if (overlaps(outs[i], tbytes, ins[j], tbytes)) return NYS_ERR_ALIAS;
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], tbytes, outs[j], tbytes)) return NYS_ERR_ALIAS;
  }
  const BwdLayout L = make_bwd_layout(desc, m, iters, conv_w ? conv_k : 0);
  cudaStream_t stream = (cudaStream_t)stream_;
  if (workspace) {
    if (workspace_bytes < L.total) return NYS_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255) != 0) return NYS_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
      if (overlaps(outs[i], tbytes, workspace, L.total)) return NYS_ERR_ALIAS;
  }
  char *ws = (char *)workspace;
  bool owned = false;
  if (!ws) {
    if (cudaMallocAsync((void **)&ws, L.total, stream) != cudaSuccess) return NYS_ERR_CUDA;
    owned = true;
  }
  if (cudaMemsetAsync(ws + L.err, 0, L.ready - L.err + (size_t)desc->batch * desc->heads * 4,
                      stream) != cudaSuccess)
    st = NYS_ERR_CUDA;
  if (st == NYS_OK) {
    const int mb = L.mb;
    if (desc->dtype == NYS_F32) {
      const float *q = (const float *)Q, *k = (const float *)K, *v = (const float *)V,
                  *g = (const float *)dO;
      float *dq = (float *)dQ, *dk = (float *)dK, *dv = (float *)dV;
      st = mb == 32 ? launch_bwd<float, 32>(q, k, v, desc, m, iters, conv_w, conv_k, g, dq, dk,
                                            dv, dconv_w, ws, L, stream)
                    : launch_bwd<float, 64>(q, k, v, desc, m, iters, conv_w, conv_k, g, dq, dk,
                                            dv, dconv_w, ws, L, stream);
    } else {
      typedef __nv_bfloat16 B;
      const B *q = (const B *)Q, *k = (const B *)K, *v = (const B *)V, *g = (const B *)dO;
      B *dq = (B *)dQ, *dk = (B *)dK, *dv = (B *)dV;
      st = mb == 32   ? launch_bwd<B, 32>(q, k, v, desc, m, iters, conv_w, conv_k, g, dq, dk, dv,
                                          dconv_w, ws, L, stream)
           : mb == 64 ? launch_bwd<B, 64>(q, k, v, desc, m, iters, conv_w, conv_k, g, dq, dk, dv,
                                          dconv_w, ws, L, stream)
                      : launch_bwd<B, 128>(q, k, v, desc, m, iters, conv_w, conv_k, g, dq, dk,
                                           dv, dconv_w, ws, L, stream);
    }
  }
  if (owned && cudaFreeAsync(ws, stream) != cudaSuccess && st == NYS_OK) st = NYS_ERR_CUDA;
  return st;
}

// ---------------------------------------------------------------------------
// nys_attn_forward_static: the forward with its scratch in a fixed device
// array instead of a caller-provided or stream-ordered workspace, for callers
// that cannot allocate device memory (see the header).  The array lives in
// this library's module: every device that loads the library holds it until
// the process exits.  Host code cannot pass the array's name to a kernel (on
// the host it is only a stand-in for the symbol), so its device address is
// looked up with cudaGetSymbolAddress, with the device current (below).
static __device__ __align__(256) unsigned char g_static_scratch[NYS_STATIC_SCRATCH_BYTES];

namespace {
// The array's device address belongs to the module as loaded in one CUDA
// context: a context that is destroyed and created again (cudaDeviceReset,
// for instance) may load the module at another address.  So the address is
// looked up again on every call outside stream capture, and the lookup is
// remembered per context (by its unique id) for calls made while a stream is
// capturing, when no lookup should run.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

constexpr int kMaxContexts = 64;
struct StaticAddr {
  unsigned long long ctx_id;
  void *addr;
};
StaticAddr g_static_addr[kMaxContexts];
int g_static_n = 0;
std::mutex g_static_mu;

// The id of the calling thread's current context; if the thread has none
// yet, the current device's primary context is made current first
// (cudaSetDevice initialises it).
nys_status current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!get_ctx || !get_id) {
    void *p = nullptr, *q = nullptr;
    cudaDriverEntryPointQueryResult r1, r2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) != cudaSuccess ||
        r1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
        r2 != cudaDriverEntryPointSuccess)
      return NYS_ERR_CUDA;
    get_ctx = (CtxGetCurrentFn)p;
    get_id = (CtxGetIdFn)q;
  }
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return NYS_ERR_CUDA;
  if (!ctx) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess ||
        get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
      return NYS_ERR_CUDA;
  }
  if (get_id(ctx, id) != CUDA_SUCCESS) return NYS_ERR_CUDA;
  return NYS_OK;
}

// Device address of g_static_scratch in the current context.
nys_status static_scratch(cudaStream_t stream, void **addr) {
  unsigned long long id = 0;
  nys_status st = current_context_id(&id);
  if (st != NYS_OK) return st;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return NYS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  int slot = -1;
  for (int i = 0; i < g_static_n; ++i)
    if (g_static_addr[i].ctx_id == id) slot = i;
  if (cs == cudaStreamCaptureStatusNone || slot < 0) {
    if (cs != cudaStreamCaptureStatusNone) return NYS_ERR_CUDA;   // first call inside a capture
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return NYS_ERR_CUDA;
    if (slot < 0) {
      if (g_static_n == kMaxContexts) return NYS_ERR_UNSUPPORTED;
      slot = g_static_n++;
      g_static_addr[slot].ctx_id = id;
    }
    g_static_addr[slot].addr = p;
  }
  *addr = g_static_addr[slot].addr;
  return NYS_OK;
}
}  // namespace

NYS_ATTN_API nys_status nys_attn_forward_static(const void *Q, const void *K, const void *V,
                                                const nys_desc *desc, int m, int iters,
                                                const float *conv_w, int conv_k, void *out,
                                                nys_stream_t stream) {
  nys_status st = validate_call(Q, K, V, desc, m, iters, conv_w, conv_k, out);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) return NYS_OK;
  if (make_layout(desc, m).total > (size_t)NYS_STATIC_SCRATCH_BYTES)
    return NYS_ERR_WORKSPACE;   // the problem needs more scratch than the fixed array holds
  void *ws = nullptr;
  st = static_scratch((cudaStream_t)stream, &ws);
  if (st != NYS_OK) return st;
  // the error word and the per-head counters are cleared by forward_impl
  return forward_impl(Q, K, V, desc, m, iters, conv_w, conv_k, out, ws,
                      (size_t)NYS_STATIC_SCRATCH_BYTES, stream, nullptr, 0);
}

NYS_ATTN_API nys_status nys_attn_forward_timed(const void *Q, const void *K, const void *V,
                                               const nys_desc *desc, int m, int iters,
                                               const float *conv_w, int conv_k, void *out,
                                               void *workspace, size_t workspace_bytes,
                                               nys_stream_t stream, void *const *events,
                                               int n_events) {
  if (!events) return NYS_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return NYS_ERR_INVALID_ARG;
  return forward_impl(Q, K, V, desc, m, iters, conv_w, conv_k, out, workspace, workspace_bytes,
                      stream, events, n_events);
}

NYS_ATTN_API nys_status nys_attn_check_error(void *workspace, const nys_desc *desc, int m,
                                             nys_stream_t stream_) {
  if (!workspace) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) return NYS_OK;
  Layout L = make_layout(desc, m);
  cudaStream_t stream = (cudaStream_t)stream_;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, (char *)workspace + L.err, 4, cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return NYS_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync((char *)workspace + L.err, 0, 4, stream) != cudaSuccess)
      return NYS_ERR_CUDA;
    return (nys_status)word;
  }
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_check_error_static(const nys_desc *desc, int m,
                                                    nys_stream_t stream_) {
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) return NYS_OK;
  if (make_layout(desc, m).total > (size_t)NYS_STATIC_SCRATCH_BYTES) return NYS_ERR_WORKSPACE;
  cudaStream_t stream = (cudaStream_t)stream_;
  void *ws = nullptr;
  st = static_scratch(stream, &ws);
  if (st != NYS_OK) return st;
  return nys_attn_check_error(ws, desc, m, stream_);
}

struct HostBufLayout {
  size_t q, k, v, out, conv, ws, total;
};

static HostBufLayout host_layout(const nys_desc *desc, int m, int conv_k) {
  HostBufLayout H;
  const size_t t = (size_t)desc->batch * desc->heads * desc->seq_len * desc->head_dim *
                   elem_size(desc->dtype);
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t at = off;
    off = align256(off + b);
    return at;
  };
  H.q = take(t);
  H.k = take(t);
  H.v = take(t);
  H.out = take(t);
  H.conv = take((size_t)desc->heads * (conv_k > 0 ? conv_k : 0) * 4);
  H.ws = take(is_empty(desc) ? 0 : make_layout(desc, m).total);
  H.total = off;
  return H;
}

NYS_ATTN_API nys_status nys_attn_host_buffer_size(const nys_desc *desc, int m, int conv_k,
                                                  size_t *bytes) {
  if (!bytes) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  *bytes = host_layout(desc, m, conv_k).total;
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_forward_host(const void *Qh, const void *Kh, const void *Vh,
                                              const nys_desc *desc, int m, int iters,
                                              const float *conv_w_h, int conv_k, void *out_h,
                                              void *dbuf, size_t dbuf_bytes,
                                              nys_stream_t stream_) {
  nys_status st = validate_call(Qh, Kh, Vh, desc, m, iters, conv_w_h, conv_k, out_h);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) return NYS_OK;
  if (!dbuf) return NYS_ERR_INVALID_ARG;
  if (((uintptr_t)dbuf & 255) != 0) return NYS_ERR_INVALID_ARG;
  HostBufLayout H = host_layout(desc, m, conv_w_h ? conv_k : 0);
  if (dbuf_bytes < H.total) return NYS_ERR_WORKSPACE;
  cudaStream_t stream = (cudaStream_t)stream_;
  char *b = (char *)dbuf;
  const size_t t = (size_t)desc->batch * desc->heads * desc->seq_len * desc->head_dim *
                   elem_size(desc->dtype);
  if (cudaMemcpyAsync(b + H.q, Qh, t, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(b + H.k, Kh, t, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(b + H.v, Vh, t, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return NYS_ERR_CUDA;
  const float *cw = nullptr;
  if (conv_w_h) {
    if (cudaMemcpyAsync(b + H.conv, conv_w_h, (size_t)desc->heads * conv_k * 4,
                        cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return NYS_ERR_CUDA;
    cw = (const float *)(b + H.conv);
  }
  st = nys_attn_forward(b + H.q, b + H.k, b + H.v, desc, m, iters, cw, conv_k, b + H.out,
                        b + H.ws, H.total - H.ws, stream_);
  if (st != NYS_OK) return st;
  if (cudaMemcpyAsync(out_h, b + H.out, t, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return NYS_ERR_CUDA;
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_launch_count(const nys_desc *desc, int m, int conv_k,
                                              int *launches) {
  (void)conv_k;
  if (!launches) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  *launches = is_empty(desc) ? 0 : (desc->dtype == NYS_BF16 ? kTcLaunches : kSimtLaunches);
  return NYS_OK;
}

NYS_ATTN_API nys_status nys_attn_launch_names(const nys_desc *desc, int m, char *names,
                                              size_t names_bytes) {
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  const char *src = is_empty(desc) ? "" : (desc->dtype == NYS_BF16 ? kTcNames : kSimtNames);
  if (names) {
    if (names_bytes < strlen(src) + 1) return NYS_ERR_INVALID_ARG;
    strcpy(names, src);
  }
  return NYS_OK;
}

#if defined(NYS_TEST_HOOKS) && NYS_TEST_HOOKS
// ---------------------------------------------------------------------------
// Entry points of the test build only (not part of the product ABI):
//  nys_test_fail_launch(idx)   the launch with index idx of the next forward
//                              call is refused (see launch_smem);
//  nys_test_w_order(mode)      which block of a head forms W (see below);
//  nys_test_timeout_probe(...) one block waits on an mbarrier that nothing
//                              completes, with a limit of limit_cycles SM
//                              cycles; the bounded wait gives up, records
//                              NYS_ERR_TIMEOUT in the workspace error word and
//                              the block returns.  No copy or MMA is in flight
//                              when it gives up;
//  nys_test_hold_head_flag(on) while on, the backward's per-head kernel does
//                              not publish dY / D, so every key block's
//                              bounded flag wait (about 0.2 s) gives up and
//                              records NYS_ERR_TIMEOUT in the backward
//                              workspace's first word.
NYS_ATTN_API void nys_test_fail_launch(int idx) { g_fail_launch = idx; }

NYS_ATTN_API void nys_test_hold_head_flag(int on) { g_hold_head_flag = on != 0; }

// nys_test_w_order(mode): 1 delays every pseudoinverse block, 2 every
// Y-merging block, before it reports its W input (0: no delay), so that the
// other one forms W.
NYS_ATTN_API nys_status nys_test_w_order(int mode) {
  return cudaMemcpyToSymbol(midtc::g_test_w_order, &mode, sizeof(int)) == cudaSuccess
             ? NYS_OK
             : NYS_ERR_CUDA;
}

NYS_ATTN_API nys_status nys_test_timeout_probe(void *workspace, const nys_desc *desc, int m,
                                               long long limit_cycles, nys_stream_t stream) {
  if (!workspace || limit_cycles < 0 || limit_cycles > (1ll << 32)) return NYS_ERR_INVALID_ARG;
  nys_status st = validate_shape(desc, m);
  if (st != NYS_OK) return st;
  if (is_empty(desc)) return NYS_ERR_INVALID_ARG;
  uint32_t *err = (uint32_t *)((char *)workspace + make_layout(desc, m).err);
  return launch(timeout_probe, dim3(1), dim3(32), 0, (cudaStream_t)stream, false, err,
                limit_cycles) == cudaSuccess
             ? NYS_OK
             : NYS_ERR_CUDA;
}
#endif

#if defined(NYS_TIMELINE) && NYS_TIMELINE
// Diagnostic build only: copies up to `cap` timeline records (see trace.cuh)
// to host memory, writes how many were recorded, and clears the count when
// `reset` is set.  Synchronises the device.
NYS_ATTN_API nys_status nys_debug_timeline(void *host, size_t cap, uint32_t *count, int reset) {
  if (!count) return NYS_ERR_INVALID_ARG;
  std::vector<TraceRec> all(kTraceCap);
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(all.data(), g_trace, sizeof(TraceRec) * kTraceCap) != cudaSuccess)
    return NYS_ERR_CUDA;
  // the used slots, in slot order
  uint32_t n = 0;
  for (const TraceRec &r : all) {
    if (r.ns == 0) continue;
    if (host && n < cap) ((TraceRec *)host)[n] = r;
    ++n;
  }
  *count = n;
  if (reset) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_trace) != cudaSuccess ||
        cudaMemset(p, 0, sizeof(TraceRec) * kTraceCap) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
      return NYS_ERR_CUDA;
  }
  return NYS_OK;
}
#endif

}  // extern "C"
