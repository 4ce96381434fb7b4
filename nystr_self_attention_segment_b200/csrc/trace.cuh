// Optional device timeline of the bf16 path: with -DNYS_TIMELINE=1 (a
// separate diagnostic build of the library, never the default one) thread 0
// of a block records (global timer, SM clock, SM id, kernel / block / event)
// at the marked points, into a fixed device array read back with
// nys_debug_timeline.  Every (kernel, block, event) has its own slot, so a
// mark is one store and no atomic on a shared counter (which would add the
// latency of a contended global atomic to every marked interval).  The
// default build compiles every mark to nothing.
#pragma once

#include <stdint.h>

namespace nys {

#if defined(NYS_TIMELINE) && NYS_TIMELINE
struct TraceRec {
  uint64_t ns;        // %globaltimer (0: slot unused)
  uint64_t clk;       // clock64 of the SM
  uint32_t tag;       // kernel << 24 | event << 16 | (block & 0xffff)
  uint32_t smid;
};
// slots: kernel 1 8192 blocks x 4 events, kernels 2 and 3 512 blocks x 128
constexpr int kTraceCap = 8192 * 4 + 2 * 512 * 128;
__host__ __device__ inline int trace_slot(uint32_t kernel, uint32_t block, uint32_t event) {
  if (kernel == 1) return (block < 8192 && event < 4) ? (int)(block * 4 + event) : -1;
  if (kernel == 2 || kernel == 3)
    return (block < 512 && event < 128)
               ? (int)(8192 * 4 + (kernel - 2) * 512 * 128 + block * 128 + event)
               : -1;
  return -1;
}
__device__ TraceRec g_trace[kTraceCap];

__device__ __forceinline__ void trace_rec(uint32_t kernel, uint32_t event) {
  uint64_t ns, clk = clock64();
  uint32_t smid;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(ns));
  asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
  const uint32_t block = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  const int i = trace_slot(kernel, block, event);
  if (i >= 0)
    g_trace[i] = TraceRec{ns, clk, (kernel << 24) | (event << 16) | (block & 0xffffu), smid};
}
__device__ __forceinline__ void trace_mark(uint32_t kernel, uint32_t event) {
  if (threadIdx.x == 0) trace_rec(kernel, event);
}
// NYS_MARK: thread 0 of the block records; NYS_MARK_T: the calling thread
// records (the caller picks one thread)
#define NYS_MARK(kernel, event) ::nys::trace_mark((kernel), (event))
#define NYS_MARK_T(kernel, event) ::nys::trace_rec((kernel), (event))
#else
#define NYS_MARK(kernel, event) ((void)0)
#define NYS_MARK_T(kernel, event) ((void)0)
#endif

// kernel ids of the marks
enum : uint32_t { kTrSeg = 1, kTrMid = 2, kTrOut = 3 };

}  // namespace nys
