// Optional device timeline of the bf16 path: with -DNYS_TIMELINE=1 (a
// separate diagnostic build of the library, never the default one) thread 0
// of a block records (global timer, SM clock, SM id, kernel / block / event)
// at the marked points, into a fixed device array read back with
// nys_debug_timeline.  The default build compiles every mark to nothing.
#pragma once

#include <stdint.h>

namespace nys {

#if defined(NYS_TIMELINE) && NYS_TIMELINE
constexpr int kTraceCap = 1 << 16;
struct TraceRec {
  uint64_t ns;        // %globaltimer
  uint64_t clk;       // clock64 of the SM
  uint32_t tag;       // kernel << 24 | event << 16 | (block & 0xffff)
  uint32_t smid;
};
__device__ TraceRec g_trace[kTraceCap];
__device__ uint32_t g_trace_n;

__device__ __forceinline__ void trace_rec(uint32_t kernel, uint32_t event) {
  uint64_t ns, clk = clock64();
  uint32_t smid;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(ns));
  asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
  const uint32_t i = atomicAdd(&g_trace_n, 1u);
  if (i < kTraceCap)
    g_trace[i] = TraceRec{ns, clk, (kernel << 24) | (event << 16) | (blockIdx.x & 0xffffu), smid};
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
