// State shared by every kernel of the library.
#pragma once
#include <cstddef>
#include <cstdint>

namespace attn {

// Device-side error word: 0, or (site << 8) | kind for the first bounded wait that ran out. Read and cleared
// through attn_get_device_error / attn_clear_device_error.
__device__ uint32_t g_device_error;

// Pipeline tracing, compiled in only with -DATTN_TRACE (a profiling build; the library never defines it):
// the first kTraceCtas CTAs of a launch record SM clock64 stamps of pipeline events into g_trace, read back
// by attn_trace_dump.
#ifdef ATTN_TRACE
constexpr int kTraceCtas = 64, kTraceEvents = 16, kTraceSlots = 64;
constexpr size_t kTraceBytes = sizeof(unsigned long long) * kTraceCtas * kTraceEvents * kTraceSlots;
__device__ unsigned long long g_trace[kTraceCtas][kTraceEvents][kTraceSlots];
#define ATTN_TRACE_EVENT(ev, slot)                                                              \
  do {                                                                                          \
    if (blockIdx.x < ::attn::kTraceCtas && (slot) < ::attn::kTraceSlots)                        \
      ::attn::g_trace[blockIdx.x][(ev)][(slot)] = static_cast<unsigned long long>(clock64());   \
  } while (0)
#else
#define ATTN_TRACE_EVENT(ev, slot) \
  do {                             \
  } while (0)
#endif

}  // namespace attn
