// State shared by every kernel of the library.
#pragma once
#include <cstddef>
#include <cstdint>

namespace attn {

// Device-side error word: 0, or the OR of (site << 8) | kind over the bounded waits that ran out (kind 1) and, in
// the debug build, the address checks that failed (kind 2). Read and cleared through attn_get_device_error /
// attn_clear_device_error.
__device__ uint32_t g_device_error;

// Sites of the debug build's address checks (the bits above the kind).
enum : uint32_t {
  kSiteChkPrepIn = 0x81, kSiteChkPrepAcc = 0x82, kSiteChkPrepRow = 0x83, kSiteChkPrepLse = 0x84,
  kSiteChkDqIn = 0x85, kSiteChkDqOut = 0x86, kSiteChkBwdRows = 0x87, kSiteChkBwdReduce = 0x88,
  kSiteChkFwdLse = 0x89, kSiteChkDecQ = 0x8a, kSiteChkDecPart = 0x8d,
  kSiteChkDecComb = 0x8e, kSiteChkDecO = 0x8f, kSiteChkDecLse = 0x90, kSiteChkSelftest = 0x7e
};

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
