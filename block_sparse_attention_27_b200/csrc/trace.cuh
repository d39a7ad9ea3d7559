// trace.cuh -- optional per-CTA phase timestamps (nanoseconds of %globaltimer).
//
// Compiled out unless the library is built with -DDSA_TRACE.  A traced build
// keeps, per translation unit, a device array of kTraceEvents stamps for each of
// the first kTraceCtas CTAs of the most recent launches, and exports
// `<fn>(void *host, size_t bytes)` / `<fn>_clear()` (see DSA_TRACE_EXPORT) to
// copy it out or zero it.  Stamps are written by the thread that reaches the
// phase; nothing else changes in the kernels.
#pragma once

#include "sm100.cuh"

namespace dsa {
constexpr int kTraceEvents = 48;
constexpr int kTraceCtas = 4096;
}  // namespace dsa

#ifdef DSA_TRACE
static __device__ unsigned long long g_dsa_trace[dsa::kTraceCtas * dsa::kTraceEvents];
#define DSA_TRACE_EVENT(ev)                                                                 \
  do {                                                                                     \
    const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (cta_ < (unsigned)::dsa::kTraceCtas)                                                \
      g_dsa_trace[cta_ * ::dsa::kTraceEvents + (ev)] = ::dsa::sm100::global_ns();          \
  } while (0)
// stamp once `val` (a loaded value) is available: the empty asm consumes it
#define DSA_TRACE_AFTER(ev, val)                         \
  do {                                                   \
    asm volatile("" ::"r"((unsigned)(val)) : "memory");  \
    DSA_TRACE_EVENT(ev);                                 \
  } while (0)
// store a raw value (a duration, a count) in the event slot instead of a timestamp
#define DSA_TRACE_VALUE(ev, v)                                                              \
  do {                                                                                     \
    const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (cta_ < (unsigned)::dsa::kTraceCtas)                                                \
      g_dsa_trace[cta_ * ::dsa::kTraceEvents + (ev)] = (unsigned long long)(v);            \
  } while (0)
#define DSA_TRACE_EXPORT(fn)                                                         \
  extern "C" int fn(void *host, size_t bytes) {                                     \
    if (bytes > sizeof(g_dsa_trace)) bytes = sizeof(g_dsa_trace);                   \
    return cudaMemcpyFromSymbol(host, g_dsa_trace, bytes) == cudaSuccess ? 0 : -1;  \
  }                                                                                 \
  extern "C" int fn##_clear(void) {                                                 \
    void *p = nullptr;                                                              \
    if (cudaGetSymbolAddress(&p, g_dsa_trace) != cudaSuccess) return -1;            \
    return cudaMemset(p, 0, sizeof(g_dsa_trace)) == cudaSuccess ? 0 : -1;           \
  }
#else
#define DSA_TRACE_EVENT(ev) \
  do {                      \
  } while (0)
#define DSA_TRACE_AFTER(ev, val) \
  do {                           \
  } while (0)
#define DSA_TRACE_VALUE(ev, v) \
  do {                         \
  } while (0)
#define DSA_TRACE_EXPORT(fn)
#endif
