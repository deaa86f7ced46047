// marks.cuh — the timeline hooks of the engine's profiling build (force-included when
// engine.cu is compiled by timeline.py; the library build leaves FMOE_MARK empty).
// Records, for CTAs 0 and 77 (every CTA up to 148 with FMOE_TRACE_ALL_CTAS) and the first 64
// units of a launch, the %globaltimer time at which one role reached event `ev` of unit u (the
// last writer of a slot wins).
#include <cuda_runtime.h>
#define FMOE_TRACE_UNITS 64
#define FMOE_TRACE_EV 88
#ifdef FMOE_TRACE_ALL_CTAS
#define FMOE_TRACE_CTAS 148
__device__ __forceinline__ int fmoe_trace_cta() {
  return blockIdx.x < FMOE_TRACE_CTAS ? (int)blockIdx.x : -1;
}
#else
#define FMOE_TRACE_CTAS 2
__device__ __forceinline__ int fmoe_trace_cta() {
  return blockIdx.x == 0 ? 0 : (blockIdx.x == 77 ? 1 : -1);
}
#endif
__device__ unsigned long long g_fmoe_trace[FMOE_TRACE_CTAS][FMOE_TRACE_UNITS][FMOE_TRACE_EV];
#define FMOE_MARK(u, ev)                                                                  \
  do {                                                                                    \
    const int c_ = fmoe_trace_cta();                                                      \
    if (c_ >= 0 && (u) < FMOE_TRACE_UNITS && (threadIdx.x & 31) == 0) {                   \
      unsigned long long t_;                                                              \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                              \
      g_fmoe_trace[c_][(u)][(ev)] = t_;                                                   \
    }                                                                                     \
  } while (0)
extern "C" int fmoe_trace_read(void* host, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(host, g_fmoe_trace, bytes);
}
