// Optional timeline trace of the persistent FFN kernels (compiled only with -DMOE_TRACE:
// python -m nvfp4_expert_ffn_b200.build --trace). Each CTA records events into a __device__
// array of its translation unit: record 0 = globaltimer at entry, record 1 = clock64 at entry,
// then (SM cycles since entry << 32) | event << 24 | tile. The host reads a kernel's records
// with moe_trace_fetch(kernel, ...), which also clears them. Without the flag every hook
// compiles to nothing.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

enum TraceEvent : uint32_t {
  kEvSetupDone = 1,   // barriers, TMEM and shared-memory operands ready
  kEvProdTile = 2,    // producer starts a tile (unit)
  kEvProdDone1 = 3,   // producer: the tile's inputs from other CTAs are complete
  kEvMmaFirst = 4,    // first stage of a tile landed
  kEvMmaLast = 5,     // last MMA of a tile issued
  kEvEpiStart = 6,    // accumulator ready for the epilogue
  kEvEpiEnd = 7,      // epilogue of a tile done
  kEvExit = 8,
  kEvDnFirst = 9,     // first down-projection stage of a unit landed
  kEvDnLast = 10,     // last down-projection MMA of a unit issued
  kEvDrainEnd = 11,   // epilogue finished adding a unit's down projection
  kEvProdIssue = 12,  // producer issued the copies of ring stage `tile`
  kEvMmaFull = 13,    // MMA issuer: stage `tile` landed
  kEvMmaSlot = 14,    // MMA issuer: its scale slot is free
  kEvMmaIssued = 15,  // MMA issuer: the stage's MMAs are issued
  kEvMmaCps = 16,     // MMA issuer: the stage's scale-factor copies are issued
};

constexpr int kTraceCtas = 160, kTraceCap = 254;

#ifdef MOE_TRACE
#define TC_TRACE_ARRAY(name) static __device__ unsigned long long name[kTraceCtas][kTraceCap + 2];
#define TC_TRACE_DECL __shared__ unsigned int s_trace_n; __shared__ long long s_trace_clk0;
#define TC_TRACE_BEGIN(arr)                                                         \
  do {                                                                              \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas) {                              \
      s_trace_n = 0;                                                                \
      s_trace_clk0 = clock64();                                                     \
      arr[blockIdx.x][0] = globaltimer_ns();                                        \
      arr[blockIdx.x][1] = (unsigned long long)s_trace_clk0;                        \
    }                                                                               \
  } while (0)
#define TC_TRACE_AT(arr, ev, tile)                                                              \
  do {                                                                                          \
    if (blockIdx.x < kTraceCtas) {                                                              \
      const unsigned int i_ = atomicAdd(&s_trace_n, 1u);                                        \
      if (i_ < (unsigned)kTraceCap)                                                             \
        arr[blockIdx.x][2 + i_] = ((unsigned long long)(clock64() - s_trace_clk0) << 32) |     \
                                  ((unsigned long long)(ev) << 24) | ((tile) & 0xFFFFFF);       \
    }                                                                                           \
  } while (0)

// copy a trace array to the host (at most `bytes`) and clear it; -1 on a CUDA error
template <typename A>
int64_t trace_fetch(A& arr, void* host, size_t bytes) {
  const size_t n = sizeof(arr) < bytes ? sizeof(arr) : bytes;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(host, arr, n) != cudaSuccess) return -1;
  static const unsigned long long zeros[(size_t)kTraceCtas * (kTraceCap + 2)] = {};
  static_assert(sizeof(arr) <= sizeof(zeros), "trace array larger than the zero buffer");
  if (cudaMemcpyToSymbol(arr, zeros, sizeof(arr)) != cudaSuccess) return -1;
  return (int64_t)n;
}
// short kernels: globaltimer stamps [kernel][cta][event] (event 0 = entry)
constexpr int kRtKernels = 8, kRtEvents = 8;
#define RT_TRACE_ARRAY(name) static __device__ unsigned long long name[kRtKernels][kTraceCtas][kRtEvents];
#define RT_TRACE(arr, kern, ev)                                                                   \
  do {                                                                                           \
    if (threadIdx.x == 0 && blockIdx.x < kTraceCtas) arr[kern][blockIdx.x][ev] = globaltimer_ns(); \
  } while (0)
#else
#define RT_TRACE_ARRAY(name)
#define RT_TRACE(arr, kern, ev) do { } while (0)
#define TC_TRACE_ARRAY(name)
#define TC_TRACE_DECL
#define TC_TRACE_BEGIN(arr) do { } while (0)
#define TC_TRACE_AT(arr, ev, tile) do { } while (0)
#endif

}  // namespace moe
