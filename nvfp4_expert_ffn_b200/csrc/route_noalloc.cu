// moe_route_noalloc: the routing call for callers that cannot hand the library any device
// memory to use as scratch.
//
// Who needs it: a serving process that reserves all of HBM for weights and KV cache at
// start-up and forbids later allocations, a plain C host without a device allocator of its
// own, or code that is in the middle of capturing a CUDA graph (cudaMalloc may not be called
// there). moe_route needs a workspace for the router logits; this variant keeps that
// scratch in one fixed array compiled into the library instead.
//
// The array below lives in every GPU that loads the library, for as long as the process
// runs. All calls share it: it keeps whatever the last call left there, and two calls whose
// work overlaps on the GPU (different streams, or different host threads) race on it.
// Nothing in it has to start at zero: each call overwrites the part it reads.
#include <mutex>
#include <string>

#include "../../include/moe_nvfp4.h"
#include "kernels.h"

namespace moe {

// Scratch of one call: the router logits (T*E float32, padded to 256 bytes), plus the
// permutation's per-chunk histograms when there are more than 4096 assignments (T*k).
// With at most 4096 assignments the array holds up to 65536 logits: T*E <= 65536.
constexpr size_t kNoAllocScratchBytes = 256 * 1024;

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev] = {};
std::mutex g_scratch_mu;

// Device address of g_route_scratch on the current device, looked up once per device.
// The symbol's name in host code is only a handle, never a device pointer.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_noalloc(const uint16_t* x_bf16, int32_t T, int32_t d, const float* Wr,
                                        const float* br, int32_t E, int32_t k, int32_t* topk_idx,
                                        float* topk_w, int32_t* counts, int32_t* offsets,
                                        int32_t* sorted_assign, int32_t* assign_pos, void* stream) {
  if (T < 0 || E <= 0 || k <= 0 || d <= 0) {
    // let moe_route report the precise argument problem (it validates before launching)
    return moe_route(x_bf16, T, d, Wr, br, E, k, topk_idx, topk_w, counts, offsets, sorted_assign,
                     assign_pos, nullptr, 0, stream);
  }
  const size_t need = route_ws_bytes(T, d, E, k);
  if (need > kNoAllocScratchBytes) {
    set_last_error("moe_route_noalloc: this call needs " + std::to_string(need) +
                   " bytes of scratch, more than the built-in " + std::to_string(kNoAllocScratchBytes) +
                   " (T*E too large); use moe_route with a workspace");
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    set_last_error(std::string("moe_route_noalloc: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return moe_route(x_bf16, T, d, Wr, br, E, k, topk_idx, topk_w, counts, offsets, sorted_assign,
                   assign_pos, scratch, kNoAllocScratchBytes, stream);
}
