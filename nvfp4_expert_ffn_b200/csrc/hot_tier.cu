// The hot tier of an expert group: a compact copy of the most-routed experts' decode-pack
// units, which the one-kernel decode layer reads instead of the decode pack and marks as
// persisting in L2 for its launch.
//
// "Basalt" project page, section "Expert tiers": the busiest experts are kept in the
// fastest memory, and the tiers follow the conversation as it shifts. On one B200 every
// expert is in HBM and the fastest level is the 126 MB L2, which an access-policy window
// can keep a range of addresses in; the experts' decode packs are spread over the whole
// group, so the hot experts are first copied into one range. The ranking comes from the
// cumulative histogram (moe_expert_hist), most routed first.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Block 0 rewrites the slot map (-1, then slot i for expert rank[i]); every block copies its
// share of the hot experts' units, 16 bytes at a time (a unit's bytes are contiguous, and so
// are an expert's units). Ranks outside [0, E) are skipped: their slots keep -1 and their
// copies are not made.
__global__ void __launch_bounds__(512) hot_tier_kernel(const uint8_t* __restrict__ dec_pack,
                                                       const int32_t* __restrict__ rank, int E, int n_hot,
                                                       size_t expert_bytes, uint8_t* __restrict__ hot_pack,
                                                       int32_t* __restrict__ hot_slot) {
  MOE_PDL_PROLOGUE();
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) hot_slot[e] = -1;
    __syncthreads();
    for (int i = threadIdx.x; i < n_hot; i += blockDim.x) {
      const int r = rank[i];
      if (r >= 0 && r < E) hot_slot[r] = i;
    }
  }
  const size_t per = expert_bytes / 16;  // 16-byte pieces of one expert
  const size_t n = (size_t)n_hot * per;
  const uint4* src = reinterpret_cast<const uint4*>(dec_pack);
  uint4* dst = reinterpret_cast<uint4*>(hot_pack);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t slot = i / per, off = i % per;
    const int r = rank[slot];
    if (r >= 0 && r < E) dst[i] = __ldcs(src + (size_t)r * per + off);
  }
}

cudaError_t launch_hot_tier(const uint8_t* dec_pack, const int32_t* rank, int E, int d, int I, int n_hot,
                            uint8_t* hot_pack, int32_t* hot_slot, int num_sms, cudaStream_t st) {
  const size_t expert_bytes = dec_pack_bytes(1, d, I);
  return launch_pdl(hot_tier_kernel, dim3(num_sms), dim3(512), 0, st, dec_pack, rank, E, n_hot, expert_bytes,
                    hot_pack, hot_slot);
}

}  // namespace moe
