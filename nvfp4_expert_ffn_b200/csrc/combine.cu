// Weighted combine of expert outputs and cast to bf16 (last step of the MoE layer).
//
// Basalt pages: "What Basalt changes in a Blackwell local inference stack", section
// "Experts can move without becoming free" (a token's output comes from its selected
// experts). Reading: y[t] = sum_j w[t,j] * o[t,j] + o_shared[t] (shared expert ungated,
// weight 1). One CTA per token row; HBM-bound (reads k float32 rows, writes one bf16 row).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

MOE_DEV uint32_t f32_to_bf16_bits(float v) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <int MODE>
MOE_DEV float combine_value(int t, int n, int d, int k, const float* __restrict__ eo,
                            const float* __restrict__ so, const float* __restrict__ w,
                            const int32_t* __restrict__ pos) {
  if (MODE == 0) return eo[(size_t)t * d + n];
  float acc = so ? so[(size_t)t * d + n] : 0.0f;
  for (int j = 0; j < k; ++j) {
    const int a = t * k + j;
    acc = fmaf(w[a], eo[(size_t)pos[a] * d + n], acc);
  }
  return acc;
}

template <int MODE>
__global__ void __launch_bounds__(256) combine_kernel(int T, int d, int k, const float* __restrict__ eo,
                                                      const float* __restrict__ so,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ pos, int rms,
                                                      uint16_t* __restrict__ y) {
  MOE_PDL_PROLOGUE();
  const int t = blockIdx.x;
  float scale = 1.0f;
  if (rms) {
    float ss = 0.0f;
    for (int n = threadIdx.x; n < d; n += blockDim.x) {
      const float v = combine_value<MODE>(t, n, d, k, eo, so, w, pos);
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    __shared__ float red[32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
      float v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
      v = warp_sum(v);
      if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float ms = red[0] / (float)d;
    scale = ms > 0.0f ? rsqrtf(ms) : 0.0f;
  }
  for (int n2 = threadIdx.x; n2 < d / 2; n2 += blockDim.x) {
    const float v0 = combine_value<MODE>(t, 2 * n2, d, k, eo, so, w, pos) * scale;
    const float v1 = combine_value<MODE>(t, 2 * n2 + 1, d, k, eo, so, w, pos) * scale;
    reinterpret_cast<uint32_t*>(y + (size_t)t * d)[n2] = f32_to_bf16_bits(v0) | (f32_to_bf16_bits(v1) << 16);
  }
}

cudaError_t launch_combine(int T, int d, int k, int mode, const float* eo, const float* so,
                           const float* w, const int32_t* pos, int rms, uint16_t* y,
                           cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (mode == 0)
    return launch_pdl(combine_kernel<0>, dim3(T), dim3(256), 0, st, T, d, k, eo, so, w, pos, rms, y);
  else
    return launch_pdl(combine_kernel<1>, dim3(T), dim3(256), 0, st, T, d, k, eo, so, w, pos, rms, y);
}

}  // namespace moe
