// NVFP4 quantisation of bf16 matrices (activation quantisation step of the MoE layer).
//
// Format reading (the Basalt pages name NVFP4 but do not define it; "Basalt" project page,
// "All the numbers", "Engines: commit, and what is not NVIDIA's weights"): E2M1 codes, one
// E4M3 scale per 16 elements, float32 tensor scale ts = amax/(6*448) unless a static scale
// (the pages' input_scale) is given. Two passes over x: a grid-wide amax, then one thread
// per 16-element block. Both are bound by HBM bandwidth: 2 bytes read per element in the
// amax pass, 2 read + 0.5625 written in the quantise pass.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// max |x| of bf16 values as the integer maximum of their magnitude bits
MOE_DEV uint32_t bf16x2_absmax(uint32_t m, uint32_t w) { return __vmaxu2(m, w & 0x7FFF7FFFu); }

__global__ void __launch_bounds__(256) amax_partial_kernel(const uint4* __restrict__ x, int64_t nvec,
                                                           float* __restrict__ partials) {
  MOE_PDL_PROLOGUE();
  uint32_t m = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nvec;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint4 v = __ldg(x + i);
    m = bf16x2_absmax(m, v.x);
    m = bf16x2_absmax(m, v.y);
    m = bf16x2_absmax(m, v.z);
    m = bf16x2_absmax(m, v.w);
  }
  float f = fmaxf(bf16_to_f32(m & 0xFFFFu), bf16_to_f32(m >> 16));
  f = warp_max(f);
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = f;
  __syncthreads();
  if (threadIdx.x < 32) {
    float g = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
    g = warp_max(g);
    if (threadIdx.x == 0) partials[blockIdx.x] = g;
  }
}

// Tensor scale from the partial maxima (or the static scale), computed by one warp.
MOE_DEV float resolve_ts(const float* ts_in, const float* partials, int npart) {
  if (ts_in) return *ts_in;
  float m = 0.0f;
  for (int i = threadIdx.x & 31; i < npart; i += 32) m = fmaxf(m, partials[i]);
  m = warp_max(m);
  return m > 0.0f ? __fdiv_rn(m, kE2M1Max * kE4M3Max) : 1.0f;
}

// One thread per 16-element block; block index b covers x[b*16 .. b*16+15] of the
// row-major matrix (cols % 16 == 0, so blocks never straddle rows).
__global__ void __launch_bounds__(256) quant_blocks_kernel(const uint4* __restrict__ x, int64_t nblk,
                                                           const float* __restrict__ ts_in,
                                                           const float* __restrict__ partials,
                                                           int npart, uint2* __restrict__ codes,
                                                           uint8_t* __restrict__ scales,
                                                           float* __restrict__ ts_out) {
  MOE_PDL_PROLOGUE();
  __shared__ float s_ts;
  if (threadIdx.x < 32) {
    float ts = resolve_ts(ts_in, partials, npart);
    if (threadIdx.x == 0) s_ts = ts;
  }
  __syncthreads();
  const float ts = s_ts;
  if (blockIdx.x == 0 && threadIdx.x == 0 && ts_out) *ts_out = ts;
  for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblk;
       b += (int64_t)gridDim.x * blockDim.x) {
    uint4 p0 = __ldg(x + 2 * b), p1 = __ldg(x + 2 * b + 1);
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_to_f32(w[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_to_f32(w[i] >> 16);
    }
    uint2 c;
    scales[b] = (uint8_t)quantize_block16(v, ts, &c);
    codes[b] = c;
  }
}

// Small inputs: one CTA computes the amax and quantises (saves a launch on the decode path).
__global__ void __launch_bounds__(1024) quant_small_kernel(const uint4* __restrict__ x, int64_t nblk,
                                                           const float* __restrict__ ts_in,
                                                           uint2* __restrict__ codes,
                                                           uint8_t* __restrict__ scales,
                                                           float* __restrict__ ts_out) {
  MOE_PDL_PROLOGUE();
  __shared__ float red[32];
  __shared__ float s_ts;
  if (!ts_in) {
    uint32_t m = 0;
    for (int64_t i = threadIdx.x; i < 2 * nblk; i += blockDim.x) {
      uint4 v = __ldg(x + i);
      m = bf16x2_absmax(m, v.x);
      m = bf16x2_absmax(m, v.y);
      m = bf16x2_absmax(m, v.z);
      m = bf16x2_absmax(m, v.w);
    }
    float f = warp_max(fmaxf(bf16_to_f32(m & 0xFFFFu), bf16_to_f32(m >> 16)));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = f;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float ts = resolve_ts(ts_in, red, ts_in ? 0 : (int)(blockDim.x >> 5));
    if (threadIdx.x == 0) {
      s_ts = ts;
      if (ts_out) *ts_out = ts;
    }
  }
  __syncthreads();
  const float ts = s_ts;
  for (int64_t b = threadIdx.x; b < nblk; b += blockDim.x) {
    uint4 p0 = __ldg(x + 2 * b), p1 = __ldg(x + 2 * b + 1);
    const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_to_f32(w[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_to_f32(w[i] >> 16);
    }
    uint2 c;
    scales[b] = (uint8_t)quantize_block16(v, ts, &c);
    codes[b] = c;
  }
}

__global__ void write_ts_kernel(const float* ts_in, float* ts_out) {
  MOE_PDL_PROLOGUE();
  if (threadIdx.x == 0 && ts_out) *ts_out = ts_in ? *ts_in : 1.0f;
}

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int cols, const float* ts_in,
                            uint8_t* codes, uint8_t* scales, float* ts_out, void* ws,
                            int num_sms, cudaStream_t st) {
  const int64_t nblk = rows * (int64_t)(cols / kBlock);
  if (nblk == 0) {
    return launch_pdl(write_ts_kernel, dim3(1), dim3(32), 0, st, ts_in, ts_out);
  }
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  if (nblk <= 4096) {
    return launch_pdl(quant_small_kernel, dim3(1), dim3(1024), 0, st, xv, nblk, ts_in,
                      reinterpret_cast<uint2*>(codes), scales, ts_out);
  }
  float* partials = reinterpret_cast<float*>(ws);
  int npart = 0;
  if (!ts_in) {
    const int64_t nvec = nblk * 2;
    int64_t want = (nvec + 255) / 256;
    npart = (int)(want < (int64_t)num_sms * 4 ? want : (int64_t)num_sms * 4);
    if (npart > kMaxPartials) npart = kMaxPartials;
    cudaError_t e = launch_pdl(amax_partial_kernel, dim3(npart), dim3(256), 0, st, xv, nvec, partials);
    if (e != cudaSuccess) return e;
  }
  int64_t want = (nblk + 255) / 256;
  int grid = (int)(want < (int64_t)num_sms * 8 ? want : (int64_t)num_sms * 8);
  return launch_pdl(quant_blocks_kernel, dim3(grid), dim3(256), 0, st, xv, nblk, ts_in,
                    (const float*)partials, npart, reinterpret_cast<uint2*>(codes), scales, ts_out);
}

}  // namespace moe
