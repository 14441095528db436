// Device helpers shared by the sm_100a kernels of this library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

constexpr int kBlock = 16;          // NVFP4 elements per E4M3 scale
constexpr float kE2M1Max = 6.0f;
constexpr float kE4M3Max = 448.0f;
constexpr int kMaxPartials = 1024;  // per-CTA partial amax values kept in the workspace

// Programmatic dependent launch: let the next kernel on the stream start launching, and
// wait until the previous kernel's writes are visible (no-ops without the launch attribute).
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
MOE_DEV void pdl_grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
#define MOE_PDL_PROLOGUE() \
  do {                     \
    pdl_trigger();         \
    pdl_grid_wait();       \
  } while (0)

MOE_DEV float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// E4M3 ("fn") byte -> float; exact. (Byte 0x7F is NaN in the format; never produced here.)
MOE_DEV float e4m3_to_f32(uint32_t b) {
  uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0) ? float(m) * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (b & 0x80u) ? -v : v;
}

// float (finite, >= 0) -> E4M3 byte, round to nearest even, saturating at 448.
MOE_DEV uint32_t f32_to_e4m3_sat(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Two floats -> one byte of two E2M1 codes (lo in bits 0-3, hi in bits 4-7), round to
// nearest even, saturating at 6. The sign bit of each code is taken from the input's sign
// bit, so a negative value that rounds to zero becomes code 0x8.
MOE_DEV uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
      "cvt.u32.u8 %0, q;\n\t}"
      : "=r"(r) : "f"(fabsf(lo)), "f"(fabsf(hi)));
  r |= ((__float_as_uint(lo) >> 31) << 3) | ((__float_as_uint(hi) >> 31) << 7);
  return r;
}

// Four bytes (8 E2M1 codes, element 2i in the low nibble of byte i) -> four f16x2 words,
// word i = (element 2i in the low half, element 2i+1 in the high half). Exact.
MOE_DEV void e2m1x8_to_f16x2x4(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3]) : "r"(w));
}

MOE_DEV uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// sum of the two f16 halves as float (exact for the integer-quarter sums used here)
MOE_DEV float f16x2_hsum(uint32_t v) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(v));
  return lo + hi;
}

// NVFP4 quantisation of one 16-element block with tensor scale ts (IEEE float32 steps):
//   sb = (amax/6)/ts, s = E4M3(sb), denom = E4M3value(s)*ts, q_i = E2M1(x_i/denom).
// Writes 8 code bytes (element 2i low nibble) into *codes and returns the scale byte.
MOE_DEV uint32_t quantize_block16(const float v[16], float ts, uint2* codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float sb = __fdiv_rn(__fdiv_rn(amax, kE2M1Max), ts);
  const uint32_t s = f32_to_e4m3_sat(sb);
  const float sval = e4m3_to_f32(s);
  uint32_t lo = 0, hi = 0;
  if (sval != 0.0f) {
    const float denom = __fmul_rn(sval, ts);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo |= f32x2_to_e2m1x2(__fdiv_rn(v[2 * i], denom), __fdiv_rn(v[2 * i + 1], denom)) << (8 * i);
      hi |= f32x2_to_e2m1x2(__fdiv_rn(v[8 + 2 * i], denom), __fdiv_rn(v[8 + 2 * i + 1], denom))
            << (8 * i);
    }
  }
  *codes = make_uint2(lo, hi);
  return s;
}

// h = silu(g) * u for 16 consecutive columns (g, u: float32 sums, scaled by sg and su), then
// the NVFP4 quantisation of that block of h with tensor scale 1. Returns the scale byte.
MOE_DEV uint32_t swiglu_quant16(const uint32_t (&g)[16], const uint32_t (&u)[16], float sg, float su, uint2* codes) {
  float h[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float gv = __uint_as_float(g[i]) * sg, uv = __uint_as_float(u[i]) * su;
    h[i] = __fdiv_rn(gv, 1.0f + expf(-gv)) * uv;
  }
  return quantize_block16(h, 1.0f, codes);
}

// ---------------------------------------------------------------- warp / block reductions
MOE_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

MOE_DEV double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Ordered exclusive scan of one int per thread over the whole block (blockDim <= 1024).
// `tmp` must hold 32 ints. Returns the exclusive prefix; *total gets the block sum.
MOE_DEV int block_exclusive_scan(int v, int* tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < nwarps) ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;  // inclusive prefix over warps
  }
  __syncthreads();
  const int warp_base = warp ? tmp[warp - 1] : 0;
  if (total) *total = tmp[nwarps - 1];
  __syncthreads();
  return warp_base + x - v;
}

}  // namespace moe
