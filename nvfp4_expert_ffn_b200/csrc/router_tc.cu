// Router for many tokens on the tcgen05 tensor cores, with an exact top-k.
//
// The router of the Basalt pages' MoE layer ("What Basalt changes in a Blackwell local
// inference stack", section "Experts can move without becoming free": each token selects
// a subset of experts) is read here as logits = x Wr^T + br in float32, top-k by logit with
// ties to the lower expert id, weights = softmax restricted to the top-k and renormalised.
//
// For thousands of tokens the float32 product is 2*T*E*d flops (34 GFLOP at 16384 tokens,
// d = 2048, E = 512), half a millisecond or more on the CUDA cores. Here it runs in three
// launches:
//   1. router_pack_kernel: Wr (float32) -> [Wr_hi | Wr_lo] as bf16 [E][2d], where
//      Wr_hi = bf16(Wr) and Wr_lo = bf16(Wr - Wr_hi). x is bf16, so every product x*Wr_hi
//      and x*Wr_lo is exact in float32, and Wr_hi + Wr_lo is Wr within 2^-17 relative.
//   2. router_tc_kernel: approximate logits = [x | x] . [Wr_hi | Wr_lo]^T + br, a bf16 GEMM
//      with K = 2d on tcgen05 (kind::f16, float32 accumulators in TMEM), tiles of 128 tokens
//      x 256 (or 128) experts, operands by TMA.
//   3. topk_refine_kernel, one warp per token: the k-th largest approximate logit tau; every
//      expert whose approximate logit is within 2*delta of tau gets its logit recomputed
//      exactly as the decode router does (blocked float32 sums, error ~1e-7); the top-k and
//      its weights are then taken over those exact logits (the others count as -inf).
//      As long as every approximate logit is within delta of its exact value, an expert left
//      out is below at least k candidates, so the result is the top-k of the exact logits.
//      delta = 2e-3, against an approximation error that stays near 1e-5 for these sums (the
//      product split contributes at most 2^-17 of sum |x w|, the tensor core's float32
//      accumulation the rest); the GPU tests check the approximate logits against the oracle.
//      With more than 32 candidates the warp recomputes every logit of the token exactly.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "route_core.cuh"
#include "sm100.cuh"
#include "tmap.h"

namespace moe {

constexpr int kRtM = 128;      // tokens per tile (MMA M)
constexpr int kRtBK = 64;      // bf16 elements of K per stage (one 128-byte swizzled row)
constexpr int kRtStages = 3;
constexpr int kRtThreads = 192;  // warp 0 producer, warp 1 MMA, warps 2-5 epilogue
constexpr float kRefineDelta = 2e-3f;
constexpr int kRtMinT = 256;   // below this many tokens the CUDA-core GEMM is used

struct RouterTcMaps {
  CUtensorMap x;   // [T][d] bf16, boxes of 64 x 128
  CUtensorMap w2;  // [E][2d] bf16, boxes of 64 x N
};

// ---------------------------------------------------------------- 1. pack
__global__ void __launch_bounds__(256) router_pack_kernel(const float* __restrict__ Wr, int E, int d,
                                                          uint16_t* __restrict__ w2) {
  MOE_PDL_PROLOGUE();
  const size_t n = (size_t)E * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float w = Wr[i];
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(w));
    const float r = __fsub_rn(w, bf16_to_f32(hi));  // exact: w - bf16(w) fits in float32
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(r));
    const size_t e = i / d, c = i % d;
    w2[e * 2 * d + c] = (uint16_t)hi;
    w2[e * 2 * d + d + c] = (uint16_t)lo;
  }
}

// ---------------------------------------------------------------- 2. approximate logits
__global__ void __launch_bounds__(kRtThreads, 1) router_tc_kernel(const __grid_constant__ RouterTcMaps maps, int T,
                                                                   int d, int E, int N, const float* __restrict__ br,
                                                                   float* __restrict__ logits, int32_t* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kRtStages], empty[kRtStages], acc_full;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRtM, n0 = blockIdx.y * N;
  const uint32_t a_bytes = kRtM * kRtBK * 2, b_bytes = (uint32_t)N * kRtBK * 2;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const int nks = 2 * d / kRtBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    fence_barrier_init();
    s_abort = 0;
    prefetch_tensormap(&maps.x);
    prefetch_tensormap(&maps.w2);
  }
  if (warp == 1) tmem_alloc(&s_tmem, (uint32_t)N);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  MOE_PDL_PROLOGUE();

  if (warp == 0) {
    if (lane == 0) {
      int ks = 0;
      for (; ks < nks; ++ks) {
        const int s = ks % kRtStages;
        if (!mbar_wait(&empty[s], ((ks / kRtStages) & 1) ^ 1, &s_abort, status)) break;
        uint8_t* st = smem + (size_t)s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        // K' = 2d: columns [0, d) pair x with Wr_hi, [d, 2d) pair x again with Wr_lo
        tma_load_2d(st, &maps.x, &full[s], (ks * kRtBK) % d, m0);
        tma_load_2d(st + a_bytes, &maps.w2, &full[s], ks * kRtBK, n0);
      }
      // no copy may still be landing when the CTA exits
      for (int j = ks > kRtStages ? ks - kRtStages : 0; j < ks; ++j) {
        volatile int no_abort = 0;
        mbar_wait(&full[j % kRtStages], (j / kRtStages) & 1, &no_abort, status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kRtM, N);
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks) {
        const int s = ks % kRtStages;
        if (!mbar_wait(&full[s], (ks / kRtStages) & 1, &s_abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aA = smem_u32(smem + (size_t)s * stage_bytes), aB = aA + a_bytes;
#pragma unroll
        for (int kk = 0; kk < kRtBK / 16; ++kk)
          mma_bf16(tmem, sdesc_sw128(aA + 32 * kk), sdesc_sw128(aB + 32 * kk), idesc, (ks | kk) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      // the accumulator barrier completes once every MMA issued above has (also on abort,
      // so that TMEM is released only after the tensor core is done with it)
      mma_commit(&acc_full);
      if (!ok) s_abort = 1;
    }
    __syncwarp();
  } else {
    // epilogue: TMEM lane quarter q = token rows 32q..32q+31 of the tile
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const int t = m0 + row;
    int go = 1;
    if (lane == 0) {
      volatile int no_abort = 0;
      go = mbar_wait(&acc_full, 0, &no_abort, status) ? 1 : 0;
    }
    go = __shfl_sync(0xffffffffu, go, 0) && !s_abort;
    tc_fence_after();
    if (go) {
      for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + c0, v);
        tmem_ld_wait();
        if (t < T) {
          float4* dst = reinterpret_cast<float4*>(logits + (size_t)t * E + n0 + c0);
          float b[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) b[i] = br ? __ldg(br + n0 + c0 + i) : 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]) + b[4 * i], __uint_as_float(v[4 * i + 1]) + b[4 * i + 1],
                                 __uint_as_float(v[4 * i + 2]) + b[4 * i + 2],
                                 __uint_as_float(v[4 * i + 3]) + b[4 * i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)N);
  }
}

// ---------------------------------------------------------------- 3. exact top-k
// Exact logit of expert e for token t: each lane sums its float4 columns c = lane, lane + 32,
// ... in order, then the 32 lane sums are added in a fixed tree; + the bias. The row's loads
// go out 16 at a time before their products, so a logit costs about one L2 round trip per
// 16 float4 of each lane rather than one per float4. xr: the token's bf16 row.
constexpr int kExactUnroll = 16;
MOE_DEV float exact_logit(const uint16_t* __restrict__ xr, const float* __restrict__ Wr, const float* br, int d,
                          int e) {
  const int lane = threadIdx.x & 31;
  const float4* w4 = reinterpret_cast<const float4*>(Wr + (size_t)e * d);
  const uint2* x4 = reinterpret_cast<const uint2*>(xr);
  const int nvec = d / 4;
  float acc = 0.0f;
  for (int c0 = lane; c0 < nvec; c0 += 32 * kExactUnroll) {
    float4 w[kExactUnroll];
    uint2 xv[kExactUnroll];
#pragma unroll
    for (int u = 0; u < kExactUnroll; ++u) {
      const int c = c0 + 32 * u;
      w[u] = c < nvec ? __ldg(w4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      xv[u] = c < nvec ? __ldg(x4 + c) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kExactUnroll; ++u) {
      if (c0 + 32 * u < nvec) {
        acc = fmaf(bf16_to_f32(xv[u].x & 0xFFFFu), w[u].x, acc);
        acc = fmaf(bf16_to_f32(xv[u].x >> 16), w[u].y, acc);
        acc = fmaf(bf16_to_f32(xv[u].y & 0xFFFFu), w[u].z, acc);
        acc = fmaf(bf16_to_f32(xv[u].y >> 16), w[u].w, acc);
      }
    }
  }
  return warp_sum(acc) + (br ? __ldg(br + e) : 0.0f);
}

constexpr int kRefineWarps = 8;

template <int NPER>
__global__ void __launch_bounds__(32 * kRefineWarps) topk_refine_kernel(const float* __restrict__ approx,
                                                                        const uint16_t* __restrict__ x,
                                                                        const float* __restrict__ Wr,
                                                                        const float* __restrict__ br, int T, int d,
                                                                        int E, int k, int32_t* __restrict__ topk_idx,
                                                                        float* __restrict__ topk_w) {
  __shared__ float s_row[kRefineWarps][32 * NPER];
  __shared__ int s_idx[kRefineWarps][32];
  __shared__ uint32_t s_scr[kRefineWarps][64];
  MOE_PDL_PROLOGUE();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRefineWarps + warp;
  if (t >= T) return;
  const float* arow = approx + (size_t)t * E;
  const uint16_t* xr = x + (size_t)t * d;
  float* row = s_row[warp];
  // the k-th largest approximate logit
  topk_token<NPER>(arow, E, k, nullptr, nullptr, s_idx[warp], nullptr, s_scr[warp]);
  __syncwarp();
  const float tau = arow[s_idx[warp][k - 1]];
  const float lim = tau - 2.0f * kRefineDelta;
  __syncwarp();  // every lane has read s_idx before it is reused for the candidates
  // candidates (approximate logit within 2 delta of tau, or above), listed in s_idx
  int ncand = 0;
#pragma unroll
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    const bool c = e < E && arow[e] >= lim;
    const uint32_t m = __ballot_sync(0xffffffffu, c);
    const int pos = ncand + __popc(m & ((1u << lane) - 1u));
    if (c && pos < 32) s_idx[warp][pos] = e;
    ncand += __popc(m);
  }
  __syncwarp();
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    if (e < E) row[e] = -INFINITY;
  }
  __syncwarp();
  if (ncand <= 32) {
    for (int i = 0; i < ncand; ++i) {
      const int e = s_idx[warp][i];
      const float v = exact_logit(xr, Wr, br, d, e);
      if (lane == 0) row[e] = v;
    }
  } else {
    // too many near-equal approximate logits: every logit of this token exactly
    for (int e = 0; e < E; ++e) {
      const float v = exact_logit(xr, Wr, br, d, e);
      if (lane == 0) row[e] = v;
    }
  }
  __syncwarp();
  topk_token<NPER>(row, E, k, topk_idx + (size_t)t * k, topk_w + (size_t)t * k, nullptr, nullptr, s_scr[warp]);
}

// ---------------------------------------------------------------- host side
bool router_tc_supported(int64_t T, int d, int E) {
  return T >= kRtMinT && d % kRtBK == 0 && E % 128 == 0 && E <= 1024 && d <= 8192;
}

size_t router_tc_ws_bytes(int d, int E) { return ((size_t)E * 2 * d * sizeof(uint16_t) + 255) & ~(size_t)255; }

static size_t router_tc_smem_bytes(int N) { return (size_t)kRtStages * (kRtM + N) * kRtBK * 2 + 1024; }

cudaError_t set_wait_limit_router_tc(unsigned long long ns) { return set_wait_limit_here(ns); }

cudaError_t init_router_tc_attributes() {
  return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)router_tc_smem_bytes(256));
}

cudaError_t launch_router_tc(const uint16_t* x, int T, int d, const float* Wr, const float* br, int E, int k,
                             int32_t* topk_idx, float* topk_w, float* logits, uint16_t* w2, int num_sms,
                             int32_t* status, cudaStream_t st) {
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  const int N = E % 256 == 0 ? 256 : 128;
  RouterTcMaps maps;
  {
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {(cuuint32_t)kRtBK, (cuuint32_t)kRtM};
    if ((e = encode_u16(&maps.x, x, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)(2 * d), (cuuint64_t)E};
    cuuint64_t strides[1] = {(cuuint64_t)d * 4};
    cuuint32_t box[2] = {(cuuint32_t)kRtBK, (cuuint32_t)N};
    if ((e = encode_u16(&maps.w2, w2, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
  if ((e = launch_pdl(router_pack_kernel, dim3(num_sms * 4), dim3(256), 0, st, Wr, E, d, w2)) != cudaSuccess)
    return e;
  if ((e = launch_pdl(router_tc_kernel, dim3((T + kRtM - 1) / kRtM, E / N), dim3(kRtThreads),
                      router_tc_smem_bytes(N), st, maps, T, d, E, N, br, logits, status)) != cudaSuccess)
    return e;
  const dim3 grid((T + kRefineWarps - 1) / kRefineWarps);
  const dim3 block(32 * kRefineWarps);
  if (E <= 256)
    return launch_pdl(topk_refine_kernel<8>, grid, block, 0, st, (const float*)logits, x, Wr, br, T, d, E, k,
                      topk_idx, topk_w);
  if (E <= 512)
    return launch_pdl(topk_refine_kernel<16>, grid, block, 0, st, (const float*)logits, x, Wr, br, T, d, E, k,
                      topk_idx, topk_w);
  return launch_pdl(topk_refine_kernel<32>, grid, block, 0, st, (const float*)logits, x, Wr, br, T, d, E, k,
                    topk_idx, topk_w);
}

}  // namespace moe
