// Router (logits), softmax/top-k/renormalisation, token permutation and expert histogram.
//
// Basalt pages: "What Basalt changes in a Blackwell local inference stack", section
// "Experts can move without becoming free" (each token selects a subset of experts) and
// the "Basalt" project page, section "Expert tiers" (the most routed experts are the hot
// ones). Reading used here: logits = x Wr^T + br in float32, top-k by logit with ties to
// the lower expert id, weights = softmax restricted to the top-k and renormalised; the
// permutation is a stable counting sort of assignments a = t*k + j by expert.
//
// Precision: a float32 sum of d = 2048 products accumulated in one running total carries
// ~1e-6 of rounding error, the size of the top-k tie margin. Sums are therefore blocked:
// the decode GEMV adds 64 products per lane and then reduces the 32 lane sums in a tree;
// the prefill GEMM sums 32 products per K tile and folds the tile sums into a compensated
// (Kahan) total. Both leave ~1e-7 of error. Float64 arithmetic is avoided on purpose: the
// B200 CUDA cores run it at a small fraction of the float32 rate.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "route_core.cuh"
#include "trace.cuh"

namespace moe {

// ---------------------------------------------------------------- router GEMV (T <= 8)
// x (T x d bf16) is staged in shared memory; each warp owns expert rows of Wr and keeps
// 16 float4 loads per lane in flight (a full 8 KB row at d = 2048) before using them.
RT_TRACE_ARRAY(g_route_trace)

constexpr int kGemvMaxT = 8;
constexpr int kGemvUnroll = 16;

__global__ void __launch_bounds__(256) router_gemv_kernel(const uint16_t* __restrict__ x, int T, int d,
                                                          const float* __restrict__ Wr,
                                                          const float* __restrict__ br, int E,
                                                          float* __restrict__ logits) {
  RT_TRACE(g_route_trace, 0, 0);
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_route_trace, 0, 1);
  extern __shared__ __align__(16) uint16_t xs[];  // [T][d]
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int nvec = d / 4;
  int e = blockIdx.x * warps + (threadIdx.x >> 5);
  // first row's weights in flight while x is staged
  float4 w[kGemvUnroll];
  auto load_w = [&](int row, int c0) {
    const float4* w4 = reinterpret_cast<const float4*>(Wr + (size_t)row * d);
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int c = c0 + 32 * u;
      w[u] = c < nvec ? __ldg(w4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  if (e < E) load_w(e, lane);
  // stage x with every load of a round in flight before the stores (one round trip per 8)
  const int nx = T * d / 8;
  for (int i0 = threadIdx.x; i0 < nx; i0 += 8 * blockDim.x) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < nx) v[u] = __ldg(reinterpret_cast<const uint4*>(x) + i);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < nx) reinterpret_cast<uint4*>(xs)[i] = v[u];
    }
  }
  __syncthreads();
  RT_TRACE(g_route_trace, 0, 2);
  for (; e < E; e += gridDim.x * warps) {
    float acc[kGemvMaxT];
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) acc[t] = 0.0f;
    for (int c0 = lane; c0 < nvec; c0 += 32 * kGemvUnroll) {
      if (c0 != lane) load_w(e, c0);
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        const int c = c0 + 32 * u;
        if (c < nvec) {
#pragma unroll
          for (int t = 0; t < kGemvMaxT; ++t) {
            if (t < T) {
              const uint2 xv = *reinterpret_cast<const uint2*>(xs + t * d + 4 * c);
              acc[t] = fmaf(bf16_to_f32(xv.x & 0xFFFFu), w[u].x, acc[t]);
              acc[t] = fmaf(bf16_to_f32(xv.x >> 16), w[u].y, acc[t]);
              acc[t] = fmaf(bf16_to_f32(xv.y & 0xFFFFu), w[u].z, acc[t]);
              acc[t] = fmaf(bf16_to_f32(xv.y >> 16), w[u].w, acc[t]);
            }
          }
        }
      }
    }
    const float b = br ? __ldg(br + e) : 0.0f;
#pragma unroll
    for (int t = 0; t < kGemvMaxT; ++t) {
      if (t < T) {
        const float s = warp_sum(acc[t]);
        if (lane == 0) logits[(size_t)t * E + e] = s + b;
      }
    }
    const int en = e + gridDim.x * warps;
    if (en < E) load_w(en, lane);
  }
  RT_TRACE(g_route_trace, 0, 3);
}

// ---------------------------------------------------------------- router GEMM (large T)
// 64 tokens x 64 experts per CTA, 256 threads with 4x4 outputs each, K tiles of 32.
constexpr int kRgBM = 64, kRgBN = 64, kRgBK = 32;

__global__ void __launch_bounds__(256) router_gemm_kernel(const uint16_t* __restrict__ x, int T, int d,
                                                          const float* __restrict__ Wr,
                                                          const float* __restrict__ br, int E,
                                                          float* __restrict__ logits) {
  MOE_PDL_PROLOGUE();
  __shared__ float xs[kRgBK][kRgBM + 4];
  __shared__ float ws[kRgBK][kRgBN + 4];
  const int m0 = blockIdx.y * kRgBM, n0 = blockIdx.x * kRgBN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float tot[4][4], cmp[4][4], acc[4][4];  // compensated total, its error term, tile sum
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[i][j] = 0.0f, cmp[i][j] = 0.0f, acc[i][j] = 0.0f;
  for (int k0 = 0; k0 < d; k0 += kRgBK) {
    // x tile: 64 rows x 32 cols bf16 = 256 x 8 elements
    {
      const int r = threadIdx.x >> 2, c8 = (threadIdx.x & 3) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m0 + r < T && k0 + c8 < d) v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(m0 + r) * d + k0 + c8));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xs[c8 + 2 * i][r] = bf16_to_f32(w[i] & 0xFFFFu);
        xs[c8 + 2 * i + 1][r] = bf16_to_f32(w[i] >> 16);
      }
    }
    // W tile: 64 rows x 32 cols fp32 = 256 x 8 elements
    {
      const int r = threadIdx.x >> 2, c8 = (threadIdx.x & 3) * 8;
      float4 a = make_float4(0, 0, 0, 0), b = a;
      if (n0 + r < E && k0 + c8 < d) {
        const float4* p = reinterpret_cast<const float4*>(Wr + (size_t)(n0 + r) * d + k0 + c8);
        a = __ldg(p);
        b = __ldg(p + 1);
      }
      ws[c8 + 0][r] = a.x; ws[c8 + 1][r] = a.y; ws[c8 + 2][r] = a.z; ws[c8 + 3][r] = a.w;
      ws[c8 + 4][r] = b.x; ws[c8 + 5][r] = b.y; ws[c8 + 6][r] = b.z; ws[c8 + 7][r] = b.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRgBK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float y = __fsub_rn(acc[i][j], cmp[i][j]);
        const float t = __fadd_rn(tot[i][j], y);
        cmp[i][j] = __fsub_rn(__fsub_rn(t, tot[i][j]), y);
        tot[i][j] = t;
        acc[i][j] = 0.0f;
      }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < E) logits[(size_t)m * E + n] = __fsub_rn(tot[i][j], cmp[i][j]) + (br ? br[n] : 0.0f);
    }
  }
}

// ---------------------------------------------------------------- top-k + weights
// (topk_token / topk_dispatch in route_core.cuh)
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                   int32_t* __restrict__ topk_idx,
                                                   float* __restrict__ topk_w) {
  __shared__ uint32_t scratch[8][64];
  MOE_PDL_PROLOGUE();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_dispatch(logits + (size_t)t * E, E, k, topk_idx + (size_t)t * k, topk_w + (size_t)t * k, nullptr, nullptr,
                scratch[threadIdx.x >> 5]);
}

// ---------------------------------------------------------------- permutation
// Stable counting sort of n = T*k assignments by expert. Chunk c covers assignments
// [c*kPermChunk, (c+1)*kPermChunk). Pass 1: per-chunk histograms (warp-aggregated shared
// atomics). Pass 2: counts, offsets and each chunk's base per expert. Pass 3: each chunk
// assigns positions in assignment order (warps in turn, lanes ranked with match_any).
constexpr int kPermChunk = 4096;
constexpr int kPermThreads = 512;

MOE_DEV void warp_aggregated_add(int* hist, int e) {
  const uint32_t peers = __match_any_sync(__activemask(), e);
  const int leader = __ffs(peers) - 1;
  if ((threadIdx.x & 31) == leader) atomicAdd(hist + e, __popc(peers));
}

MOE_DEV void chunk_histogram(const int32_t* idx, int n, int c, int E, int* sh) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int beg = c * kPermChunk, end = min(n, beg + kPermChunk);
  for (int a = beg + threadIdx.x; a < end; a += blockDim.x) warp_aggregated_add(sh, idx[a]);
  __syncthreads();
}

// Positions for chunk c given run[e] = first free position of expert e for this chunk.
MOE_DEV void chunk_scatter(const int32_t* idx, int n, int c, int* run, int32_t* sorted_assign,
                           int32_t* assign_pos) {
  const int beg = c * kPermChunk, end = min(n, beg + kPermChunk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = beg; base < end; base += blockDim.x) {
    const int a = base + threadIdx.x;
    const bool valid = a < end;
    const int e = valid ? idx[a] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const bool last = (peers >> lane) == 1u;  // highest lane of its group
    for (int w = 0; w < nw; ++w) {
      if (warp == w && valid) {
        const int p = run[e] + rank;
        sorted_assign[p] = a;
        assign_pos[a] = p;
      }
      __syncthreads();
      if (warp == w && valid && last) run[e] += __popc(peers);
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(const int32_t* __restrict__ idx, int n,
                                                                 int E, int32_t* __restrict__ chunk_hist) {
  MOE_PDL_PROLOGUE();
  extern __shared__ int sh[];
  chunk_histogram(idx, n, blockIdx.x, E, sh);
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)blockIdx.x * E + e] = sh[e];
}

// One CTA: counts, offsets, and chunk_hist[c][e] := base position of chunk c for expert e.
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ chunk_hist, int nchunk,
                                                         int E, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets) {
  MOE_PDL_PROLOGUE();
  __shared__ int tmp[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int run = 0;
    if (e < E) {
      for (int c = 0; c < nchunk; ++c) {
        const int h = chunk_hist[(size_t)c * E + e];
        chunk_hist[(size_t)c * E + e] = run;
        run += h;
      }
    }
    int total;
    const int excl = block_exclusive_scan(run, tmp, &total) + carry;
    if (e < E) {
      counts[e] = run;
      offsets[e] = excl;
      for (int c = 0; c < nchunk; ++c) chunk_hist[(size_t)c * E + e] += excl;
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) offsets[E] = carry;
}

__global__ void __launch_bounds__(kPermThreads) perm_scatter_kernel(const int32_t* __restrict__ idx, int n,
                                                                    int E,
                                                                    const int32_t* __restrict__ chunk_base,
                                                                    int32_t* __restrict__ sorted_assign,
                                                                    int32_t* __restrict__ assign_pos) {
  MOE_PDL_PROLOGUE();
  extern __shared__ int run[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = chunk_base[(size_t)blockIdx.x * E + e];
  __syncthreads();
  chunk_scatter(idx, n, blockIdx.x, run, sorted_assign, assign_pos);
}

// Single CTA for n <= kPermChunk: histogram, scan and scatter in one launch.
__global__ void __launch_bounds__(kPermThreads) perm_small_kernel(const int32_t* __restrict__ idx, int n,
                                                                  int E, int32_t* __restrict__ counts,
                                                                  int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ sorted_assign,
                                                                  int32_t* __restrict__ assign_pos) {
  MOE_PDL_PROLOGUE();
  extern __shared__ int sh[];  // [E]
  __shared__ int tmp[32];
  __shared__ int carry;
  chunk_histogram(idx, n, 0, E, sh);
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int h = e < E ? sh[e] : 0;
    int total;
    const int excl = block_exclusive_scan(h, tmp, &total) + carry;
    if (e < E) {
      counts[e] = h;
      offsets[e] = excl;
      sh[e] = excl;
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) offsets[E] = carry;
  __syncthreads();
  chunk_scatter(idx, n, 0, sh, sorted_assign, assign_pos);
}

// Decode-sized calls (T <= 32 tokens, T*k <= 4096): top-k of every token (one warp each)
// and the whole permutation in one CTA.
__global__ void __launch_bounds__(1024) topk_perm_small_kernel(const float* __restrict__ logits, int T,
                                                               int E, int k, int32_t* __restrict__ topk_idx,
                                                               float* __restrict__ topk_w,
                                                               int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ sorted_assign,
                                                               int32_t* __restrict__ assign_pos) {
  RT_TRACE(g_route_trace, 1, 0);
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_route_trace, 1, 1);
  extern __shared__ int sh[];  // [E] counts / running positions, then [T*k] chosen experts
  int* sidx = sh + E;
  const int warp = threadIdx.x >> 5;
  if (warp < T)
    topk_dispatch(logits + (size_t)warp * E, E, k, topk_idx + (size_t)warp * k, topk_w + (size_t)warp * k,
                  sidx + warp * k);
  __syncthreads();
  RT_TRACE(g_route_trace, 1, 2);
  if (warp != 0) return;
  perm_small_warp(sidx, T * k, E, sh, counts, offsets, sorted_assign, assign_pos);
  RT_TRACE(g_route_trace, 1, 3);
}

__global__ void zero_counts_kernel(int E, int32_t* counts, int32_t* offsets) {
  MOE_PDL_PROLOGUE();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    if (e < E) counts[e] = 0;
    offsets[e] = 0;
  }
}

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_assign, int32_t* assign_pos,
                           void* ws, cudaStream_t st) {
  const int n = T * k;
  if (n == 0) {
    return launch_pdl(zero_counts_kernel, dim3(1), dim3(1024), 0, st, E, counts, offsets);
  }
  const size_t smem = (size_t)E * sizeof(int);
  if (n <= kPermChunk) {
    return launch_pdl(perm_small_kernel, dim3(1), dim3(kPermThreads), smem, st, idx, n, E, counts, offsets,
                      sorted_assign, assign_pos);
  }
  const int nchunk = (n + kPermChunk - 1) / kPermChunk;
  int32_t* chunk_hist = reinterpret_cast<int32_t*>(ws);
  cudaError_t e = launch_pdl(perm_hist_kernel, dim3(nchunk), dim3(kPermThreads), smem, st, idx, n, E, chunk_hist);
  if (e != cudaSuccess) return e;
  e = launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), 0, st, chunk_hist, nchunk, E, counts, offsets);
  if (e != cudaSuccess) return e;
  return launch_pdl(perm_scatter_kernel, dim3(nchunk), dim3(kPermThreads), smem, st, idx, n, E,
                    (const int32_t*)chunk_hist, sorted_assign, assign_pos);
}

// Per-chunk histograms of the three-kernel permutation; the single-CTA permutation of at
// most kPermChunk assignments keeps its histogram in shared memory and needs none.
size_t permute_ws_bytes(int64_t T, int k, int E) {
  const int64_t n = T * k;
  if (n <= kPermChunk) return 0;
  const int64_t nchunk = (n + kPermChunk - 1) / kPermChunk;
  return (size_t)(nchunk * E * sizeof(int32_t));
}

// Workspace: the router logits [T][E] float32; with the tensor-core router the bf16 split
// of Wr [E][2d]; then the permutation's chunk histograms.
size_t route_ws_bytes(int64_t T, int d, int E, int k) {
  const size_t logits = ((size_t)T * E * sizeof(float) + 255) & ~(size_t)255;
  const size_t w2 = router_tc_supported(T, d, E) ? router_tc_ws_bytes(d, E) : 0;
  return logits + w2 + permute_ws_bytes(T, k, E);
}

cudaError_t launch_route(const uint16_t* x, int T, int d, const float* Wr, const float* br,
                         int E, int k, int32_t* topk_idx, float* topk_w, int32_t* counts,
                         int32_t* offsets, int32_t* sorted_assign, int32_t* assign_pos, void* ws,
                         int num_sms, int32_t* status, cudaStream_t st) {
  if (T == 0) return launch_permute(nullptr, 0, k, E, counts, offsets, sorted_assign, assign_pos,
                                    nullptr, st);
  float* logits = reinterpret_cast<float*>(ws);
  const size_t logits_bytes = ((size_t)T * E * sizeof(float) + 255) & ~(size_t)255;
  if (router_tc_supported(T, d, E)) {
    uint16_t* w2 = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(ws) + logits_bytes);
    void* perm_ws = reinterpret_cast<char*>(ws) + logits_bytes + router_tc_ws_bytes(d, E);
    cudaError_t e0 = launch_router_tc(x, T, d, Wr, br, E, k, topk_idx, topk_w, logits, w2, num_sms, status, st);
    if (e0 != cudaSuccess) return e0;
    return launch_permute(topk_idx, T, k, E, counts, offsets, sorted_assign, assign_pos, perm_ws, st);
  }
  void* perm_ws = reinterpret_cast<char*>(ws) + logits_bytes;
  if (T <= kGemvMaxT) {
    // 4 warps (one expert row each) per CTA: E = 512 spreads the router matrix over 128 SMs
    const int grid = (E + 3) / 4;
    cudaError_t e0 = launch_pdl(router_gemv_kernel, dim3(grid), dim3(128), (size_t)T * d * sizeof(uint16_t), st,
                                x, T, d, Wr, br, E, logits);
    if (e0 != cudaSuccess) return e0;
  } else {
    dim3 grid((E + kRgBN - 1) / kRgBN, (T + kRgBM - 1) / kRgBM);
    cudaError_t e0 = launch_pdl(router_gemm_kernel, grid, dim3(256), 0, st, x, T, d, Wr, br, E, logits);
    if (e0 != cudaSuccess) return e0;
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (T <= 32 && T * k <= kPermChunk) {
    return launch_pdl(topk_perm_small_kernel, dim3(1), dim3(1024), (size_t)(E + T * k) * sizeof(int), st,
                      (const float*)logits, T, E, k, topk_idx, topk_w, counts, offsets, sorted_assign, assign_pos);
  }
  err = launch_pdl(topk_kernel, dim3((T + 7) / 8), dim3(256), 0, st, (const float*)logits, T, E, k, topk_idx,
                   topk_w);
  if (err != cudaSuccess) return err;
  return launch_permute(topk_idx, T, k, E, counts, offsets, sorted_assign, assign_pos, perm_ws, st);
}

// ---------------------------------------------------------------- cumulative histogram
// One CTA: cum[e] += counts[e] (or = on reset); then a bitonic sort in shared memory of
// keys (cum descending, id ascending) packed into 64 bits: key = (2^51-1-cum) << 12 | e
// (E <= 4096, checked by the caller).

__global__ void __launch_bounds__(1024) hist_kernel(const int32_t* __restrict__ counts, int E,
                                                    int64_t* __restrict__ cum,
                                                    int32_t* __restrict__ rank_out, int reset) {
  extern __shared__ unsigned long long keys[];  // [n], n = next power of two >= E
  int n = 1;
  while (n < E) n <<= 1;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    if (e < E) {
      const long long v = (reset ? 0 : cum[e]) + counts[e];
      cum[e] = v;
      keys[e] = ((((1ull << 51) - 1ull) - (unsigned long long)v) << 12) | (unsigned long long)e;
    } else {
      keys[e] = ~0ull;
    }
  }
  __syncthreads();
  if (!rank_out) return;
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == up) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int r = threadIdx.x; r < E; r += blockDim.x) rank_out[r] = (int32_t)(keys[r] & 0xFFFull);
}

cudaError_t launch_hist(const int32_t* counts, int E, int64_t* cum, int32_t* rank_out, int reset,
                        cudaStream_t st) {
  int n = 1;
  while (n < E) n <<= 1;
  return launch_pdl(hist_kernel, dim3(1), dim3(1024), (size_t)n * sizeof(unsigned long long), st, counts, E,
                    cum, rank_out, reset);
}

cudaError_t init_route_attributes() {
  return cudaFuncSetAttribute(router_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kGemvMaxT * 8192 * (int)sizeof(uint16_t));
}


}  // namespace moe

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_route(void* host, size_t bytes) { return trace_fetch(g_route_trace, host, bytes); }
}  // namespace moe
#endif
