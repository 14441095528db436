// Expert SwiGLU FFN, CUDA-core path for few tokens per expert (decode, 1-64 tokens).
//
// The MoE layer of the Basalt pages ("What Basalt changes in a Blackwell local inference
// stack", section "Experts can move without becoming free") runs each selected expert on
// its tokens; for decode this is a GEMV per expert, bound by HBM bandwidth on the 4-bit
// weight stream (0.5625 bytes per weight element). Reading used for the FFN: SwiGLU,
// h = silu(x Wg^T) * (x Wu^T), h re-quantised to NVFP4 (tensor scale 1.0) before the down
// projection.
//
// Dot products: an E2M1 x E2M1 product is a multiple of 1/4 with magnitude <= 36, so the
// sum of eight of them (<= 288) is exact in f16. Weights and activations are decoded to
// f16x2 with the hardware E2M1 converter and multiplied with f16x2 FMAs; each 16-element
// block's exact integer-quarter sum is then scaled by the two E4M3 block scales in
// float32. Work units are (active expert, 16 h-rows) for gate/up and (active expert, 32
// output rows) for down; active experts are those with tokens, found by every CTA from
// the offsets array.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kTokChunk = 8;      // tokens processed together per unit pass
constexpr int kFfnThreads = 256;  // 8 warps
constexpr int kDownRows = 32;     // output rows per down unit (4 per warp)

__host__ __device__ __forceinline__ size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

// Compacted list of experts with tokens (routed ids in increasing order, then E for the
// shared expert). Returns the count; identical in every CTA.
MOE_DEV int build_active_list(const FfnArgs& a, int* s_act, int* tmp) {
  int n = 0;
  for (int e0 = 0; e0 < a.E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int c = (e < a.E) ? (a.offsets[e + 1] - a.offsets[e]) : 0;
    const int flag = c > 0 ? 1 : 0;
    int total;
    const int pos = block_exclusive_scan(flag, tmp, &total);
    if (flag) s_act[n + pos] = e;
    n += total;
  }
  if (a.has_shared && a.T > 0) {
    if (threadIdx.x == 0) s_act[n] = a.E;
    n += 1;
  }
  __syncthreads();
  return n;
}

struct UnitExpert {
  const ExpertGroup* G;
  int eloc, cnt, off;
  bool shared;
};

MOE_DEV UnitExpert unit_expert(const FfnArgs& a, int e) {
  UnitExpert u;
  u.shared = (e == a.E);
  u.G = u.shared ? &a.shared : &a.routed;
  u.eloc = u.shared ? 0 : e;
  u.cnt = u.shared ? a.T : (a.offsets[e + 1] - a.offsets[e]);
  u.off = u.shared ? 0 : a.offsets[e];
  return u;
}

// dot of one weight block (8 code bytes, decoded) with one activation block in shared
// memory (8 f16x2 words): exact sum of the 16 E2M1 products, as float
MOE_DEV float block_dot(const uint32_t wf[8], const uint32_t* xblk) {
  const uint4 xa = *reinterpret_cast<const uint4*>(xblk);
  const uint4 xb = *reinterpret_cast<const uint4*>(xblk + 4);
  uint32_t acc = 0;
  acc = hfma2(wf[0], xa.x, acc);
  acc = hfma2(wf[1], xa.y, acc);
  acc = hfma2(wf[2], xa.z, acc);
  acc = hfma2(wf[3], xa.w, acc);
  acc = hfma2(wf[4], xb.x, acc);
  acc = hfma2(wf[5], xb.y, acc);
  acc = hfma2(wf[6], xb.z, acc);
  acc = hfma2(wf[7], xb.w, acc);
  return f16x2_hsum(acc);
}

// Stage nt rows of NVFP4 (codes [.][K/2], scales [.][K/16]) into shared memory as f16x2
// words [nt][K/2] and float scales [nt][K/16]; row j comes from src row rows[j].
MOE_DEV void stage_rows(const uint8_t* codes, const uint8_t* scales, int K, const int* rows, int nt,
                        uint32_t* s_f16, float* s_sc) {
  const int q_per_row = K / 8;  // 32-bit words of codes per row
  for (int i = threadIdx.x; i < nt * q_per_row; i += blockDim.x) {
    const int j = i / q_per_row, q = i - j * q_per_row;
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(codes + (size_t)rows[j] * (K / 2)) + q);
    uint32_t o[4];
    e2m1x8_to_f16x2x4(w, o);
    *reinterpret_cast<uint4*>(s_f16 + (size_t)j * (K / 2) + 4 * q) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  const int nb = K / kBlock;
  for (int i = threadIdx.x; i < nt * nb; i += blockDim.x) {
    const int j = i / nb, b = i - j * nb;
    s_sc[i] = e4m3_to_f32(__ldg(scales + (size_t)rows[j] * nb + b));
  }
}

// Partial dot products of one weight row (K elements, NVFP4) with nt staged rows.
MOE_DEV void row_dots(const uint8_t* wc, const uint8_t* wsc, int K, const uint32_t* s_f16,
                      const float* s_sc, int nt, float part[kTokChunk]) {
  const int lane = threadIdx.x & 31;
  const int nb = K / kBlock;
  for (int b = lane; b < nb; b += 32) {
    const uint2 cw = __ldg(reinterpret_cast<const uint2*>(wc) + b);
    const float sw = e4m3_to_f32(__ldg(wsc + b));
    uint32_t wf[8];
    e2m1x8_to_f16x2x4(cw.x, wf);
    e2m1x8_to_f16x2x4(cw.y, wf + 4);
#pragma unroll
    for (int j = 0; j < kTokChunk; ++j) {
      if (j < nt) {
        const float s = block_dot(wf, s_f16 + (size_t)j * (K / 2) + 8 * b);
        part[j] = fmaf(s, sw * s_sc[j * nb + b], part[j]);
      }
    }
  }
}

// ---------------------------------------------------------------- gate/up + SwiGLU + h quant
__global__ void __launch_bounds__(kFfnThreads) ffn_gateup_decode_kernel(FfnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int d = a.d, I = a.I;
  int* s_act = reinterpret_cast<int*>(smem);
  size_t off = align16((size_t)(a.E + 1) * sizeof(int));
  uint32_t* s_x = reinterpret_cast<uint32_t*>(smem + off);
  off += align16((size_t)kTokChunk * (d / 2) * sizeof(uint32_t));
  float* s_xs = reinterpret_cast<float*>(smem + off);
  off += align16((size_t)kTokChunk * (d / kBlock) * sizeof(float));
  __shared__ float s_g[kTokChunk][16], s_u[kTokChunk][16];
  __shared__ int s_rows[kTokChunk], s_slot[kTokChunk];
  __shared__ int tmp[32];

  // ACCUMULATE mode: zero y_acc here; the down kernel runs after this grid completes.
  if (a.mode == 0) {
    const size_t n4 = (size_t)a.T * d / 4;
    float4* o4 = reinterpret_cast<float4*>(a.out);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x)
      o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  const int n_act = build_active_list(a, s_act, tmp);
  const int nhb = I / kBlock;
  const int units = n_act * nhb;
  const float ts_x = *a.xq_ts;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int hb = u % nhb;
    const UnitExpert ue = unit_expert(a, s_act[u / nhb]);
    const ExpertGroup& G = *ue.G;
    const float ts_g = G.gu_ts[2 * ue.eloc] * ts_x;
    const float ts_u = G.gu_ts[2 * ue.eloc + 1] * ts_x;
    // this warp's rows: h-rows i0, i0+1 (gate rows i, up rows I+i); 8 warps x 2 = 16
    const int i0 = hb * kBlock + 2 * warp;
    const size_t rowstride_c = (size_t)(d / 2), rowstride_s = (size_t)(d / kBlock);
    const size_t ebase = (size_t)ue.eloc * 2 * I;
    for (int c0 = 0; c0 < ue.cnt; c0 += kTokChunk) {
      const int nt = min(kTokChunk, ue.cnt - c0);
      __syncthreads();
      if (threadIdx.x < nt) {
        const int j = threadIdx.x;
        if (ue.shared) {
          s_rows[j] = c0 + j;
          s_slot[j] = a.T * a.k + c0 + j;
        } else {
          s_rows[j] = a.sorted_assign[ue.off + c0 + j] / a.k;
          s_slot[j] = ue.off + c0 + j;
        }
      }
      __syncthreads();
      stage_rows(a.xq_codes, a.xq_scales, d, s_rows, nt, s_x, s_xs);
      __syncthreads();
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + (r & 1);
        const int row = (r < 2) ? i : I + i;
        float part[kTokChunk];
#pragma unroll
        for (int j = 0; j < kTokChunk; ++j) part[j] = 0.0f;
        row_dots(G.gu_codes + (ebase + row) * rowstride_c, G.gu_scales + (ebase + row) * rowstride_s,
                 d, s_x, s_xs, nt, part);
#pragma unroll
        for (int j = 0; j < kTokChunk; ++j) {
          const float v = warp_sum(part[j]);
          if (lane == 0 && j < nt) {
            if (r < 2) s_g[j][2 * warp + (r & 1)] = v * ts_g;
            else s_u[j][2 * warp + (r & 1)] = v * ts_u;
          }
        }
      }
      __syncthreads();
      // SwiGLU + NVFP4 quantisation of h (tensor scale 1.0): 16 lanes per token
      if (threadIdx.x < kTokChunk * 16) {
        const int j = threadIdx.x >> 4, ii = threadIdx.x & 15;
        const float g = s_g[j][ii], uu = s_u[j][ii];
        const float h = __fdiv_rn(g, 1.0f + expf(-g)) * uu;
        float amax = fabsf(h);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o, 16));
        const uint32_t s = f32_to_e4m3_sat(__fdiv_rn(__fdiv_rn(amax, kE2M1Max), 1.0f));
        const float sval = e4m3_to_f32(s);
        const float q = (sval != 0.0f) ? __fdiv_rn(h, __fmul_rn(sval, 1.0f)) : 0.0f;
        uint32_t code = f32x2_to_e2m1x2(q, 0.0f) & 0xFu;
        if (sval == 0.0f) code = 0;
        uint32_t b = code | (__shfl_down_sync(0xffffffffu, code, 1, 16) << 4);
        b |= __shfl_down_sync(0xffffffffu, b, 2, 16) << 8;
        b |= __shfl_down_sync(0xffffffffu, b, 4, 16) << 16;
        const uint32_t hi = __shfl_down_sync(0xffffffffu, b, 8, 16);
        if (ii == 0 && j < nt) {
          const size_t slot = (size_t)s_slot[j];
          *reinterpret_cast<uint2*>(a.h_codes + slot * (I / 2) + hb * 8) = make_uint2(b, hi);
          a.h_scales[slot * (I / kBlock) + hb] = (uint8_t)s;
        }
      }
    }
  }
}

// ---------------------------------------------------------------- down projection
__global__ void __launch_bounds__(kFfnThreads) ffn_down_decode_kernel(FfnArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int d = a.d, I = a.I;
  int* s_act = reinterpret_cast<int*>(smem);
  size_t off = align16((size_t)(a.E + 1) * sizeof(int));
  uint32_t* s_h = reinterpret_cast<uint32_t*>(smem + off);
  off += align16((size_t)kTokChunk * (I / 2) * sizeof(uint32_t));
  float* s_hs = reinterpret_cast<float*>(smem + off);
  __shared__ int s_rows[kTokChunk], s_tok[kTokChunk];
  __shared__ float s_w[kTokChunk];
  __shared__ int tmp[32];

  const int n_act = build_active_list(a, s_act, tmp);
  const int ntile = (d + kDownRows - 1) / kDownRows;
  const int units = n_act * ntile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int tile = u % ntile;
    const UnitExpert ue = unit_expert(a, s_act[u / ntile]);
    const ExpertGroup& G = *ue.G;
    const float ts_o = G.dn_ts[ue.eloc];  // h tensor scale is 1.0
    for (int c0 = 0; c0 < ue.cnt; c0 += kTokChunk) {
      const int nt = min(kTokChunk, ue.cnt - c0);
      __syncthreads();
      if (threadIdx.x < nt) {
        const int j = threadIdx.x;
        if (ue.shared) {
          s_rows[j] = a.T * a.k + c0 + j;
          s_tok[j] = c0 + j;
          s_w[j] = 1.0f;
        } else {
          const int p = ue.off + c0 + j;
          const int asg = a.sorted_assign[p];
          s_rows[j] = p;
          s_tok[j] = asg / a.k;
          s_w[j] = a.topk_w[asg];
        }
      }
      __syncthreads();
      stage_rows(a.h_codes, a.h_scales, I, s_rows, nt, s_h, s_hs);
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kDownRows / 8; ++r) {
        const int n = tile * kDownRows + warp * (kDownRows / 8) + r;
        if (n >= d) continue;  // warp-uniform: d % 16 == 0 but not always % 32
        const size_t row = (size_t)ue.eloc * d + n;
        float part[kTokChunk];
#pragma unroll
        for (int j = 0; j < kTokChunk; ++j) part[j] = 0.0f;
        row_dots(G.dn_codes + row * (I / 2), G.dn_scales + row * (I / kBlock), I, s_h, s_hs, nt, part);
#pragma unroll
        for (int j = 0; j < kTokChunk; ++j) {
          const float v = warp_sum(part[j]);
          if (lane == j && j < nt) {
            const float o = v * ts_o;
            if (a.mode == 0) {
              atomicAdd(a.out + (size_t)s_tok[j] * d + n, s_w[j] * o);
            } else if (ue.shared) {
              a.shared_out[(size_t)s_tok[j] * d + n] = o;
            } else {
              a.out[(size_t)s_rows[j] * d + n] = o;
            }
          }
        }
      }
    }
  }
}

size_t ffn_decode_smem_gateup(int d, int E) {
  return align16((size_t)(E + 1) * sizeof(int)) + align16((size_t)kTokChunk * (d / 2) * 4) +
         align16((size_t)kTokChunk * (d / kBlock) * 4);
}

size_t ffn_decode_smem_down(int I, int E) {
  return align16((size_t)(E + 1) * sizeof(int)) + align16((size_t)kTokChunk * (I / 2) * 4) +
         align16((size_t)kTokChunk * (I / kBlock) * 4);
}

size_t ffn_decode_ws_bytes(int64_t T, int d, int E, int k, int I) {
  const size_t slots = (size_t)(T * k + T);
  return ((slots * (I / 2) + 255) & ~(size_t)255) + ((slots * (I / kBlock) + 255) & ~(size_t)255);
}

cudaError_t launch_ffn_decode(const FfnArgs& a, int num_sms, cudaStream_t st) {
  const int max_act = (a.T * a.k < a.E ? a.T * a.k : a.E) + (a.has_shared ? 1 : 0);
  const int gu_units = max_act * (a.I / kBlock);
  const int dn_units = max_act * ((a.d + kDownRows - 1) / kDownRows);
  int g1 = gu_units < num_sms * 4 ? gu_units : num_sms * 4;
  int g2 = dn_units < num_sms * 4 ? dn_units : num_sms * 4;
  if (a.mode == 0) {
    // the gate/up grid also zeroes y_acc: make sure it covers it reasonably
    if (g1 < num_sms) g1 = num_sms;
  }
  if (g1 < 1) g1 = 1;
  if (g2 < 1) g2 = 1;
  ffn_gateup_decode_kernel<<<g1, kFfnThreads, ffn_decode_smem_gateup(a.d, a.E), st>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ffn_down_decode_kernel<<<g2, kFfnThreads, ffn_decode_smem_down(a.I, a.E), st>>>(a);
  return cudaGetLastError();
}

cudaError_t init_ffn_decode_attributes() {
  cudaError_t e = cudaFuncSetAttribute(ffn_gateup_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ffn_decode_smem_gateup(8192, 1024));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ffn_down_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)ffn_decode_smem_down(8192, 1024));
}

}  // namespace moe
