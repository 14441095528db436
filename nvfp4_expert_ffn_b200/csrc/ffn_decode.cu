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
#include "sm100.cuh"

namespace moe {

constexpr int kTokChunk = 8;      // tokens processed together per unit pass

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

// ---------------------------------------------------------------- fused persistent kernel
// One CTA per SM. Warp 8 is the producer: it streams the weights of this CTA's work units
// into a ring of shared-memory stages with cp.async.bulk. Warps 0-7 consume:
//   phase 1 unit (active expert a, 16 h-rows): gate and up rows -> SwiGLU -> NVFP4 h, written
//     to the workspace; then the unit is counted in done[a];
//   phase 2 unit (active expert a, r2 output rows): waits until done[a] == I/16 (all of the
//     expert's h is written), then the down projection and the weighted scatter into y.
// Every CTA takes a contiguous range of phase-1 units, then a contiguous range of phase-2
// units, so a CTA reaches phase 2 only after finishing its phase-1 work; all CTAs are
// resident (grid <= SM count, one CTA per SM), so the waits always end.
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kFusedThreads = kConsumers + 32;
constexpr int kMaxStages = 6;

struct DecodeCfg {
  int stage_bytes;  // bytes of one stage (phase-1 unit: 32 rows x (d/2 + d/16))
  int nstages;
  int r2;           // output rows per phase-2 unit
  int kmax;         // max(d, I): staged activation row length
  int32_t* done;    // [E+1] phase-1 units finished per active slot (zeroed before launch)
  int32_t* status;  // device status word
};

struct UnitRange {
  int beg, end;
};

MOE_DEV UnitRange block_range(int n, int cta, int ncta) {
  return UnitRange{(int)((long long)n * cta / ncta), (int)((long long)n * (cta + 1) / ncta)};
}

MOE_DEV int32_t ld_acquire(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Stage nt rows of NVFP4 written earlier in this kernel by other CTAs (read through L2).
MOE_DEV void stage_rows_cg(const uint8_t* codes, const uint8_t* scales, int K, const int* rows, int nt,
                           uint32_t* s_f16, float* s_sc, int tid, int nthr) {
  const int q_per_row = K / 8;
  for (int i = tid; i < nt * q_per_row; i += nthr) {
    const int j = i / q_per_row, q = i - j * q_per_row;
    const uint32_t w = __ldcg(reinterpret_cast<const uint32_t*>(codes + (size_t)rows[j] * (K / 2)) + q);
    uint32_t o[4];
    e2m1x8_to_f16x2x4(w, o);
    *reinterpret_cast<uint4*>(s_f16 + (size_t)j * (K / 2) + 4 * q) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  const int nb = K / kBlock;
  for (int i = tid; i < nt * nb; i += nthr) {
    const int j = i / nb, b = i - j * nb;
    s_sc[i] = e4m3_to_f32(__ldcg(scales + (size_t)rows[j] * nb + b));
  }
}

MOE_DEV void stage_rows_nc(const uint8_t* codes, const uint8_t* scales, int K, const int* rows, int nt,
                           uint32_t* s_f16, float* s_sc, int tid, int nthr) {
  const int q_per_row = K / 8;
  for (int i = tid; i < nt * q_per_row; i += nthr) {
    const int j = i / q_per_row, q = i - j * q_per_row;
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(codes + (size_t)rows[j] * (K / 2)) + q);
    uint32_t o[4];
    e2m1x8_to_f16x2x4(w, o);
    *reinterpret_cast<uint4*>(s_f16 + (size_t)j * (K / 2) + 4 * q) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  const int nb = K / kBlock;
  for (int i = tid; i < nt * nb; i += nthr) {
    const int j = i / nb, b = i - j * nb;
    s_sc[i] = e4m3_to_f32(__ldg(scales + (size_t)rows[j] * nb + b));
  }
}

// Partial dots of one smem weight row (codes, scales) with nt staged rows.
MOE_DEV void row_dots_smem(const uint8_t* wc, const uint8_t* wsc, int K, const uint32_t* s_f16,
                           const float* s_sc, int nt, float part[kTokChunk]) {
  const int lane = threadIdx.x & 31;
  const int nb = K / kBlock;
  for (int b = lane; b < nb; b += 32) {
    const uint2 cw = *reinterpret_cast<const uint2*>(wc + 8 * b);
    const float sw = e4m3_to_f32(wsc[b]);
    uint32_t wf[8];
    e2m1x8_to_f16x2x4(cw.x, wf);
    e2m1x8_to_f16x2x4(cw.y, wf + 4);
#pragma unroll
    for (int j = 0; j < kTokChunk; ++j) {
      if (j < nt) {
        const float sdot = block_dot(wf, s_f16 + (size_t)j * (K / 2) + 8 * b);
        part[j] = fmaf(sdot, sw * s_sc[j * nb + b], part[j]);
      }
    }
  }
}

__global__ void __launch_bounds__(kFusedThreads, 1) ffn_decode_fused_kernel(FfnArgs a, DecodeCfg c) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int d = a.d, I = a.I;
  const int nst = c.nstages;
  uint8_t* stages = smem;
  size_t off = (size_t)nst * c.stage_bytes;
  uint32_t* s_x = reinterpret_cast<uint32_t*>(smem + off);
  off += align16((size_t)kTokChunk * (c.kmax / 2) * sizeof(uint32_t));
  float* s_xs = reinterpret_cast<float*>(smem + off);
  off += align16((size_t)kTokChunk * (c.kmax / kBlock) * sizeof(float));
  int* s_act = reinterpret_cast<int*>(smem + off);
  off += align16((size_t)(a.E + 1) * sizeof(int));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  uint64_t* empty = full + kMaxStages;
  __shared__ float s_g[kTokChunk][16], s_u[kTokChunk][16];
  __shared__ int s_rows[kTokChunk], s_slot[kTokChunk], s_tok[kTokChunk];
  __shared__ float s_w[kTokChunk];
  __shared__ int tmp[32];
  __shared__ volatile int s_abort;
  __shared__ int s_go[2];  // decision of the waiting thread, by unit parity

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_barrier_init();
    s_abort = 0;
  }
  const int n_act = build_active_list(a, s_act, tmp);  // contains __syncthreads
  const int nhb = I / kBlock;
  const int nrt = (d + c.r2 - 1) / c.r2;
  const UnitRange r1 = block_range(n_act * nhb, blockIdx.x, gridDim.x);
  const UnitRange r2 = block_range(n_act * nrt, blockIdx.x, gridDim.x);
  const int n_units = (r1.end - r1.beg) + (r2.end - r2.beg);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      for (; it < n_units && !s_abort; ++it) {
        const int s = it % nst;
        if (!mbar_wait(&empty[s], ((it / nst) & 1) ^ 1, &s_abort, c.status)) break;
        uint8_t* dst = stages + (size_t)s * c.stage_bytes;
        const bool ph1 = it < (r1.end - r1.beg);
        const int v = ph1 ? r1.beg + it : r2.beg + (it - (r1.end - r1.beg));
        const int e = s_act[ph1 ? v / nhb : v / nrt];
        const bool sh = (e == a.E);
        const ExpertGroup& G = sh ? a.shared : a.routed;
        const size_t eloc = sh ? 0 : (size_t)e;
        if (ph1) {
          const int i0 = (v % nhb) * kBlock;
          const uint32_t cb = 16u * (uint32_t)(d / 2), sb = 16u * (uint32_t)(d / kBlock);
          mbar_arrive_expect_tx(&full[s], 2 * cb + 2 * sb);
          bulk_g2s(dst, G.gu_codes + (eloc * 2 * I + i0) * (d / 2), cb, &full[s]);
          bulk_g2s(dst + cb, G.gu_codes + (eloc * 2 * I + I + i0) * (d / 2), cb, &full[s]);
          bulk_g2s(dst + 2 * cb, G.gu_scales + (eloc * 2 * I + i0) * (d / kBlock), sb, &full[s]);
          bulk_g2s(dst + 2 * cb + sb, G.gu_scales + (eloc * 2 * I + I + i0) * (d / kBlock), sb, &full[s]);
        } else {
          const int n0 = (v % nrt) * c.r2;
          const int R = min(c.r2, d - n0);
          const uint32_t cb = (uint32_t)R * (I / 2), sb = (uint32_t)R * (I / kBlock);
          mbar_arrive_expect_tx(&full[s], cb + sb);
          bulk_g2s(dst, G.dn_codes + (eloc * d + n0) * (I / 2), cb, &full[s]);
          bulk_g2s(dst + (size_t)c.r2 * (I / 2), G.dn_scales + (eloc * d + n0) * (I / kBlock), sb,
                   &full[s]);
        }
      }
      // never leave copies in flight: wait for the last issued stage of each slot
      for (int j = (it > nst ? it - nst : 0); j < it; ++j) {
        volatile int no_abort = 0;
        mbar_wait(&full[j % nst], (j / nst) & 1, &no_abort, c.status);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int tid = threadIdx.x;
    int staged_e = -1, staged_c0 = -1;
    const float ts_x = *a.xq_ts;
    for (int it = 0; it < n_units; ++it) {
      const int s = it % nst;
      // one thread waits, the barrier publishes both the data and the decision
      if (tid == 0) s_go[it & 1] = mbar_wait(&full[s], (it / nst) & 1, &s_abort, c.status) ? 1 : 0;
      named_bar_sync(1, kConsumers);
      if (!s_go[it & 1]) break;
      const uint8_t* st = stages + (size_t)s * c.stage_bytes;
      const bool ph1 = it < (r1.end - r1.beg);
      const int v = ph1 ? r1.beg + it : r2.beg + (it - (r1.end - r1.beg));
      const int ai = ph1 ? v / nhb : v / nrt;
      const UnitExpert ue = unit_expert(a, s_act[ai]);
      const ExpertGroup& G = *ue.G;
      if (ph1) {
        const int hb = v % nhb;
        const float ts_g = G.gu_ts[2 * ue.eloc] * ts_x;
        const float ts_u = G.gu_ts[2 * ue.eloc + 1] * ts_x;
        const uint8_t* gc = st;
        const uint8_t* uc = st + 16 * (d / 2);
        const uint8_t* gs = st + 32 * (d / 2);
        const uint8_t* us = gs + 16 * (d / kBlock);
        for (int c0 = 0; c0 < ue.cnt; c0 += kTokChunk) {
          const int nt = min(kTokChunk, ue.cnt - c0);
          if (staged_e != s_act[ai] || staged_c0 != c0) {
            named_bar_sync(1, kConsumers);
            if (tid < nt) {
              const int j = tid;
              s_rows[j] = ue.shared ? c0 + j : a.sorted_assign[ue.off + c0 + j] / a.k;
            }
            named_bar_sync(1, kConsumers);
            stage_rows_nc(a.xq_codes, a.xq_scales, d, s_rows, nt, s_x, s_xs, tid, kConsumers);
            if (tid < nt) s_slot[tid] = ue.shared ? a.T * a.k + c0 + tid : ue.off + c0 + tid;
            named_bar_sync(1, kConsumers);
            staged_e = s_act[ai];
            staged_c0 = c0;
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int rr = 2 * warp + (r & 1);  // row within the unit's 16 h-rows
            float part[kTokChunk];
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) part[j] = 0.0f;
            if (r < 2)
              row_dots_smem(gc + rr * (d / 2), gs + rr * (d / kBlock), d, s_x, s_xs, nt, part);
            else
              row_dots_smem(uc + rr * (d / 2), us + rr * (d / kBlock), d, s_x, s_xs, nt, part);
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) {
              const float vsum = warp_sum(part[j]);
              if (lane == 0 && j < nt) {
                if (r < 2) s_g[j][rr] = vsum * ts_g;
                else s_u[j][rr] = vsum * ts_u;
              }
            }
          }
          named_bar_sync(1, kConsumers);
          if (tid < kTokChunk * 16) {
            const int j = tid >> 4, ii = tid & 15;
            const float g = s_g[j][ii], uu = s_u[j][ii];
            const float h = __fdiv_rn(g, 1.0f + expf(-g)) * uu;
            float amax = fabsf(h);
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o, 16));
            const uint32_t sbyte = f32_to_e4m3_sat(__fdiv_rn(__fdiv_rn(amax, kE2M1Max), 1.0f));
            const float sval = e4m3_to_f32(sbyte);
            uint32_t code = 0;
            if (sval != 0.0f) code = f32x2_to_e2m1x2(__fdiv_rn(h, __fmul_rn(sval, 1.0f)), 0.0f) & 0xFu;
            uint32_t b = code | (__shfl_down_sync(0xffffffffu, code, 1, 16) << 4);
            b |= __shfl_down_sync(0xffffffffu, b, 2, 16) << 8;
            b |= __shfl_down_sync(0xffffffffu, b, 4, 16) << 16;
            const uint32_t hi = __shfl_down_sync(0xffffffffu, b, 8, 16);
            if (ii == 0 && j < nt) {
              const size_t slot = (size_t)s_slot[j];
              *reinterpret_cast<uint2*>(a.h_codes + slot * (I / 2) + hb * 8) = make_uint2(b, hi);
              a.h_scales[slot * (I / kBlock) + hb] = (uint8_t)sbyte;
            }
            __threadfence();
          }
          named_bar_sync(1, kConsumers);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (tid == 0) atomicAdd(c.done + ai, 1);
      } else {
        // phase 2: wait for all h-blocks of this expert
        const int rt = v % nrt;
        const int n0 = rt * c.r2;
        const int R = min(c.r2, d - n0);
        if (tid == 0) {
          int ok = 1;
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire(c.done + ai) < nhb) {
            if (s_abort) {
              ok = 0;
              break;
            }
            if (globaltimer_ns() - t0 > wait_limit_ns()) {
              s_abort = 1;
              atomicExch(c.status, kStatusTimeout);
              ok = 0;
              break;
            }
          }
          s_go[it & 1] = ok;
        }
        named_bar_sync(1, kConsumers);
        if (!s_go[it & 1]) break;
        __threadfence();
        const float ts_o = G.dn_ts[ue.eloc];
        const uint8_t* dc = st;
        const uint8_t* ds = st + (size_t)c.r2 * (I / 2);
        for (int c0 = 0; c0 < ue.cnt; c0 += kTokChunk) {
          const int nt = min(kTokChunk, ue.cnt - c0);
          named_bar_sync(1, kConsumers);
          if (tid < nt) {
            const int j = tid;
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
          named_bar_sync(1, kConsumers);
          stage_rows_cg(a.h_codes, a.h_scales, I, s_rows, nt, s_x, s_xs, tid, kConsumers);
          named_bar_sync(1, kConsumers);
          staged_e = -1;  // s_x now holds h, not x
          for (int rr = warp; rr < R; rr += kConsumerWarps) {
            const int n = n0 + rr;
            float part[kTokChunk];
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) part[j] = 0.0f;
            row_dots_smem(dc + (size_t)rr * (I / 2), ds + (size_t)rr * (I / kBlock), I, s_x, s_xs, nt, part);
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) {
              const float vsum = warp_sum(part[j]);
              if (lane == j && j < nt) {
                const float o = vsum * ts_o;
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
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
  }
  __syncthreads();
}

size_t ffn_decode_smem_fused(int d, int I, int E, int stage_bytes, int nstages) {
  const int kmax = d > I ? d : I;
  return (size_t)nstages * stage_bytes + align16((size_t)kTokChunk * (kmax / 2) * 4) +
         align16((size_t)kTokChunk * (kmax / kBlock) * 4) + align16((size_t)(E + 1) * sizeof(int)) +
         2 * kMaxStages * sizeof(uint64_t);
}

constexpr size_t kFusedSmemLimit = 227 * 1024 - 2048;  // leave room for static shared memory

size_t ffn_decode_ws_bytes(int64_t T, int d, int E, int k, int I) {
  const size_t slots = (size_t)(T * k + T);
  return ((slots * (I / 2) + 255) & ~(size_t)255) + ((slots * (I / kBlock) + 255) & ~(size_t)255) +
         (((size_t)(E + 1) * sizeof(int32_t) + 255) & ~(size_t)255);
}

cudaError_t launch_ffn_decode(const FfnArgs& a, int num_sms, int32_t* status, cudaStream_t st) {
  DecodeCfg c;
  c.stage_bytes = 32 * (a.d / 2 + a.d / kBlock);  // 16 gate + 16 up rows
  c.kmax = a.d > a.I ? a.d : a.I;
  int r2 = c.stage_bytes / (a.I / 2 + a.I / kBlock);
  r2 = r2 > 256 ? 256 : r2;
  r2 = (r2 / 16) * 16;
  if (r2 < 16) {
    // very wide I: grow the stage to hold 16 down rows
    r2 = 16;
    c.stage_bytes = 16 * (a.I / 2 + a.I / kBlock);
  }
  c.r2 = r2;
  int nst = kMaxStages;
  while (nst > 2 && ffn_decode_smem_fused(a.d, a.I, a.E, c.stage_bytes, nst) > kFusedSmemLimit) --nst;
  if (ffn_decode_smem_fused(a.d, a.I, a.E, c.stage_bytes, nst) > kFusedSmemLimit)
    return cudaErrorInvalidConfiguration;
  c.nstages = nst;
  const size_t slots = (size_t)a.T * a.k + a.T;
  c.done = reinterpret_cast<int32_t*>(a.h_codes + (((slots * (a.I / 2) + 255) & ~(size_t)255) +
                                                   ((slots * (a.I / kBlock) + 255) & ~(size_t)255)));
  c.status = status;
  cudaError_t e = cudaMemsetAsync(c.done, 0, (size_t)(a.E + 1) * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  if (a.mode == 0) {
    e = cudaMemsetAsync(a.out, 0, (size_t)a.T * a.d * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  const int max_act = (a.T * a.k < a.E ? a.T * a.k : a.E) + (a.has_shared ? 1 : 0);
  const int units = max_act * (a.I / kBlock);
  const int grid = units < num_sms ? (units > 0 ? units : 1) : num_sms;
  const size_t smem = ffn_decode_smem_fused(a.d, a.I, a.E, c.stage_bytes, nst);
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  ffn_decode_fused_kernel<<<grid, kFusedThreads, smem, st>>>(a, c);
  return cudaGetLastError();
}

cudaError_t set_wait_limit_ffn_decode(unsigned long long ns) { return set_wait_limit_here(ns); }

cudaError_t init_ffn_decode_attributes() {
  return cudaFuncSetAttribute(ffn_decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kFusedSmemLimit);
}

}  // namespace moe
