// One MoE layer forward for at most 8 tokens in one persistent kernel: activation
// quantisation (A4), router (A1), top-k and weights (A2), permutation and per-call
// histogram (A3), the expert FFN with the shared expert (A5-A8, the unit core of
// dec_core.cuh) and the combine into bf16 (A9).
//
// With a handful of tokens every step but the expert FFN is a few microseconds of work,
// and as separate kernels each costs a launch and a chain of dependent memory round trips.
// Here one CTA per SM (all but one SM, left to a side-stream kernel such as the cumulative
// histogram) runs:
//   prologue (before the kernel waits on its predecessor) the CTA's router rows are copied
//            into shared memory and, with a shared expert, CTA j < I/64 starts bringing its
//            shared-expert unit (slice j) into L2: neither depends on the previous kernel.
//   phase 1  every CTA loads x, takes the global amax itself (the NVFP4 tensor scale),
//            quantises its share of the 64-element groups into the xq output buffers, and
//            computes the router logits of its expert rows; CTA 0 zeroes y_acc.
//   barrier
//   phase 2  warp t < T reads token t's logits from L2 and runs its top-k while the other
//            warps read all tokens' codes and scales into the MMA operand tiles (one round
//            of loads); then warp 0 derives this CTA's units from the bitmap of chosen
//            experts, and the last CTA also writes the routing outputs (top-k, counts,
//            offsets, permutation).
//   phase 3  the units (expert, 64-column slice of I), adding into y_acc.
//   phase 4  each CTA counts itself done; the one that comes last converts y_acc to bf16
//            (optionally RMS-renormalised). The others exit without waiting.
// The barrier and the done count share one 64-bit workspace word that must be zero before
// the first call; every call adds 2G to it (G CTAs). A CTA that gives up at a bounded wait
// marks the workspace (a second word), since the count may then be left between multiples
// of G; later calls on a marked workspace do nothing but report MOE_ERR_WORKSPACE until the
// caller zeroes it. A third word, which the library never writes, makes CTA 0 hold back its
// barrier arrival while it is nonzero: a test sets it to make the other CTAs' bounded waits
// run out. The launch is cooperative: it fails rather than start a grid whose CTAs cannot
// all be resident, so the barrier cannot wait on a CTA that has not started.
#include <cuda_bf16.h>

#include "dec_core.cuh"
#include "route_core.cuh"

namespace moe {

constexpr int kLayerMaxK = 32;
constexpr int kLayerMaxRows = kDecThreads / 32;  // router rows per CTA (the host checks E <= grid * this)

RT_TRACE_ARRAY(g_layer_trace)

struct LayerArgs {
  const uint16_t* x;   // [T][d] bf16
  const float* ts_in;  // static activation tensor scale, or NULL
  const float* Wr;     // [E][d]
  const float* br;     // [E] or NULL
  ExpertGroup routed, shared;
  int has_shared;
  int E, d, I, T, k;
  int nstages, group_chunks;
  int rms;
  // outputs
  uint8_t* xq_codes;   // [T][d/2]
  uint8_t* xq_scales;  // [T][d/16]
  float* xq_ts;        // [1]
  int32_t* topk_idx;   // [T][k]
  float* topk_w;       // [T][k]
  int32_t* counts;     // [E]
  int32_t* offsets;    // [E+1]
  int32_t* sorted_assign;  // [T*k]
  int32_t* assign_pos;     // [T*k]
  float* y_acc;        // [T][d]
  uint16_t* y;         // [T][d] bf16
  // workspace
  float* logits;       // [T][E]
  unsigned long long* sync;  // arrival counter of the grid barrier (zero before the first call)
  unsigned int* poison;      // nonzero once a call on this workspace gave up at a bounded wait
  const unsigned int* hold;  // nonzero: CTA 0 does not arrive at the barrier (set only by tests)
  int32_t* status;
};

// Grid-wide barrier on a 64-bit arrival counter that only grows: thread 0 of each CTA adds
// one and waits (bounded) until the count reaches the next multiple of the grid size. The
// counter starts at zero and every call adds two multiples (the barrier's arrivals, then
// phase 4's done count), so it stays aligned. Writes
// before the arrival are visible to every CTA after the wait; the CTA may work between the
// two halves.
//
// Arrival (every thread calls it): returns, in thread 0, the count to wait for (0 if the
// kernel is aborting and did not arrive).
MOE_DEV unsigned long long grid_arrive(unsigned long long* count, volatile int* abort) {
  __syncthreads();
  unsigned long long target = 0;
  if (threadIdx.x == 0 && !*abort) {
    const unsigned long long G = gridDim.x;
    __threadfence();
    const unsigned long long old = atomicAdd(count, 1ull);
    target = (old / G + 1) * G;
  }
  return target;
}

// Wait (every thread calls it, thread 0 with the arrival's target): false after an abort or
// a timeout.
MOE_DEV bool grid_wait(unsigned long long* count, unsigned long long target, volatile int* abort, int32_t* status) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    int ok = target != 0 && !*abort ? 1 : 0;
    const uint64_t t0 = globaltimer_ns();
    while (ok) {
      unsigned long long c;
      asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(c) : "l"(count) : "memory");
      if (c >= target) break;
      if (*abort) {
        ok = 0;
      } else if (globaltimer_ns() - t0 > wait_limit_ns()) {
        *abort = 1;
        atomicExch(status, kStatusTimeout);
        ok = 0;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

MOE_DEV bool grid_sync(unsigned long long* count, volatile int* abort, int32_t* status) {
  return grid_wait(count, grid_arrive(count, abort), abort, status);
}

// Shared-memory scratch of phases 1 and 2, on the weight ring (not in use before phase 3):
// the bf16 activations (phase 1), the top-k of each token, the permutation's counters, the
// router's partial sums and rows.
struct LayerScratch {
  uint16_t* xb;   // [8][d] (phase 1)
  int* tidx;      // [8][32] expert ids of each token's top-k
  float* tw;      // [8][32] their weights
  int* perm;      // [1024] counters of the permutation
  int* sidx;      // [256] top-k expert ids, assignment order
  float* part;    // [kDecThreads] router partial sums (phase 1)
  uint32_t* tks;  // [8][64] top-k scratch of each token's warp
  int* hslot;     // [1024] the routed group's hot-tier slots (with a hot tier)
  float* wr;      // [rows][d] this CTA's router rows (phase 1)
};

__host__ __device__ inline size_t layer_scratch_head(int d) { return 16 * (size_t)d; }

MOE_DEV LayerScratch layer_scratch(uint8_t* ring, int d) {
  LayerScratch s;
  s.xb = reinterpret_cast<uint16_t*>(ring);
  s.tidx = reinterpret_cast<int*>(ring + layer_scratch_head(d));
  s.tw = reinterpret_cast<float*>(s.tidx + kDecMaxT * kLayerMaxK);
  s.perm = reinterpret_cast<int*>(s.tw + kDecMaxT * kLayerMaxK);
  s.sidx = s.perm + 1024;
  s.part = reinterpret_cast<float*>(s.sidx + 256);
  s.tks = reinterpret_cast<uint32_t*>(s.part + kDecThreads);
  s.hslot = reinterpret_cast<int*>(s.tks + kDecMaxT * 64);
  s.wr = reinterpret_cast<float*>(s.hslot + 1024);
  return s;
}
// bytes of scratch past the head
constexpr size_t kLayerScratchTail =
    2 * kDecMaxT * kLayerMaxK * 4 + (1024 + 256 + kDecThreads + kDecMaxT * 64 + 1024) * 4;
static_assert(kLayerScratchTail % 16 == 0, "router rows must start 16-byte aligned");

__global__ void __launch_bounds__(kDecThreads, 1) layer_dec_kernel(LayerArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ DecBars bar;
  __shared__ int s_ue[kDecMaxUnits], s_uj[kDecMaxUnits];
  __shared__ float s_uw[kDecMaxUnits * kDecMaxT];
  __shared__ float s_red[32];
  __shared__ uint32_t s_bits[32];  // experts chosen by some token (E <= 1024)
  __shared__ int s_nu;
  const DecSmem sm = dec_smem(align1024(smem_raw), p.d, p.nstages);
  const LayerScratch sc = layer_scratch(sm.ring, p.d);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, T = p.T, E = p.E, k = p.k;
  const int G = (int)gridDim.x, b = (int)blockIdx.x;
  const int nvec = d / 4;  // float4 per router row
  volatile int* abort = reinterpret_cast<volatile int*>(&bar.abort);

  RT_TRACE(g_layer_trace, 0, 0);
  // this CTA's router rows b, b + G, ... are copied into shared memory before the kernel
  // waits on its predecessor (the router weights are not written by anything)
  const int nrows = b < E ? (E - 1 - b) / G + 1 : 0;
  __shared__ uint64_t s_wbar, s_hbar;
  __shared__ float s_bias[kLayerMaxRows];
  __shared__ const uint8_t* s_ub[kDecMaxUnits];  // where each unit's stages start
  __shared__ int s_hot;                           // the hot-tier slots are on their way
  if (threadIdx.x == 0) {
    mbar_init(&s_wbar, 1);
    mbar_init(&s_hbar, 1);
  }
  if (threadIdx.x < 32) s_bits[threadIdx.x] = 0u;
  if (threadIdx.x < nrows) s_bias[threadIdx.x] = p.br ? __ldg(p.br + b + threadIdx.x * G) : 0.0f;
  dec_init(bar, p.nstages);  // includes the barrier-init fence
  if (threadIdx.x == 0 && nrows > 0) {
    mbar_arrive_expect_tx(&s_wbar, (uint32_t)(nrows * d * 4));
    for (int r = 0; r < nrows; ++r)
      bulk_g2s(sc.wr + (size_t)r * d, p.Wr + (size_t)(b + r * G) * d, (uint32_t)(d * 4), &s_wbar);
  }
  // units 0 .. I/64 - 1 are the shared expert's slices and go to CTAs 0 .. I/64 - 1 (the unit
  // table of phase 2): such a CTA starts its unit's stages on their way into L2 now
  if (threadIdx.x == 32 && p.has_shared && b < p.I / 64) {
    const uint32_t unit_bytes = (uint32_t)((d / 256 + d / 512) * kDecStageBytes);
    prefetch_l2_bulk(p.shared.dec_pack + (size_t)b * unit_bytes, unit_bytes);
  }
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_layer_trace, 0, 1);
  // a workspace marked by an earlier call that gave up: report it and do nothing (the mark is
  // written by the predecessor kernels this one has just waited for)
  __shared__ int s_live;
  if (threadIdx.x == 0) {
    s_live = 1;
    s_hot = 0;
    if (*reinterpret_cast<volatile unsigned int*>(p.poison) != 0u) {
      s_live = 0;
      *abort = 1;
      atomicExch(p.status, kStatusWorkspace);
    } else {
      if (b == 0 && *reinterpret_cast<const volatile unsigned int*>(p.hold) != 0u)
        *abort = 1;  // held back: no arrival, so every other CTA's barrier wait runs out
      if (p.routed.n_hot > 0) {
        // the routed group's hot-tier slots (written by the update that came before this
        // call, so only now), needed when the unit table is built
        s_hot = 1;
        mbar_arrive_expect_tx(&s_hbar, (uint32_t)(E * 4));
        bulk_g2s(sc.hslot, p.routed.hot_slot, (uint32_t)(E * 4), &s_hbar);
      }
    }
  }
  __syncthreads();
  const bool live = s_live != 0;
  float ts = 1.0f;

  // ---------------------------------------------------------------- phase 1
  if (live) {
  // x -> shared memory (every load of a round in flight before the stores), with each
  // thread's running maximum of |x| (bf16 magnitudes order like their bit patterns)
  uint32_t mx2 = 0;
  {
    const int nx = T * d / 8;
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x);
    uint4* xb4 = reinterpret_cast<uint4*>(sc.xb);
    for (int i0 = threadIdx.x; i0 < nx; i0 += 8 * blockDim.x) {
      // all of a round's loads in flight together (past the end: piece 0, not used)
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x;
        v[u] = __ldg(x4 + (i < nx ? i : 0));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < nx) {
          xb4[i] = v[u];
          mx2 = __vmaxu2(mx2, v[u].x & 0x7FFF7FFFu);
          mx2 = __vmaxu2(mx2, v[u].y & 0x7FFF7FFFu);
          mx2 = __vmaxu2(mx2, v[u].z & 0x7FFF7FFFu);
          mx2 = __vmaxu2(mx2, v[u].w & 0x7FFF7FFFu);
        }
      }
    }
  }
  // NVFP4 tensor scale: amax / (6 * 448) over all T tokens (every CTA computes the same), or
  // the static scale
  {
    float f = warp_max(fmaxf(bf16_to_f32(mx2 & 0xFFFFu), bf16_to_f32(mx2 >> 16)));
    if (lane == 0) s_red[warp] = f;
    __syncthreads();  // also: x is in shared memory
    RT_TRACE(g_layer_trace, 0, 2);
    if (p.ts_in) {
      ts = *p.ts_in;
    } else {
      f = lane < (int)(blockDim.x >> 5) ? s_red[lane] : 0.0f;
      f = warp_max(f);
      ts = f > 0.0f ? __fdiv_rn(f, kE2M1Max * kE4M3Max) : 1.0f;
    }
  }
  RT_TRACE(g_layer_trace, 2, 0);
  // this CTA's share of the 64-element groups (b, b + G, ...), one warp per group of four
  // 16-element blocks, two elements per lane (the steps of quantize_block16): the group's 32
  // code bytes and its 4 scale bytes leave as whole 32-bit words
  {
    const int gpr = d / 64;  // groups per token row
    const int ngrp = T * gpr;
    const int nw = (int)(blockDim.x >> 5);
    for (int g = b + G * warp; g < ngrp; g += G * nw) {
      const int t = g / gpr, c = g % gpr;
      const uint32_t xv = *reinterpret_cast<const uint32_t*>(sc.xb + (size_t)t * d + 64 * c + 2 * lane);
      const float v0 = bf16_to_f32(xv & 0xFFFFu), v1 = bf16_to_f32(xv >> 16);
      float amax = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const uint32_t sbyte = f32_to_e4m3_sat(__fdiv_rn(__fdiv_rn(amax, kE2M1Max), ts));
      const float sval = e4m3_to_f32(sbyte);
      uint32_t cb = 0u;
      if (sval != 0.0f) {
        const float den = __fmul_rn(sval, ts);
        cb = f32x2_to_e2m1x2(__fdiv_rn(v0, den), __fdiv_rn(v1, den)) & 0xFFu;
      }
      const uint32_t word = cb | (__shfl_down_sync(0xffffffffu, cb, 1) << 8) |
                            (__shfl_down_sync(0xffffffffu, cb, 2) << 16) | (__shfl_down_sync(0xffffffffu, cb, 3) << 24);
      const uint32_t swd = sbyte | (__shfl_down_sync(0xffffffffu, sbyte, 8) << 8) |
                           (__shfl_down_sync(0xffffffffu, sbyte, 16) << 16) |
                           (__shfl_down_sync(0xffffffffu, sbyte, 24) << 24);
      if ((lane & 3) == 0) reinterpret_cast<uint32_t*>(p.xq_codes)[8 * g + (lane >> 2)] = word;
      if (lane == 0) reinterpret_cast<uint32_t*>(p.xq_scales)[g] = swd;
    }
    if (b == G - 1 && threadIdx.x == 0) *p.xq_ts = ts;
  }
  RT_TRACE(g_layer_trace, 2, 1);
  // router logits of this CTA's rows b + r*G, four rows at a time: thread i takes float4
  // columns i, i + blockDim.x, ... of every row and token (32 partial sums), a warp
  // reduce-scatter leaves lane l with the warp's sum of (row l / 8, token l % 8), and warp 0
  // adds the warps' sums
  if (nrows > 0) {
    {
      volatile int no_abort = 0;  // the rows' copies land before anything else happens
      if (!mbar_wait(&s_wbar, 0, &no_abort, p.status)) *abort = 1;
    }
    RT_TRACE(g_layer_trace, 2, 3);
    for (int r0 = 0; r0 < nrows; r0 += 4) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.0f;
      for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
        float xf[kDecMaxT][4];
#pragma unroll
        for (int t = 0; t < kDecMaxT; ++t) {
          uint2 xv = make_uint2(0u, 0u);
          if (t < T) xv = *reinterpret_cast<const uint2*>(sc.xb + (size_t)t * d + 4 * c);
          xf[t][0] = bf16_to_f32(xv.x & 0xFFFFu);
          xf[t][1] = bf16_to_f32(xv.x >> 16);
          xf[t][2] = bf16_to_f32(xv.y & 0xFFFFu);
          xf[t][3] = bf16_to_f32(xv.y >> 16);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (r0 + r < nrows) {
            const float4 wv = reinterpret_cast<const float4*>(sc.wr + (size_t)(r0 + r) * d)[c];
#pragma unroll
            for (int t = 0; t < kDecMaxT; ++t) {
              float a = v[8 * r + t];
              a = fmaf(xf[t][0], wv.x, a);
              a = fmaf(xf[t][1], wv.y, a);
              a = fmaf(xf[t][2], wv.z, a);
              a = fmaf(xf[t][3], wv.w, a);
              v[8 * r + t] = a;
            }
          }
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = upper ? v[i] : v[i + o];
          const float keep = upper ? v[i + o] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      sc.part[threadIdx.x] = v[0];
      __syncthreads();
      if (warp == 0) {
        float sum = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += sc.part[32 * w + lane];
        const int r = r0 + (lane >> 3), t = lane & 7;
        if (r < nrows && t < T) p.logits[(size_t)t * E + b + r * G] = sum + s_bias[r];
      }
      __syncthreads();
    }
  }
  RT_TRACE(g_layer_trace, 2, 2);
  // y_acc starts at zero: the units add into it after the barrier
  if (b == 0) {
    float4* y4 = reinterpret_cast<float4*>(p.y_acc);
    for (int i = threadIdx.x; i < T * d / 4; i += blockDim.x) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  } else if (nrows > 0) {
    // marked workspace: only wait for the router rows' copies, which must land before exit
    volatile int no_abort = 0;
    mbar_wait(&s_wbar, 0, &no_abort, p.status);
  }
  RT_TRACE(g_layer_trace, 0, 3);
  bool ok = grid_sync(p.sync, abort, p.status);
  RT_TRACE(g_layer_trace, 0, 4);
  if (threadIdx.x == 0 && s_hot) {
    // long landed by now; waited for on every path, as it must land before the CTA exits
    volatile int no_abort = 0;
    if (!mbar_wait(&s_hbar, 0, &no_abort, p.status)) {
      *abort = 1;
      ok = false;
    }
  }

  // ---------------------------------------------------------------- phase 2
  // Data written by other CTAs before the barrier is read with plain loads: the barrier's
  // acquire, fence and block barrier make it visible, and plain loads are all in flight
  // together (ld.global.cg loads were measured to complete one after another).
  const int nt1 = p.I / 64;
  const bool writer = b == G - 1;  // the CTA with the fewest units writes the routing outputs
  int nu = 0;
  if (ok) {
    if (warp < T) {
      // token `warp`: its logits straight from L2 into the top-k; the chosen experts are
      // marked in s_bits
      unsigned long long* stamps = nullptr;
#ifdef MOE_TRACE
      if (warp == 0 && b < kTraceCtas) stamps = &g_layer_trace[4][b][0];
#endif
      topk_dispatch(p.logits + (size_t)warp * E, E, k, writer ? p.topk_idx + (size_t)warp * k : nullptr,
                    writer ? p.topk_w + (size_t)warp * k : nullptr, sc.tidx + warp * kLayerMaxK,
                    sc.tw + warp * kLayerMaxK, sc.tks + warp * 64, stamps);
      RT_TRACE(g_layer_trace, 3, 0);
      __syncwarp();
      if (lane < k) {
        const int e = sc.tidx[warp * kLayerMaxK + lane];
        atomicOr(&s_bits[e >> 5], 1u << (e & 31));
      }
    } else {
      // the other warps: all tokens' codes -> the 8-row tiles (rows >= T zero) and their
      // scale words -> the atoms (word kc of token t goes to rows t, t + 8, t + 16, t + 24 of
      // atom kc), each thread's loads of a round in flight together. Every CTA reads the same
      // few lines right after the barrier, so each starts the codes at its own place.
      const int tid = (int)threadIdx.x - 32 * T, nth = (int)blockDim.x - 32 * T;
      const int cpr = d / 32, q4 = d / 256;       // 16-byte code / scale pieces of a token row
      const int nc = kDecMaxT * cpr, ns = kDecMaxT * q4;
      const int rot_c = (b * 37) % nc;
      auto code_piece = [&](int iu) { return iu + rot_c < nc ? iu + rot_c : iu + rot_c - nc; };
      for (int i0 = tid; i0 < nc + ns; i0 += 8 * nth) {
        // every load of the round in flight together: pieces of rows >= T and past the end
        // read piece 0 of the codes and are replaced by zeros
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int iu = i0 + u * nth;
          const uint4* src = reinterpret_cast<const uint4*>(p.xq_codes);
          if (iu < nc) {
            const int i = code_piece(iu), t = i / cpr;
            if (t < T) src = reinterpret_cast<const uint4*>(p.xq_codes + (size_t)t * (d / 2)) + i % cpr;
          } else if (iu < nc + ns) {
            const int t = (iu - nc) / q4;
            if (t < T) src = reinterpret_cast<const uint4*>(p.xq_scales + (size_t)t * (d / kBlock)) + (iu - nc) % q4;
          }
          v[u] = *src;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int iu = i0 + u * nth;
          const bool real = iu < nc ? code_piece(iu) / cpr < T : (iu < nc + ns && (iu - nc) / q4 < T);
          if (!real) v[u] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int iu = i0 + u * nth;
          if (iu < nc) {
            const int i = code_piece(iu);
            *reinterpret_cast<uint4*>(sm.xs + dec_xs_offset(i / cpr, i % cpr)) = v[u];
          } else if (iu < nc + ns) {
            const int t = (iu - nc) / q4, c4 = (iu - nc) % q4;
            const uint32_t wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
              for (int r1 = 0; r1 < 4; ++r1) dec_xsf_store(sm.xsf, 4 * c4 + w, t + 8 * r1, wv[w]);
          }
        }
      }
    }
    fence_proxy_async_smem();  // the tiles and atoms are read by tcgen05 (async proxy)
    __syncthreads();
    RT_TRACE(g_layer_trace, 3, 1);
    if (warp == 0) {
      // This CTA's units are b, b + G, ... of nslots * nt1 (slot 0 the shared expert, then the
      // experts in use in id order; unit ug is slice ug % nt1 of slot ug / nt1). Lane w holds
      // bitmap word w and the inclusive count of experts in use up to it; lane u finds its
      // unit's expert as the n-th chosen bit.
      const int nwd = (E + 31) >> 5;
      const uint32_t word = lane < nwd ? s_bits[lane] : 0u;
      int incl = __popc(word);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int nslots = __shfl_sync(0xffffffffu, incl, 31) + p.has_shared;
      const int nunits = nslots * nt1;
      int n = b < nunits ? (nunits - 1 - b) / G + 1 : 0;
      if (n > kDecMaxUnits) {  // the host checks the worst case, so this does not happen
        if (lane == 0) atomicExch(p.status, kStatusUnsupported);
        n = kDecMaxUnits;
      }
      const int ug = b + lane * G;
      const int rnk = ug / nt1 - p.has_shared;  // rank among the experts in use (< 0: shared)
      int lo = 0;                                // the first word whose inclusive count exceeds rnk
#pragma unroll
      for (int step = 16; step >= 1; step >>= 1)
        if (__shfl_sync(0xffffffffu, incl, lo + step - 1) <= rnk) lo += step;
      // (every lane takes part in every shuffle)
      uint32_t wd = __shfl_sync(0xffffffffu, word, lo);
      const int prev = __shfl_sync(0xffffffffu, incl, lo > 0 ? lo - 1 : 0);
      const int below = lo > 0 ? prev : 0;
      if (lane < n) {
        int e = E;
        if (rnk >= 0) {
          for (int i = 0; i < rnk - below; ++i) wd &= wd - 1u;
          e = 32 * lo + __ffs(wd) - 1;
        }
        s_ue[lane] = e;
        s_uj[lane] = ug % nt1;
        // the unit's stages: the shared expert's, a hot expert's copy, or its decode pack
        const size_t unit_bytes = (size_t)(d / 256 + d / 512) * kDecStageBytes;
        int hs = (e < E && s_hot) ? sc.hslot[e] : -1;
        if (hs >= p.routed.n_hot) hs = -1;  // not a slot of this tier: read the decode pack
        s_ub[lane] = e == E ? p.shared.dec_pack + (size_t)(ug % nt1) * unit_bytes
                     : hs >= 0 ? p.routed.hot_pack + ((size_t)hs * nt1 + ug % nt1) * unit_bytes
                               : p.routed.dec_pack + ((size_t)e * nt1 + ug % nt1) * unit_bytes;
      }
      if (lane == 0) s_nu = n;
      RT_TRACE(g_layer_trace, 3, 4);
      __syncwarp();
      for (int i = lane; i < n * kDecMaxT; i += 32) {
        const int u = i / kDecMaxT, t = i % kDecMaxT;
        const int e = s_ue[u];
        float wt = 0.0f;
        if (t < T) {
          if (e == E) {
            wt = 1.0f;
          } else {
            for (int j = 0; j < k; ++j)
              if (sc.tidx[t * kLayerMaxK + j] == e) wt = sc.tw[t * kLayerMaxK + j];
          }
        }
        s_uw[u * kDecMaxT + t] = wt;
      }
      RT_TRACE(g_layer_trace, 3, 3);
    } else if (warp == 1 && writer) {
      // the routing outputs: assignment a = t*k + j in expert order
      for (int a = lane; a < T * k; a += 32) sc.sidx[a] = sc.tidx[(a / k) * kLayerMaxK + a % k];
      __syncwarp();
      perm_small_warp(sc.sidx, T * k, E, sc.perm, p.counts, p.offsets, p.sorted_assign, p.assign_pos);
    }
    __syncthreads();
    nu = s_nu;
    RT_TRACE(g_layer_trace, 3, 2);
  }
  fence_proxy_async_smem();  // the bulk copies of phase 3 overwrite the scratch written above
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  RT_TRACE(g_layer_trace, 0, 5);
  // ---------------------------------------------------------------- phase 3
  DecArgs a;
  a.routed = p.routed;
  a.shared = p.shared;
  a.has_shared = p.has_shared;
  a.E = E; a.d = d; a.I = p.I; a.T = T;
  a.nstages = p.nstages;
  a.group_chunks = p.group_chunks;
  a.ts_x = ts;
  a.xsf_loaded = 0;  // the MMA issuers copy the activation scale atoms to TMEM
  a.out = p.y_acc;
  a.status = p.status;
  dec_run(a, sm, bar, DecUnits{nu, s_ue, s_uj, s_uw, s_ub});
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(bar.tmem, 512);
  }

  RT_TRACE(g_layer_trace, 0, 6);
  // ---------------------------------------------------------------- phase 4
  // Each CTA that finished its units counts itself on the barrier word (the call's second G
  // arrivals); the one whose arrival completes the multiple of G has seen every other CTA's
  // additions into y_acc and converts it: row t by warp t, to bf16, optionally scaled to
  // unit root-mean-square. The others exit at once.
  __shared__ int s_last;
  __syncthreads();  // every unit's additions are issued and complete
  if (threadIdx.x == 0) {
    s_last = 0;
    if (ok && !*abort) {
      __threadfence();
      const unsigned long long old = atomicAdd(p.sync, 1ull);
      s_last = old % (unsigned long long)G == (unsigned long long)(G - 1) ? 1 : 0;
      __threadfence();
    }
  }
  __syncthreads();
  RT_TRACE(g_layer_trace, 1, 0);
  if (s_last && warp < T) {
    const int t = warp, n4 = d / 4;
    const float4* row = reinterpret_cast<const float4*>(p.y_acc + (size_t)t * d);
    uint2* out = reinterpret_cast<uint2*>(p.y + (size_t)t * d);
    float scale = 1.0f;
    if (p.rms) {
      float ss = 0.0f;
      for (int c0 = lane; c0 < n4; c0 += 32 * 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = row[c0 + 32 * u < n4 ? c0 + 32 * u : 0];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (c0 + 32 * u < n4) {
            ss = fmaf(v[u].x, v[u].x, ss);
            ss = fmaf(v[u].y, v[u].y, ss);
            ss = fmaf(v[u].z, v[u].z, ss);
            ss = fmaf(v[u].w, v[u].w, ss);
          }
        }
      }
      const float ms = warp_sum(ss) / (float)d;
      scale = ms > 0.0f ? rsqrtf(ms) : 0.0f;
    }
    auto bf2 = [&](float lo, float hi) {
      return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo * scale)) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi * scale)) << 16);
    };
    for (int c0 = lane; c0 < n4; c0 += 32 * 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = row[c0 + 32 * u < n4 ? c0 + 32 * u : 0];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (c0 + 32 * u < n4) out[c0 + 32 * u] = make_uint2(bf2(v[u].x, v[u].y), bf2(v[u].z, v[u].w));
    }
  }
  // a CTA that gave up (or found the workspace marked) marks it for the calls that follow
  if (threadIdx.x == 0 && *abort) atomicExch(p.poison, 1u);
  RT_TRACE(g_layer_trace, 1, 1);
}

// ---------------------------------------------------------------- host side
namespace {
size_t a256l(size_t v) { return (v + 255) & ~(size_t)255; }
int layer_grid(int num_sms) { return num_sms > 1 ? num_sms - 1 : 1; }
}  // namespace

// workspace: the barrier word, the mark and the hold word (each on its own line), then the
// logits
constexpr size_t kLayerWsHeader = 2048, kLayerWsPoison = 1024, kLayerWsHold = 1536;
size_t layer_dec_ws_bytes(int64_t T, int E) { return kLayerWsHeader + a256l((size_t)T * E * 4); }

bool layer_dec_supported(int64_t T, int d, int I, int E, int k, int has_shared, int num_sms) {
  const int G = layer_grid(num_sms);
  if (!dec_shape_ok(T, d, I) || k < 1 || k > kLayerMaxK || E < k || E > 1024) return false;
  if (E > G * (kDecThreads / 32)) return false;  // router rows: one per warp
  const int nst = dec_stages(d);
  const size_t rows = (size_t)(E + G - 1) / G;  // router rows of one CTA, staged in the ring
  if ((size_t)nst * kDecStageBytes < layer_scratch_head(d) + kLayerScratchTail + rows * d * 4) return false;
  const int64_t slots = (T * k < E ? T * k : E) + has_shared;
  return (slots * (I / 64) + G - 1) / G <= kDecMaxUnits;
}

cudaError_t set_wait_limit_layer_dec(unsigned long long ns) { return set_wait_limit_here(ns); }

cudaError_t init_layer_dec_attributes() {
  return cudaFuncSetAttribute(layer_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecSmemBudget);
}

cudaError_t launch_layer_dec(const LayerDecArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st) {
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  LayerArgs p;
  p.x = a.x;
  p.ts_in = a.ts_in;
  p.Wr = a.Wr;
  p.br = a.br;
  p.routed = a.routed;
  p.shared = a.shared;
  p.has_shared = a.has_shared;
  p.E = a.E; p.d = a.d; p.I = a.I; p.T = a.T; p.k = a.k;
  p.nstages = dec_stages(a.d);
  p.group_chunks = dec_group_chunks(a.d);
  p.rms = a.rms;
  p.xq_codes = a.xq_codes;
  p.xq_scales = a.xq_scales;
  p.xq_ts = a.xq_ts;
  p.topk_idx = a.topk_idx;
  p.topk_w = a.topk_w;
  p.counts = a.counts;
  p.offsets = a.offsets;
  p.sorted_assign = a.sorted_assign;
  p.assign_pos = a.assign_pos;
  p.y_acc = a.y_acc;
  p.y = a.y;
  p.sync = reinterpret_cast<unsigned long long*>(w);
  p.poison = reinterpret_cast<unsigned int*>(w + kLayerWsPoison);
  p.hold = reinterpret_cast<const unsigned int*>(w + kLayerWsHold);
  p.logits = reinterpret_cast<float*>(w + kLayerWsHeader);
  p.status = status;
  // a hot tier: its copies are read as persisting in L2, everything else as streaming
  cudaAccessPolicyWindow win = {};
  const cudaAccessPolicyWindow* wp = nullptr;
  if (a.routed.n_hot > 0) {
    int dev = 0, max_win = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&max_win, cudaDevAttrMaxAccessPolicyWindowSize, dev);
    if (e != cudaSuccess) return e;
    const size_t bytes = (size_t)a.routed.n_hot * (a.I / 64) * (a.d / 256 + a.d / 512) * kDecStageBytes;
    win.base_ptr = const_cast<uint8_t*>(a.routed.hot_pack);
    win.num_bytes = bytes < (size_t)max_win ? bytes : (size_t)max_win;
    win.hitRatio = 1.0f;
    win.hitProp = cudaAccessPropertyPersisting;
    win.missProp = cudaAccessPropertyStreaming;
    if (win.num_bytes > 0) wp = &win;
  }
  return launch_pdl_coop(layer_dec_kernel, dim3(layer_grid(num_sms)), dim3(kDecThreads), dec_smem_bytes(a.d), st,
                         wp, p);
}

}  // namespace moe

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_layer(void* host, size_t bytes) { return trace_fetch(g_layer_trace, host, bytes); }
int64_t trace_fetch_layer_core(void* host, size_t bytes) { return trace_fetch(g_dec_trace, host, bytes); }
}  // namespace moe
#endif
