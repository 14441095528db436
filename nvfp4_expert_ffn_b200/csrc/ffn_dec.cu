// Decode expert FFN (at most 8 tokens) on the tcgen05 tensor cores, split over the
// intermediate dimension so that every unit of work is independent.
//
// The MoE layer of the Basalt pages ("What Basalt changes in a Blackwell local inference
// stack", section "Experts can move without becoming free": each token runs a small subset
// of the experts; "Basalt" project page, "Engines": routed experts are NVFP4) computes per
// chosen expert h = silu(x Wg^T) * (x Wu^T), h re-quantised to NVFP4 (tensor scale 1, blocks
// of 16 along I), o = h Wd^T, and y += w * o. With a handful of tokens the cost is reading
// the chosen experts' weights once, so this kernel is built to stream weights and nothing
// else:
//
//   * a unit is (expert, 64-column slice j of I). Its gate/up product needs weight rows
//     64j..64j+63 of the gate and of the up matrix; SwiGLU and the NVFP4 quantisation of h
//     are local to the slice (4 blocks of 16); and the slice's share of the down projection,
//     h[:, slice] Wd[:, slice]^T, is added into y (float32 reductions). Units of one expert
//     never wait for each other, so there is no phase barrier between the two GEMMs.
//   * the activations of all T <= 8 tokens are the A operand of every unit: the CTA keeps
//     them in shared memory for the whole kernel as one 8-row, 128-byte-swizzled tile per
//     256 columns, and the MMA reads it as a 128-row operand whose 8-row groups all start
//     at the same address (row r holds token r % 8). The scale atoms of A repeat the same 8
//     tokens' scales. h is written by the epilogue the same way (32-byte swizzled rows).
//     Tokens that an expert does not use are computed and discarded.
//   * the ring of shared-memory stages therefore carries only weights: one stage is either
//     a 64-gate + 64-up row x 256-column tile of the stacked gate/up matrix (TMA, 128-byte
//     swizzle) or four 128-row x 64-column tiles of the down matrix (TMA, 32-byte swizzle),
//     each with its scale atoms (one bulk copy). The down tiles come from the slice-grouped
//     copy of the down matrix (moe_pack_experts), where a slice's 32-byte rows are
//     contiguous: read from the natural layout, each row's 32 bytes sit 256 bytes apart and
//     the stream runs at about half the HBM bandwidth.
//
// Warp roles (320 threads, one CTA per SM): warp 0 lane 0 issues the copies; warp 1 owns
// TMEM and lane 0 issues tcgen05.cp / tcgen05.mma; warps 2-9 run the epilogue. The MMA
// order is gu(0), gu(1), dn(0), gu(2), dn(1), ..., dn(n-1) so the gate/up product of the
// next unit overlaps the SwiGLU of the current one. TMEM: columns 0-127 the gate/up
// accumulator, 128-383 two 128-column down accumulators, 384-511 four scale slots.
//
// A small preparation kernel (one CTA) runs first: it zeroes y and lists the experts in
// use (the shared expert first) with each token's routing weight for each of them.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"
#include "trace.cuh"

namespace moe {

constexpr int kDecMaxT = 8;
constexpr int kDecThreads = 352;  // producer, two MMA issuers, 8 epilogue warps
constexpr int kDecEpiWarps = 8;
constexpr int kDecMaxStages = 12;
constexpr int kDecMinStages = 4;
constexpr int kDecAtom = 512;                          // scale atom: 128 rows x 4 blocks
constexpr int kDecBBytes = 16384;                      // weight bytes of one stage
constexpr int kDecStageBytes = kDecBBytes + 4 * kDecAtom;
constexpr int kDecSfSlots = 4;
constexpr int kDecDnN = 16;                                // 16 token columns (8 tokens read twice)
constexpr uint32_t kDecIdescT = idesc_mxf4nvf4(128, kDecDnN);  // 128 weight rows x 16 token columns
constexpr int kDecHBytes = 1024;                       // h codes (8 rows x 32 B) + its atom at +512

TC_TRACE_ARRAY(g_dec_trace)

struct DecParams {
  const uint8_t* xq_codes;
  const uint8_t* xq_scales;
  const float* xq_ts;
  const int32_t* offsets;
  const int32_t* sorted_assign;
  const float* topk_w;
  ExpertGroup routed, shared;
  int has_shared;
  int E, d, I, T, k;
  int nstages;
  int group_chunks;    // down chunks accumulated in TMEM at a time
  float* out;          // y [T][d] float32
  int32_t* nslots;     // workspace: experts in use (shared expert included)
  int32_t* slots;      // [E + 1] expert ids (E = the shared expert)
  float* slot_w;       // [E + 1][8] routing weight of each token (0: not routed)
  int32_t* status;
};

struct DecMaps {
  CUtensorMap b1, b1s;  // gate/up codes {d/2, I, 2, E}, boxes {128, 64, 2, 1}, 128-byte swizzle
  CUtensorMap b2, b2s;  // down codes by I-slice {32, 128, d/128, E*I/64}, boxes {32, 128, 4, 1}, 32-byte swizzle
};

// ---------------------------------------------------------------- preparation (one CTA)
// One pass over the experts (E <= 1024 = blockDim) lists those in use after the shared
// expert; then one thread per routed assignment writes its token's weight into its
// expert's row of slot_w (rows cleared first).
RT_TRACE_ARRAY(g_prep_trace)

__global__ void __launch_bounds__(1024) ffn_dec_prep_kernel(DecParams p) {
  RT_TRACE(g_prep_trace, 0, 0);
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_prep_trace, 0, 1);
  __shared__ int tmp[32];
  __shared__ int s_off[1025];
  __shared__ int s_slot[1024];
  const size_t n4 = (size_t)p.T * p.d / 4;
  float4* y4 = reinterpret_cast<float4*>(p.out);
  for (size_t i = threadIdx.x; i < n4; i += blockDim.x) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) s_off[e] = p.offsets[e];
  __syncthreads();
  const int e = threadIdx.x;
  const bool active = e < p.E && s_off[e + 1] > s_off[e];
  int total;
  const int slot = block_exclusive_scan(active ? 1 : 0, tmp, &total) + p.has_shared;
  if (e < p.E) s_slot[e] = active ? slot : -1;
  if (active) p.slots[slot] = e;
  const int nslots = total + p.has_shared;
  if (threadIdx.x == 0) {
    *p.nslots = nslots;
    if (p.has_shared) p.slots[0] = p.E;
  }
  for (int i = threadIdx.x; i < nslots * kDecMaxT; i += blockDim.x)
    p.slot_w[i] = (p.has_shared && i < kDecMaxT && i < p.T) ? 1.0f : 0.0f;
  __syncthreads();
  const int n = p.T * p.k;
  for (int q = threadIdx.x; q < n; q += blockDim.x) {
    int lo = 0, hi = p.E - 1;  // the expert e with s_off[e] <= q < s_off[e + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= q) lo = mid;
      else hi = mid - 1;
    }
    const int a = p.sorted_assign[q];
    p.slot_w[(size_t)s_slot[lo] * kDecMaxT + a / p.k] = p.topk_w[a];
  }
  RT_TRACE(g_prep_trace, 0, 2);
}

// ---------------------------------------------------------------- the FFN kernel
MOE_DEV uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~(uintptr_t)1023);
}

// TMEM columns (512 allocated): gate/up accumulators of the two MMA issuers, h scale slots
// (per issuer, per unit parity), the weight-scale ring, the resident activation scales
// (d/16 columns), then the down accumulators (16 columns per 128-row chunk).
constexpr uint32_t kColD1 = 0, kColH = 32, kColSf = 48, kColX = 112;
__host__ __device__ inline uint32_t dec_col_d2(int d) { return (kColX + (uint32_t)d / 16 + 15u) & ~15u; }

__global__ void __launch_bounds__(kDecThreads, 1) ffn_dec_kernel(const __grid_constant__ DecMaps maps, DecParams p) {
  TC_TRACE_DECL
  TC_TRACE_BEGIN(g_dec_trace);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  __shared__ uint64_t full[kDecMaxStages], empty[kDecMaxStages];
  __shared__ uint64_t xsf_ready, acc1_full, acc1_empty, h_full[2], acc2_full, acc2_empty, final_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_go;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, I = p.I, NST = p.nstages, T = p.T;
  const int nt1 = I / 64;    // units per expert
  const int nks1 = d / 256;  // gate/up stages per unit
  const int nch = d / 128;   // down chunks per unit
  const int nks2 = nch / 4;  // down stages per unit
  const int gch = p.group_chunks;  // down chunks accumulated in TMEM at a time (multiple of 4)
  const int gst = gch / 4;         // down stages per group
  const uint32_t col_d2 = dec_col_d2(d);

  uint8_t* ring = smem;                                    // NST x 18 KB
  uint8_t* xs = ring + (size_t)NST * kDecStageBytes;       // [d/256][8 rows x 128 B], swizzled
  uint8_t* xsf = xs + (size_t)nks1 * 1024;                 // [d/64] scale atoms of x
  uint8_t* hb = xsf + (size_t)(d / 64) * kDecAtom;         // [2] h tiles (codes + scale atom)
  float* s_gu = reinterpret_cast<float*>(hb + 2 * kDecHBytes);  // [128][8] gate/up sums of a unit

  // setup, overlapping the previous kernel's tail
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&xsf_ready, 2);
    mbar_init(&acc1_full, 2);
    mbar_init(&acc1_empty, kDecEpiWarps);
    mbar_init(&h_full[0], 1);
    mbar_init(&h_full[1], 1);
    mbar_init(&acc2_full, 2);
    mbar_init(&acc2_empty, kDecEpiWarps);
    mbar_init(&final_bar, 2);
    fence_barrier_init();
    s_abort = 0;
    prefetch_tensormap(&maps.b1);
    prefetch_tensormap(&maps.b2);
    if (p.has_shared) {
      prefetch_tensormap(&maps.b1s);
      prefetch_tensormap(&maps.b2s);
    }
  }
  if (warp == 1) tmem_alloc(&s_tmem, 512);
  RT_TRACE(g_prep_trace, 1, 0);
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_prep_trace, 1, 1);

  // x codes -> 8-row 128-byte-swizzled tiles (rows >= T are zero); chunk c of a row goes to
  // 16-byte slot c ^ row within its 128-byte line
  for (int i = threadIdx.x; i < kDecMaxT * (d / 32); i += blockDim.x) {
    const int t = i / (d / 32), c = i % (d / 32);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t < T) v = __ldg(reinterpret_cast<const uint4*>(p.xq_codes + (size_t)t * (d / 2)) + c);
    *reinterpret_cast<uint4*>(xs + (c >> 3) * 1024 + t * 128 + (((c & 7) ^ t) << 4)) = v;
  }
  // x scale atoms: row r = 32*r1 + r0 is token r0 % 8; byte r0*16 + r1*4 + b = scale of block b
  for (int i = threadIdx.x; i < (d / 64) * 32; i += blockDim.x) {
    const int kc = i / 32, r0 = i % 32, t = r0 & 7;
    uint32_t w = 0u;
    if (t < T) w = __ldg(reinterpret_cast<const uint32_t*>(p.xq_scales + (size_t)t * (d / kBlock)) + kc);
    *reinterpret_cast<uint4*>(xsf + (size_t)kc * kDecAtom + r0 * 16) = make_uint4(w, w, w, w);
  }
  fence_proxy_async_smem();  // generic writes above are read by tcgen05 (async proxy)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int nunits = *p.nslots * nt1;
  // this CTA's units: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int nu = (int)blockIdx.x < nunits ? (nunits - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto unit = [&](int u, int& slot, int& e, int& j) {
    const int ug = (int)blockIdx.x + u * (int)gridDim.x;
    slot = ug / nt1;
    j = ug % nt1;
    e = p.slots[slot];
  };
  // Gate/up K blocks are visited in an order rotated per CTA and unit (the sum does not
  // depend on the order).
  auto unit_rot = [&](int u) { return (int)((blockIdx.x + 3 * u) % nks1); };
  // job jb of 2*nu: gu(0), then pairs (gu(s), dn(s-1)) for s = 1..nu-1, then dn(nu-1), so the
  // SwiGLU of unit s overlaps the gate/up product of unit s+1
  auto job_is_gu = [&](int jb) { return jb == 0 || (jb < 2 * nu - 1 && (jb & 1)); };
  auto job_unit = [&](int jb) {
    if (jb == 0) return 0;
    if (jb == 2 * nu - 1) return nu - 1;
    return (jb & 1) ? (jb + 1) / 2 : jb / 2 - 1;
  };
  if (threadIdx.x == 0) TC_TRACE_AT(g_dec_trace, kEvSetupDone, nu);

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // jobs in the order the MMAs consume them: gu(0), gu(1), dn(0), gu(2), dn(1), ..., dn(n-1)
    if (lane == 0) {
      uint32_t it = 0;
      bool alive = true;
      for (int jb = 0; jb < 2 * nu && alive; ++jb) {
        const bool gu = job_is_gu(jb);
        const int u = job_unit(jb);
        int slot, e, j;
        unit(u, slot, e, j);
        const bool sh = e == p.E;
        const int el = sh ? 0 : e;
        const ExpertGroup& G = sh ? p.shared : p.routed;
        if (gu) TC_TRACE_AT(g_dec_trace, kEvProdTile, u);
        const int rot = unit_rot(u);
        const int q0 = gu ? 0 : nks1, q1 = gu ? nks1 : nks1 + nks2;
        for (int q = q0; q < q1; ++q, ++it) {
          const int st = (int)(it % (uint32_t)NST);
          if (!mbar_wait(&empty[st], ((it / NST) & 1) ^ 1, &s_abort, p.status)) {
            alive = false;
            break;
          }
          uint8_t* sb = ring + (size_t)st * kDecStageBytes;
          if (it < 40) TC_TRACE_AT(g_dec_trace, kEvProdIssue, it);
          mbar_arrive_expect_tx(&full[st], kDecStageBytes);
          if (q < nks1) {
            const int kq = (q + rot) % nks1;  // K block of this stage
            tma_load_4d(sb, sh ? &maps.b1s : &maps.b1, &full[st], kq * 128, 64 * j, 0, el);
            bulk_g2s(sb + kDecBBytes, G.gu_sf_tiled + (((size_t)el * nt1 + j) * (d / 64) + 4 * kq) * kDecAtom,
                     4 * kDecAtom, &full[st]);
          } else {
            // four 128-row chunks of slice j (16 KB contiguous) and their scale atoms (2 KB)
            const int q2 = q - nks1;
            tma_load_4d(sb, sh ? &maps.b2s : &maps.b2, &full[st], 0, 0, 4 * q2, el * nt1 + j);
            bulk_g2s(sb + kDecBBytes, G.dn_sf_slice + (((size_t)el * nt1 + j) * nch + 4 * q2) * kDecAtom,
                     4 * kDecAtom, &full[st]);
          }
        }
      }
      // no copy may still be landing when the CTA exits
      for (uint32_t jj = it > (uint32_t)NST ? it - NST : 0; jj < it; ++jj) {
        volatile int no_abort = 0;
        mbar_wait(&full[jj % NST], (jj / NST) & 1, &no_abort, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------------ MMA issuers
    // Two threads issue tcgen05 work, each for the ring stages of its parity: issuing a
    // scale copy or an MMA takes tens of nanoseconds, and one thread alone would pace the
    // weight stream. Gate/up is computed transposed, D1[weight row][token] (weights are the
    // 128-row A operand, the tokens a 16-column B operand whose two 8-row groups both read
    // the 8 tokens), each issuer into its own 16 columns; the epilogue adds the two.
    const int who = warp - 1;
    if (lane == 0) {
      // the activation scale atoms stay in TMEM for the whole kernel (each issuer copies
      // half of them; both wait for all)
      for (int a = who; a < d / 64; a += 2) tmem_cp_sf(tmem + kColX + 4 * a, sdesc_sf(smem_u32(xsf + (size_t)a * kDecAtom)));
      mma_commit(&xsf_ready);
      bool ok = mbar_wait(&xsf_ready, 0, &s_abort, p.status);
      tc_fence_after();
      uint32_t it = 0, gc = 0;
      // stage `itx` has landed and the scale slot it reuses (last used by stage itx - 4, of
      // the same issuer) is no longer read by an MMA in flight
      auto stage_in = [&](uint32_t itx) -> bool {
        if (!mbar_wait(&full[itx % NST], (itx / NST) & 1, &s_abort, p.status)) return false;
        if (itx < 40) TC_TRACE_AT(g_dec_trace, kEvMmaFull, itx);
        if (itx >= (uint32_t)kDecSfSlots) {
          const uint32_t pv = itx - kDecSfSlots;
          if (!mbar_wait(&empty[pv % NST], (pv / NST) & 1, &s_abort, p.status)) return false;
        }
        tc_fence_after();
        return true;
      };
      const uint32_t d1 = tmem + kColD1 + 16 * who;
      for (int jb = 0; jb < 2 * nu && ok; ++jb) {
        const int u = job_unit(jb);
        if (job_is_gu(jb)) {
        if (!mbar_wait(&acc1_empty, (u & 1) ^ 1, &s_abort, p.status)) break;
        tc_fence_after();
        const int rot = unit_rot(u);
        bool first = true;
        for (int q = 0; q < nks1; ++q, ++it) {
          if ((int)(it & 1) != who) continue;
          if (!stage_in(it)) {
            ok = false;
            break;
          }
          if (who == 0 && first) TC_TRACE_AT(g_dec_trace, kEvMmaFirst, u);
          const int kq = (q + rot) % nks1;
          const uint8_t* sb = ring + (size_t)(it % NST) * kDecStageBytes;
          const uint32_t sf = tmem + kColSf + 16 * (it % kDecSfSlots);
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) tmem_cp_sf(sf + 4 * kc, sdesc_sf(smem_u32(sb + kDecBBytes + kc * kDecAtom)));
          if (it < 40) TC_TRACE_AT(g_dec_trace, kEvMmaCps, it);
#pragma unroll
          for (int kc = 0; kc < 4; ++kc)
            mma_mxf4nvf4(d1, sdesc_kmajor(smem_u32(sb + 32 * kc), 1024, kSwizzle128B),
                         sdesc_kmajor(smem_u32(xs + kq * 1024 + 32 * kc), 0, kSwizzle128B), kDecIdescT, sf + 4 * kc,
                         tmem + kColX + 4 * (4 * kq + kc), (!first || kc) ? 1u : 0u);
          first = false;
          mma_commit(&empty[it % NST]);
          if (it < 40) TC_TRACE_AT(g_dec_trace, kEvMmaIssued, it);
        }
        if (!ok) break;
        if (who == 0) TC_TRACE_AT(g_dec_trace, kEvMmaLast, u);
        mma_commit(&acc1_full);
        continue;
        }
        // down projection of unit u, transposed: D2[output row][token] = Wd chunk x h^T, one
        // 16-column accumulator per 128-row chunk, gch chunks (one group) at a time
        const uint8_t* hbuf = hb + (u & 1) * kDecHBytes;
        if (!mbar_wait(&h_full[u & 1], (u >> 1) & 1, &s_abort, p.status)) break;
        tc_fence_after();
        const uint32_t hsf = tmem + kColH + 8 * who + 4 * (u & 1);
        tmem_cp_sf(hsf, sdesc_sf(smem_u32(hbuf + 512)));
        for (int q = 0; q < nks2; ++q, ++it) {
          if (q % gst == 0) {  // a new group: the epilogue has read the previous one
            if (!mbar_wait(&acc2_empty, (gc & 1) ^ 1, &s_abort, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if ((int)(it & 1) == who) {
            if (!stage_in(it)) {
              ok = false;
              break;
            }
            if (who == 0 && q == 0) TC_TRACE_AT(g_dec_trace, kEvDnFirst, u);
            const uint8_t* sb = ring + (size_t)(it % NST) * kDecStageBytes;
            const uint32_t sf = tmem + kColSf + 16 * (it % kDecSfSlots);
#pragma unroll
            for (int i = 0; i < 4; ++i) tmem_cp_sf(sf + 4 * i, sdesc_sf(smem_u32(sb + kDecBBytes + i * kDecAtom)));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int cl = (4 * q + i) % gch;
              mma_mxf4nvf4(tmem + col_d2 + kDecDnN * cl, sdesc_kmajor(smem_u32(sb + 4096 * i), 256, kSwizzle32B),
                           sdesc_kmajor(smem_u32(hbuf), 0, kSwizzle32B), kDecIdescT, sf + 4 * i, hsf, 0u);
            }
            mma_commit(&empty[it % NST]);
            if (it < 40) TC_TRACE_AT(g_dec_trace, kEvMmaIssued, it);
          }
          if (q % gst == gst - 1 || q == nks2 - 1) {
            mma_commit(&acc2_full);
            ++gc;
          }
        }
        if (!ok) break;
        if (who == 0) TC_TRACE_AT(g_dec_trace, kEvDnLast, u);
      }
      // every issued tensor-core operation has completed before TMEM is released
      mma_commit(&final_bar);
      volatile int no_abort = 0;
      mbar_wait(&final_bar, 0, &no_abort, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quarter q4 = w % 4. Every epilogue warp runs the same sequence
    // of named barriers whatever happens (after an abort the waits return at once and
    // nothing is written), so none can be left behind.
    const int ew = warp - 3;
    const int q4 = warp & 3;
    const int half = ew >> 2;
    const float ts_x = *p.xq_ts;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t gc = 0;
    for (int jb = 0; jb < 2 * nu; ++jb) {
      const int u = job_unit(jb);
      int slot, e, j;
      unit(u, slot, e, j);
      const bool sh = e == p.E;
      const int el = sh ? 0 : e;
      const ExpertGroup& G = sh ? p.shared : p.routed;
      if (job_is_gu(jb)) {
        // ---- SwiGLU of unit u. D1 lane r < 64 holds gate row r of the slice, lane 64 + r up
        // row r (h column r); columns 0..7 are the tokens, each issuer's sums 16 columns apart.
        // Every warp copies its quarter's sums to shared memory (one warp of each quarter), then
        // warp ew computes token ew: lane l takes h columns l and l + 32.
        if (ew == 0 && lane == 0) s_go = mbar_wait(&acc1_full, u & 1, &s_abort, p.status) ? 1 : 0;
        named_bar_sync(2, 32 * kDecEpiWarps);
        const bool go = s_go != 0;
        if (ew == 0 && lane == 0) TC_TRACE_AT(g_dec_trace, kEvEpiStart, u);
        tc_fence_after();
        uint32_t va[8], vb[8];
        tmem_ld8(lane_base + kColD1, va);
        tmem_ld8(lane_base + kColD1 + 16, vb);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc1_empty);
        if (half == 0) {
          float4* dst = reinterpret_cast<float4*>(s_gu + (32 * q4 + lane) * 8);
          dst[0] = make_float4(__uint_as_float(va[0]) + __uint_as_float(vb[0]), __uint_as_float(va[1]) + __uint_as_float(vb[1]),
                               __uint_as_float(va[2]) + __uint_as_float(vb[2]), __uint_as_float(va[3]) + __uint_as_float(vb[3]));
          dst[1] = make_float4(__uint_as_float(va[4]) + __uint_as_float(vb[4]), __uint_as_float(va[5]) + __uint_as_float(vb[5]),
                               __uint_as_float(va[6]) + __uint_as_float(vb[6]), __uint_as_float(va[7]) + __uint_as_float(vb[7]));
        }
        named_bar_sync(2, 32 * kDecEpiWarps);
        uint8_t* hbuf = hb + (u & 1) * kDecHBytes;
        const int t = ew;  // token of this warp
        const float sg = G.gu_ts[2 * el] * ts_x, su = G.gu_ts[2 * el + 1] * ts_x;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = lane + 32 * hh;  // h column within the slice
          const float gv = s_gu[i * 8 + t] * sg, uv = s_gu[(64 + i) * 8 + t] * su;
          const float h = __fdiv_rn(gv, 1.0f + expf(-gv)) * uv;
          // NVFP4 block of 16 h columns (16 lanes), tensor scale 1
          float amax = fabsf(h);
#pragma unroll
          for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          const uint32_t sbyte = f32_to_e4m3_sat(__fdiv_rn(amax, kE2M1Max));
          const float sval = e4m3_to_f32(sbyte);
          const uint32_t nib = sval != 0.0f ? (f32x2_to_e2m1x2(__fdiv_rn(h, sval), 0.0f) & 0xFu) : 0u;
          // byte of columns (i, i+1) on even lanes, then 4 bytes (8 columns) on lanes i % 8 == 0
          const uint32_t b = nib | (__shfl_down_sync(0xffffffffu, nib, 1) << 4);
          const uint32_t b1 = __shfl_down_sync(0xffffffffu, b, 2), b2 = __shfl_down_sync(0xffffffffu, b, 4),
                         b3 = __shfl_down_sync(0xffffffffu, b, 6);
          if (go && (lane & 7) == 0) {
            const uint32_t word = (b & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
            // row t of the 32-byte swizzled h tile: bytes i/2 .. i/2+3 in 16-byte half (i >> 5)
            *reinterpret_cast<uint32_t*>(hbuf + t * 32 + ((hh ^ (t >> 2)) & 1) * 16 + ((i >> 1) & 15)) = word;
          }
          if (go && (lane & 15) < 4) {
            // h scale atom: rows r0 = t + 8r (token t), all four r1, block i / 16 (lanes
            // 0..3 and 16..19 each write one r)
            const int r = lane & 3;
#pragma unroll
            for (int r1 = 0; r1 < 4; ++r1) hbuf[512 + (t + 8 * r) * 16 + r1 * 4 + (i >> 4)] = (uint8_t)sbyte;
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 32 * kDecEpiWarps);
        if (ew == 0 && lane == 0) {
          mbar_arrive(&h_full[u & 1]);
          TC_TRACE_AT(g_dec_trace, kEvEpiEnd, u);
        }
      } else {
        // ---- down projection of unit u: D2 lane 32*q4 + l is output row 128c + 32*q4 + l of
        // chunk c; column 16*(c % gch) + t is token t. Warp (q4, half) takes the chunks of
        // parity `half`.
        const float ts_o = G.dn_ts[el];
        float wf[kDecMaxT];
#pragma unroll
        for (int t = 0; t < kDecMaxT; ++t) wf[t] = p.slot_w[(size_t)slot * kDecMaxT + t] * ts_o;
        for (int g0 = 0; g0 < nch; g0 += gch, ++gc) {
          const int ng = nch - g0 < gch ? nch - g0 : gch;
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&acc2_full, gc & 1, &s_abort, p.status) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          tc_fence_after();
          for (int cl = half; cl < ng; cl += 2) {
            uint32_t v[8];
            tmem_ld8(lane_base + col_d2 + kDecDnN * cl, v);
            tmem_ld_wait();
            if (ok) {
              float* dst = p.out + (size_t)128 * (g0 + cl) + 32 * q4 + lane;
#pragma unroll
              for (int t = 0; t < kDecMaxT; ++t)
                if (t < T && wf[t] != 0.0f) red_add_f32(dst + (size_t)t * d, __uint_as_float(v[t]) * wf[t]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc2_empty);
        }
        if (ew == 0 && lane == 0) TC_TRACE_AT(g_dec_trace, kEvDrainEnd, u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) TC_TRACE_AT(g_dec_trace, kEvExit, 0);
  RT_TRACE(g_prep_trace, 1, 2);
}

// ---------------------------------------------------------------- host side
namespace {

constexpr size_t kDecSmemBudget = 226 * 1024;  // dynamic shared memory; the rest of 227 KB is static

size_t dec_fixed_smem(int d) {
  // x tiles, x scale atoms, two h tiles, the gate/up sums exchange, alignment slack
  return (size_t)(d / 256) * 1024 + (size_t)(d / 64) * kDecAtom + 2 * kDecHBytes + 128 * 8 * 4 + 1024;
}

// down chunks whose 16-column accumulators fit in TMEM next to everything else
int dec_group_chunks(int d) {
  const int avail = (512 - (int)dec_col_d2(d)) / kDecDnN;
  const int g = avail & ~3;
  return g < d / 128 ? g : d / 128;
}

int dec_stages(int d) {
  const size_t budget = kDecSmemBudget;
  const size_t fixed = dec_fixed_smem(d);
  if (fixed >= budget) return 0;
  const size_t n = (budget - fixed) / kDecStageBytes;
  return n > (size_t)kDecMaxStages ? kDecMaxStages : (int)n;
}

size_t dec_smem_bytes(int d) { return (size_t)dec_stages(d) * kDecStageBytes + dec_fixed_smem(d); }

size_t a256d(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

bool ffn_dec_supported(int64_t T, int d, int I, int mode) {
  return T >= 1 && T <= kDecMaxT && mode == 0 && d % 512 == 0 && I % 64 == 0 && d <= 4096 && I <= 16384 &&
         dec_stages(d) >= kDecMinStages && dec_group_chunks(d) >= 4;
}

size_t ffn_dec_ws_bytes(int E) { return 256 + a256d((size_t)(E + 1) * 4) + a256d((size_t)(E + 1) * kDecMaxT * 4); }

cudaError_t init_ffn_dec_attributes() {
  // the largest configuration; launches use at most this much
  return cudaFuncSetAttribute(ffn_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecSmemBudget);
}

cudaError_t launch_ffn_dec(const FfnArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st) {
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  DecParams p;
  p.xq_codes = a.xq_codes;
  p.xq_scales = a.xq_scales;
  p.xq_ts = a.xq_ts;
  p.offsets = a.offsets;
  p.sorted_assign = a.sorted_assign;
  p.topk_w = a.topk_w;
  p.routed = a.routed;
  p.shared = a.shared;
  p.has_shared = a.has_shared;
  p.E = a.E; p.d = a.d; p.I = a.I; p.T = (int)a.T; p.k = a.k;
  p.nstages = dec_stages(a.d);
  p.group_chunks = dec_group_chunks(a.d);
  p.out = a.out;
  p.nslots = reinterpret_cast<int32_t*>(w);
  p.slots = reinterpret_cast<int32_t*>(w + 256);
  p.slot_w = reinterpret_cast<float*>(w + 256 + a256d((size_t)(a.E + 1) * 4));
  p.status = status;

  DecMaps maps;
  const int d = a.d, I = a.I;
  for (int which = 0; which < 2; ++which) {
    const ExpertGroup& g = which ? a.shared : a.routed;
    const int E = which ? 1 : a.E;
    CUtensorMap* m1 = which ? &maps.b1s : &maps.b1;
    CUtensorMap* m2 = which ? &maps.b2s : &maps.b2;
    if (which && !a.has_shared) {
      *m1 = maps.b1;
      *m2 = maps.b2;
      continue;
    }
    cuuint64_t dims1[4] = {(cuuint64_t)(d / 2), (cuuint64_t)I, 2, (cuuint64_t)E};
    cuuint64_t str1[3] = {(cuuint64_t)(d / 2), (cuuint64_t)I * (d / 2), (cuuint64_t)2 * I * (d / 2)};
    cuuint32_t box1[4] = {128, 64, 2, 1};
    if ((e = encode_u8(m1, g.gu_codes, 4, dims1, str1, box1, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    cuuint64_t dims2[4] = {32, 128, (cuuint64_t)(d / 128), (cuuint64_t)E * (I / 64)};
    cuuint64_t str2[3] = {32, 128 * 32, (cuuint64_t)d * 32};
    cuuint32_t box2[4] = {32, 128, 4, 1};
    if ((e = encode_u8(m2, g.dn_codes_slice, 4, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_32B)) != cudaSuccess) return e;
  }
  if ((e = launch_pdl(ffn_dec_prep_kernel, dim3(1), dim3(1024), 0, st, p)) != cudaSuccess) return e;
  return launch_pdl(ffn_dec_kernel, dim3(num_sms), dim3(kDecThreads), dec_smem_bytes(d), st, maps, p);
}

}  // namespace moe

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_dec(void* host, size_t bytes) { return trace_fetch(g_dec_trace, host, bytes); }
int64_t trace_fetch_prep(void* host, size_t bytes) { return trace_fetch(g_prep_trace, host, bytes); }
}  // namespace moe
#endif
