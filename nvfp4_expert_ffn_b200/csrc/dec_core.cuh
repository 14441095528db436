// The expert-FFN core for at most 8 tokens on the tcgen05 tensor cores, shared by the decode
// FFN kernel (ffn_dec.cu) and the fused decode-layer kernel (layer_dec.cu).
//
// The MoE layer of the Basalt pages ("What Basalt changes in a Blackwell local inference
// stack", section "Experts can move without becoming free": each token runs a small subset
// of the experts; "Basalt" project page, "Engines": routed experts are NVFP4) computes per
// chosen expert h = silu(x Wg^T) * (x Wu^T), h re-quantised to NVFP4 (tensor scale 1, blocks
// of 16 along I), o = h Wd^T, and y += w * o. With a handful of tokens the cost is reading the
// chosen experts' weights once, so the core is built to stream weights and nothing else:
//
//   * a unit is (expert, 64-column slice j of I). Its gate/up product needs weight rows
//     64j..64j+63 of the gate and of the up matrix; SwiGLU and the NVFP4 quantisation of h
//     are local to the slice (4 blocks of 16); and the slice's share of the down projection,
//     h[:, slice] Wd[:, slice]^T, is added into y (float32 reductions). Units never wait for
//     each other, so there is no phase barrier between the two GEMMs.
//   * the activations of all T <= 8 tokens are an operand of every unit: the CTA keeps them
//     in shared memory as one 8-row, 128-byte-swizzled tile per 256 columns, read by the MMA
//     as a 16-row operand whose two 8-row groups start at the same address (row r is token
//     r % 8); their scale atoms (rows r -> token r % 8) are copied to TMEM once. h is written
//     by the epilogue the same way (32-byte swizzled rows). Tokens an expert does not use are
//     computed and discarded.
//   * both products are computed transposed, D[weight row][token]: the weight tile is the
//     128-row A operand, the tokens a 16-column B operand, so an accumulator takes 16 TMEM
//     columns and a unit's 16 down chunks accumulate side by side.
//   * the ring of shared-memory stages carries only weights, each stage one 18 KB block of
//     the decode pack (moe_pack_experts) moved by one bulk copy: a 64-gate + 64-up row x
//     256-column tile already in the 128-byte swizzle, or four 128-row x 64-column down
//     chunks already in the 32-byte swizzle, followed by the stage's 4 scale atoms. A unit's
//     blocks are contiguous, so HBM streams whole runs, and one copy per stage leaves the
//     per-SM copy engine, which also executes the tcgen05 scale copies, as free as it can be.
//   * the down accumulators form two buffers of group_chunks chunks; down groups alternate
//     between them, so one group's MMAs overlap the epilogue's reading of the previous one.
//
// Warp roles (352 threads, one CTA per SM): warp 0 lane 0 issues the copies; warps 1 and 2
// (lane 0) issue tcgen05 copies and MMAs for alternate ring stages (an issued tcgen05
// instruction costs the issuing thread tens of nanoseconds; one thread alone would pace the
// stream); warp 1 owns TMEM; warps 3-10 run SwiGLU and add the down results into y. Jobs run
// gu(0), gu(1), dn(0), gu(2), dn(1), ..., dn(n-1), so SwiGLU overlaps the next gate/up.
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "trace.cuh"

namespace moe {

constexpr int kDecMaxT = 8;
constexpr int kDecThreads = 352;  // producer, two MMA issuers, 8 epilogue warps
constexpr int kDecEpiWarps = 8;
constexpr int kDecMaxStages = 12;
constexpr int kDecMinStages = 4;
constexpr int kDecMaxUnits = 32;                       // units per CTA
constexpr int kDecAtom = 512;                          // scale atom: 128 rows x 4 blocks
constexpr int kDecBBytes = 16384;                      // weight bytes of one stage
constexpr int kDecStageBytes = kDecBBytes + 4 * kDecAtom;
constexpr int kDecSfSlots = 4;
constexpr int kDecDnN = 16;                                    // 16 token columns (8 tokens read twice)
constexpr uint32_t kDecIdescT = idesc_mxf4nvf4(128, kDecDnN);  // 128 weight rows x 16 token columns
constexpr int kDecHBytes = 1024;                       // h codes (8 rows x 32 B) + its atom at +512
constexpr size_t kDecSmemBudget = 224 * 1024;          // dynamic shared memory; the rest is static
// The weight stream is read once per call: its L2 lines go first, so that the activations,
// logits, router rows and the kernel's own code stay in L2 while it passes.
constexpr bool kDecStreamEvictFirst = true;

// TMEM columns (512 allocated): gate/up accumulators of the two MMA issuers, h scale slots
// (per issuer, per unit parity), the weight-scale ring, the resident activation scales
// (d/16 columns), then the down accumulators (16 columns per 128-row chunk).
constexpr uint32_t kColD1 = 0, kColH = 32, kColSf = 48, kColX = 112;
__host__ __device__ inline uint32_t dec_col_d2(int d) { return (kColX + (uint32_t)d / 16 + 15u) & ~15u; }


// What the unit loop needs besides its units.
struct DecArgs {
  ExpertGroup routed, shared;
  int has_shared;
  int E, d, I, T;
  int nstages;       // ring stages
  int group_chunks;  // down chunks accumulated in TMEM at a time (multiple of 4)
  float ts_x;        // tensor scale of the activations
  int xsf_loaded;    // the activation scale atoms are in TMEM already (xsf_ready completes)
  float* out;        // y [T][d] float32, added into
  int32_t* status;
};

// This CTA's units, in shared memory: expert id (E = the shared expert), slice j, and the
// routing weight of each of the 8 tokens (0: token not routed to the expert); optionally
// where each unit's stages start (else the unit's place in the group's decode pack).
struct DecUnits {
  int n;
  const int* e;
  const int* j;
  const float* w;  // [n][8]
  const uint8_t* const* base = nullptr;
};

struct DecBars {
  uint64_t full[kDecMaxStages], empty[kDecMaxStages];
  uint64_t xsf_ready, acc1_full, acc1_empty, h_full[2], acc2_full[2], acc2_empty[2], final_bar;
  uint32_t tmem;
  int abort;
  int go;
};

// Shared-memory carve-up (from a 1024-byte aligned base).
struct DecSmem {
  uint8_t* ring;  // nstages x 18 KB
  uint8_t* xs;    // [d/256][8 rows x 128 B], 128-byte swizzled
  uint8_t* xsf;   // [d/64] scale atoms of x
  uint8_t* hb;    // [2] h tiles (codes + scale atom)
  float* s_gu;    // [128][8] gate/up sums of a unit
};

MOE_DEV uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~(uintptr_t)1023);
}

MOE_DEV DecSmem dec_smem(uint8_t* base, int d, int nst) {
  DecSmem s;
  s.ring = base;
  s.xs = s.ring + (size_t)nst * kDecStageBytes;
  s.xsf = s.xs + (size_t)(d / 256) * 1024;
  s.hb = s.xsf + (size_t)(d / 64) * kDecAtom;
  s.s_gu = reinterpret_cast<float*>(s.hb + 2 * kDecHBytes);
  return s;
}

// Barriers (thread 0) and TMEM (warp 1); called by every thread before the first
// __syncthreads of the kernel, so it can run before the kernel waits on its predecessor.
MOE_DEV void dec_init(DecBars& b, int nst) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&b.full[s], 1);
      mbar_init(&b.empty[s], 1);
    }
    mbar_init(&b.xsf_ready, 2);
    mbar_init(&b.acc1_full, 2);
    mbar_init(&b.acc1_empty, kDecEpiWarps);
    mbar_init(&b.h_full[0], 1);
    mbar_init(&b.h_full[1], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.acc2_full[i], 2);
      mbar_init(&b.acc2_empty[i], kDecEpiWarps);
    }
    mbar_init(&b.final_bar, 2);
    fence_barrier_init();
    b.abort = 0;
  }
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&b.tmem, 512);
}

// Byte offset of 16-byte chunk c (of a token row's codes, 16 chunks per 256 columns) of
// token t in the x tiles: tile c / 8, row t, 128-byte-swizzled slot (c % 8) ^ t.
MOE_DEV uint32_t dec_xs_offset(int t, int c) { return (uint32_t)((c >> 3) * 1024 + t * 128 + (((c & 7) ^ t) << 4)); }

// x scale atom kc (scale blocks 4kc..4kc+3) from the 8 tokens' 4-byte scale words: row
// r = 32*r1 + r0 is token r0 % 8, byte r0*16 + r1*4 + b = scale of block b. Called for
// (kc, r0) pairs by any threads.
MOE_DEV void dec_xsf_store(uint8_t* xsf, int kc, int r0, uint32_t word_of_token) {
  *reinterpret_cast<uint4*>(xsf + (size_t)kc * kDecAtom + r0 * 16) =
      make_uint4(word_of_token, word_of_token, word_of_token, word_of_token);
}

// Runs this CTA's units. Preconditions: dec_init() done and visible (a __syncthreads), the
// x tiles and x scale atoms written to shared memory and made visible to the async proxy
// (with p.xsf_loaded, the atoms already copied to TMEM by tcgen05.cp with two commits on
// xsf_ready),
// y zeroed (or holding what the units should add to). Every thread of the CTA calls it; it
// returns once every unit's results have been added into p.out and every tensor-core
// operation has completed. TMEM stays allocated (the caller releases it).
TC_TRACE_ARRAY(g_dec_trace)

MOE_DEV void dec_run(const DecArgs& p, const DecSmem& sm, DecBars& bar, const DecUnits& U) {
  TC_TRACE_DECL
  TC_TRACE_BEGIN(g_dec_trace);
  __syncthreads();
  uint64_t* full = bar.full;
  uint64_t* empty = bar.empty;
  uint64_t& xsf_ready = bar.xsf_ready;
  uint64_t& acc1_full = bar.acc1_full;
  uint64_t& acc1_empty = bar.acc1_empty;
  uint64_t* h_full = bar.h_full;
  uint64_t* acc2_full = bar.acc2_full;    // per down-accumulator buffer
  uint64_t* acc2_empty = bar.acc2_empty;
  uint64_t& final_bar = bar.final_bar;
  volatile int& s_abort = *reinterpret_cast<volatile int*>(&bar.abort);
  int& s_go = bar.go;
  const uint32_t tmem = bar.tmem;
  uint8_t* const ring = sm.ring;
  uint8_t* const xs = sm.xs;
  uint8_t* const xsf = sm.xsf;
  uint8_t* const hb = sm.hb;
  float* const s_gu = sm.s_gu;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, I = p.I, NST = p.nstages, T = p.T;
  const int nt1 = I / 64;          // units per expert
  const int nks1 = d / 256;        // gate/up stages per unit
  const int nch = d / 128;         // down chunks per unit
  const int nks2 = nch / 4;        // down stages per unit
  // down chunks accumulated in TMEM at a time (multiple of 4); groups alternate between two
  // accumulator buffers, so the MMAs of one group overlap the epilogue's reading of the last
  const int gch = p.group_chunks;
  const int gst = gch / 4;         // down stages per group
  const uint32_t col_d2 = dec_col_d2(d);
  const int nu = U.n;
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
      const uint64_t pol = l2_policy_evict_first();
      for (int jb = 0; jb < 2 * nu && alive; ++jb) {
        const bool gu = job_is_gu(jb);
        const int u = job_unit(jb);
        const int e = U.e[u], j = U.j[u];
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
          // one contiguous 18 KB block of the decode pack: the stage's swizzled codes and its
          // four scale atoms (gate/up K block (q + rot) % nks1, or down chunks 4(q - nks1)..+3)
          const int qp = q < nks1 ? (q + rot) % nks1 : q;
          mbar_arrive_expect_tx(&full[st], kDecStageBytes);
          const uint8_t* ub =
              U.base ? U.base[u] : G.dec_pack + ((size_t)el * nt1 + j) * (nks1 + nks2) * kDecStageBytes;
          const uint8_t* src = ub + (size_t)qp * kDecStageBytes;
          if (kDecStreamEvictFirst) bulk_g2s_hint(sb, src, kDecStageBytes, &full[st], pol);
          else bulk_g2s(sb, src, kDecStageBytes, &full[st]);
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
      if (!p.xsf_loaded) {
        for (int a = who; a < d / 64; a += 2)
          tmem_cp_sf(tmem + kColX + 4 * a, sdesc_sf(smem_u32(xsf + (size_t)a * kDecAtom)));
        mma_commit(&xsf_ready);
      }
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
          if (q % gst == 0) {  // a new group: the epilogue has read this buffer's last group
            if (!mbar_wait(&acc2_empty[gc & 1], ((gc >> 1) & 1) ^ 1, &s_abort, p.status)) {
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
              mma_mxf4nvf4(tmem + col_d2 + (gc & 1) * gch * kDecDnN + kDecDnN * cl,
                           sdesc_kmajor(smem_u32(sb + 4096 * i), 256, kSwizzle32B),
                           sdesc_kmajor(smem_u32(hbuf), 0, kSwizzle32B), kDecIdescT, sf + 4 * i, hsf, 0u);
            }
            mma_commit(&empty[it % NST]);
            if (it < 40) TC_TRACE_AT(g_dec_trace, kEvMmaIssued, it);
          }
          if (q % gst == gst - 1 || q == nks2 - 1) {
            mma_commit(&acc2_full[gc & 1]);
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
    const float ts_x = p.ts_x;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t gc = 0;
    for (int jb = 0; jb < 2 * nu; ++jb) {
      const int u = job_unit(jb);
      const int e = U.e[u];
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
        for (int t = 0; t < kDecMaxT; ++t) wf[t] = U.w[u * kDecMaxT + t] * ts_o;
        for (int g0 = 0; g0 < nch; g0 += gch, ++gc) {
          const int ng = nch - g0 < gch ? nch - g0 : gch;
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&acc2_full[gc & 1], (gc >> 1) & 1, &s_abort, p.status) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          tc_fence_after();
          for (int cl = half; cl < ng; cl += 2) {
            uint32_t v[8];
            tmem_ld8(lane_base + col_d2 + (gc & 1) * gch * kDecDnN + kDecDnN * cl, v);
            tmem_ld_wait();
            // lanes 4i..4i+3 hold output rows 4i..4i+3 of the chunk: lane 4i adds the four
            // values of a token with one vector reduction (a quarter of the atomic operations)
            float* dst = p.out + (size_t)128 * (g0 + cl) + 32 * q4 + lane;
#pragma unroll
            for (int t = 0; t < kDecMaxT; ++t) {
              if (t < T && wf[t] != 0.0f) {  // the same for every lane of the warp
                const float a = __uint_as_float(v[t]) * wf[t];
                const float a1 = __shfl_down_sync(0xffffffffu, a, 1);
                const float a2 = __shfl_down_sync(0xffffffffu, a, 2);
                const float a3 = __shfl_down_sync(0xffffffffu, a, 3);
                if (ok && (lane & 3) == 0) red_add_v4(dst + (size_t)t * d, a, a1, a2, a3);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc2_empty[gc & 1]);
        }
        if (ew == 0 && lane == 0) TC_TRACE_AT(g_dec_trace, kEvDrainEnd, u);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TC_TRACE_AT(g_dec_trace, kEvExit, 0);
}

// ---------------------------------------------------------------- host-side sizing
inline size_t dec_fixed_smem(int d) {
  // x tiles, x scale atoms, two h tiles, the gate/up sums exchange, alignment slack
  return (size_t)(d / 256) * 1024 + (size_t)(d / 64) * kDecAtom + 2 * kDecHBytes + 128 * 8 * 4 + 1024;
}

// down chunks whose 16-column accumulators fit in TMEM next to everything else
inline int dec_group_chunks(int d) {
  const int avail = (512 - (int)dec_col_d2(d)) / kDecDnN / 2;  // two buffers
  const int g = avail & ~3;
  return g < d / 128 ? g : d / 128;
}

inline int dec_stages(int d, size_t extra = 0) {
  const size_t fixed = dec_fixed_smem(d) + extra;
  if (fixed >= kDecSmemBudget) return 0;
  const size_t n = (kDecSmemBudget - fixed) / kDecStageBytes;
  return n > (size_t)kDecMaxStages ? kDecMaxStages : (int)n;
}

inline size_t dec_smem_bytes(int d, size_t extra = 0) {
  return (size_t)dec_stages(d, extra) * kDecStageBytes + dec_fixed_smem(d) + extra;
}

// Shapes the core handles: T <= 8 tokens, d a multiple of 512 up to 4096, I a multiple of 64.
inline bool dec_shape_ok(int64_t T, int d, int I) {
  return T >= 1 && T <= kDecMaxT && d % 512 == 0 && I % 64 == 0 && d <= 4096 && I <= 16384 &&
         dec_stages(d) >= kDecMinStages && dec_group_chunks(d) >= 4;
}

}  // namespace moe
