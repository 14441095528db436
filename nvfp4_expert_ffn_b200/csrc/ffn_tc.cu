// Expert SwiGLU FFN on the tcgen05 tensor cores: block-scaled NVFP4 x NVFP4 grouped GEMMs.
//
// The MoE layer of the Basalt pages ("What Basalt changes in a Blackwell local inference
// stack", section "Experts can move without becoming free": each token runs a subset of
// experts; "Basalt" project page, "Engines": routed experts are NVFP4) computes, per
// expert, h = silu(x Wg^T) * (x Wu^T), h re-quantised to NVFP4 (tensor scale 1), then
// o = h Wd^T, and y += w * o. Here both products are tcgen05.mma kind::mxf4nvf4 with the
// E4M3 block scales staged into tensor memory: the tensor core consumes E2M1 codes and
// scales directly, nothing is decoded on the CUDA cores.
//
// Two launches per call (three for more than 64 tokens):
//   1. tc_schedule_kernel: CTA 0 lays out 128-row m-tiles over each expert's tokens (the
//      shared expert is slot E) and zeroes the per-m-tile completion counters; the other
//      CTAs zero y in accumulate mode.
//   1b. (more than 64 tokens) tc_row_gather_kernel: copies each m-tile's activation rows
//      and scale bytes into contiguous per-m-tile buffers, read once per phase-1 tile.
//   2. tc_ffn_kernel (persistent, one CTA per SM, warp-specialised):
//        warp 0    producer: for few tokens, gathers each m-tile's activation rows
//                  straight from the quantised activations with TMA tile::gather4 (their
//                  scale bytes with cp.async into 128x4 scale atoms); for many, one TMA
//                  box of the gathered rows per stage; TMA-loads weight tiles and their
//                  pre-tiled scale atoms, into a 4-stage shared-memory ring
//        warp 1    TMEM allocation and the MMA issuer (single thread)
//        warps 2-9 epilogue: TMEM -> registers; two warps per TMEM lane quarter, each
//                  taking half of the tile's columns
//      phase-1 tiles (m-tile, 64 gate + 64 up rows): SwiGLU and NVFP4 h quantisation in
//      the epilogue, h written to the workspace; phase-2 tiles (m-tile, 128 output rows)
//      wait until all phase-1 tiles of their m-tile are done (bounded wait; their weights
//      are already streaming), then the down GEMM, whose epilogue stages each token row of
//      w * o in shared memory and adds it into y with a bulk reduction
//      (cp.reduce.async.bulk .add.f32), or stores o.
//      Accumulators are double-buffered in TMEM so an epilogue overlaps the next tile.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tmap.h"
#include "trace.cuh"

namespace moe {

constexpr int kTcStages = 4;
constexpr int kTileM = 128;                // tokens per m-tile (MMA M)
constexpr int kTileN = 128;                // weight rows per tile (MMA N)
constexpr int kStageK = 256;               // elements of K per pipeline stage (4 MMAs)
constexpr int kAtom = 512;                 // bytes of one 128-row x 4-block scale atom
constexpr int kABytes = kTileM * kStageK / 2;   // 16 KB
constexpr int kBBytes = kTileN * kStageK / 2;   // 16 KB
constexpr int kSfBytes = 4 * kAtom;             // 2 KB per operand per stage
constexpr int kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
constexpr int kEpiWarps = 8;
constexpr int kTcThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiRowFloats = 36;              // staged row stride: 144 B keeps rows 16 B aligned and
                                               // spreads 8 consecutive rows over all 32 banks
constexpr int kEpiStageBytes = 32 * kEpiRowFloats * 4;  // one warp's 32 rows x 32 float32 columns
constexpr int kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_mxf4nvf4(kTileM, kTileN);
constexpr int kSmallT = 64;  // up to this many tokens the producer copies activation scales itself



TC_TRACE_ARRAY(g_tc_trace)

struct TcParams {
  // schedule and gathered rows (workspace)
  int32_t* n_mtiles;
  int32_t* mt_expert;
  int32_t* mt_valid;
  int32_t* mt_first;  // local row index (within its expert) of the m-tile's first row
  int32_t* done1;
  int32_t* row_token;
  float* row_weight;
  int32_t* row_slot;
  uint8_t* a1;        // [rows_cap][d/2] x codes gathered per m-tile row (large T), or NULL
  uint8_t* sfa1;      // [m][d/64][512] x scale atoms gathered per m-tile (large T), or NULL
  uint8_t* h_codes;   // [rows_cap][I/2]
  uint8_t* sfa2;      // [m][I/64][512]
  int max_m;
  // inputs
  const uint8_t* xq_codes;
  const uint8_t* xq_scales;
  const float* xq_ts;
  const uint16_t* x_bf16;  // static input scales: rows are quantised from here (else NULL)
  const float* in_gu;      // [E + 1] static activation scale of each expert (shared at E)
  const float* in_dn;      // [E + 1] static h scale of each expert, or NULL (1.0)
  const int32_t* offsets;
  const int32_t* sorted_assign;
  const float* topk_w;
  ExpertGroup routed, shared;
  int has_shared;
  int E, d, I, T, k, mode;
  float* out;
  float* shared_out;
  int32_t* status;
};

// ---------------------------------------------------------------- 1. schedule
MOE_DEV void schedule_body(const TcParams& p) {
  __shared__ int tmp[32];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int nslots = p.E + (p.has_shared ? 1 : 0);
  for (int e0 = 0; e0 < nslots; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    int cnt = 0;
    if (e < p.E) cnt = p.offsets[e + 1] - p.offsets[e];
    else if (e < nslots) cnt = p.T;
    const int nm = (cnt + kTileM - 1) / kTileM;
    int total;
    const int base = block_exclusive_scan(nm, tmp, &total) + carry;
    for (int i = 0; i < nm; ++i) {
      const int m = base + i;
      if (m < p.max_m) {
        p.mt_expert[m] = e;
        p.mt_valid[m] = min(kTileM, cnt - i * kTileM);
        p.mt_first[m] = i * kTileM;
        p.done1[m] = 0;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) *p.n_mtiles = min(carry, p.max_m);
}

__global__ void __launch_bounds__(1024) tc_schedule_kernel(TcParams p) {
  MOE_PDL_PROLOGUE();
  if (blockIdx.x == 0) {
    schedule_body(p);
    return;
  }
  // accumulate mode: y is summed into by the FFN kernel, so it starts at zero
  const size_t n4 = (size_t)p.T * p.d / 4;
  float4* o4 = reinterpret_cast<float4*>(p.out);
  for (size_t i = (blockIdx.x - 1) * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)(gridDim.x - 1) * blockDim.x)
    o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------- 1b. row gather (large T)
// With many rows per m-tile, every phase-1 tile of an m-tile would gather the same rows
// again, 4 rows per TMA request; instead the rows' d/2 code bytes are copied into a
// contiguous [m-tile row][d/2] buffer (one TMA box per stage then), their d/16 scale bytes
// into the m-tile's scale atoms, and each row's (token, weight, output slot) is written.
// A warp takes 32 rows of one m-tile: lane r resolves row r's token through the expert's
// offset and the sorted assignment, so the 32 rows' chains of dependent index loads overlap;
// the warp then copies the rows kGatherRows at a time, all their loads issued before the
// stores.
constexpr int kGatherRows = 8;
constexpr int kGatherQuantMaxD = 2048;  // static input scales need the m-tile kernel: d <= its limit

// QUANT: the static-input-scale form (rows quantised from p.x_bf16), a kernel of its own so
// that its registers do not lower the plain copy's occupancy.
template <bool QUANT>
__global__ void __launch_bounds__(256, QUANT ? 2 : 3) tc_row_gather_kernel(TcParams p) {
  MOE_PDL_PROLOGUE();
  const int n_m = *p.n_mtiles;
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int d = p.d;
  for (int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < n_m * (kTileM / 32); g += nw) {
    const int m = g / (kTileM / 32), r0 = 32 * (g % (kTileM / 32));
    const int valid = p.mt_valid[m];
    if (r0 >= valid) continue;
    const int e = p.mt_expert[m];
    const int nr = min(32, valid - r0);
    const int r = r0 + lane;
    int t = 0;
    if (lane < nr) {
      const int i = p.mt_first[m] + r;
      int slot = -1;
      float wgt = 1.0f;
      t = i;
      if (e < p.E) {
        const int q = p.offsets[e] + i;
        const int a = p.sorted_assign[q];
        t = a / p.k;
        wgt = p.topk_w[a];
        slot = q;
      }
      const size_t prow = (size_t)m * kTileM + r;
      p.row_token[prow] = t;
      p.row_weight[prow] = wgt;
      p.row_slot[prow] = slot;
    }
    if constexpr (QUANT) {
      // static input scales: each token's bf16 row quantised with its expert's own tensor
      // scale. Lane l takes 16-element blocks l, l + 32, ...: its 8 code bytes go to the
      // gathered row, its scale byte into the m-tile's scale atom.
      // (d <= kGatherQuantMaxD: at most kQBlk blocks per lane; the loads of two rows go out first)
      constexpr int kQBlk = kGatherQuantMaxD / kBlock / 32;
      const float ts = p.in_gu[e];
      const int nblk = d / kBlock;
      for (int j0 = 0; j0 < nr; j0 += 2) {
        uint4 raw[2][kQBlk][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int tj = __shfl_sync(0xffffffffu, t, (j0 + u) & 31);
          const uint4* xsrc = reinterpret_cast<const uint4*>(p.x_bf16 + (size_t)tj * d);
#pragma unroll
          for (int b = 0; b < kQBlk; ++b) {
            const int blk = lane + 32 * b;
            const bool ld = j0 + u < nr && blk < nblk;
            raw[u][b][0] = ld ? __ldg(xsrc + 2 * blk) : make_uint4(0u, 0u, 0u, 0u);
            raw[u][b][1] = ld ? __ldg(xsrc + 2 * blk + 1) : make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rj = r0 + j0 + u;
          if (j0 + u >= nr) break;
          uint2* cdst = reinterpret_cast<uint2*>(p.a1 + ((size_t)m * kTileM + rj) * (d / 2));
#pragma unroll
          for (int b = 0; b < kQBlk; ++b) {
            const int blk = lane + 32 * b;
            if (blk >= nblk) break;
            const uint4 lo = raw[u][b][0], hi = raw[u][b][1];
            const uint32_t wv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
            float v[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              v[2 * i] = __uint_as_float(wv[i] << 16);
              v[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
            }
            uint2 cw;
            const uint32_t sb = quantize_block16(v, ts, &cw);
            cdst[blk] = cw;
            p.sfa1[((size_t)m * (d / 64) + blk / 4) * kAtom + (rj % 32) * 16 + (rj / 32) * 4 + blk % 4] = (uint8_t)sb;
          }
        }
      }
    } else {
      for (int j0 = 0; j0 < nr; j0 += kGatherRows) {
        int tj[kGatherRows];
#pragma unroll
        for (int u = 0; u < kGatherRows; ++u) tj[u] = __shfl_sync(0xffffffffu, t, (j0 + u) & 31);
        if (p.a1) {
          for (int c = lane; c < d / 32; c += 32) {
            uint4 v[kGatherRows];
#pragma unroll
            for (int u = 0; u < kGatherRows; ++u)
              if (j0 + u < nr) v[u] = __ldg(reinterpret_cast<const uint4*>(p.xq_codes + (size_t)tj[u] * (d / 2)) + c);
#pragma unroll
            for (int u = 0; u < kGatherRows; ++u)
              if (j0 + u < nr) reinterpret_cast<uint4*>(p.a1 + ((size_t)m * kTileM + r0 + j0 + u) * (d / 2))[c] = v[u];
          }
        }
        for (int kc = lane; kc < d / 64; kc += 32) {
          uint32_t v[kGatherRows];
#pragma unroll
          for (int u = 0; u < kGatherRows; ++u)
            if (j0 + u < nr) v[u] = __ldg(reinterpret_cast<const uint32_t*>(p.xq_scales + (size_t)tj[u] * (d / kBlock)) + kc);
#pragma unroll
          for (int u = 0; u < kGatherRows; ++u) {
            const int rj = r0 + j0 + u;
            if (j0 + u < nr)
              *reinterpret_cast<uint32_t*>(p.sfa1 + ((size_t)m * (d / 64) + kc) * kAtom + (rj % 32) * 16 + (rj / 32) * 4) = v[u];
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- pack weight scales
// gate/up: [E][I/64][d/64][512], atom row r < 64 -> gate row 64j + r, else up row 64j + r - 64
// down:    [E][d/128][I/64][512], atom row r -> down row 128j + r
// Within an atom, row r = 32*r1 + r0 and block kb of the 4-block chunk sit at r0*16+r1*4+kb.
__global__ void pack_sf_kernel(const uint8_t* __restrict__ gu_scales, const uint8_t* __restrict__ dn_scales,
                               int E, int d, int I, uint8_t* __restrict__ gu_t, uint8_t* __restrict__ dn_t) {
  const size_t n_gu = (size_t)E * (I / 64) * (d / 64) * 128;  // 32-bit words
  const size_t n_dn = (size_t)E * (d / 128) * (I / 64) * 128;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < n_gu + n_dn;
       w += (size_t)gridDim.x * blockDim.x) {
    if (w < n_gu) {
      const size_t atom = w / 128;
      const int slot = (int)(w % 128);  // r0 * 4 + r1
      const int r = (slot % 4) * 32 + slot / 4;
      const int kc = (int)(atom % (d / 64));
      const int j = (int)((atom / (d / 64)) % (I / 64));
      const size_t e = atom / ((size_t)(d / 64) * (I / 64));
      const int row = r < 64 ? 64 * j + r : I + 64 * j + (r - 64);
      const uint32_t v = *reinterpret_cast<const uint32_t*>(gu_scales + (e * 2 * I + row) * (d / kBlock) + 4 * kc);
      *reinterpret_cast<uint32_t*>(gu_t + atom * kAtom + (slot / 4) * 16 + (slot % 4) * 4) = v;
    } else {
      const size_t ww = w - n_gu;
      const size_t atom = ww / 128;
      const int slot = (int)(ww % 128);
      const int r = (slot % 4) * 32 + slot / 4;
      const int kc = (int)(atom % (I / 64));
      const int j = (int)((atom / (I / 64)) % (d / 128));
      const size_t e = atom / ((size_t)(I / 64) * (d / 128));
      const int row = 128 * j + r;
      const uint32_t v = *reinterpret_cast<const uint32_t*>(dn_scales + (e * d + row) * (I / kBlock) + 4 * kc);
      *reinterpret_cast<uint32_t*>(dn_t + atom * kAtom + (slot / 4) * 16 + (slot % 4) * 4) = v;
    }
  }
}

// ---------------------------------------------------------------- 3. persistent FFN kernel
struct TcMaps {
  CUtensorMap xg;    // x codes [T][d/2], one-row boxes for tile::gather4
  CUtensorMap a1;    // gathered x codes [rows_cap][d/2] (large T)
  CUtensorMap a2;    // h codes           [rows_cap][I/2]
  CUtensorMap b1;    // routed gate/up    {d/2, I, 2, E}
  CUtensorMap b1s;   // shared gate/up    {d/2, I, 2, 1}
  CUtensorMap b2;    // routed down       {I/2, d, E}
  CUtensorMap b2s;   // shared down       {I/2, d, 1}
};

struct TileInfo {
  int phase, m, j;
};

MOE_DEV TileInfo decode_tile(int t, int n_m, int nt1, int nt2) {
  TileInfo ti;
  if (t < n_m * nt1) {
    ti.phase = 1;
    ti.m = t / nt1;
    ti.j = t % nt1;
  } else {
    const int u = t - n_m * nt1;
    ti.phase = 2;
    ti.m = u / nt2;
    ti.j = u % nt2;
  }
  return ti;
}

__global__ void __launch_bounds__(kTcThreads, 1) tc_ffn_kernel(const __grid_constant__ TcMaps maps, TcParams p) {
  TC_TRACE_DECL
  MOE_PDL_PROLOGUE();
  TC_TRACE_BEGIN(g_tc_trace);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kTcStages], empty[kTcStages], acc_full[2], acc_empty[2], final_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, I = p.I;
  const int nt1 = I / 64, nt2 = d / kTileN;
  const int nks1 = d / kStageK, nks2 = I / kStageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // producer lane 0 (expect_tx) + 32 cp.async arrivals
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(&final_bar, 1);
    fence_barrier_init();
    s_abort = 0;
    prefetch_tensormap(p.a1 ? &maps.a1 : &maps.xg);
    prefetch_tensormap(&maps.a2);
    prefetch_tensormap(&maps.b1);
    prefetch_tensormap(&maps.b2);
  }
  if (warp == 1) tmem_alloc(&s_tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_m = *p.n_mtiles;
  const int total = n_m * (nt1 + nt2);
  if (threadIdx.x == 0) TC_TRACE_AT(g_tc_trace, kEvSetupDone, n_m);

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // All 32 lanes: lane 0 waits on barriers, arms them and issues weight / h copies; each
    // lane gathers 4 activation rows (rows 4*lane .. 4*lane+3 of the m-tile) and copies
    // their scale bytes, then signals the stage's barrier when its cp.async copies land.
    uint32_t it = 0;
    bool alive = true;
    // Token ids of the 4 rows this lane gathers, for a phase-1 tile; the loads for the next
    // tile are started before the current tile's copies are issued, so their latency hides.
    auto load_rowtok = [&](int tt, int (&rt)[4]) {
      const TileInfo tn = decode_tile(tt, n_m, nt1, nt2);
      if (tt >= total || tn.phase != 1 || p.a1) return;
      const int en = p.mt_expert[tn.m];
      const int vn = p.mt_valid[tn.m];
      const int first = p.mt_first[tn.m];
      const int off = en == p.E ? 0 : p.offsets[en];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * lane + i;
        rt[i] = r < vn ? (en == p.E ? first + r : p.sorted_assign[off + first + r]) : -1;
      }
    };
    int next_tok[4] = {-1, -1, -1, -1};
    load_rowtok(blockIdx.x, next_tok);
    for (int t = blockIdx.x; t < total && alive; t += gridDim.x) {
      const TileInfo ti = decode_tile(t, n_m, nt1, nt2);
      const int e = p.mt_expert[ti.m];
      const bool sh = (e == p.E);
      const int eloc = sh ? 0 : e;
      const int valid = p.mt_valid[ti.m];
      const ExpertGroup& G = sh ? p.shared : p.routed;
      const int nks = ti.phase == 1 ? nks1 : nks2;
      if (lane == 0) TC_TRACE_AT(g_tc_trace, kEvProdTile, t);
      int rowtok[4] = {0, 0, 0, 0};
      int ngather = 0;
      if (ti.phase == 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i)  // assignment ids -> token ids (the shared expert's are tokens)
          rowtok[i] = next_tok[i] < 0 ? -1 : (sh ? next_tok[i] : next_tok[i] / p.k);
        const int tok0 = __shfl_sync(0xffffffffu, rowtok[0], 0);  // row 0 always exists
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (rowtok[i] < 0) rowtok[i] = tok0;  // padding rows of a gather group repeat a real row
        ngather = (valid + 3) / 4;
      }
      load_rowtok(t + gridDim.x, next_tok);
      const int nq = (valid + 31) / 32;
      const uint32_t stage_tx =
          ti.phase == 1 ? (p.a1 ? (uint32_t)(kABytes + kBBytes + 2 * kSfBytes)
                                : (uint32_t)(ngather * 512 + kBBytes + kSfBytes))
                        : (uint32_t)(nq * 4096 + kBBytes + 2 * kSfBytes);
      auto wait_empty = [&](uint32_t itx) -> bool {
        int ok = 1;
        if (lane == 0)
          ok = mbar_wait(&empty[itx % kTcStages], ((itx / kTcStages) & 1) ^ 1, &s_abort, p.status) ? 1 : 0;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
      };
      auto arm_and_issue_b = [&](int ks, uint32_t s) {
        if (lane != 0) return;
        uint8_t* st = smem + (size_t)s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], stage_tx);
        if (ti.phase == 1) {
          tma_load_4d(st + kABytes, sh ? &maps.b1s : &maps.b1, &full[s], ks * 128, 64 * ti.j, 0, eloc);
          bulk_g2s(st + kABytes + kBBytes + kSfBytes,
                   G.gu_sf_tiled + (((size_t)eloc * nt1 + ti.j) * (d / 64) + 4 * ks) * kAtom, kSfBytes, &full[s]);
        } else {
          tma_load_3d(st + kABytes, sh ? &maps.b2s : &maps.b2, &full[s], ks * 128, kTileN * ti.j, eloc);
          bulk_g2s(st + kABytes + kBBytes + kSfBytes,
                   G.dn_sf_tiled + (((size_t)eloc * nt2 + ti.j) * (I / 64) + 4 * ks) * kAtom, kSfBytes, &full[s]);
        }
      };
      auto issue_a = [&](int ks, uint32_t s) {
        uint8_t* st = smem + (size_t)s * kStageBytes;
        uint8_t* sSFA = st + kABytes + kBBytes;
        if (ti.phase == 1 && p.a1) {
          if (lane == 0) {
            tma_load_2d(st, &maps.a1, &full[s], ks * 128, ti.m * kTileM);
            bulk_g2s(sSFA, p.sfa1 + ((size_t)ti.m * (d / 64) + 4 * ks) * kAtom, kSfBytes, &full[s]);
          }
        } else if (ti.phase == 1) {
          if (4 * lane < valid) {
            tma_gather4(st + 4 * lane * 128, &maps.xg, &full[s], ks * 128, rowtok[0], rowtok[1], rowtok[2],
                        rowtok[3]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 4 * lane + i;
              if (r < valid) {
                const uint8_t* src = p.xq_scales + (size_t)rowtok[i] * (d / kBlock) + 16 * ks;
#pragma unroll
                for (int kc = 0; kc < 4; ++kc)
                  cp_async4(sSFA + kc * kAtom + (r % 32) * 16 + (r / 32) * 4, src + 4 * kc);
              }
            }
          }
        } else if (lane == 0) {
          for (int q = 0; q < nq; ++q)
            tma_load_2d(st + q * 4096, &maps.a2, &full[s], ks * 128, ti.m * kTileM + 32 * q);
          bulk_g2s(sSFA, p.sfa2 + ((size_t)ti.m * (I / 64) + 4 * ks) * kAtom, kSfBytes, &full[s]);
        }
        cp_async_arrive(&full[s]);
      };
      int ks0 = 0;
      if (ti.phase == 2) {
        // the down weights do not depend on phase 1: start streaming them, then wait
        // until every phase-1 tile of this m-tile has written its h rows
        const int npre = nks < kTcStages ? nks : kTcStages;
        for (int ks = 0; ks < npre && alive; ++ks) {
          if (!wait_empty(it + ks)) alive = false;
          else arm_and_issue_b(ks, (it + ks) % kTcStages);
        }
        if (!alive) break;
        int ok = 1;
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu(p.done1 + ti.m) < nt1) {
            if (s_abort) {
              ok = 0;
              break;
            }
            if (globaltimer_ns() - t0 > wait_limit_ns()) {
              s_abort = 1;
              atomicExch(p.status, kStatusTimeout);
              ok = 0;
              break;
            }
          }
          fence_proxy_async_global();
          TC_TRACE_AT(g_tc_trace, kEvProdDone1, t);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        for (int ks = 0; ks < npre; ++ks) issue_a(ks, (it + ks) % kTcStages);
        it += npre;
        ks0 = npre;
      }
      for (int ks = ks0; ks < nks; ++ks, ++it) {
        const uint32_t s = it % kTcStages;
        if (!wait_empty(it)) {
          alive = false;
          break;
        }
        arm_and_issue_b(ks, s);
        issue_a(ks, s);
      }
    }
    // no copies left in flight: the last issued stage of each slot has landed
    if (lane == 0) {
      for (uint32_t j = (it > (uint32_t)kTcStages ? it - kTcStages : 0); j < it; ++j) {
        volatile int no_abort = 0;
        mbar_wait(&full[j % kTcStages], (j / kTcStages) & 1, &no_abort, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      for (int t = blockIdx.x; t < total && !s_abort; t += gridDim.x, ++tc) {
        const TileInfo ti = decode_tile(t, n_m, nt1, nt2);
        const int buf = tc & 1;
        if (!mbar_wait(&acc_empty[buf], ((tc >> 1) & 1) ^ 1, &s_abort, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * kTileN;
        const int nks = ti.phase == 1 ? nks1 : nks2;
        bool ok = true;
        for (int ks = 0; ks < nks; ++ks, ++it) {
          const int s = it % kTcStages;
          if (!mbar_wait(&full[s], (it / kTcStages) & 1, &s_abort, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (ks == 0) TC_TRACE_AT(g_tc_trace, kEvMmaFirst, t);
          fence_proxy_async_smem();  // scale bytes arrived through cp.async (generic proxy)
          const uint8_t* st = smem + (size_t)s * kStageBytes;
          const uint32_t aA = smem_u32(st), aB = smem_u32(st + kABytes);
          const uint32_t aSFA = smem_u32(st + kABytes + kBBytes), aSFB = aSFA + kSfBytes;
          const uint32_t sfa_col = tmem + 256 + 32 * s, sfb_col = sfa_col + 16;
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            tmem_cp_sf(sfa_col + 4 * kc, sdesc_sf(aSFA + kAtom * kc));
            tmem_cp_sf(sfb_col + 4 * kc, sdesc_sf(aSFB + kAtom * kc));
          }
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            mma_mxf4nvf4(d_tmem, sdesc_sw128(aA + 32 * kc), sdesc_sw128(aB + 32 * kc), kIdesc,
                         sfa_col + 4 * kc, sfb_col + 4 * kc, (ks | kc) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        TC_TRACE_AT(g_tc_trace, kEvMmaLast, t);
        mma_commit(&acc_full[buf]);
      }
      // all issued tensor-core work has completed before TMEM is released
      mma_commit(&final_bar);
      volatile int no_abort = 0;
      mbar_wait(&final_bar, 0, &no_abort, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    // one thread waits for the accumulator; a named barrier publishes data and decision
    __shared__ int s_epi_go[2];  // by tile parity: a slow warp never reads the next tile's value
    const int q = warp & 3;            // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;  // which half of the tile's columns this warp takes
    const int row = 32 * q + lane;     // accumulator row = token row of the m-tile
    const float ts_x = *p.xq_ts;
    // two 4 KB staging buffers per warp for the bulk reductions of phase 2
    float* stage_f = reinterpret_cast<float*>(smem + (size_t)kTcStages * kStageBytes) +
                     (size_t)(warp - 2) * 2 * (kEpiStageBytes / 4);
    uint32_t tc = 0, nbulk = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tc) {
      const TileInfo ti = decode_tile(t, n_m, nt1, nt2);
      const int buf = tc & 1;
      if (warp == 2 && lane == 0)
        s_epi_go[buf] = mbar_wait(&acc_full[buf], (tc >> 1) & 1, &s_abort, p.status) ? 1 : 0;
      named_bar_sync(2, 32 * kEpiWarps);
      if (!s_epi_go[buf]) break;
      if (warp == 2 && lane == 0) TC_TRACE_AT(g_tc_trace, kEvEpiStart, t);
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + buf * kTileN;
      const int e = p.mt_expert[ti.m];
      const bool sh = (e == p.E);
      const int eloc = sh ? 0 : e;
      const ExpertGroup& G = sh ? p.shared : p.routed;
      const bool valid = row < p.mt_valid[ti.m];
      const size_t prow = (size_t)ti.m * kTileM + row;
      if (ti.phase == 1) {
        // columns 32*half .. +31 of gate (0..63) and of up (64..127): 32 h values
        const float sg = G.gu_ts[2 * eloc] * ts_x, su = G.gu_ts[2 * eloc + 1] * ts_x;
        uint32_t g[32], u[32];
        tmem_ld32(taddr + 32 * half, g);
        tmem_ld32(taddr + 64 + 32 * half, u);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
        // SwiGLU and the NVFP4 quantisation of h (tensor scale 1), IEEE float32 steps as in the
        // activation quantiser
        uint32_t packed[8];
        uint32_t sbytes = 0;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gv = __uint_as_float(g[16 * b + i]) * sg, uv = __uint_as_float(u[16 * b + i]) * su;
            h[i] = __fdiv_rn(gv, 1.0f + expf(-gv)) * uv;
          }
          uint2 cw;
          sbytes |= quantize_block16(h, 1.0f, &cw) << (8 * b);
          packed[4 * b] = cw.x;      // elements 0-7 of the block
          packed[4 * b + 2] = cw.y;  // elements 8-15
        }
        if (valid) {
          // 32 codes = 16 bytes at h columns 64j + 32*half
          *reinterpret_cast<uint4*>(p.h_codes + prow * (I / 2) + 32 * ti.j + 16 * half) =
              make_uint4(packed[0], packed[2], packed[4], packed[6]);
          *reinterpret_cast<uint16_t*>(p.sfa2 + ((size_t)ti.m * (I / 64) + ti.j) * kAtom + (row % 32) * 16 +
                                       (row / 32) * 4 + 2 * half) = (uint16_t)sbytes;
        }
        if (!p.a1 && ti.j == 0 && half == 0 && valid) {
          // token, routing weight and output slot of this row, for the phase-2 epilogue
          const int i = p.mt_first[ti.m] + row;
          int tokr = i, slotr = -1;
          float wr = 1.0f;
          if (!sh) {
            const int q = p.offsets[e] + i;
            const int asg = p.sorted_assign[q];
            tokr = asg / p.k;
            wr = p.topk_w[asg];
            slotr = q;
          }
          p.row_token[prow] = tokr;
          p.row_weight[prow] = wr;
          p.row_slot[prow] = slotr;
        }
        // publish h of this tile: generic writes -> visible to other CTAs' TMA reads
        fence_proxy_async_global();
        __threadfence();
        named_bar_sync(2, 32 * kEpiWarps);
        if (warp == 2 && lane == 0) {
          atomicAdd(p.done1 + ti.m, 1);
          TC_TRACE_AT(g_tc_trace, kEvEpiEnd, t);
        }
      } else {
        const float ts_o = G.dn_ts[eloc];  // h tensor scale is 1
        int tok = 0, slot = 0;
        float wgt = 0.0f;
        if (valid) {  // written by another CTA's phase-1 epilogue: read through L2
          tok = __ldcg(p.row_token + prow);
          wgt = __ldcg(p.row_weight + prow);
          slot = __ldcg(p.row_slot + prow);
        }
        const float f = p.mode == 0 ? wgt * ts_o : ts_o;
        uint32_t v[2][32];
        tmem_ld32(taddr + 64 * half, v[0]);
        tmem_ld32(taddr + 64 * half + 32, v[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
#pragma unroll
        for (int c = 0; c < 2; ++c, ++nbulk) {
          float* sb = stage_f + (nbulk & 1) * (kEpiStageBytes / 4);
          bulk_wait_read<1>();  // the buffer used two chunks ago has been read
          __syncwarp();
          float4* rowp = reinterpret_cast<float4*>(sb + kEpiRowFloats * lane);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            rowp[i] = make_float4(__uint_as_float(v[c][4 * i]) * f, __uint_as_float(v[c][4 * i + 1]) * f,
                                  __uint_as_float(v[c][4 * i + 2]) * f, __uint_as_float(v[c][4 * i + 3]) * f);
          fence_proxy_async_smem();
          if (valid) {
            const int n0 = kTileN * ti.j + 64 * half + 32 * c;
            if (p.mode == 0)
              bulk_reduce_add_f32(p.out + (size_t)tok * d + n0, rowp, 128);
            else
              bulk_s2g((sh ? p.shared_out + (size_t)tok * d : p.out + (size_t)slot * d) + n0, rowp, 128);
          }
          bulk_commit();
        }
        if (warp == 2 && lane == 0) TC_TRACE_AT(g_tc_trace, kEvEpiEnd, t);
      }
    }
    bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) TC_TRACE_AT(g_tc_trace, kEvExit, 0);
}

// ---------------------------------------------------------------- 4. m-tile kernel
// One job = the whole FFN of one m-tile (up to 128 rows of one expert), run by one CTA:
//   gate/up: I/128 tiles of N = 256 weight rows (gate and up rows of two 64-row slices of I,
//            in the order the scale atoms hold them), K = d; SwiGLU and the NVFP4
//            quantisation of h in the epilogue, h written into this CTA's shared memory in
//            the layout the down GEMM reads as its token operand;
//   down:    d/256 tiles of 256 output rows, K = I, computed transposed (the two 128-row
//            weight boxes as A, that h tile as the N = 128 B operand); the epilogue adds
//            w * o into y with reductions from registers (or stores o).
// The activation scale atoms of the m-tile (K = d) and then those of h (K = I) stay in TMEM
// for all of the job's tiles, so a K = 64 step needs only the two weight scale copies next to
// its N = 256 MMA (each tcgen05.cp takes the tensor pipe about as long as a 128-column MMA).
// One N = 256 accumulator (TMEM has no room for a second one beside the scales): the
// epilogue takes its columns into registers first and releases it before its own math; 16
// epilogue warps (four per TMEM lane quarter, 64 columns each) keep that math short.
// y of every token the call covers receives about k + 1 float32 reductions, 128 contiguous
// bytes of one row per warp instruction (the down tiles are computed transposed).
constexpr int kMtN = 256;
constexpr int kMtStages = 3;
constexpr int kMtEpiWarps = 16;
constexpr int kMtThreads = 64 + 32 * kMtEpiWarps;
constexpr int kMtABytes = kTileM * kStageK / 2;      // 16 KB: gathered activation rows
constexpr int kMtBBytes = kMtN * kStageK / 2;        // 32 KB: weight rows
constexpr int kMtSfbBytes = 8 * kAtom;               // 4 KB: two atoms per K = 64 step
constexpr int kMtStageBytes = kMtABytes + kMtBBytes + kMtSfbBytes;
constexpr int kMtColSfa = 256, kMtColSfb = 384;      // TMEM columns (accumulator at 0)
constexpr int kMtMaxD = 2048, kMtMaxI = 768;
static_assert(kMtMaxD <= kGatherQuantMaxD, "the row gather quantises rows of up to kGatherQuantMaxD");
constexpr size_t kMtSmemMax = 225 * 1024;  // + 2 KB of static shared memory = the 227 KB limit
constexpr uint32_t kMtIdesc = idesc_mxf4nvf4(kTileM, kMtN);
// Down tiles computed transposed, D[output column][token] (weights the A operand, two M = 128
// halves of a 256-column tile; h the N = 128 B operand): each thread of the epilogue then
// holds one output column for 32 tokens, and a warp's reduction covers 32 consecutive floats
// (128 bytes) of one token's row of y.
constexpr uint32_t kMtIdescDownT = idesc_mxf4nvf4(128, kTileM);
constexpr bool kMtPregather = true;  // above 64 tokens: one TMA box of pre-gathered rows per stage

__host__ __device__ inline size_t mt_h_bytes(int I) { return (size_t)(I / kStageK) * kMtABytes; }
__host__ __device__ inline size_t mt_smem_bytes(int d, int I) {
  return (size_t)kMtStages * kMtStageBytes + mt_h_bytes(I) + (size_t)(I / 64) * kAtom + (size_t)(d / 64) * kAtom + 1024;
}

// trace id of tile `t` (0..nt1-1 gate/up, then down) of this CTA's job `jc` (first 2 jobs only)
#define MT_TRACE(ev, jc, t)                                        \
  do {                                                             \
    if ((jc) < 2) TC_TRACE_AT(g_tc_trace, ev, (jc) * 64 + (t));    \
  } while (0)

__global__ void __launch_bounds__(kMtThreads, 1) tc_ffn_mt_kernel(const __grid_constant__ TcMaps maps, TcParams p) {
  TC_TRACE_DECL
  MOE_PDL_PROLOGUE();
  TC_TRACE_BEGIN(g_tc_trace);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t full[kMtStages], empty[kMtStages], acc_full, acc_empty, sfa_full, sfa_empty, h_ready,
      final_bar;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_epi_go[2];
  __shared__ int s_orow[kTileM];  // this job's rows: output row (-1: padding) and factor, for the
  __shared__ float s_f[kTileM];   // transposed down read-out

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, I = p.I;
  const int nt1 = I / 128, nt2 = d / kMtN;      // tiles per job
  const int nks1 = d / kStageK, nks2 = I / kStageK;
  // CTAs that work on the same expert at the same time visit its weight tiles and K stages in
  // orders rotated by their index, so that they do not all request the same lines from L2 at
  // once (the sums do not depend on the order)
  const int rj = blockIdx.x % nt1, rn = blockIdx.x % nt2;
  const int rk1 = (blockIdx.x / nt1) % nks1, rk2 = (blockIdx.x / nt2) % nks2;
  uint8_t* const ring = smem;
  uint8_t* const htile = smem + (size_t)kMtStages * kMtStageBytes;   // [I/256][128 rows][128 B]
  uint8_t* const hsf = htile + mt_h_bytes(I);                         // [I/64][512]
  uint8_t* const xsf = hsf + (size_t)(I / 64) * kAtom;                // [d/64][512]

  if (threadIdx.x == 0) {
    for (int st = 0; st < kMtStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, kMtEpiWarps);
    mbar_init(&sfa_full, 1);
    mbar_init(&sfa_empty, 1);
    mbar_init(&h_ready, 1);
    mbar_init(&final_bar, 1);
    fence_barrier_init();
    s_abort = 0;
    prefetch_tensormap(p.a1 ? &maps.a1 : &maps.xg);
    prefetch_tensormap(&maps.b1);
    prefetch_tensormap(&maps.b2);
  }
  if (warp == 1) tmem_alloc(&s_tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_m = *p.n_mtiles;
  if (threadIdx.x == 0) TC_TRACE_AT(g_tc_trace, kEvSetupDone, n_m);

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    uint32_t it = 0, jc = 0;
    bool alive = true;
    auto wait_empty = [&](uint32_t itx) -> bool {
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait(&empty[itx % kMtStages], ((itx / kMtStages) & 1) ^ 1, &s_abort, p.status) ? 1 : 0;
      return __shfl_sync(0xffffffffu, ok, 0) != 0;
    };
    for (int m = blockIdx.x; m < n_m && alive; m += gridDim.x, ++jc) {
      const int e = p.mt_expert[m];
      const bool sh = (e == p.E);
      const int eloc = sh ? 0 : e;
      const ExpertGroup& G = sh ? p.shared : p.routed;
      const int valid = p.mt_valid[m];
      const int ngather = (valid + 3) / 4;
      // the 4 rows this lane gathers (padding rows of a group repeat the m-tile's first row)
      int rowtok[4];
      const int tok0 = p.row_token[(size_t)m * kTileM];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 4 * lane + i;
        rowtok[i] = r < valid ? p.row_token[(size_t)m * kTileM + r] : tok0;
      }
      // the m-tile's activation scale atoms (pre-gathered) for the whole of K = d
      if (lane == 0) {
        if (!mbar_wait(&sfa_empty, (jc & 1) ^ 1, &s_abort, p.status)) alive = false;
        else {
          mbar_arrive_expect_tx(&sfa_full, (uint32_t)(d / 64) * kAtom);
          bulk_g2s(xsf, p.sfa1 + (size_t)m * (d / 64) * kAtom, (uint32_t)(d / 64) * kAtom, &sfa_full);
        }
      }
      alive = __shfl_sync(0xffffffffu, alive ? 1 : 0, 0) != 0;
      // gate/up stages: activation rows by gather4, two 64-row gate+up boxes, their scales
      for (int jq = 0; jq < nt1 && alive; ++jq) {
        const int j = (jq + rj) % nt1;
        for (int kq = 0; kq < nks1; ++kq, ++it) {
          const int ks = (kq + rk1) % nks1;
          const uint32_t st = it % kMtStages;
          if (!wait_empty(it)) {
            alive = false;
            break;
          }
          if (kq == 0 && lane == 0) MT_TRACE(kEvProdTile, jc, jq);
          uint8_t* sb = ring + (size_t)st * kMtStageBytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[st], (uint32_t)((p.a1 ? kMtABytes : ngather * 512) + kMtBBytes + kMtSfbBytes));
            if (p.a1) tma_load_2d(sb, &maps.a1, &full[st], ks * 128, m * kTileM);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              tma_load_4d(sb + kMtABytes + hh * (kMtBBytes / 2), sh ? &maps.b1s : &maps.b1, &full[st], ks * 128,
                          64 * (2 * j + hh), 0, eloc);
              bulk_g2s(sb + kMtABytes + kMtBBytes + hh * (kMtSfbBytes / 2),
                       G.gu_sf_tiled + (((size_t)eloc * (I / 64) + 2 * j + hh) * (d / 64) + 4 * ks) * kAtom,
                       kMtSfbBytes / 2, &full[st]);
            }
          }
          __syncwarp();
          if (!p.a1 && lane < ngather)
            tma_gather4(sb + 4 * lane * 128, &maps.xg, &full[st], ks * 128, rowtok[0], rowtok[1], rowtok[2],
                        rowtok[3]);
        }
      }
      // down stages: two 128-row boxes of output rows and their scales
      for (int nq = 0; nq < nt2 && alive; ++nq) {
        const int n = (nq + rn) % nt2;
        for (int kq = 0; kq < nks2; ++kq, ++it) {
          const int ks = (kq + rk2) % nks2;
          const uint32_t st = it % kMtStages;
          if (!wait_empty(it)) {
            alive = false;
            break;
          }
          if (kq == 0 && lane == 0) MT_TRACE(kEvProdTile, jc, nt1 + nq);
          uint8_t* sb = ring + (size_t)st * kMtStageBytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[st], (uint32_t)(kMtBBytes + kMtSfbBytes));
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              tma_load_3d(sb + kMtABytes + hh * (kMtBBytes / 2), sh ? &maps.b2s : &maps.b2, &full[st], ks * 128,
                          kMtN * n + 128 * hh, eloc);
              bulk_g2s(sb + kMtABytes + kMtBBytes + hh * (kMtSfbBytes / 2),
                       G.dn_sf_tiled + (((size_t)eloc * (d / 128) + 2 * n + hh) * (I / 64) + 4 * ks) * kAtom,
                       kMtSfbBytes / 2, &full[st]);
            }
          }
          __syncwarp();
        }
      }
    }
    // no copy may still be landing when the CTA exits
    if (lane == 0) {
      for (uint32_t jj = (it > (uint32_t)kMtStages ? it - kMtStages : 0); jj < it; ++jj) {
        volatile int no_abort = 0;
        mbar_wait(&full[jj % kMtStages], (jj / kMtStages) & 1, &no_abort, p.status);
      }
      if (jc > 0) {
        volatile int no_abort = 0;
        mbar_wait(&sfa_full, (jc - 1) & 1, &no_abort, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0, jc = 0;
      bool ok = true;
      int tix = 0;  // tile index within the job, for the trace
      auto tile = [&](int nks, bool phase1) -> bool {
        if (!mbar_wait(&acc_empty, (tc & 1) ^ 1, &s_abort, p.status)) return false;
        tc_fence_after();
        MT_TRACE(kEvMmaSlot, jc, tix);
        const int rk = phase1 ? rk1 : rk2;
        for (int kq = 0; kq < nks; ++kq, ++it) {
          const int ks = (kq + rk) % nks;  // the producer's order
          const uint32_t st = it % kMtStages;
          if (!mbar_wait(&full[st], (it / kMtStages) & 1, &s_abort, p.status)) return false;
          tc_fence_after();
          if (kq == 0) MT_TRACE(kEvMmaFirst, jc, tix);
          const uint8_t* sb = ring + (size_t)st * kMtStageBytes;
          const uint32_t aB = smem_u32(sb + kMtABytes);
          const uint32_t aA = phase1 ? smem_u32(sb) : smem_u32(htile + (size_t)ks * kMtABytes);
          const uint32_t aS = smem_u32(sb + kMtABytes + kMtBBytes);
          const uint32_t sfb = tmem + kMtColSfb + 32 * st;
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            tmem_cp_sf(sfb + 8 * kc, sdesc_sf(aS + kAtom * kc));                        // rows 0-127
            tmem_cp_sf(sfb + 8 * kc + 4, sdesc_sf(aS + kMtSfbBytes / 2 + kAtom * kc));  // rows 128-255
          }
          if (phase1) {
#pragma unroll
            for (int kc = 0; kc < 4; ++kc)
              mma_mxf4nvf4(tmem, sdesc_sw128(aA + 32 * kc), sdesc_sw128(aB + 32 * kc), kMtIdesc,
                           tmem + kMtColSfa + 4 * (4 * ks + kc), sfb + 8 * kc, (kq | kc) ? 1u : 0u);
          } else {
            // output rows 0-127 and 128-255 of the tile (the two boxes) as A, h as B, into
            // accumulator columns 0-127 and 128-255; the weight scales are the A scales
#pragma unroll
            for (int kc = 0; kc < 4; ++kc)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
                mma_mxf4nvf4(tmem + 128 * hh, sdesc_sw128(aB + hh * (kMtBBytes / 2) + 32 * kc),
                             sdesc_sw128(aA + 32 * kc), kMtIdescDownT, sfb + 8 * kc + 4 * hh,
                             tmem + kMtColSfa + 4 * (4 * ks + kc), (kq | kc) ? 1u : 0u);
          }
          mma_commit(&empty[st]);
        }
        mma_commit(&acc_full);
        MT_TRACE(kEvMmaLast, jc, tix);
        ++tc;
        ++tix;
        return true;
      };
      for (int m = blockIdx.x; m < n_m && ok; m += gridDim.x, ++jc) {
        tix = 0;
        // activation scale atoms of the m-tile -> TMEM for the job's gate/up tiles
        if (!mbar_wait(&sfa_full, jc & 1, &s_abort, p.status)) break;
        tc_fence_after();
        for (int a = 0; a < d / 64; ++a) tmem_cp_sf(tmem + kMtColSfa + 4 * a, sdesc_sf(smem_u32(xsf + (size_t)a * kAtom)));
        mma_commit(&sfa_empty);
        for (int j = 0; j < nt1 && ok; ++j) ok = tile(nks1, true);
        if (!ok) break;
        // h (written by the epilogue into shared memory) and its scale atoms -> TMEM
        if (!mbar_wait(&h_ready, jc & 1, &s_abort, p.status)) break;
        tc_fence_after();
        MT_TRACE(kEvProdDone1, jc, 0);
        for (int a = 0; a < I / 64; ++a) tmem_cp_sf(tmem + kMtColSfa + 4 * a, sdesc_sf(smem_u32(hsf + (size_t)a * kAtom)));
        for (int n = 0; n < nt2 && ok; ++n) ok = tile(nks2, false);
      }
      // all issued tensor-core work has completed before TMEM is released
      mma_commit(&final_bar);
      volatile int no_abort = 0;
      mbar_wait(&final_bar, 0, &no_abort, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    // warp w takes TMEM lane quarter q = w % 4 (m-tile rows 32q..32q+31) and column quarter
    // cq = (w - 2) / 4: accumulator columns [64cq, 64cq + 64) in the down tiles; in the
    // gate/up tiles the gate and up columns of 32 h columns (see below). One thread waits; a
    // named barrier publishes its decision.
    const int ew = warp - 2;
    const int q = warp & 3;
    const int cq = ew >> 2;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const float ts_call = p.x_bf16 ? 1.0f : *p.xq_ts;  // per-call activation scale
    uint32_t tc = 0, jc = 0;
    bool go = true;
    int tix = 0;
    auto wait_acc = [&]() -> bool {
      if (ew == 0 && lane == 0) {
        s_epi_go[tc & 1] = mbar_wait(&acc_full, tc & 1, &s_abort, p.status) ? 1 : 0;
        MT_TRACE(kEvEpiStart, jc, tix);
      }
      named_bar_sync(2, 32 * kMtEpiWarps);
      const bool g = s_epi_go[tc & 1] != 0;
      tc_fence_after();
      return g;
    };
    // two 32-column groups of this thread's row, at columns c0 and c1
    auto drain = [&](uint32_t c0, uint32_t c1, uint32_t (&v)[2][32]) {
      tmem_ld32(lane_base + c0, v[0]);
      tmem_ld32(lane_base + c1, v[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty);
      if (ew == 0 && lane == 0) MT_TRACE(kEvDrainEnd, jc, tix);
      ++tc;
    };
    for (int m = blockIdx.x; m < n_m && go; m += gridDim.x, ++jc) {
      tix = 0;
      const int e = p.mt_expert[m];
      const bool sh = (e == p.E);
      const int eloc = sh ? 0 : e;
      const ExpertGroup& G = sh ? p.shared : p.routed;
      const bool valid = row < p.mt_valid[m];
      const size_t prow = (size_t)m * kTileM + row;
      // ---- gate/up tiles: SwiGLU and NVFP4 h into the shared-memory h tile. Tile j holds gate
      // rows of slice s = 2j + (cq >> 1) at columns 128(cq >> 1) .. +63 and its up rows 64
      // columns later; this thread takes h columns 32(cq & 1) .. +31 of that slice.
      // tensor scales of this expert's activations and h: static per expert, or the call's
      // activation scale and 1.0
      const float ts_x = p.x_bf16 ? p.in_gu[e] : ts_call;
      const float ts_h = p.in_dn ? p.in_dn[e] : 1.0f;
      const float sg = G.gu_ts[2 * eloc] * ts_x, su = G.gu_ts[2 * eloc + 1] * ts_x;
      const uint32_t cg = 128 * (cq >> 1) + 32 * (cq & 1);
      for (int jq = 0; jq < nt1 && go; ++jq) {
        const int j = (jq + rj) % nt1;
        if (!(go = wait_acc())) break;
        uint32_t v[2][32];
        drain(cg, cg + 64, v);
        uint32_t packed[4];
        uint32_t sbytes = 0;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gv = __uint_as_float(v[0][16 * b + i]) * sg;
            const float uv = __uint_as_float(v[1][16 * b + i]) * su;
            h[i] = __fdiv_rn(gv, 1.0f + expf(-gv)) * uv;
          }
          uint2 cw;
          sbytes |= quantize_block16(h, ts_h, &cw) << (8 * b);
          packed[2 * b] = cw.x;
          packed[2 * b + 1] = cw.y;
        }
        if (!valid) packed[0] = packed[1] = packed[2] = packed[3] = sbytes = 0u;
        // 16 code bytes at h column hc: K stage hc / 256, 16-byte piece (hc % 256) / 32 of the
        // row (128-byte swizzle: piece c of row r at r*128 + (c ^ (r % 8))*16)
        const int hc = 128 * j + 64 * (cq >> 1) + 32 * (cq & 1);
        uint8_t* hrow = htile + (size_t)(hc / kStageK) * kMtABytes + (size_t)row * 128;
        const int pc = (hc % kStageK) / 32;
        *reinterpret_cast<uint4*>(hrow + ((pc ^ (row & 7)) * 16)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        // the two scale bytes: blocks (hc % 64) / 16 and the next of atom hc / 64
        *reinterpret_cast<uint16_t*>(hsf + (size_t)(hc / 64) * kAtom + (row % 32) * 16 + (row / 32) * 4 +
                                     (hc % 64) / 16) = (uint16_t)sbytes;
        if (ew == 0 && lane == 0) MT_TRACE(kEvEpiEnd, jc, tix);
        ++tix;
      }
      if (!go) break;
      // h complete: visible to the tensor core (async proxy), then released to the MMA issuer
      fence_proxy_async_smem();
      named_bar_sync(2, 32 * kMtEpiWarps);
      if (ew == 0 && lane == 0) mbar_arrive(&h_ready);
      // ---- down tiles: w * o added into y (or o stored)
      const float ts_o = G.dn_ts[eloc] * ts_h;
      int orow = -1;  // output row of this thread's m-tile row (lane = row), -1 if padding
      float f = 0.0f;
      if (valid) {
        const int tok = p.row_token[prow];
        orow = (p.mode == 0 || sh) ? tok : p.row_slot[prow];
        f = p.mode == 0 ? p.row_weight[prow] * ts_o : ts_o;
      }
      float* const obase = (p.mode != 0 && sh) ? p.shared_out : p.out;
      // D[output column][token]: thread = output column 32q + lane of each 128-column half,
      // its 32 registers = tokens 32cq .. 32cq + 31 (their output rows and factors from
      // shared memory, published by the first tile's barrier)
      if (cq == 0) {
        s_orow[row] = orow;
        s_f[row] = f;
      }
      for (int nq = 0; nq < nt2 && go; ++nq) {
        const int n = (nq + rn) % nt2;
        if (!(go = wait_acc())) break;
        uint32_t v[2][32];
        tmem_ld32(lane_base + 32 * cq, v[0]);
        tmem_ld32(lane_base + 128 + 32 * cq, v[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty);
        if (ew == 0 && lane == 0) MT_TRACE(kEvDrainEnd, jc, tix);
        ++tc;
        const int ocol = kMtN * n + 32 * q + lane;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int orr = s_orow[32 * cq + j];
          const float fr = s_f[32 * cq + j];
          if (orr >= 0) {
            float* o = obase + (size_t)orr * d + ocol;
            const float a0 = __uint_as_float(v[0][j]) * fr, a1 = __uint_as_float(v[1][j]) * fr;
            if (p.mode == 0) {
              red_add_f32(o, a0);
              red_add_f32(o + 128, a1);
            } else {
              o[0] = a0;
              o[128] = a1;
            }
          }
        }
        if (ew == 0 && lane == 0) MT_TRACE(kEvEpiEnd, jc, tix);
        ++tix;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) TC_TRACE_AT(g_tc_trace, kEvExit, 0);
}

// ---------------------------------------------------------------- host side
namespace {

size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

struct TcLayout {
  int max_m;
  size_t rows_cap;
  size_t off_hdr, off_expert, off_valid, off_first, off_done, off_tok, off_w, off_slot, off_a1, off_sfa1, off_h,
      off_sfa2, total;
};

bool mt_supported(int d, int I) {
  return d <= kMtMaxD && I <= kMtMaxI && d % kStageK == 0 && I % kStageK == 0 && mt_smem_bytes(d, I) <= kMtSmemMax;
}

TcLayout tc_layout(int64_t T, int d, int E, int k, int I, bool per_expert_rows = false) {
  TcLayout L;
  const int64_t n = T * k;
  L.max_m = (int)((n + kTileM - 1) / kTileM + (n < E ? n : E) + (T + kTileM - 1) / kTileM + 2);
  L.rows_cap = (size_t)L.max_m * kTileM;
  size_t o = 0;
  L.off_hdr = o; o += 256;
  L.off_expert = o; o += a256((size_t)L.max_m * 4);
  L.off_valid = o; o += a256((size_t)L.max_m * 4);
  L.off_first = o; o += a256((size_t)L.max_m * 4);
  L.off_done = o; o += a256((size_t)L.max_m * 4);
  L.off_tok = o; o += a256(L.rows_cap * 4);
  L.off_w = o; o += a256(L.rows_cap * 4);
  L.off_slot = o; o += a256(L.rows_cap * 4);
  // the previous kernel gathers activation rows for large T; the m-tile kernel needs only the
  // rows' scale atoms (every T)
  const bool mt = mt_supported(d, I);
  const bool big = T > kSmallT;
  L.off_a1 = o; o += ((big && (!mt || kMtPregather)) || per_expert_rows) ? a256(L.rows_cap * (d / 2)) : 0;
  L.off_sfa1 = o; o += (big || mt) ? a256(L.rows_cap * (d / kBlock)) : 0;
  L.off_h = o; o += a256(L.rows_cap * (I / 2));
  L.off_sfa2 = o; o += a256(L.rows_cap * (I / kBlock));
  L.total = o;
  return L;
}

}  // namespace

size_t ffn_tc_ws_bytes(int64_t T, int d, int E, int k, int I) {
  if (d % kStageK || I % kStageK) return 0;
  return tc_layout(T, d, E, k, I).total;
}

size_t ffn_tc_static_ws_bytes(int64_t T, int d, int E, int k, int I) {
  if (!mt_supported(d, I)) return 0;
  return tc_layout(T, d, E, k, I, true).total;
}

bool ffn_tc_supported(int d, int I) { return d % kStageK == 0 && I % kStageK == 0 && d <= 16384 && I <= 16384; }

size_t ffn_tc_smem_bytes() { return (size_t)kTcStages * kStageBytes + (size_t)kEpiWarps * 2 * kEpiStageBytes + 1024; }

cudaError_t set_wait_limit_ffn_tc(unsigned long long ns) { return set_wait_limit_here(ns); }

cudaError_t init_ffn_tc_attributes() {
  cudaError_t e = cudaFuncSetAttribute(tc_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ffn_tc_smem_bytes());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(tc_ffn_mt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMtSmemMax);
}

cudaError_t launch_pack_sf(const ExpertGroup& g, int E, int d, int I, uint8_t* gu_t, uint8_t* dn_t, int num_sms,
                           cudaStream_t st) {
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  pack_sf_kernel<<<num_sms * 4, 256, 0, st>>>(g.gu_scales, g.dn_scales, E, d, I, gu_t, dn_t);
  return cudaGetLastError();
}


cudaError_t launch_ffn_tc(const FfnArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st) {
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  const bool per_expert = a.x_bf16 != nullptr;  // static input scales: rows quantised per expert
  const TcLayout L = tc_layout(a.T, a.d, a.E, a.k, a.I, per_expert);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  TcParams p;
  p.n_mtiles = reinterpret_cast<int32_t*>(w + L.off_hdr);
  p.mt_expert = reinterpret_cast<int32_t*>(w + L.off_expert);
  p.mt_valid = reinterpret_cast<int32_t*>(w + L.off_valid);
  p.mt_first = reinterpret_cast<int32_t*>(w + L.off_first);
  p.done1 = reinterpret_cast<int32_t*>(w + L.off_done);
  p.row_token = reinterpret_cast<int32_t*>(w + L.off_tok);
  p.row_weight = reinterpret_cast<float*>(w + L.off_w);
  p.row_slot = reinterpret_cast<int32_t*>(w + L.off_slot);
  const bool mt = mt_supported(a.d, a.I);
  if (per_expert && !mt) return cudaErrorInvalidValue;  // the caller checks the shapes
  p.a1 = ((a.T > kSmallT && (!mt || kMtPregather)) || per_expert) ? w + L.off_a1 : nullptr;
  p.sfa1 = (a.T > kSmallT || mt) ? w + L.off_sfa1 : nullptr;
  p.h_codes = w + L.off_h;
  p.sfa2 = w + L.off_sfa2;
  p.max_m = L.max_m;
  p.xq_codes = a.xq_codes;
  p.xq_scales = a.xq_scales;
  p.xq_ts = a.xq_ts;
  p.x_bf16 = a.x_bf16;
  p.in_gu = a.in_gu;
  p.in_dn = a.in_dn;
  p.offsets = a.offsets;
  p.sorted_assign = a.sorted_assign;
  p.topk_w = a.topk_w;
  p.routed = a.routed;
  p.shared = a.shared;
  p.has_shared = a.has_shared;
  p.E = a.E; p.d = a.d; p.I = a.I; p.T = a.T; p.k = a.k; p.mode = a.mode;
  p.out = a.out;
  p.shared_out = a.shared_out;
  p.status = status;

  TcMaps maps;
  const int d = a.d, I = a.I;
  if (a.xq_codes) {
    cuuint64_t dims[2] = {(cuuint64_t)(d / 2), (cuuint64_t)a.T};
    cuuint64_t strides[1] = {(cuuint64_t)(d / 2)};
    cuuint32_t box[2] = {128, 1};
    if ((e = encode_u8(&maps.xg, a.xq_codes, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
  if (p.a1) {
    cuuint64_t dims[2] = {(cuuint64_t)(d / 2), (cuuint64_t)L.rows_cap};
    cuuint64_t strides[1] = {(cuuint64_t)(d / 2)};
    cuuint32_t box[2] = {128, 128};
    if ((e = encode_u8(&maps.a1, p.a1, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
    if (!a.xq_codes) maps.xg = maps.a1;  // not read: the rows come from a1
  } else {
    maps.a1 = maps.xg;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)(I / 2), (cuuint64_t)L.rows_cap};
    cuuint64_t strides[1] = {(cuuint64_t)(I / 2)};
    cuuint32_t box[2] = {128, 32};
    if ((e = encode_u8(&maps.a2, p.h_codes, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
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
    cuuint64_t dims2[3] = {(cuuint64_t)(I / 2), (cuuint64_t)d, (cuuint64_t)E};
    cuuint64_t str2[2] = {(cuuint64_t)(I / 2), (cuuint64_t)d * (I / 2)};
    cuuint32_t box2[3] = {128, 128, 1};
    if ((e = encode_u8(m2, g.dn_codes, 3, dims2, str2, box2, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess) return e;
  }
  int zc = 0;
  if (a.mode == 0) {
    const size_t n4 = (size_t)a.T * a.d / 4;
    zc = (int)((n4 + 4095) / 4096);
    if (zc > num_sms) zc = num_sms;
  }
  if ((e = launch_pdl(tc_schedule_kernel, dim3(1 + zc), dim3(1024), 0, st, p)) != cudaSuccess) return e;
  if (mt) {
    // m-tile kernel: rows gathered once per m-tile, then one job per m-tile
    e = per_expert ? launch_pdl(tc_row_gather_kernel<true>, dim3(num_sms * 8), dim3(256), 0, st, p)
                   : launch_pdl(tc_row_gather_kernel<false>, dim3(num_sms * 8), dim3(256), 0, st, p);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_ffn_mt_kernel, dim3(num_sms), dim3(kMtThreads), mt_smem_bytes(a.d, a.I), st, maps, p);
  }
  if (p.a1 && (e = launch_pdl(tc_row_gather_kernel<false>, dim3(num_sms * 8), dim3(256), 0, st, p)) != cudaSuccess)
    return e;
  return launch_pdl(tc_ffn_kernel, dim3(num_sms), dim3(kTcThreads), ffn_tc_smem_bytes(), st, maps, p);
}

}  // namespace moe

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_tc(void* host, size_t bytes) { return trace_fetch(g_tc_trace, host, bytes); }
}  // namespace moe
#endif
