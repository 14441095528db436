// Decode expert FFN (moe_expert_ffn with at most 8 tokens) on the tcgen05 tensor cores:
// the per-(expert, I-slice) unit core of dec_core.cuh, fed from the routing outputs of
// moe_route and the quantised activations of nvfp4_quantize_act.
//
// Two launches per call: a one-CTA preparation kernel zeroes y and lists the experts in use
// (the shared expert first) with each token's routing weight for each of them; then the
// persistent kernel (one CTA per SM) stages the activation codes into its shared-memory
// tiles, reads its own units from those lists and runs them.
#include "dec_core.cuh"

namespace moe {

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
__global__ void __launch_bounds__(kDecThreads, 1) ffn_dec_kernel(DecParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ DecBars bar;
  __shared__ int s_ue[kDecMaxUnits], s_uj[kDecMaxUnits];
  __shared__ float s_uw[kDecMaxUnits * kDecMaxT];
  const DecSmem sm = dec_smem(align1024(smem_raw), p.d, p.nstages);
  const int d = p.d, T = p.T, nt1 = p.I / 64;

  dec_init(bar, p.nstages);  // overlaps the previous kernel's tail
  RT_TRACE(g_prep_trace, 1, 0);
  MOE_PDL_PROLOGUE();
  RT_TRACE(g_prep_trace, 1, 1);

  // x codes -> the 8-row swizzled tiles (rows >= T zero); x scales -> atoms
  for (int i = threadIdx.x; i < kDecMaxT * (d / 32); i += blockDim.x) {
    const int t = i / (d / 32), c = i % (d / 32);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t < T) v = __ldg(reinterpret_cast<const uint4*>(p.xq_codes + (size_t)t * (d / 2)) + c);
    *reinterpret_cast<uint4*>(sm.xs + dec_xs_offset(t, c)) = v;
  }
  // scale words: token t's row as d/256 16-byte pieces; word kc goes to rows t, t + 8, t + 16,
  // t + 24 of atom kc (one load per piece: every CTA reads these same few lines)
  const int q4 = d / 256;
  if (threadIdx.x < kDecMaxT * q4) {
    const int t = threadIdx.x / q4, c4 = threadIdx.x % q4;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t < T) v = __ldg(reinterpret_cast<const uint4*>(p.xq_scales + (size_t)t * (d / kBlock)) + c4);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) dec_xsf_store(sm.xsf, 4 * c4 + w, t + 8 * r1, wv[w]);
  }
  // this CTA's units (blockIdx.x, blockIdx.x + gridDim.x, ...) from the preparation lists
  const int nunits = *p.nslots * nt1;
  int nu = (int)blockIdx.x < nunits ? (nunits - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  if (nu > kDecMaxUnits) {  // the host checks the worst case, so this does not happen
    if (threadIdx.x == 0) atomicExch(p.status, kStatusUnsupported);
    nu = kDecMaxUnits;
  }
  for (int i = threadIdx.x; i < nu * (kDecMaxT + 1); i += blockDim.x) {
    const int u = i / (kDecMaxT + 1), f = i % (kDecMaxT + 1);
    const int ug = (int)blockIdx.x + u * (int)gridDim.x;
    const int slot = ug / nt1;
    if (f == kDecMaxT) {
      s_ue[u] = p.slots[slot];
      s_uj[u] = ug % nt1;
    } else {
      s_uw[u * kDecMaxT + f] = p.slot_w[(size_t)slot * kDecMaxT + f];
    }
  }
  fence_proxy_async_smem();  // generic writes above are read by tcgen05 (async proxy)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  DecArgs a;
  a.routed = p.routed;
  a.shared = p.shared;
  a.has_shared = p.has_shared;
  a.E = p.E; a.d = d; a.I = p.I; a.T = T;
  a.nstages = p.nstages;
  a.group_chunks = p.group_chunks;
  a.ts_x = *p.xq_ts;
  a.xsf_loaded = 0;
  a.out = p.out;
  a.status = p.status;
  dec_run(a, sm, bar, DecUnits{nu, s_ue, s_uj, s_uw});
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(bar.tmem, 512);
  }
  RT_TRACE(g_prep_trace, 1, 2);
}

// ---------------------------------------------------------------- the decode pack
// Per unit (expert e, 64-wide slice j of I): d/256 gate/up stages, then d/512 down stages,
// each an 18 KB block that one bulk copy moves into a ring stage as the MMAs read it:
//   gate/up stage kb: 128 rows x 128 bytes (rows 0-63 gate rows 64j.., rows 64-127 up rows
//     64j..; bytes 128kb.. of each row) in the 128-byte swizzle (16-byte piece c of row r at
//     r*128 + ((c ^ (r % 8)) * 16)), then the 4 scale atoms 4kb..4kb+3 of (e, j);
//   down stage q: four 128-row chunks c = 4q..4q+3 (rows 128c.. of the down matrix, bytes
//     32j..32j+31), each 128 x 32 bytes in the 32-byte swizzle (piece c' of row r at
//     r*32 + ((c' ^ ((r / 4) % 2)) * 16)), then the scale atoms of those chunks for slice j.
// One thread per 16-byte piece of the output.
__global__ void pack_dec_kernel(const uint8_t* __restrict__ gu_codes, const uint8_t* __restrict__ dn_codes,
                                const uint8_t* __restrict__ gu_sf, const uint8_t* __restrict__ dn_sf, int E, int d,
                                int I, uint8_t* __restrict__ out) {
  const int nt1 = I / 64, nks1 = d / 256, nks2 = d / 512, nsu = nks1 + nks2;
  constexpr int kPieces = kDecStageBytes / 16;  // 1152 per stage, 1024 of them codes
  const size_t n = (size_t)E * nt1 * nsu * kPieces;
  for (size_t w = blockIdx.x * (size_t)blockDim.x + threadIdx.x; w < n; w += (size_t)gridDim.x * blockDim.x) {
    const int pc = (int)(w % kPieces);
    const size_t us = w / kPieces;
    const int q = (int)(us % nsu);
    const size_t unit = us / nsu;
    const int j = (int)(unit % nt1);
    const size_t e = unit / nt1;
    const uint8_t* src;
    if (pc < kDecBBytes / 16) {
      if (q < nks1) {
        const int r = pc / 8, c = (pc % 8) ^ (r % 8);
        const size_t row = e * 2 * I + (r < 64 ? 64 * j + r : I + 64 * j + r - 64);
        src = gu_codes + row * (d / 2) + 128 * q + 16 * c;
      } else {
        const int ch = 4 * (q - nks1) + pc / 256, r = (pc % 256) / 2, c = (pc % 2) ^ ((r / 4) % 2);
        src = dn_codes + (e * d + 128 * ch + r) * (I / 2) + 32 * j + 16 * c;
      }
    } else {
      const int a = (pc - kDecBBytes / 16) / 32, pa = (pc - kDecBBytes / 16) % 32;
      const size_t atom = q < nks1 ? (e * nt1 + j) * (d / 64) + 4 * q + a
                                   : (e * (d / 128) + 4 * (q - nks1) + a) * nt1 + j;
      src = (q < nks1 ? gu_sf : dn_sf) + atom * kDecAtom + 16 * pa;
    }
    *reinterpret_cast<uint4*>(out + w * 16) = *reinterpret_cast<const uint4*>(src);
  }
}

// ---------------------------------------------------------------- host side
size_t dec_pack_bytes(int E, int d, int I) {
  return (size_t)E * (I / 64) * (d / 256 + d / 512) * kDecStageBytes;
}

cudaError_t launch_pack_dec(const ExpertGroup& g, int E, int d, int I, const uint8_t* gu_sf_tiled,
                            const uint8_t* dn_sf_tiled, uint8_t* dec_pack, int num_sms, cudaStream_t st) {
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  pack_dec_kernel<<<num_sms * 4, 256, 0, st>>>(g.gu_codes, g.dn_codes, gu_sf_tiled, dn_sf_tiled, E, d, I, dec_pack);
  return cudaGetLastError();
}

namespace {
size_t a256d(size_t v) { return (v + 255) & ~(size_t)255; }
}  // namespace

// Units per CTA in the worst case (every routed assignment on its own expert) must fit the
// shared-memory unit table.
bool ffn_dec_supported(int64_t T, int d, int I, int mode, int E, int k, int has_shared, int grid) {
  if (mode != 0 || !dec_shape_ok(T, d, I) || grid <= 0) return false;
  const int64_t slots = (T * k < E ? T * k : E) + has_shared;
  const int64_t units = slots * (I / 64);
  return (units + grid - 1) / grid <= kDecMaxUnits;
}

size_t ffn_dec_ws_bytes(int E) { return 256 + a256d((size_t)(E + 1) * 4) + a256d((size_t)(E + 1) * kDecMaxT * 4); }

cudaError_t set_wait_limit_ffn_dec(unsigned long long ns) { return set_wait_limit_here(ns); }

cudaError_t init_ffn_dec_attributes() {
  // the largest configuration; launches use at most this much
  return cudaFuncSetAttribute(ffn_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecSmemBudget);
}

cudaError_t launch_ffn_dec(const FfnArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st) {
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
  cudaError_t e = launch_pdl(ffn_dec_prep_kernel, dim3(1), dim3(1024), 0, st, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(ffn_dec_kernel, dim3(num_sms), dim3(kDecThreads), dec_smem_bytes(a.d), st, p);
}

}  // namespace moe

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_dec(void* host, size_t bytes) { return trace_fetch(g_dec_trace, host, bytes); }
int64_t trace_fetch_prep(void* host, size_t bytes) { return trace_fetch(g_prep_trace, host, bytes); }
}  // namespace moe
#endif
