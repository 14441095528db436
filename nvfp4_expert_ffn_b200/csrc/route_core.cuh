// Device routines of the routing step shared by the routing kernels and the fused decode
// layer kernel: per-token top-k with renormalised weights, and the stable counting sort of a
// few hundred assignments by one warp.
//
// Basalt pages: "What Basalt changes in a Blackwell local inference stack", section
// "Experts can move without becoming free" (each token selects a subset of experts).
// Reading: top-k by logit with ties to the lower expert id; weights = softmax restricted to
// the top-k and renormalised, exp(l_j - l_max) / sum over the chosen k; the permutation is a
// stable counting sort of assignments a = t*k + j by expert.
#pragma once

#include "common.cuh"

namespace moe {

// float -> unsigned key with the same order; -0.0 and +0.0 get the same key (they are equal
// logits, so the lower expert id goes first)
MOE_DEV uint32_t ordered_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// One warp per token. Lane L holds logits L, L+32, ... (keys that order like the floats).
// Outputs (each may be NULL): idx_out / w_out in global memory, idx_smem / w_smem in shared
// memory, k entries each, in descending logit order, ties to the lower expert id. The logits
// are read with plain loads: a row written by other CTAs of the same kernel is visible once
// the grid barrier (acquire, fence, block barrier) has passed, and plain loads pipeline where
// ld.global.cg loads were measured to complete one after another.
//
// With a 64-word shared scratch and k <= 32 the selection first takes a threshold: the k-th
// largest of the 32 lane maxima. At least k logits reach it (those k maxima), so every logit
// of the top k is among the candidates at or above it; when there are at most 32 candidates
// (the usual case: about k + 2 for independent logits) they are gathered one per lane and
// each candidate's rank is counted against the other 31. Otherwise k rounds of a warp
// arg-max pick the winners one at a time, and only the winning lane rescans its entries.
// Both give the same picks in the same order.
// stamps (trace builds only): lane 0 records globaltimer after the loads, the threshold, the
// selection and the weights into stamps[0..3], and the SM cycles since the previous point
// (the first since entry) into stamps[4..7]
#ifdef MOE_TRACE
#define TOPK_STAMP(i)                                                    \
  do {                                                                   \
    if (stamps != nullptr && lane == 0) {                                \
      stamps[i] = globaltimer_ns_rc();                                   \
      const unsigned long long c_ = clock64();                           \
      stamps[4 + (i)] = c_ - clk_prev;                                   \
      clk_prev = c_;                                                     \
    }                                                                    \
  } while (0)
MOE_DEV unsigned long long globaltimer_ns_rc() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#else
#define TOPK_STAMP(i) do { } while (0)
#endif
template <int NPER>
MOE_DEV void topk_token(const float* __restrict__ row, int E, int k, int32_t* idx_out, float* w_out,
                        int* idx_smem = nullptr, float* w_smem = nullptr, uint32_t* scratch = nullptr,
                        unsigned long long* stamps = nullptr) {
  const int lane = threadIdx.x & 31;
#ifdef MOE_TRACE
  unsigned long long clk_prev = clock64();
#endif
  // every load first (entries past E read entry 0 and are masked below), so that they are
  // all in flight together, then the keys
  float val[NPER];
#pragma unroll
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    const float* src = row + (e < E ? e : 0);
    val[j] = *src;
  }
  uint32_t key[NPER];
#pragma unroll
  for (int j = 0; j < NPER; ++j) key[j] = lane + 32 * j < E ? ordered_key(val[j]) : 0u;  // 0: below every key
  // does (ka, ea) come before (kb, eb): larger key, or equal key and lower index
  auto before = [](uint32_t ka, int ea, uint32_t kb, int eb) { return ka > kb || (ka == kb && ea < eb); };
  uint32_t taken = 0;
  // this lane's best remaining entry: largest key, lowest index among equal keys
  auto local_best = [&](uint32_t& bk, int& be) {
    bk = 0u;
    be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPER; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && before(key[j], e, bk, be)) bk = key[j], be = e;
    }
  };
  uint32_t top_key = 0, my_key = 0;  // lane r < k ends with the r-th pick
  int my_e = 0;
  bool done = false;
  if (scratch != nullptr && k <= 32) {
    // the lane's largest key (a tree, so the steps do not wait on one another)
    uint32_t m[NPER];
#pragma unroll
    for (int j = 0; j < NPER; ++j) m[j] = key[j];
#pragma unroll
    for (int w = NPER / 2; w >= 1; w /= 2)
#pragma unroll
      for (int j = 0; j < w; ++j) m[j] = max(m[j], m[j + w]);
    const uint32_t lmax = m[0];
    TOPK_STAMP(0);
    // threshold: the k-th largest lane maximum = the smallest maximum with fewer than k
    // maxima strictly above it (lanes without entries hold 0, below every key)
    int above = 0;
#pragma unroll 8
    for (int o = 1; o < 32; ++o) above += __shfl_sync(0xffffffffu, lmax, (lane + o) & 31) > lmax ? 1 : 0;
    const uint32_t th = __reduce_min_sync(0xffffffffu, above < k ? lmax : 0xffffffffu);
    TOPK_STAMP(1);
    int c = 0;
#pragma unroll
    for (int j = 0; j < NPER; ++j) c += (lane + 32 * j < E && key[j] >= th) ? 1 : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= 32) {
      int pos = incl - c;
#pragma unroll
      for (int j = 0; j < NPER; ++j) {
        const int e = lane + 32 * j;
        if (e < E && key[j] >= th) {
          scratch[pos] = key[j];
          scratch[32 + pos] = (uint32_t)e;
          ++pos;
        }
      }
      __syncwarp();
      const uint32_t ck = lane < total ? scratch[lane] : 0u;
      const int ce = lane < total ? (int)scratch[32 + lane] : 0x7fffffff;
      __syncwarp();
      // rank of each candidate: keys strictly above it, then (only when two candidates share
      // a key) the equal keys of lower expert id
      int r = 0;
#pragma unroll 8
      for (int o = 1; o < 32; ++o) r += __shfl_sync(0xffffffffu, ck, (lane + o) & 31) > ck ? 1 : 0;
      const uint32_t same = __match_any_sync(0xffffffffu, ck);
      if (__any_sync(0xffffffffu, lane < total && __popc(same) > 1)) {
        for (int o = 1; o < 32; ++o) {
          const int src = (lane + o) & 31;
          const uint32_t ok = __shfl_sync(0xffffffffu, ck, src);
          const int oe = __shfl_sync(0xffffffffu, ce, src);
          r += (ok == ck && oe < ce) ? 1 : 0;
        }
      }
      if (lane < total && r < k) {
        scratch[r] = ck;
        scratch[32 + r] = (uint32_t)ce;
      }
      __syncwarp();
      if (lane < k) {
        my_key = scratch[lane];
        my_e = (int)scratch[32 + lane];
      }
      top_key = __shfl_sync(0xffffffffu, my_key, 0);
      __syncwarp();
      done = true;
    }
  }
  if (!done) {
    uint32_t lbk;
    int lbe;
    local_best(lbk, lbe);
    for (int r = 0; r < k; ++r) {
      const uint32_t mk = __reduce_max_sync(0xffffffffu, lbk);
      const int me = (int)__reduce_min_sync(0xffffffffu, lbk == mk ? (uint32_t)lbe : 0x7fffffffu);
      if (r == 0) top_key = mk;
      if (lane == r) my_key = mk, my_e = me;
      if ((me & 31) == lane) {
        taken |= 1u << (me >> 5);
        local_best(lbk, lbe);
      }
    }
  }
  TOPK_STAMP(2);
  auto key_to_float = [](uint32_t kk) {
    return __uint_as_float((kk & 0x80000000u) ? (kk & 0x7fffffffu) : ~kk);
  };
  const float ex = (lane < k) ? expf(key_to_float(my_key) - key_to_float(top_key)) : 0.0f;
  const float sum = warp_sum(ex);
  if (lane < k) {
    const float w = ex / sum;
    if (idx_out) idx_out[lane] = my_e;
    if (w_out) w_out[lane] = w;
    if (idx_smem) idx_smem[lane] = my_e;
    if (w_smem) w_smem[lane] = w;
  }
  TOPK_STAMP(3);
}

// scratch: NULL, or 64 words of shared memory for this warp
MOE_DEV void topk_dispatch(const float* row, int E, int k, int32_t* idx, float* w, int* idx_smem = nullptr,
                           float* w_smem = nullptr, uint32_t* scratch = nullptr,
                           unsigned long long* stamps = nullptr) {
  if (E <= 256) topk_token<8>(row, E, k, idx, w, idx_smem, w_smem, scratch, stamps);
  else if (E <= 512) topk_token<16>(row, E, k, idx, w, idx_smem, w_smem, scratch, stamps);
  else topk_token<32>(row, E, k, idx, w, idx_smem, w_smem, scratch, stamps);
}

// The permutation of n <= 32*k assignments by one warp, without block-wide barriers:
// histogram of sidx[0..n) (match_any leaders), warp scan of the counts, then a stable
// scatter in assignment order, 32 at a time. sh: E ints of shared scratch.
MOE_DEV void perm_small_warp(const int* sidx, int n, int E, int* sh, int32_t* counts, int32_t* offsets,
                             int32_t* sorted_assign, int32_t* assign_pos) {
  const int lane = threadIdx.x & 31;
  for (int e = lane; e < E; e += 32) sh[e] = 0;
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int a = base + lane;
    const int e = a < n ? sidx[a] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (a < n && (peers & ((1u << lane) - 1u)) == 0) sh[e] += __popc(peers);
    __syncwarp();
  }
  // exclusive scan of sh[0..E): lane L owns the contiguous range [L*per, (L+1)*per)
  const int per = (E + 31) / 32;
  int local = 0;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < E) local += sh[e];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - local;
  for (int i = 0; i < per; ++i) {
    const int e = lane * per + i;
    if (e < E) {
      const int c = sh[e];
      counts[e] = c;
      offsets[e] = run;
      sh[e] = run;
      run += c;
    }
  }
  if (lane == 31) offsets[E] = incl;
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int a = base + lane;
    const int e = a < n ? sidx[a] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (a < n) {
      const int pos = sh[e] + rank;
      sorted_assign[pos] = a;
      assign_pos[a] = pos;
    }
    __syncwarp();
    if (a < n && (peers >> lane) == 1u) sh[e] += __popc(peers);  // highest lane of its group
    __syncwarp();
  }
}

}  // namespace moe
