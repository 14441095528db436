// Internal launchers (host side) of the sm_100a kernels. Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <string>

namespace moe {

// Kernels enqueued by this library in this process (host side; see moe_launch_count).
extern std::atomic<uint64_t> g_launch_count;

// Launch with programmatic dependent launch allowed: the kernel may start while the
// previous kernel on the stream drains; every kernel of this library calls
// griddepcontrol.wait before it reads anything a predecessor wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// As launch_pdl, and cooperative: the launch fails instead of starting unless every CTA of
// the grid can be resident at once (kernels that wait at grid-wide barriers). With `win`,
// the launch also carries that L2 access-policy window.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_coop(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t st, const cudaAccessPolicyWindow* win, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (win) {
    attr[2].id = cudaLaunchAttributeAccessPolicyWindow;
    attr[2].val.accessPolicyWindow = *win;
    cfg.numAttrs = 3;
  }
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// per-thread detail string returned by moe_last_error()
void set_last_error(const std::string& msg);

// Device-side view of one expert group (natural NVFP4 layout, see moe_nvfp4.h).
struct ExpertGroup {
  const uint8_t* gu_codes;
  const uint8_t* gu_scales;
  const float* gu_ts;
  const uint8_t* dn_codes;
  const uint8_t* dn_scales;
  const float* dn_ts;
  const uint8_t* gu_sf_tiled;
  const uint8_t* dn_sf_tiled;
  const uint8_t* dec_pack;  // [E][I/64][d/256 + d/512][18432]: decode stages (moe_pack_experts)
  const uint8_t* hot_pack;  // [n_hot][I/64][d/256 + d/512][18432]: copies of the hot experts' units
  const int32_t* hot_slot;  // [E]: slot in hot_pack, or -1
  int n_hot;
};

struct FfnArgs {
  const uint8_t* xq_codes;
  const uint8_t* xq_scales;
  const float* xq_ts;
  // static per-expert input scales (tcgen05 m-tile path only): the bf16 activations, which
  // each expert's rows are quantised from with in_gu[e], and h's scale in_dn[e]; NULL for the
  // per-call quantised activations above and h scale 1
  const uint16_t* x_bf16 = nullptr;
  const float* in_gu = nullptr;
  const float* in_dn = nullptr;
  int T, d, I, E, k;
  ExpertGroup routed, shared;
  int has_shared;
  const int32_t* offsets;
  const int32_t* sorted_assign;
  const float* topk_w;
  int mode;  // 0 accumulate, 1 per-assignment
  float* out;
  float* shared_out;
  // workspace: NVFP4 h of every (assignment slot, h-block); slots 0..T*k-1 are sorted
  // positions of routed assignments, T*k + t is token t of the shared expert
  uint8_t* h_codes;   // [(T*k + T)][I/2]
  uint8_t* h_scales;  // [(T*k + T)][I/16]
};

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int cols, const float* ts_in,
                            uint8_t* codes, uint8_t* scales, float* ts_out, void* ws, int num_sms,
                            cudaStream_t st);

cudaError_t launch_route(const uint16_t* x, int T, int d, const float* Wr, const float* br, int E,
                         int k, int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                         int32_t* sorted_assign, int32_t* assign_pos, void* ws, int num_sms,
                         int32_t* status, cudaStream_t st);
// tensor-core router (many tokens): approximate bf16-split logits, then an exact top-k
bool router_tc_supported(int64_t T, int d, int E);
size_t router_tc_ws_bytes(int d, int E);
cudaError_t launch_router_tc(const uint16_t* x, int T, int d, const float* Wr, const float* br, int E, int k,
                             int32_t* topk_idx, float* topk_w, float* logits, uint16_t* w2, int num_sms,
                             int32_t* status, cudaStream_t st);
size_t route_ws_bytes(int64_t T, int d, int E, int k);

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* counts,
                           int32_t* offsets, int32_t* sorted_assign, int32_t* assign_pos, void* ws,
                           cudaStream_t st);
size_t permute_ws_bytes(int64_t T, int k, int E);

cudaError_t launch_hist(const int32_t* counts, int E, int64_t* cum, int32_t* rank_out, int reset,
                        cudaStream_t st);

cudaError_t launch_ffn_decode(const FfnArgs& a, int num_sms, int32_t* status, cudaStream_t st);
size_t ffn_decode_ws_bytes(int64_t T, int d, int E, int k, int I);

cudaError_t launch_combine(int T, int d, int k, int mode, const float* expert_out,
                           const float* shared_out, const float* topk_w, const int32_t* assign_pos,
                           int rms, uint16_t* y, cudaStream_t st);

// tensor-core (tcgen05) FFN path
bool ffn_tc_supported(int d, int I);
size_t ffn_tc_ws_bytes(int64_t T, int d, int E, int k, int I);
// the m-tile kernel's workspace when rows are quantised per expert (static input scales);
// 0 when the m-tile kernel does not take these shapes
size_t ffn_tc_static_ws_bytes(int64_t T, int d, int E, int k, int I);
cudaError_t launch_ffn_tc(const FfnArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st);
// tcgen05 decode FFN (at most 8 tokens)
bool ffn_dec_supported(int64_t T, int d, int I, int mode, int E, int k, int has_shared, int grid);
size_t ffn_dec_ws_bytes(int E);
cudaError_t launch_ffn_dec(const FfnArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st);
// fused decode layer (at most 8 tokens): quantise, route, expert FFN and combine in one kernel
struct LayerDecArgs {
  const uint16_t* x;
  const float* ts_in;
  const float* Wr;
  const float* br;
  ExpertGroup routed, shared;
  int has_shared;
  int E, d, I, T, k;
  int rms;
  uint8_t* xq_codes;
  uint8_t* xq_scales;
  float* xq_ts;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_assign;
  int32_t* assign_pos;
  float* y_acc;
  uint16_t* y;
};
bool layer_dec_supported(int64_t T, int d, int I, int E, int k, int has_shared, int num_sms);
size_t layer_dec_ws_bytes(int64_t T, int E);
cudaError_t launch_layer_dec(const LayerDecArgs& a, void* ws, int num_sms, int32_t* status, cudaStream_t st);
cudaError_t launch_pack_dec(const ExpertGroup& g, int E, int d, int I, const uint8_t* gu_sf_tiled,
                            const uint8_t* dn_sf_tiled, uint8_t* dec_pack, int num_sms, cudaStream_t st);
size_t dec_pack_bytes(int E, int d, int I);
cudaError_t launch_hot_tier(const uint8_t* dec_pack, const int32_t* rank, int E, int d, int I, int n_hot,
                            uint8_t* hot_pack, int32_t* hot_slot, int num_sms, cudaStream_t st);
cudaError_t launch_pack_sf(const ExpertGroup& g, int E, int d, int I, uint8_t* gu_t, uint8_t* dn_t,
                           int num_sms, cudaStream_t st);

// the bounded-wait limit of each translation unit with device-side waits, on the current device
cudaError_t set_wait_limit_ffn_decode(unsigned long long ns);
cudaError_t set_wait_limit_ffn_tc(unsigned long long ns);
cudaError_t set_wait_limit_ffn_dec(unsigned long long ns);
cudaError_t set_wait_limit_layer_dec(unsigned long long ns);
cudaError_t set_wait_limit_router_tc(unsigned long long ns);
inline cudaError_t set_wait_limits(unsigned long long ns) {
  cudaError_t e = set_wait_limit_ffn_decode(ns);
  if (e == cudaSuccess) e = set_wait_limit_router_tc(ns);
  if (e == cudaSuccess) e = set_wait_limit_ffn_tc(ns);
  if (e == cudaSuccess) e = set_wait_limit_ffn_dec(ns);
  if (e == cudaSuccess) e = set_wait_limit_layer_dec(ns);
  return e;
}

// one-time per-device kernel attribute setup (dynamic shared memory limits)
cudaError_t init_route_attributes();
cudaError_t init_router_tc_attributes();
cudaError_t init_ffn_decode_attributes();
cudaError_t init_ffn_tc_attributes();
cudaError_t init_ffn_dec_attributes();
cudaError_t init_layer_dec_attributes();
inline cudaError_t init_kernel_attributes() {
  cudaError_t e = init_route_attributes();
  if (e != cudaSuccess) return e;
  e = init_router_tc_attributes();
  if (e != cudaSuccess) return e;
  e = init_ffn_decode_attributes();
  if (e != cudaSuccess) return e;
  e = init_ffn_tc_attributes();
  if (e != cudaSuccess) return e;
  e = init_ffn_dec_attributes();
  if (e != cudaSuccess) return e;
  return init_layer_dec_attributes();
}

}  // namespace moe
