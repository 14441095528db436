// C ABI entry points (declared in include/moe_nvfp4.h): argument validation on the host,
// workspace carving, and kernel launches on the caller's stream.
#include <mutex>
#include <string>

#include "../../include/moe_nvfp4.h"
#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ int32_t g_device_status = 0;

namespace {

thread_local std::string t_last_error;

moe_status fail(moe_status s, const std::string& msg) {
  t_last_error = msg;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  t_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int kMaxDevices = 64;
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int32_t* status = nullptr;  // device address of g_device_status on this device
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device one-time setup: SM count and dynamic shared memory limits.
moe_status device_info(int* num_sms, int32_t** status = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(MOE_ERR_CUDA, "this library is built for sm_100a (B200); device is sm_" +
                                    std::to_string(major * 10 + minor));
    e = cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = init_kernel_attributes();
    if (e != cudaSuccess) return cuda_fail(e, "kernel attribute setup");
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&di.status), g_device_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_device_status)");
    di.ready = true;
  }
  *num_sms = di.num_sms;
  if (status) *status = di.status;
  return MOE_OK;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

size_t quant_ws_bytes() { return align256(kMaxPartials * sizeof(float)); }

size_t ffn_ws_bytes(int64_t T, int d, int E, int k, int I) {
  const size_t a = ffn_decode_ws_bytes(T, d, E, k, I);
  const size_t b = ffn_tc_ws_bytes(T, d, E, k, I);
  const size_t c = ffn_dec_ws_bytes(E);
  const size_t ab = a > b ? a : b;
  return ab > c ? ab : c;
}

moe_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return MOE_OK;
  if (!ws || ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) + " bytes, got " +
                                       std::to_string(ws_bytes));
  if (((uintptr_t)ws & 255u) != 0) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return MOE_OK;
}

// The tensor scales are always needed. The natural-layout codes and scales may all be NULL
// when the group carries its decode pack (which holds the same bytes), for the calls that read
// only the pack; `natural` reports whether they are present.
moe_status check_weights(const moe_expert_weights_t& w, const char* name, int E, int d, int I, bool* natural) {
  const std::string n(name);
  if (w.E != E || w.d != d || w.I != I) return fail(MOE_ERR_INVALID_ARG, n + ": inconsistent E/d/I");
  const void* ts[2] = {w.gu_ts, w.dn_ts};
  for (const void* p : ts) {
    if (!p) return fail(MOE_ERR_INVALID_ARG, n + ": null tensor-scale pointer");
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, n + ": weight pointer not 16-byte aligned");
  }
  const void* nat[4] = {w.gu_codes, w.gu_scales, w.dn_codes, w.dn_scales};
  int present = 0;
  for (const void* p : nat) {
    if (p && !aligned16(p)) return fail(MOE_ERR_INVALID_ARG, n + ": weight pointer not 16-byte aligned");
    present += p ? 1 : 0;
  }
  if (present != 0 && present != 4)
    return fail(MOE_ERR_INVALID_ARG, n + ": the natural-layout codes and scales must all be given or all NULL");
  if (present == 0 && !w.dec_pack)
    return fail(MOE_ERR_INVALID_ARG, n + ": null weight pointer (neither the natural layout nor the decode pack)");
  if (w.dec_pack && !aligned16(w.dec_pack)) return fail(MOE_ERR_INVALID_ARG, n + ": dec_pack not 16-byte aligned");
  *natural = present == 4;
  return MOE_OK;
}

ExpertGroup to_group(const moe_expert_weights_t& w) {
  return ExpertGroup{w.gu_codes, w.gu_scales,   w.gu_ts,       w.dn_codes, w.dn_scales, w.dn_ts,
                     w.gu_sf_tiled, w.dn_sf_tiled, w.dec_pack, w.hot_pack, w.hot_slot, w.n_hot};
}

}  // namespace

void set_last_error(const std::string& msg) { t_last_error = msg; }

std::atomic<uint64_t> g_launch_count{0};

}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_version(void) { return 100; }

uint64_t moe_launch_count(void) { return g_launch_count.load(std::memory_order_relaxed); }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_WORKSPACE: return "workspace too small, misaligned, or marked by a call that gave up";
  }
  return "unknown status";
}

const char* moe_last_error(void) { return t_last_error.c_str(); }

size_t moe_workspace_size(int32_t op, int64_t T, int32_t d, int32_t E, int32_t k, int32_t I) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || I <= 0) return 0;
  const size_t q = quant_ws_bytes();
  const size_t r = align256(route_ws_bytes(T, d, E, k));
  const size_t f = align256(ffn_ws_bytes(T, d, E, k, I));
  switch (op) {
    case MOE_OP_QUANT: return q;
    case MOE_OP_ROUTE: return r;
    case MOE_OP_FFN: return f;
    case MOE_OP_LAYER: {
      size_t m = q > r ? q : r;
      return m > f ? m : f;
    }
    case MOE_OP_LAYER_DECODE: return layer_dec_ws_bytes(T, E);
    case MOE_OP_FFN_STATIC: return align256(ffn_tc_static_ws_bytes(T, d, E, k, I));
  }
  return 0;
}

moe_status nvfp4_quantize_act(const uint16_t* x, int64_t rows, int32_t cols, const float* ts_in,
                              uint8_t* codes, uint8_t* scales, float* ts_out, void* ws,
                              size_t ws_bytes, void* stream) {
  if (rows < 0 || cols <= 0) return fail(MOE_ERR_INVALID_ARG, "rows must be >= 0 and cols > 0");
  if (cols % kBlock) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "cols must be a multiple of 16");
  if (rows > 0) {
    if (!x || !codes || !scales) return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(x) || !aligned16(codes))
      return fail(MOE_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  }
  if (ts_in && !aligned16(ts_in)) return fail(MOE_ERR_INVALID_ARG, "ts_in must be 16-byte aligned");
  const int64_t nblk = rows * (int64_t)(cols / kBlock);
  if (nblk > 4096 && !ts_in) {
    moe_status s = check_ws(ws, ws_bytes, quant_ws_bytes());
    if (s != MOE_OK) return s;
  }
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_quantize(x, rows, cols, ts_in, codes, scales, ts_out, ws, sms,
                                  (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "nvfp4_quantize_act launch");
}

static moe_status check_route_common(int32_t T, int32_t E, int32_t k, int32_t* counts,
                                     int32_t* offsets, int32_t* sorted_assign,
                                     int32_t* assign_pos) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (k < 1 || k > 32) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "k must be in [1, 32]");
  if (E < k || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E must be in [k, 1024]");
  if ((int64_t)T * k > (int64_t)1 << 30) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  if (!counts || !offsets) return fail(MOE_ERR_INVALID_ARG, "null counts/offsets");
  if (T > 0 && (!sorted_assign || !assign_pos)) return fail(MOE_ERR_INVALID_ARG, "null permutation output");
  return MOE_OK;
}

moe_status moe_permute(const int32_t* topk_idx, int32_t T, int32_t k, int32_t E, int32_t* counts,
                       int32_t* offsets, int32_t* sorted_assign, int32_t* assign_pos, void* ws,
                       size_t ws_bytes, void* stream) {
  moe_status s = check_route_common(T, E, k, counts, offsets, sorted_assign, assign_pos);
  if (s != MOE_OK) return s;
  if (T > 0 && !topk_idx) return fail(MOE_ERR_INVALID_ARG, "null topk_idx");
  if ((int64_t)T * k > 4096) {
    s = check_ws(ws, ws_bytes, permute_ws_bytes(T, k, E));
    if (s != MOE_OK) return s;
  }
  int sms = 0;
  s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_permute(topk_idx, T, k, E, counts, offsets, sorted_assign, assign_pos, ws,
                                 (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_permute launch");
}

moe_status moe_route(const uint16_t* x, int32_t T, int32_t d, const float* Wr, const float* br,
                     int32_t E, int32_t k, int32_t* topk_idx, float* topk_w, int32_t* counts,
                     int32_t* offsets, int32_t* sorted_assign, int32_t* assign_pos, void* ws,
                     size_t ws_bytes, void* stream) {
  moe_status s = check_route_common(T, E, k, counts, offsets, sorted_assign, assign_pos);
  if (s != MOE_OK) return s;
  if (d <= 0 || d % kBlock || d > 8192) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "d must be a multiple of 16 in [16, 8192]");
  if (T > 0) {
    if (!x || !Wr || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(x) || !aligned16(Wr)) return fail(MOE_ERR_INVALID_ARG, "x and Wr must be 16-byte aligned");
    s = check_ws(ws, ws_bytes, route_ws_bytes(T, d, E, k));
    if (s != MOE_OK) return s;
  }
  int sms = 0;
  int32_t* dstatus = nullptr;
  s = device_info(&sms, &dstatus);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_route(x, T, d, Wr, br, E, k, topk_idx, topk_w, counts, offsets,
                               sorted_assign, assign_pos, ws, sms, dstatus, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route launch");
}

moe_status moe_pack_experts(const moe_expert_weights_t* W, uint8_t* gu_sf_tiled,
                            uint8_t* dn_sf_tiled, uint8_t* dec_pack, void* stream) {
  if (!W || !gu_sf_tiled || !dn_sf_tiled) return fail(MOE_ERR_INVALID_ARG, "null argument");
  if (dec_pack && (!aligned16(dec_pack) || !W->dn_codes || !aligned16(W->dn_codes) || !W->gu_codes ||
                   !aligned16(W->gu_codes)))
    return fail(MOE_ERR_INVALID_ARG, "dec_pack, dn_codes and gu_codes must be 16-byte aligned");
  if (W->E < 1 || W->d <= 0 || W->I <= 0) return fail(MOE_ERR_INVALID_ARG, "bad E/d/I");
  if (W->d % 128 || W->I % 64) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "packing needs d % 128 == 0 and I % 64 == 0");
  if (dec_pack && W->d % 512) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "the decode pack needs d % 512 == 0");
  if (!W->gu_scales || !W->dn_scales) return fail(MOE_ERR_INVALID_ARG, "null scales");
  if (!aligned16(W->gu_scales) || !aligned16(W->dn_scales) || !aligned16(gu_sf_tiled) || !aligned16(dn_sf_tiled))
    return fail(MOE_ERR_INVALID_ARG, "scale pointers must be 16-byte aligned");
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_pack_sf(to_group(*W), W->E, W->d, W->I, gu_sf_tiled, dn_sf_tiled, sms,
                                 (cudaStream_t)stream);
  if (e == cudaSuccess && dec_pack)
    e = launch_pack_dec(to_group(*W), W->E, W->d, W->I, gu_sf_tiled, dn_sf_tiled, dec_pack, sms,
                        (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_pack_experts launch");
}

moe_status moe_expert_ffn(const uint8_t* xq_codes, const uint8_t* xq_scales, const float* xq_ts,
                          int32_t T, const moe_experts_t* W, int32_t k, const int32_t* offsets,
                          const int32_t* sorted_assign, const float* topk_w, int32_t mode,
                          int32_t path, float* out, float* shared_out, void* ws, size_t ws_bytes,
                          void* stream) {
  if (!W) return fail(MOE_ERR_INVALID_ARG, "null weights");
  const int E = W->routed.E, d = W->routed.d, I = W->routed.I;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (k < 1 || k > 32 || E < k || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "need 1 <= k <= 32, k <= E <= 1024");
  if (d <= 0 || I <= 0 || d % kBlock || I % kBlock || d > 8192 || I > 8192)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "d and I must be multiples of 16 in [16, 8192]");
  if (mode != MOE_FFN_ACCUMULATE && mode != MOE_FFN_PER_ASSIGN) return fail(MOE_ERR_INVALID_ARG, "bad mode");
  if (path != MOE_PATH_AUTO && path != MOE_PATH_DECODE && path != MOE_PATH_PREFILL && path != MOE_PATH_CUDA_CORE)
    return fail(MOE_ERR_INVALID_ARG, "bad path");
  bool nat_r = false, nat_s = true;
  moe_status s = check_weights(W->routed, "routed", E, d, I, &nat_r);
  if (s != MOE_OK) return s;
  if (W->has_shared) {
    s = check_weights(W->shared, "shared", 1, d, I, &nat_s);
    if (s != MOE_OK) return s;
  }
  const bool natural = nat_r && nat_s;
  if (T == 0) return MOE_OK;
  if (!xq_codes || !xq_scales || !xq_ts || !offsets || !sorted_assign || !topk_w || !out)
    return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(xq_codes) || !aligned16(xq_scales) || !aligned16(out))
    return fail(MOE_ERR_INVALID_ARG, "xq_codes, xq_scales and out must be 16-byte aligned");
  if (mode == MOE_FFN_PER_ASSIGN && W->has_shared && !shared_out)
    return fail(MOE_ERR_INVALID_ARG, "shared_out needed in PER_ASSIGN mode with a shared expert");
  int sms = 0;
  int32_t* dstatus = nullptr;
  s = device_info(&sms, &dstatus);
  if (s != MOE_OK) return s;
  const bool packed = W->routed.gu_sf_tiled && W->routed.dn_sf_tiled &&
                      (!W->has_shared || (W->shared.gu_sf_tiled && W->shared.dn_sf_tiled));
  const bool tc_ok = ffn_tc_supported(d, I) && packed && natural;
  const bool dec_packed = W->routed.dec_pack && (!W->has_shared || W->shared.dec_pack);
  const bool dec_ok = ffn_dec_supported(T, d, I, mode, E, k, W->has_shared ? 1 : 0, sms) && dec_packed;
  if (path == MOE_PATH_PREFILL && !tc_ok)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                "tensor-core path needs d % 256 == 0, I % 256 == 0, the natural-layout weights and scales "
                "packed by moe_pack_experts");
  if (path == MOE_PATH_DECODE && !dec_ok)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                "decode path needs T <= 8, ACCUMULATE mode, d % 512 == 0, I % 64 == 0 and the decode pack");
  if (path == MOE_PATH_CUDA_CORE && !natural)
    return fail(MOE_ERR_INVALID_ARG, "the CUDA-core path reads the natural-layout weights, which are NULL");
  const int kind = path == MOE_PATH_AUTO ? (dec_ok ? MOE_PATH_DECODE : tc_ok ? MOE_PATH_PREFILL : MOE_PATH_CUDA_CORE)
                                         : path;
  if (kind == MOE_PATH_CUDA_CORE && !natural)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                "without the natural-layout weights only the DECODE path (T <= 8) can run this call");
  const size_t need = kind == MOE_PATH_DECODE    ? ffn_dec_ws_bytes(E)
                      : kind == MOE_PATH_PREFILL ? ffn_tc_ws_bytes(T, d, E, k, I)
                                                 : ffn_decode_ws_bytes(T, d, E, k, I);
  s = check_ws(ws, ws_bytes, need);
  if (s != MOE_OK) return s;
  FfnArgs a;
  a.xq_codes = xq_codes;
  a.xq_scales = xq_scales;
  a.xq_ts = xq_ts;
  a.T = T; a.d = d; a.I = I; a.E = E; a.k = k;
  a.routed = to_group(W->routed);
  a.shared = W->has_shared ? to_group(W->shared) : ExpertGroup{};
  a.has_shared = W->has_shared ? 1 : 0;
  a.offsets = offsets;
  a.sorted_assign = sorted_assign;
  a.topk_w = topk_w;
  a.mode = mode;
  a.out = out;
  a.shared_out = shared_out;
  const size_t slots = (size_t)T * k + T;
  a.h_codes = reinterpret_cast<uint8_t*>(ws);
  a.h_scales = reinterpret_cast<uint8_t*>(ws) + align256(slots * (I / 2));
  cudaError_t e = kind == MOE_PATH_DECODE    ? launch_ffn_dec(a, ws, sms, dstatus, (cudaStream_t)stream)
                  : kind == MOE_PATH_PREFILL ? launch_ffn_tc(a, ws, sms, dstatus, (cudaStream_t)stream)
                                             : launch_ffn_decode(a, sms, dstatus, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn launch");
}

moe_status moe_layer_decode(const uint16_t* x, int32_t T, const float* ts_in, const float* Wr, const float* br,
                            const moe_experts_t* W, int32_t k, uint8_t* xq_codes, uint8_t* xq_scales,
                            float* xq_ts, int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                            int32_t* sorted_assign, int32_t* assign_pos, float* y_acc, uint16_t* y,
                            int32_t rms_renorm, void* ws, size_t ws_bytes, void* stream) {
  if (!W) return fail(MOE_ERR_INVALID_ARG, "null weights");
  const int E = W->routed.E, d = W->routed.d, I = W->routed.I;
  bool nat = false;
  moe_status s = check_weights(W->routed, "routed", E, d, I, &nat);
  if (s != MOE_OK) return s;
  if (W->has_shared && (s = check_weights(W->shared, "shared", 1, d, I, &nat)) != MOE_OK) return s;
  if (!x || !Wr || !xq_codes || !xq_scales || !xq_ts || !topk_idx || !topk_w || !counts || !offsets ||
      !sorted_assign || !assign_pos || !y_acc || !y)
    return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(x) || !aligned16(Wr) || !aligned16(xq_codes) || !aligned16(xq_scales) || !aligned16(y_acc) ||
      !aligned16(y))
    return fail(MOE_ERR_INVALID_ARG, "x, Wr, xq_codes, xq_scales, y_acc and y must be 16-byte aligned");
  const bool packed = W->routed.dec_pack && (!W->has_shared || W->shared.dec_pack);
  if (!packed) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "weights need the decode pack of moe_pack_experts");
  const moe_expert_weights_t& R = W->routed;
  if (R.n_hot < 0 || R.n_hot > E) return fail(MOE_ERR_INVALID_ARG, "routed.n_hot must be in [0, E]");
  if (R.n_hot > 0) {
    if (!R.hot_pack || !R.hot_slot || !aligned16(R.hot_pack) || !aligned16(R.hot_slot))
      return fail(MOE_ERR_INVALID_ARG, "a hot tier needs 16-byte aligned hot_pack and hot_slot");
    if (E % 4 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "a hot tier needs E % 4 == 0");
  }
  int sms = 0;
  int32_t* dstatus = nullptr;
  if ((s = device_info(&sms, &dstatus)) != MOE_OK) return s;
  if (!layer_dec_supported(T, d, I, E, k, W->has_shared ? 1 : 0, sms))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                "moe_layer_decode needs 1 <= T <= 8, d % 512 == 0, d <= 4096, I % 64 == 0, 1 <= k <= 32, "
                "k <= E <= 1024 and at most 32 units per CTA");
  if ((s = check_ws(ws, ws_bytes, layer_dec_ws_bytes(T, E))) != MOE_OK) return s;
  LayerDecArgs a;
  a.x = x;
  a.ts_in = ts_in;
  a.Wr = Wr;
  a.br = br;
  a.routed = to_group(W->routed);
  a.shared = W->has_shared ? to_group(W->shared) : ExpertGroup{};
  a.has_shared = W->has_shared ? 1 : 0;
  a.E = E; a.d = d; a.I = I; a.T = T; a.k = k;
  a.rms = rms_renorm ? 1 : 0;
  a.xq_codes = xq_codes;
  a.xq_scales = xq_scales;
  a.xq_ts = xq_ts;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.counts = counts;
  a.offsets = offsets;
  a.sorted_assign = sorted_assign;
  a.assign_pos = assign_pos;
  a.y_acc = y_acc;
  a.y = y;
  cudaError_t e = launch_layer_dec(a, ws, sms, dstatus, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer_decode launch");
}

moe_status moe_expert_ffn_static(const uint16_t* x, int32_t T, const moe_experts_t* W, const float* in_gu,
                                 const float* in_dn, int32_t k, const int32_t* offsets,
                                 const int32_t* sorted_assign, const float* topk_w, int32_t mode, float* out,
                                 float* shared_out, void* ws, size_t ws_bytes, void* stream) {
  if (!W) return fail(MOE_ERR_INVALID_ARG, "null weights");
  const int E = W->routed.E, d = W->routed.d, I = W->routed.I;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (k < 1 || k > 32 || E < k || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "need 1 <= k <= 32, k <= E <= 1024");
  if (mode != MOE_FFN_ACCUMULATE && mode != MOE_FFN_PER_ASSIGN) return fail(MOE_ERR_INVALID_ARG, "bad mode");
  if (d <= 0 || I <= 0 || ffn_tc_static_ws_bytes(1, d, E, k, I) == 0)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "static input scales need d % 256 == 0, I % 256 == 0, d <= 2048, I <= 768");
  bool nat_r = false, nat_s = true;
  moe_status s = check_weights(W->routed, "routed", E, d, I, &nat_r);
  if (s != MOE_OK) return s;
  if (W->has_shared && (s = check_weights(W->shared, "shared", 1, d, I, &nat_s)) != MOE_OK) return s;
  const bool packed = W->routed.gu_sf_tiled && W->routed.dn_sf_tiled &&
                      (!W->has_shared || (W->shared.gu_sf_tiled && W->shared.dn_sf_tiled));
  if (!(nat_r && nat_s) || !packed)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "static input scales need the natural-layout weights and packed scales");
  if (T == 0) return MOE_OK;
  if (!x || !in_gu || !in_dn || !offsets || !sorted_assign || !topk_w || !out)
    return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(x) || !aligned16(out)) return fail(MOE_ERR_INVALID_ARG, "x_bf16 and out must be 16-byte aligned");
  if (mode == MOE_FFN_PER_ASSIGN && W->has_shared && !shared_out)
    return fail(MOE_ERR_INVALID_ARG, "shared_out needed in PER_ASSIGN mode with a shared expert");
  int sms = 0;
  int32_t* dstatus = nullptr;
  if ((s = device_info(&sms, &dstatus)) != MOE_OK) return s;
  if ((s = check_ws(ws, ws_bytes, ffn_tc_static_ws_bytes(T, d, E, k, I))) != MOE_OK) return s;
  FfnArgs a;
  a.xq_codes = nullptr;
  a.xq_scales = nullptr;
  a.xq_ts = nullptr;
  a.x_bf16 = x;
  a.in_gu = in_gu;
  a.in_dn = in_dn;
  a.T = T; a.d = d; a.I = I; a.E = E; a.k = k;
  a.routed = to_group(W->routed);
  a.shared = W->has_shared ? to_group(W->shared) : ExpertGroup{};
  a.has_shared = W->has_shared ? 1 : 0;
  a.offsets = offsets;
  a.sorted_assign = sorted_assign;
  a.topk_w = topk_w;
  a.mode = mode;
  a.out = out;
  a.shared_out = shared_out;
  a.h_codes = nullptr;
  a.h_scales = nullptr;
  cudaError_t e = launch_ffn_tc(a, ws, sms, dstatus, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn_static launch");
}

moe_status moe_combine(int32_t T, int32_t d, int32_t k, int32_t mode, const float* expert_out,
                       const float* shared_out, const float* topk_w, const int32_t* assign_pos,
                       int32_t rms_renorm, uint16_t* y, void* stream) {
  if (T < 0 || d <= 0 || d % kBlock) return fail(MOE_ERR_INVALID_ARG, "T >= 0 and d a positive multiple of 16");
  if (mode != MOE_FFN_ACCUMULATE && mode != MOE_FFN_PER_ASSIGN) return fail(MOE_ERR_INVALID_ARG, "bad mode");
  if (T == 0) return MOE_OK;
  if (!expert_out || !y) return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  if (mode == MOE_FFN_PER_ASSIGN && (k < 1 || !topk_w || !assign_pos))
    return fail(MOE_ERR_INVALID_ARG, "PER_ASSIGN combine needs k >= 1, topk_w and assign_pos");
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_combine(T, d, k, mode, expert_out, shared_out, topk_w, assign_pos,
                                 rms_renorm ? 1 : 0, y, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine launch");
}

moe_status moe_expert_hist(const int32_t* counts, int32_t E, int64_t* cum, int32_t* rank_out,
                           int32_t reset, void* stream) {
  if (E < 1 || E > 4096) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E must be in [1, 4096]");
  if (!counts || !cum) return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_hist(counts, E, cum, rank_out, reset ? 1 : 0, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_hist launch");
}

moe_status moe_hot_tier_update(const moe_expert_weights_t* W, const int32_t* rank, int32_t n_hot,
                               uint8_t* hot_pack, int32_t* hot_slot, void* stream) {
  if (!W) return fail(MOE_ERR_INVALID_ARG, "null weights");
  if (!W->dec_pack) return fail(MOE_ERR_INVALID_ARG, "the group needs its decode pack (moe_pack_experts)");
  if (!rank || !hot_slot || (n_hot > 0 && !hot_pack)) return fail(MOE_ERR_INVALID_ARG, "null tensor pointer");
  if (n_hot < 0 || n_hot > W->E) return fail(MOE_ERR_INVALID_ARG, "n_hot must be in [0, E]");
  if (W->E % 4 != 0 || W->d % 512 != 0 || W->I % 64 != 0)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "a hot tier needs E % 4 == 0, d % 512 == 0 and I % 64 == 0");
  if ((hot_pack && !aligned16(hot_pack)) || !aligned16(hot_slot) || !aligned16(W->dec_pack))
    return fail(MOE_ERR_INVALID_ARG, "hot_pack, hot_slot and dec_pack must be 16-byte aligned");
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = launch_hot_tier(W->dec_pack, rank, W->E, W->d, W->I, n_hot, hot_pack, hot_slot, sms,
                                  (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_hot_tier_update launch");
}

moe_status moe_set_l2_persisting(size_t bytes, size_t* bytes_out) {
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  int dev = 0, max_bytes = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&max_bytes, cudaDevAttrMaxPersistingL2CacheSize, dev);
  if (e != cudaSuccess) return cuda_fail(e, "persisting L2 maximum");
  const size_t b = bytes < (size_t)max_bytes ? bytes : (size_t)max_bytes;
  if (b == 0 && (e = cudaCtxResetPersistingL2Cache()) != cudaSuccess) return cuda_fail(e, "cudaCtxResetPersistingL2Cache");
  if ((e = cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, b)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize)");
  if (bytes_out && (e = cudaDeviceGetLimit(bytes_out, cudaLimitPersistingL2CacheSize)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetLimit(cudaLimitPersistingL2CacheSize)");
  return MOE_OK;
}

moe_status moe_set_wait_limit_ns(uint64_t ns) {
  if (ns < 1000000ull || ns > 60000000000ull)
    return fail(MOE_ERR_INVALID_ARG, "wait limit must be between 1 ms and 60 s");
  int sms = 0;
  moe_status s = device_info(&sms);
  if (s != MOE_OK) return s;
  cudaError_t e = set_wait_limits((unsigned long long)ns);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_set_wait_limit_ns");
}

moe_status moe_get_device_status(void* stream, int32_t clear, int32_t* status_out) {
  if (!status_out) return fail(MOE_ERR_INVALID_ARG, "null status_out");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  e = cudaMemcpyFromSymbol(status_out, g_device_status, sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e, "clear device status");
  }
  return MOE_OK;
}

}  // extern "C"

#ifdef MOE_TRACE
namespace moe {
int64_t trace_fetch_tc(void* host, size_t bytes);
int64_t trace_fetch_dec(void* host, size_t bytes);
int64_t trace_fetch_route(void* host, size_t bytes);
int64_t trace_fetch_prep(void* host, size_t bytes);
int64_t trace_fetch_layer(void* host, size_t bytes);
int64_t trace_fetch_layer_core(void* host, size_t bytes);
}  // namespace moe
// Trace builds only: timeline records of the last runs of the tensor-core FFN kernel
// (kernel 0: the grouped-GEMM path, 1: the decode path; 2: entry/wait/exit stamps of the
// routing kernels, 3: of the decode preparation and FFN kernels, 4: phase stamps of the
// one-kernel decode layer, 5: its unit-core records), copied to `host` and cleared.
extern "C" int64_t moe_trace_fetch(int32_t kernel, void* host, size_t bytes) {
  switch (kernel) {
    case 0: return moe::trace_fetch_tc(host, bytes);
    case 1: return moe::trace_fetch_dec(host, bytes);
    case 2: return moe::trace_fetch_route(host, bytes);
    case 4: return moe::trace_fetch_layer(host, bytes);
    case 5: return moe::trace_fetch_layer_core(host, bytes);
    default: return moe::trace_fetch_prep(host, bytes);
  }
}
#endif
