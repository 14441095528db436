/*
 * moe_nvfp4.h - C ABI of the B200 (sm_100a) NVFP4 mixture-of-experts layer library.
 *
 * The layer follows the Basalt pages:
 *   - "What Basalt changes in a Blackwell local inference stack", section "Experts can move
 *     without becoming free": the model selects a subset of its experts for each token.
 *   - "Basalt" project page, section "Expert tiers" (and FAQ "Can it use a second GPU or
 *     system RAM?"): each token uses only a few experts; the most routed experts form the
 *     hot tier.
 *   - "Basalt" project page, "All the numbers", list "Engines: commit, and what is not
 *     NVIDIA's weights": routed experts are NVIDIA's NVFP4, kept bit-exact, including an
 *     activation input_scale.
 * The pages define neither NVFP4 nor the routing rule. This library uses:
 *   NVFP4  - E2M1 codes (two per byte, element 2i in the low nibble), one E4M3 scale per 16
 *            consecutive elements of a row ([rows][cols/16] bytes), one float32 tensor scale;
 *            value = e2m1 * e4m3 * ts. Dynamic tensor scale ts = amax / (6 * 448).
 *            Conversions round to nearest even and saturate; a negative value that rounds
 *            to zero keeps its sign (code 0x8); a block whose scale rounds to 0 stores +0s.
 *   router - logits = x Wr^T + br (float32); top-k by logit, ties to the lower expert id;
 *            weights = softmax over all experts restricted to the top-k and renormalised.
 *   FFN    - SwiGLU: h = silu(x Wg^T) * (x Wu^T); h is re-quantised to NVFP4 with tensor
 *            scale 1.0; o = h Wd^T. A shared expert, if given, is added with weight 1.
 *   order  - the token permutation is a stable counting sort of assignments a = t*k + j.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers, owned by the caller; the library never
 *     allocates device memory. Scratch comes from a caller-provided workspace `ws` of
 *     `ws_bytes` bytes (see moe_workspace_size); it must be 256-byte aligned.
 *   - Tensor pointers must be 16-byte aligned. bf16 values are passed as uint16_t bits.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). Argument errors are detected on the host before anything is launched and
 *     returned synchronously; nothing is enqueued in that case.
 *   - Device-side problems (a bounded wait that ran out) are recorded in a device status
 *     word, read with moe_get_device_status (which synchronises the stream).
 *   - Functions never abort and never throw across the ABI.
 */
#ifndef MOE_NVFP4_H
#define MOE_NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, negative size, misaligned pointer ... */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* sizes outside what the kernels handle */
  MOE_ERR_CUDA = 3,               /* a CUDA runtime call failed (see moe_last_error) */
  MOE_ERR_TIMEOUT = 4,            /* a bounded device-side wait ran out */
  MOE_ERR_WORKSPACE = 5           /* ws too small or misaligned */
} moe_status;

/* FFN output modes */
#define MOE_FFN_ACCUMULATE 0  /* out = float32 y_acc [T][d] = sum_j w[t,j] o[t,j] + shared */
#define MOE_FFN_PER_ASSIGN 1  /* out = float32 [T*k][d], row p = o of sorted_assign[p];
                                 shared_out = float32 [T][d] (unweighted) */
/* FFN kernel paths */
#define MOE_PATH_AUTO 0       /* the fastest path whose requirements hold */
#define MOE_PATH_DECODE 1     /* tcgen05 split-over-I decode kernel (T <= 8) */
#define MOE_PATH_PREFILL 2    /* tcgen05 block-scaled grouped GEMM path (any T) */
#define MOE_PATH_CUDA_CORE 3  /* CUDA-core kernel on the natural layout (any shape) */

/* workspace query operations */
#define MOE_OP_LAYER 0        /* enough for every call of one layer forward */
#define MOE_OP_ROUTE 1
#define MOE_OP_QUANT 2
#define MOE_OP_FFN 3
#define MOE_OP_LAYER_DECODE 4 /* moe_layer_decode (zero-filled before its first use) */
#define MOE_OP_FFN_STATIC 5   /* moe_expert_ffn_static */

/*
 * Expert weights of one expert group (E routed experts, or E = 1 for the shared expert),
 * natural NVFP4 layout as a checkpoint stores it. All pointers are device pointers.
 *   gu_codes  [E][2I][d/2]   gate rows 0..I-1, then up rows I..2I-1
 *   gu_scales [E][2I][d/16]  E4M3 bytes
 *   gu_ts     [E][2]         float32 tensor scales (gate, up)
 *   dn_codes  [E][d][I/2]
 *   dn_scales [E][d][I/16]
 *   dn_ts     [E]            float32
 *   gu_sf_tiled, dn_sf_tiled: the same scale bytes re-tiled for the tensor-core path by
 *            moe_pack_experts (NULL if not packed; the PREFILL path then refuses).
 *   dec_pack  the decode pack written by moe_pack_experts for the DECODE path and
 *            moe_layer_decode (NULL if absent): every weight byte and scale of the group
 *            again, as the 18432-byte blocks the decode kernel copies into shared memory.
 * A group that has its decode pack may leave gu_codes, gu_scales, dn_codes, dn_scales and the
 * re-tiled scales NULL (all four natural arrays, or none): moe_layer_decode and the DECODE
 * path of moe_expert_ffn read only the pack and the tensor scales, so a decode-only model
 * holds each weight byte once. The other paths then return an error.
 */
typedef struct moe_expert_weights {
  int32_t E, d, I;
  const uint8_t* gu_codes;
  const uint8_t* gu_scales;
  const float* gu_ts;
  const uint8_t* dn_codes;
  const uint8_t* dn_scales;
  const float* dn_ts;
  const uint8_t* gu_sf_tiled;
  const uint8_t* dn_sf_tiled;
  const uint8_t* dec_pack;
  /* Optional hot tier of the group (NULL, NULL, 0 for none), read by moe_layer_decode:
   * hot_pack holds copies of n_hot experts' decode-pack units, [n_hot][I/64][d/256 +
   * d/512][18432] (slot s: the same bytes as expert hot_slot^-1(s)'s dec_pack rows), and
   * hot_slot int32 [E] (device) the slot of each expert, or -1. moe_hot_tier_update fills
   * both. */
  const uint8_t* hot_pack;
  const int32_t* hot_slot;
  int32_t n_hot;
} moe_expert_weights_t;

typedef struct moe_experts {
  moe_expert_weights_t routed;
  moe_expert_weights_t shared;  /* used when has_shared != 0; shared.E must be 1 */
  int32_t has_shared;
} moe_experts_t;

/*
 * nvfp4_quantize_act - NVFP4 quantisation of a bf16 matrix (activations, or weights at
 * load time): step A4 of the layer. Source: "Basalt" project page, "All the numbers", list
 * "Engines: commit, and what is not NVIDIA's weights" (routed experts are NVIDIA's NVFP4;
 * the llama.cpp row keeps NVIDIA's activation input_scale, the static scale ts_in here).
 * Steps: amax over the whole matrix (unless ts_in is given), then per 16-block
 *   sb = (amax_b / 6) / ts; s = E4M3(sb); q_i = E2M1(x_i / (E4M3value(s) * ts)).
 *   x_bf16  [rows][cols] device; cols % 16 == 0
 *   ts_in   device float32[1] static tensor scale, or NULL for the dynamic amax/2688
 *   codes   [rows][cols/2] out; scales [rows][cols/16] out; ts_out float32[1] out (may be
 *           NULL); ws needs moe_workspace_size(MOE_OP_QUANT, rows*cols/... ) bytes.
 * rows == 0 is allowed (writes only ts_out = 1 or *ts_in).
 */
moe_status nvfp4_quantize_act(const uint16_t* x_bf16, int64_t rows, int32_t cols,
                              const float* ts_in, uint8_t* codes, uint8_t* scales,
                              float* ts_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_route - router (A1), softmax/top-k/renormalisation (A2) and permutation (A3).
 * Source: "What Basalt changes in a Blackwell local inference stack", section "Experts can
 * move without becoming free" (each token selects a subset of the experts) and the "Basalt"
 * project page, section "Expert tiers" (each token uses only a few experts).
 *   x_bf16 [T][d]; Wr float32 [E][d]; br float32 [E] or NULL.
 *   topk_idx int32 [T][k] (descending logit), topk_w float32 [T][k],
 *   counts int32 [E], offsets int32 [E+1], sorted_assign int32 [T*k] (assignment ids
 *   a = t*k + j grouped by expert, increasing a within an expert), assign_pos int32 [T*k]
 *   (inverse of sorted_assign). 1 <= k <= 32, k <= E <= 1024, d % 16 == 0.
 * From 256 tokens on, with E % 128 == 0 and d % 64 == 0, the logits come from a bf16-split
 * tensor-core product and every expert near each token's k-th logit is recomputed exactly,
 * so the top-k is that of the float32 logits; the workspace then also holds the split
 * router matrix (moe_workspace_size accounts for it).
 */
moe_status moe_route(const uint16_t* x_bf16, int32_t T, int32_t d, const float* Wr,
                     const float* br, int32_t E, int32_t k, int32_t* topk_idx,
                     float* topk_w, int32_t* counts, int32_t* offsets,
                     int32_t* sorted_assign, int32_t* assign_pos, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * moe_permute - the permutation step (A3) alone, from given top-k indices: a stable
 * counting sort of the T*k assignments by expert, with the per-expert histogram (the
 * routing counts of "Basalt" project page, section "Expert tiers").
 * Same outputs and limits as moe_route.
 */
moe_status moe_permute(const int32_t* topk_idx, int32_t T, int32_t k, int32_t E,
                       int32_t* counts, int32_t* offsets, int32_t* sorted_assign,
                       int32_t* assign_pos, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_pack_experts - derived layouts of an expert group for the tensor-core paths, written
 * once per weight load into caller-owned buffers (set them in W afterwards). The pages have
 * no counterpart (they keep NVIDIA's NVFP4 bytes unchanged, "Basalt" project page,
 * "Engines" list); these are the same bytes rearranged for the tensor core:
 *   gu_sf_tiled (E*2I*d/16 bytes), dn_sf_tiled (E*d*I/16 bytes): the E4M3 scale bytes in
 *     512-byte atoms of 128 weight rows x 4 scale blocks, the layout the tensor core reads
 *     its scales in (gate/up atoms [E][I/64][d/64], atom rows 0-63 gate, 64-127 up; down
 *     atoms [E][d/128][I/64]);
 *   dec_pack (E*I*d*27/16 bytes; optional, NULL to skip; needs d % 512 == 0): for each
 *     unit (expert e, 64-wide slice j of I), d/256 gate/up blocks then d/512 down blocks of
 *     18432 bytes each, in that order. Gate/up block kb: the 128 x 128-byte tile of gate
 *     rows 64j..64j+63 then up rows 64j..64j+63, bytes 128kb..128kb+127 of each, stored in
 *     the 128-byte swizzle (16-byte piece c of row r at r*128 + (c ^ (r % 8))*16), then the
 *     four gate/up scale atoms 4kb..4kb+3 of (e, j). Down block q: chunks c = 4q..4q+3, each
 *     the 128 x 32-byte tile of rows 128c..128c+127, bytes 32j..32j+31, stored in the 32-byte
 *     swizzle (piece c' of row r at r*32 + (c' ^ ((r / 4) % 2))*16), then the four down
 *     scale atoms of those chunks for slice j. A block is exactly what one shared-memory
 *     stage of the decode kernel holds, so it moves with one bulk copy.
 * The natural-layout arrays stay as they are and remain in use by the CUDA-core path.
 * Requires d % 128 == 0 and I % 64 == 0.
 */
moe_status moe_pack_experts(const moe_expert_weights_t* W, uint8_t* gu_sf_tiled,
                            uint8_t* dn_sf_tiled, uint8_t* dec_pack, void* stream);

/*
 * moe_expert_ffn - expert SwiGLU FFN for all routed assignments (A5-A7) and the shared
 * expert (A8). Source: "What Basalt changes in a Blackwell local inference stack", section
 * "Experts can move without becoming free" (only the selected experts run for a token) and
 * the "Basalt" project page, "Engines" list (the experts' weights are NVFP4) and section
 * "Expert tiers" (every kernel, FP4 included, written for Blackwell).
 *   xq_codes [T][d/2], xq_scales [T][d/16], xq_ts float32[1]: the NVFP4 activation.
 *   offsets [E+1], sorted_assign [T*k], topk_w [T][k]: from moe_route / moe_permute.
 *   mode MOE_FFN_ACCUMULATE: out = float32 [T][d], set by the call to
 *        sum_j topk_w[t,j] * o[t,j] + o_shared[t] (the call zeroes it first); shared_out
 *        unused. The order of the float32 additions is not fixed.
 *   mode MOE_FFN_PER_ASSIGN: out = float32 [T*k][d] in sorted order (unweighted);
 *        shared_out = float32 [T][d] when the layer has a shared expert, else NULL.
 *   path: MOE_PATH_DECODE = tcgen05 kernel for at most 8 tokens, one CTA per (expert,
 *        64-column slice of I) computing gate/up, SwiGLU, h and that slice's share of
 *        the down projection (needs T <= 8, MOE_FFN_ACCUMULATE, d % 512 == 0,
 *        I % 64 == 0 and both groups packed by moe_pack_experts, slices included);
 *        MOE_PATH_PREFILL = tcgen05 block-scaled grouped GEMMs over 128-token tiles
 *        (any T; needs d % 256 == 0, I % 256 == 0 and packed scales);
 *        MOE_PATH_CUDA_CORE = the CUDA-core kernel on the natural layout (d % 16 == 0,
 *        I % 16 == 0); MOE_PATH_AUTO = DECODE when its requirements hold, else PREFILL
 *        when its requirements hold, else CUDA_CORE.
 * Limits: d <= 8192, I <= 8192. The workspace (moe_workspace_size(MOE_OP_FFN, ...)) holds
 * the tile schedule, the NVFP4 intermediate h and, above 64 tokens, the gathered
 * activation rows. Device waits that exceed 2 s end the kernel and set the device status
 * to MOE_ERR_TIMEOUT (read it with moe_get_device_status).
 */
moe_status moe_expert_ffn(const uint8_t* xq_codes, const uint8_t* xq_scales,
                          const float* xq_ts, int32_t T, const moe_experts_t* W, int32_t k,
                          const int32_t* offsets, const int32_t* sorted_assign,
                          const float* topk_w, int32_t mode, int32_t path, float* out,
                          float* shared_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn_static - moe_expert_ffn with static per-expert input scales: each expert
 * quantises its own token rows from the bf16 activations with its own static tensor scale,
 * and its h with its own static scale, instead of one per-call quantisation of the
 * activations and h scale 1.0. Source: "Basalt" project page, "All the numbers", list
 * "Engines: commit, and what is not NVIDIA's weights" (the llama.cpp row keeps NVIDIA's
 * experts bit-exact including their input_scale).
 *   x_bf16 [T][d] (16-byte aligned); in_scale_gu, in_scale_dn: float32 [E + has_shared]
 *   (device; the shared expert's at index E): per expert, the tensor scale of its
 *   activations and of its h (dequantisation multipliers, e.g. a calibrated amax / 2688).
 *   Block scales and codes follow nvfp4_quantize_act with ts_in = the expert's scale.
 *   Other arguments, modes and outputs as moe_expert_ffn. Always the tcgen05 PREFILL kernel
 *   (any T; needs d % 256 == 0, I % 256 == 0, d <= 2048, I <= 768, the natural-layout
 *   weights and the scales packed by moe_pack_experts), with every routed row quantised
 *   once per (token, expert) by the row-gather step. The workspace is
 *   moe_workspace_size(MOE_OP_FFN_STATIC, ...).
 */
moe_status moe_expert_ffn_static(const uint16_t* x_bf16, int32_t T, const moe_experts_t* W,
                                 const float* in_scale_gu, const float* in_scale_dn, int32_t k,
                                 const int32_t* offsets, const int32_t* sorted_assign,
                                 const float* topk_w, int32_t mode, float* out, float* shared_out,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * moe_combine - weighted combine (A9) and cast to bf16: a token's output is the sum of its
 * selected experts' outputs, weighted by the routing weights ("What Basalt changes in a
 * Blackwell local inference stack", section "Experts can move without becoming free").
 *   mode MOE_FFN_ACCUMULATE: expert_out = y_acc float32 [T][d]; y = bf16(y_acc).
 *   mode MOE_FFN_PER_ASSIGN: y[t] = sum_j topk_w[t,j] * expert_out[assign_pos[t*k+j]]
 *        + shared_out[t] (shared_out may be NULL).
 *   rms_renorm != 0: each output row is scaled to unit root-mean-square before the cast
 *        (an all-zero row stays zero); used to chain layers of a decode stack.
 *   y_bf16 [T][d] out.
 */
moe_status moe_combine(int32_t T, int32_t d, int32_t k, int32_t mode, const float* expert_out,
                       const float* shared_out, const float* topk_w,
                       const int32_t* assign_pos, int32_t rms_renorm, uint16_t* y_bf16,
                       void* stream);

/*
 * moe_layer_decode - one whole MoE layer forward for at most 8 tokens in one kernel launch:
 * activation quantisation (as nvfp4_quantize_act), router, top-k and weights, permutation
 * and per-call histogram (as moe_route), the expert FFN with the shared expert (as
 * moe_expert_ffn, MOE_FFN_ACCUMULATE, DECODE path) and the combine into bf16 (as
 * moe_combine). The same steps as those calls in that order, with the same outputs, for
 * the decode case where each of them is a few microseconds of work and their launches and
 * memory round trips would cost more than the work (Basalt pages: "What Basalt changes in a
 * Blackwell local inference stack", section "Experts can move without becoming free").
 *   x_bf16 [T][d]; ts_in float32[1] static activation scale or NULL (dynamic amax);
 *   Wr float32 [E][d]; br float32 [E] or NULL; W: both groups with the decode pack
 *   (dec_pack) of moe_pack_experts.
 *   Outputs: xq_codes [T][d/2], xq_scales [T][d/16], xq_ts [1]; topk_idx [T][k],
 *   topk_w [T][k]; counts [E], offsets [E+1], sorted_assign [T*k], assign_pos [T*k];
 *   y_acc float32 [T][d] (the unrounded output); y_bf16 [T][d]; rms_renorm as moe_combine.
 *   ws: moe_workspace_size(MOE_OP_LAYER_DECODE, ...) bytes, zero-filled before the first
 *   call. Its first 2048 bytes are a header: at byte 0 the 64-bit arrival count of the
 *   kernel's grid-wide barrier and of its final done count, which every call leaves at a
 *   multiple of the grid size; at byte 1024 a mark that a CTA sets when it gives up at a
 *   bounded wait (moe_get_device_status then reports MOE_ERR_TIMEOUT); at byte 1536 a word
 *   the library never writes: while it is nonzero, CTA 0 holds back its barrier arrival, so
 *   the other CTAs' bounded waits run out (tests use it to exercise that path). A call that
 *   finds the mark set computes nothing, writes no output and sets the device status to
 *   MOE_ERR_WORKSPACE; zero the workspace again to recover.
 * Limits: 1 <= T <= 8, d % 512 == 0, d <= 4096, I % 64 == 0, 1 <= k <= 32, k <= E <= 1024,
 * and at most 32 units per CTA in the worst case ((min(T*k, E) + shared) * I/64 units over
 * all SMs but one); otherwise MOE_ERR_UNSUPPORTED_SHAPE.
 * The kernel uses all SMs but one and waits at a grid-wide barrier. It is launched as a
 * cooperative grid, so the launch fails (MOE_ERR_CUDA) rather than start when its CTAs cannot
 * all be resident; while it runs, other kernels on the GPU get one SM.
 */
moe_status moe_layer_decode(const uint16_t* x_bf16, int32_t T, const float* ts_in, const float* Wr,
                            const float* br, const moe_experts_t* W, int32_t k, uint8_t* xq_codes,
                            uint8_t* xq_scales, float* xq_ts, int32_t* topk_idx, float* topk_w,
                            int32_t* counts, int32_t* offsets, int32_t* sorted_assign,
                            int32_t* assign_pos, float* y_acc, uint16_t* y_bf16, int32_t rms_renorm,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_hist - cumulative routing counts and hot-to-cold ranking (A10). Source:
 * "Basalt" project page, section "Expert tiers" (the busiest experts are kept in VRAM, and
 * the tiers follow the conversation as it shifts) and its FAQ "Can it use a second GPU or
 * system RAM?".
 *   counts int32 [E] (this call's histogram), cum int64 [E] in/out (cum += counts, or
 *   cum = counts when reset != 0), rank_out int32 [E] or NULL: expert ids from most to
 *   least routed, equal counts by lower id. E <= 4096.
 */
moe_status moe_expert_hist(const int32_t* counts, int32_t E, int64_t* cum, int32_t* rank_out,
                           int32_t reset, void* stream);

/*
 * moe_hot_tier_update - puts the top-ranked experts of a group into its hot tier. Source:
 * "Basalt" project page, section "Expert tiers" (the busiest experts are kept in the
 * fastest memory and the tiers follow the conversation as it shifts) and its FAQ "Can it
 * use a second GPU or system RAM?". On one B200 every expert is in HBM; the fastest tier
 * is the L2 cache, so the hot tier is a compact copy of the hot experts' decode-pack units
 * that moe_layer_decode reads instead of dec_pack and marks as persisting in L2 for its
 * launch (an access-policy window; see moe_set_l2_persisting for the set-aside it uses).
 *   W: the group, with its decode pack; rank int32 [E] device: expert ids from most to
 *   least routed (moe_expert_hist's rank_out); n_hot in [0, E];
 *   hot_pack: n_hot * (I/64) * (d/256 + d/512) * 18432 bytes, 16-byte aligned, out;
 *   hot_slot int32 [E] device out: slot i < n_hot for expert rank[i], -1 for the others.
 * Stream-ordered: calls on the same stream after it read the new tier, calls before it
 * the old one. Put the two pointers and n_hot into the group's hot_pack, hot_slot and
 * n_hot (once; later updates rewrite the same buffers). Needs E % 4 == 0 and d % 512 == 0.
 */
moe_status moe_hot_tier_update(const moe_expert_weights_t* W, const int32_t* rank, int32_t n_hot,
                               uint8_t* hot_pack, int32_t* hot_slot, void* stream);

/*
 * moe_set_l2_persisting - size of the L2 set-aside for lines accessed as persisting (the
 * hot tier's window) in this process's CUDA context on the current device, clamped to the
 * device's maximum (the driver may round it up to its granularity); 0 gives the set-aside
 * back and returns persisting lines to normal. It
 * is part of the context's state, not a setting of the GPU: it ends with the context
 * (process exit or cudaDeviceReset) and other processes do not see it. Writes the size in
 * effect to *bytes_out when not NULL.
 */
moe_status moe_set_l2_persisting(size_t bytes, size_t* bytes_out);

/*
 * moe_route_noalloc - moe_route for callers that cannot give the library any scratch
 * memory: for instance a serving process that reserves all device memory up front and
 * allows no later allocation, a C host with no device allocator of its own, or code that is
 * capturing a CUDA graph, where cudaMalloc may not be called. The Basalt pages have no
 * counterpart of this call; it exists for such callers only.
 *   Same arguments, outputs and results as moe_route, minus ws/ws_bytes. The scratch is one
 *   256 KiB array compiled into the library and held by every GPU that loads it until the
 *   process exits; calls whose scratch need (moe_workspace_size(MOE_OP_ROUTE, ...)) exceeds
 *   256 KiB return MOE_ERR_UNSUPPORTED_SHAPE. With T*k <= 4096 the scratch is the T*E float32
 *   router logits alone, so T*E <= 65536 fits (e.g. 64 tokens with 1024 experts, or 128
 *   tokens with 512 experts); above 4096 assignments per-chunk histograms are added.
 *   It allocates nothing. The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before capturing any stream. The address is
 *   kept for the life of the process, so no call may follow a cudaDeviceReset.
 *   All calls share the one array, which keeps the last call's contents (nothing in it needs
 *   to start at zero). Calls that overlap on the GPU - on different streams or from
 *   different host threads - race on it and give undefined results.
 */
moe_status moe_route_noalloc(const uint16_t* x_bf16, int32_t T, int32_t d, const float* Wr,
                             const float* br, int32_t E, int32_t k, int32_t* topk_idx,
                             float* topk_w, int32_t* counts, int32_t* offsets,
                             int32_t* sorted_assign, int32_t* assign_pos, void* stream);

/* Bytes of workspace needed by one op (MOE_OP_*) for these sizes (MOE_OP_LAYER: max). */
size_t moe_workspace_size(int32_t op, int64_t T, int32_t d, int32_t E, int32_t k, int32_t I);

/* Synchronise `stream` and return the device status word of the current device: MOE_OK,
 * MOE_ERR_TIMEOUT (a bounded device-side wait ran out; the kernel stopped early and its
 * outputs are not valid) or MOE_ERR_WORKSPACE (moe_layer_decode found its workspace marked
 * by an earlier call that gave up). `clear` != 0 resets it afterwards. */
moe_status moe_get_device_status(void* stream, int32_t clear, int32_t* status_out);

/* How long a device-side wait (for a copy, a tensor-core result, another CTA) may last before
 * the kernel gives up and reports MOE_ERR_TIMEOUT, for kernels launched on the current device
 * from now on, including replays of captured graphs. Default 2 s; allowed 1 ms .. 60 s. A
 * short limit can end a long call early: the waits of the PREFILL path last up to the length
 * of the call. */
moe_status moe_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code, and a per-thread detail of the last failure. */
const char* moe_status_string(moe_status s);
const char* moe_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t moe_version(void);

/* Number of kernels this library has enqueued in this process, counted on the host when
 * each launch is issued (all devices and streams). A launch recorded into a CUDA graph
 * counts once at capture; replays of the graph do not add to it. Instrumentation for
 * launch accounting; the Basalt pages have no counterpart. */
uint64_t moe_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_NVFP4_H */
