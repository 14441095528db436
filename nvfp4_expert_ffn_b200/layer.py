"""One MoE layer forward through the C ABI: buffers on the GPU and the five calls in order.

    quantise x -> route (router, top-k, permutation) -> expert FFN -> combine -> histogram

Each step is one call of libmoe_nvfp4.so; this module only allocates device buffers
(torch) and passes pointers.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B
from . import synth


def quantize_weights_gpu(seed: int, cfg: synth.LayerShape, layer: int = 0, device="cuda",
                         experts: Optional[range] = None, shared: bool = False,
                         ws: Optional[torch.Tensor] = None, pack: bool = True,
                         decode_only: bool = False, chunk: int = 32) -> B.ExpertWeights:
    """Generate an expert group's bf16 weights on the GPU (a chunk of experts at a time) and
    quantise each matrix (gate, up, down of every expert, one tensor scale each) with
    nvfp4_quantize_act; then re-tile the scales for the tensor-core path (moe_pack_experts)
    when the shape allows. decode_only: keep only the decode pack and the tensor scales."""
    E = 1 if shared else cfg.E
    d, I = cfg.d, cfg.I
    w = B.ExpertWeights(
        gu_codes=torch.empty(E, 2 * I, d // 2, dtype=torch.uint8, device=device),
        gu_scales=torch.empty(E, 2 * I, d // 16, dtype=torch.uint8, device=device),
        gu_ts=torch.empty(E, 2, dtype=torch.float32, device=device),
        dn_codes=torch.empty(E, d, I // 2, dtype=torch.uint8, device=device),
        dn_scales=torch.empty(E, d, I // 16, dtype=torch.uint8, device=device),
        dn_ts=torch.empty(E, dtype=torch.float32, device=device))
    if ws is None:
        ws = torch.empty(B.moe_workspace_size(B.MOE_OP_QUANT, 1, d, 1, 1, I),
                         dtype=torch.uint8, device=device)
    for e0 in range(0, E, chunk):
        ids = range(e0, min(E, e0 + chunk))
        g, u, dn = synth.make_experts_weights_bf16(seed, cfg, ids, layer, shared, device)
        for r, e in enumerate(ids):
            B.nvfp4_quantize_act(g[r], w.gu_codes[e, :I], w.gu_scales[e, :I], w.gu_ts[e, 0:1], ws=ws)
            B.nvfp4_quantize_act(u[r], w.gu_codes[e, I:], w.gu_scales[e, I:], w.gu_ts[e, 1:2], ws=ws)
            B.nvfp4_quantize_act(dn[r], w.dn_codes[e], w.dn_scales[e], w.dn_ts[e:e + 1], ws=ws)
        del g, u, dn
    if pack and d % 128 == 0 and I % 64 == 0:
        B.moe_pack_experts(w)
        if decode_only:
            w.release_natural()
    return w


class MoeLayer:
    """Device buffers for one layer and up to T_max tokens per call."""

    def __init__(self, experts: B.Experts, Wr: torch.Tensor, br: Optional[torch.Tensor], k: int,
                 T_max: int, static_ts: Optional[torch.Tensor] = None, device="cuda",
                 fused: Optional[bool] = None, input_scales: Optional[tuple] = None):
        """input_scales: optional (in_gu, in_dn) float32 [E + 1] device tensors, static
        per-expert input scales (moe_expert_ffn_static); the layer then skips the per-call
        activation quantisation and always runs the five-call path."""
        self.experts, self.Wr, self.br, self.k = experts, Wr, br, k
        self.input_scales = input_scales
        r = experts.routed
        self.E, self.d, self.I = r.E, r.d, r.I
        self.T_max = T_max
        self.static_ts = static_ts
        d, E, k, I = self.d, self.E, k, self.I
        dev = device
        self.xq_codes = torch.empty(T_max, d // 2, dtype=torch.uint8, device=dev)
        self.xq_scales = torch.empty(T_max, d // 16, dtype=torch.uint8, device=dev)
        self.xq_ts = torch.empty(4, dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty(T_max, k, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(T_max, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.sorted_assign = torch.empty(max(1, T_max * k), dtype=torch.int32, device=dev)
        self.assign_pos = torch.empty(max(1, T_max * k), dtype=torch.int32, device=dev)
        self.y_acc = torch.empty(T_max, d, dtype=torch.float32, device=dev)
        self.y = torch.empty(T_max, d, dtype=torch.int16, device=dev)
        self.cum = torch.zeros(E, dtype=torch.int64, device=dev)
        self.rank = torch.empty(E, dtype=torch.int32, device=dev)
        ws = B.moe_workspace_size(B.MOE_OP_LAYER, T_max, d, E, k, I)
        if input_scales is not None:
            ws = max(ws, B.moe_workspace_size(B.MOE_OP_FFN_STATIC, T_max, d, E, k, I))
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        # the quantiser runs concurrently with the router, so it gets its own workspace
        self.ws_q = torch.empty(B.moe_workspace_size(B.MOE_OP_QUANT, T_max, d, E, k, I),
                                dtype=torch.uint8, device=dev)
        self.path = B.MOE_PATH_AUTO
        self._side = torch.cuda.Stream(device=dev)
        self._ev = [torch.cuda.Event() for _ in range(4)]
        self._hist_pending = False  # the last call's histogram may still read self.counts
        # calls of at most 8 tokens go through the one-kernel decode layer when the shapes allow;
        # its workspace holds a barrier counter and must start zeroed
        can_fuse = (d % 512 == 0 and d <= 4096 and I % 64 == 0 and k <= 32 and E <= 1024
                    and experts.routed.dec_pack is not None
                    and (experts.shared is None or experts.shared.dec_pack is not None))
        can_fuse = can_fuse and input_scales is None
        self.fused = can_fuse if fused is None else (fused and can_fuse)
        self.ws_dec = torch.zeros(
            max(256, B.moe_workspace_size(B.MOE_OP_LAYER_DECODE, min(T_max, 8), d, E, k, I)),
            dtype=torch.uint8, device=dev) if self.fused else None

    def forward(self, x: torch.Tensor, rms_renorm: bool = False, stream=None,
                join: bool = True) -> torch.Tensor:
        """x: bf16 bits (int16 or bfloat16) [T][d] on the GPU. Returns y bf16 bits [T][d]
        (a view into this layer's output buffer). Enqueued on `stream` (default: current);
        work on the side stream (the quantiser, the expert histogram) forks from it and, with
        join=True, joins back at the end, so the call is capturable in a CUDA graph. With
        join=False the histogram may still run when the call returns; join(stream) later."""
        T, k = x.shape[0], self.k
        assert T <= self.T_max
        main = torch.cuda.current_stream() if stream is None else stream
        side, ev = self._side, self._ev
        if self._hist_pending:
            main.wait_event(ev[3])  # this call rewrites the counts the last histogram reads
        self._hist_pending = not join
        if self.fused and T <= 8:
            B.moe_layer_decode(x, self.static_ts, self.Wr, self.br, self.experts, k,
                               self.xq_codes[:T], self.xq_scales[:T], self.xq_ts[:1],
                               self.topk_idx[:T], self.topk_w[:T], self.counts, self.offsets,
                               self.sorted_assign[:T * k], self.assign_pos[:T * k],
                               self.y_acc[:T], self.y[:T], rms_renorm, self.ws_dec, stream=main)
            ev[2].record(main)
            side.wait_event(ev[2])
            B.moe_expert_hist(self.counts, self.cum, self.rank, stream=side)
            ev[3].record(side)
            if join:
                main.wait_event(ev[3])
            return self.y[:T]
        static = self.input_scales is not None
        if not static:
            ev[0].record(main)
            side.wait_event(ev[0])
            B.nvfp4_quantize_act(x, self.xq_codes[:T], self.xq_scales[:T], self.xq_ts[:1],
                                 ts_in=self.static_ts, ws=self.ws_q, stream=side)
            ev[1].record(side)
        B.moe_route(x, self.Wr, self.br, k, self.topk_idx[:T], self.topk_w[:T], self.counts,
                    self.offsets, self.sorted_assign[:T * k], self.assign_pos[:T * k], self.ws,
                    stream=main)
        ev[2].record(main)
        if static:
            B.moe_expert_ffn_static(x, self.experts, self.input_scales[0], self.input_scales[1], k,
                                    self.offsets, self.sorted_assign[:T * k], self.topk_w[:T],
                                    B.MOE_FFN_ACCUMULATE, self.y_acc[:T], None, self.ws, stream=main)
        else:
            main.wait_event(ev[1])
            B.moe_expert_ffn(self.xq_codes[:T], self.xq_scales[:T], self.xq_ts[:1], self.experts, k,
                             self.offsets, self.sorted_assign[:T * k], self.topk_w[:T],
                             B.MOE_FFN_ACCUMULATE, self.path, self.y_acc[:T], None, self.ws,
                             stream=main)
        side.wait_event(ev[2])
        B.moe_expert_hist(self.counts, self.cum, self.rank, stream=side)
        ev[3].record(side)
        B.moe_combine(T, self.d, k, B.MOE_FFN_ACCUMULATE, self.y_acc[:T], None, self.topk_w[:T],
                      self.assign_pos[:T * k], rms_renorm, self.y[:T], stream=main)
        if join:
            main.wait_event(ev[3])
        return self.y[:T]

    def update_hot_tier(self, n_hot: int, stream=None) -> None:
        """Refill the routed group's hot tier with the n_hot experts this layer has routed most
        so far (the ranking of its cumulative histogram); 0 turns the tier off. Enqueued on
        `stream` (default: current) after this layer's outstanding histogram. The one-kernel
        decode layer then reads those experts' units from the tier, as persisting in L2 (the
        process's set-aside: binding.moe_set_l2_persisting)."""
        main = torch.cuda.current_stream() if stream is None else stream
        self.join(main)
        B.moe_hot_tier_update(self.experts.routed, self.rank, n_hot, stream=main)

    def join(self, stream=None) -> None:
        """Make `stream` (default: current) wait for the side-stream work of the last
        forward(join=False) of this layer, if one is outstanding (otherwise nothing to do)."""
        if self._hist_pending:
            (torch.cuda.current_stream() if stream is None else stream).wait_event(self._ev[3])
            self._hist_pending = False

    def graphed(self, T: int, n_slots: int = 1, stream=None) -> "GraphedMoeLayer":
        """A replayable CUDA graph of forward() with its host copies, for a fixed token count."""
        return GraphedMoeLayer(self, T, n_slots=n_slots, stream=stream)


class GraphedMoeLayer:
    """forward() of one layer for a fixed token count, captured once as a CUDA graph together
    with its host copies: each replay copies one pinned host input slot to the device, runs
    the layer and copies y back to a pinned host buffer - one launch per step.

    Write a step's input (bf16 bits [T][d]) into ``x_host[slot]`` before ``run(slot)``, and
    read ``y_host`` after synchronising ``stream``. All replays go to ``stream``."""

    def __init__(self, layer: MoeLayer, T: int, rms_renorm: bool = False, n_slots: int = 1,
                 stream: Optional[torch.cuda.Stream] = None):
        self.layer, self.T = layer, T
        dev = layer.xq_codes.device
        self.x = torch.zeros(T, layer.d, dtype=torch.int16, device=dev)
        self.x_host = [torch.zeros(T, layer.d, dtype=torch.int16).pin_memory() for _ in range(n_slots)]
        self.y_host = torch.zeros(T, layer.d, dtype=torch.int16).pin_memory()
        self.stream = stream if stream is not None else torch.cuda.Stream(device=dev)
        with torch.cuda.stream(self.stream):
            layer.forward(self.x, rms_renorm)  # first calls do per-device set-up
        self.stream.synchronize()
        self.graphs = []
        for slot in range(n_slots):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.x.copy_(self.x_host[slot], non_blocking=True)
                y = layer.forward(self.x, rms_renorm, join=False)
                self.y_host.copy_(y, non_blocking=True)  # y does not wait for the histogram
                layer.join(self.stream)
            self.graphs.append(g)

    def run(self, slot: int = 0) -> None:
        """Asynchronous on self.stream: x_host[slot] -> device, the layer, y -> y_host."""
        with torch.cuda.stream(self.stream):  # a graph replays on the current stream
            self.graphs[slot].replay()

    def step(self, x_host: torch.Tensor, y_host: torch.Tensor) -> None:
        """Copy a host batch into slot 0 (synchronising the stream first, since the last
        replay may still be reading it), run, and copy y_host out after the replay ends."""
        self.stream.synchronize()
        self.x_host[0].copy_(x_host)
        self.run(0)
        self.stream.synchronize()
        y_host.copy_(self.y_host)
