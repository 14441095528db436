"""Mixture-of-experts layer forward, plain and slow (oracle; test infrastructure only).

Sources on the Basalt pages:
  * "What Basalt changes in a Blackwell local inference stack", section "Experts can move
    without becoming free": experts are parameter groups, and the model selects a subset of
    them for each token.
  * "Basalt" project page, section "Expert tiers" and FAQ "Can it use a second GPU or system
    RAM?": each token uses a few experts; the most routed experts are the hot tier.
The routing rule, the FFN form and the permutation are not written on the pages; readings
R4-R7 (package docstring) are used. Each function below states its reading.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

F32 = np.float32


# --------------------------------------------------------------------------- router (A1, A2)

def router_logits(x_f32, Wr, br=None) -> np.ndarray:
    """Reading R4: logits[t, e] = sum_i x[t, i] * Wr[e, i] + br[e], summed in float64 and
    rounded once to float32. x is the bf16 activation widened exactly to float32."""
    x64 = np.asarray(x_f32, dtype=np.float64)
    W64 = np.asarray(Wr, dtype=np.float64)
    logits = x64 @ W64.T
    if br is not None:
        logits = logits + np.asarray(br, dtype=np.float64)[None, :]
    return logits.astype(F32)


def topk(logits, k: int) -> np.ndarray:
    """Reading R4: the k largest float32 logits of each token, in descending order; equal
    logits are ordered by the lower expert index. Returns int32 [T][k]."""
    logits = np.asarray(logits, dtype=F32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    order_key = np.arange(E)
    for t in range(T):
        # sort by (-logit, index): descending logit, ascending index among equals
        order = sorted(order_key, key=lambda e: (-float(logits[t, e]), e))
        idx[t] = order[:k]
    return idx


def topk_fast(logits, k: int) -> np.ndarray:
    """Same result as ``topk`` for large T (vectorised with a stable sort on -logit)."""
    logits = np.asarray(logits, dtype=F32)
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def routing_weights(logits, idx) -> np.ndarray:
    """Reading R4: softmax over all E logits, restricted to the chosen k and renormalised.
    The common factor cancels, so w_j = exp(l_j - m) / sum_{j' in top-k} exp(l_j' - m)
    with m the largest chosen logit; float64, rounded once to float32."""
    l = np.take_along_axis(np.asarray(logits, dtype=np.float64), np.asarray(idx), axis=1)
    if l.shape[1] == 0:
        return l.astype(F32)
    m = np.max(l, axis=1, keepdims=True)
    e = np.exp(l - m)
    return (e / np.sum(e, axis=1, keepdims=True)).astype(F32)


# --------------------------------------------------------------------------- permutation (A3)

def permute(idx, E: int):
    """Reading R6: stable counting sort of the T*k assignments a = t*k + j by expert.

    Returns counts int32 [E], offsets int32 [E+1] (exclusive prefix sum of counts),
    sorted_assign int32 [T*k] (assignment ids grouped by expert, increasing a inside an
    expert) and assign_pos int32 [T*k] (position of assignment a in sorted_assign)."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    n = flat.size
    counts = np.zeros(E, dtype=np.int64)
    for a in range(n):
        counts[flat[a]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:E].copy()
    sorted_assign = np.empty(n, dtype=np.int64)
    assign_pos = np.empty(n, dtype=np.int64)
    for a in range(n):
        e = flat[a]
        sorted_assign[fill[e]] = a
        assign_pos[a] = fill[e]
        fill[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            sorted_assign.astype(np.int32), assign_pos.astype(np.int32))


# --------------------------------------------------------------------------- expert FFN (A5-A8)

def silu(g):
    """silu(g) = g / (1 + exp(-g)), float64."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


class Expert:
    """One expert's NVFP4 weights: gate and up [I][d] (stored as one [2I][d] matrix, gate
    rows first), down [d][I], each with its own float32 tensor scale."""

    def __init__(self, gu_codes, gu_scales, gate_ts, up_ts, dn_codes, dn_scales, dn_ts):
        self.gu_codes, self.gu_scales = np.asarray(gu_codes), np.asarray(gu_scales)
        self.gate_ts, self.up_ts, self.dn_ts = F32(gate_ts), F32(up_ts), F32(dn_ts)
        self.dn_codes, self.dn_scales = np.asarray(dn_codes), np.asarray(dn_scales)
        self.I = self.gu_codes.shape[0] // 2

    @classmethod
    def from_f32(cls, gate, up, down):
        """Quantise float32 gate/up/down matrices (one tensor scale per matrix)."""
        gc, gs, gts = nvfp4.quantize(np.asarray(gate, dtype=F32))
        uc, us, uts = nvfp4.quantize(np.asarray(up, dtype=F32))
        dc, ds, dts = nvfp4.quantize(np.asarray(down, dtype=F32))
        return cls(np.concatenate([gc, uc]), np.concatenate([gs, us]), gts, uts, dc, ds, dts)

    def dense(self):
        """Exact float64 (gate [I][d], up [I][d], down [d][I])."""
        I = self.I
        g = nvfp4.dequantize(self.gu_codes[:I], self.gu_scales[:I], self.gate_ts)
        u = nvfp4.dequantize(self.gu_codes[I:], self.gu_scales[I:], self.up_ts)
        dn = nvfp4.dequantize(self.dn_codes, self.dn_scales, self.dn_ts)
        return g, u, dn


def expert_ffn(x_hat, expert: Expert, dense=None, h_ts=1.0):
    """Reading R5 for a batch of dequantised token rows x_hat float64 [n][d]:
        g = x_hat Wg^T, u = x_hat Wu^T         (float64)
        h = silu(g) * u                        (float64, rounded once to float32)
        h_hat = NVFP4(h) with tensor scale h_ts (blocks of 16 along I); h_ts is 1.0 unless
                the expert has a static input scale for its down projection (R13)
        o = h_hat Wd^T                         (float64)
    Returns o float64 [n][d]."""
    Wg, Wu, Wd = dense if dense is not None else expert.dense()
    x_hat = np.asarray(x_hat, dtype=np.float64)
    if x_hat.shape[0] == 0:
        return np.zeros((0, Wd.shape[0]))
    g = x_hat @ Wg.T
    u = x_hat @ Wu.T
    h = (silu(g) * u).astype(F32)
    hc, hs, hts = nvfp4.quantize(h, ts=F32(h_ts))
    h_hat = nvfp4.dequantize(hc, hs, hts)
    return h_hat @ Wd.T


def expert_ffn_static(x_f32, expert: Expert, in_gu, in_dn, dense=None):
    """Reading R13, static per-expert input scales ("Basalt" project page, "All the numbers",
    list "Engines: commit, and what is not NVIDIA's weights": NVIDIA's NVFP4 experts come
    with their input_scale): the expert's token rows x (float32 [n][d], the bf16
    activations) are quantised to NVFP4 with the expert's own static tensor scale in_gu
    instead of the per-call dynamic one, and h with the expert's static scale in_dn; the
    rest is expert_ffn. Returns o float64 [n][d]."""
    xc, xs, xts = nvfp4.quantize(np.asarray(x_f32, dtype=F32), ts=F32(in_gu))
    return expert_ffn(nvfp4.dequantize(xc, xs, xts), expert, dense, h_ts=in_dn)


def ffn_static_forward(x_bits, idx, w, experts, shared, in_gu, in_dn, tokens=None):
    """The expert FFN and the combine (A5-A9) with static per-expert input scales (R13) for a
    given routing: y[t] = sum_j w[t, j] * o_{idx[t, j]}(x_t) + o_shared(x_t), every o from
    expert_ffn_static with that expert's scales (the shared expert's at index E of in_gu and
    in_dn). x_bits: bf16 bit patterns [T][d]; idx, w: [T][k]. Rows outside `tokens` (default
    all) are NaN. Returns y float64 [T][d]."""
    x_bits = np.asarray(x_bits)
    T, d = x_bits.shape
    E = len(experts)
    k = np.asarray(idx).shape[1]
    x_f32 = (x_bits.astype(np.uint16).astype(np.uint32) << 16).view(F32).reshape(T, d)
    tokens = np.arange(T) if tokens is None else np.asarray(sorted(set(tokens)))
    idx, w = np.asarray(idx), np.asarray(w)
    o = {}
    for e in range(E):
        rows = [(t, j) for t in tokens for j in range(k) if idx[t, j] == e]
        if rows:
            oe = expert_ffn_static(x_f32[[t for t, _ in rows]], experts[e], in_gu[e], in_dn[e])
            for (t, j), r in zip(rows, oe):
                o[(t, j)] = r
    o_shared = None
    if shared is not None:
        o_shared = np.zeros((T, d))
        o_shared[tokens] = expert_ffn_static(x_f32[tokens], shared, in_gu[E], in_dn[E])
    y = np.full((T, d), np.nan)
    if tokens.size:
        o_assign = np.concatenate([np.stack([o[(t, j)] for j in range(k)]) for t in tokens])
        y[tokens] = combine(len(tokens), d, idx[tokens], w[tokens], o_assign,
                            None if o_shared is None else o_shared[tokens])
    return y


# --------------------------------------------------------------------------- combine (A9)

def combine(T: int, d: int, idx, w, o_assign, o_shared=None):
    """y[t] = sum_j w[t, j] * o[t*k + j] + o_shared[t]   (float64). Reading R5: the shared
    expert is an ungated add with weight 1. o_assign is indexed by assignment id t*k + j."""
    k = np.asarray(idx).shape[1] if T else 0
    y = np.zeros((T, d))
    w64 = np.asarray(w, dtype=np.float64)
    for t in range(T):
        for j in range(k):
            y[t] += w64[t, j] * o_assign[t * k + j]
    if o_shared is not None:
        y += o_shared
    return y


def rms_renorm(y):
    """Per-token RMS normalisation to 1 (used to chain layers of the decode stack);
    an all-zero row stays zero."""
    y = np.asarray(y, dtype=np.float64)
    ms = np.mean(y * y, axis=1, keepdims=True)
    return np.where(ms > 0, y / np.sqrt(np.where(ms > 0, ms, 1.0)), 0.0)


# --------------------------------------------------------------------------- histogram (A10)

def hist_update(counts, cum=None, reset=False):
    """Reading R7: cum += counts (int64); rank lists expert ids from most to least routed,
    equal counts ordered by the lower id."""
    counts = np.asarray(counts, dtype=np.int64)
    cum = np.zeros_like(counts) if (cum is None or reset) else np.asarray(cum, np.int64)
    cum = cum + counts
    E = counts.size
    rank = sorted(range(E), key=lambda e: (-int(cum[e]), e))
    return cum, np.asarray(rank, dtype=np.int32)


# --------------------------------------------------------------------------- whole layer

def layer_forward(x_bits, Wr, br, k, experts, shared=None, ts_x=None, assign_subset=None):
    """One MoE layer forward (steps A1-A10 in order).

    x_bits: bf16 bit patterns int16/uint16 [T][d]. experts: list of Expert. shared: Expert
    or None. ts_x: static activation tensor scale or None (dynamic). assign_subset: optional
    token ids; when given, the FFN and combine run only for those tokens (routing and the
    permutation always cover all tokens).

    Returns a dict with the quantised activation, routing outputs, permutation, y (float64
    [T][d], rows outside the subset are NaN) and the per-call counts."""
    x_bits = np.asarray(x_bits)
    T, d = x_bits.shape
    E = len(experts)
    x_f32 = (x_bits.astype(np.uint16).astype(np.uint32) << 16).view(F32).reshape(T, d)
    xc, xs, xts = nvfp4.quantize(x_f32, ts=ts_x)
    logits = router_logits(x_f32, Wr, br)
    idx = topk_fast(logits, k)
    w = routing_weights(logits, idx)
    counts, offsets, sorted_assign, assign_pos = permute(idx, E)
    x_hat = nvfp4.dequantize(xc, xs, xts)

    tokens = np.arange(T) if assign_subset is None else np.asarray(sorted(set(assign_subset)))
    want = np.zeros(T, dtype=bool)
    want[tokens] = True
    o_assign = np.full((T * k, d), np.nan)
    for e in range(E):
        seg = sorted_assign[offsets[e]:offsets[e + 1]]
        seg = seg[want[seg // k]]
        if seg.size == 0:
            continue
        o_assign[seg] = expert_ffn(x_hat[seg // k], experts[e])
    o_shared = None
    if shared is not None:
        o_shared = np.full((T, d), np.nan)
        o_shared[tokens] = expert_ffn(x_hat[tokens], shared)
    y = np.full((T, d), np.nan)
    if tokens.size:
        sub_idx = idx[tokens]
        sub_w = w[tokens]
        sub_o = np.concatenate([o_assign[t * k:(t + 1) * k] for t in tokens])
        y[tokens] = combine(len(tokens), d, sub_idx, sub_w, sub_o,
                            None if o_shared is None else o_shared[tokens])
    return dict(x_codes=xc, x_scales=xs, x_ts=xts, logits=logits, idx=idx, w=w,
                counts=counts, offsets=offsets, sorted_assign=sorted_assign,
                assign_pos=assign_pos, y=y, tokens=tokens)
