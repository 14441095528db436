"""Shared test helpers: build the same layer on both sides, compare with the tolerances.

Weights: synth draws bf16 weights; the oracle quantises them on the CPU, the CUDA path
quantises them on the GPU (or receives the oracle's codes for small cases). Nothing the
oracle uses ever comes from the CUDA path.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe as omoe
from oracle import nvfp4 as onv
from oracle.weights import OracleWeights, expert_from_bf16  # noqa: F401
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import synth

F32 = np.float32

# float tolerance of the layer output (against the float64 oracle before bf16 rounding)
REL_L2_TOL = 5e-3
MAX_ABS_TOL_RMS = 2e-2
# top-k comparisons excuse tokens whose k-th/(k+1)-th float32 logit margin is below this
TIE_MARGIN = 1e-6


def bits_to_f32(bits) -> np.ndarray:
    b = np.asarray(bits)
    return (b.astype(np.uint16).astype(np.uint32) << 16).view(F32)


def assert_close_layer(y_gpu, y_ref, what=""):
    """rel-L2 <= 5e-3 and max-abs <= 2e-2 * RMS(y_ref)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y_gpu.shape == y_ref.shape, (y_gpu.shape, y_ref.shape)
    if y_ref.size == 0:
        return
    assert np.all(np.isfinite(y_gpu)), what
    nrm = np.linalg.norm(y_ref)
    rel = np.linalg.norm(y_gpu - y_ref) / max(nrm, 1e-300)
    rms = nrm / np.sqrt(y_ref.size)
    mabs = np.max(np.abs(y_gpu - y_ref))
    assert rel <= REL_L2_TOL, f"{what}: rel-L2 {rel:.3e} > {REL_L2_TOL}"
    assert mabs <= MAX_ABS_TOL_RMS * rms, f"{what}: max-abs {mabs:.3e} > {MAX_ABS_TOL_RMS}*{rms:.3e}"
    return rel, mabs / rms


oracle_expert_from_bf16 = expert_from_bf16


def weights_to_gpu(experts, device="cuda", pack=False) -> B.ExpertWeights:
    """Upload a list of oracle Expert objects (their codes) as one GPU expert group;
    optionally re-tile its scales for the tensor-core path."""
    gu_c = np.stack([e.gu_codes for e in experts])
    gu_s = np.stack([e.gu_scales for e in experts])
    gu_t = np.array([[e.gate_ts, e.up_ts] for e in experts], dtype=F32)
    dn_c = np.stack([e.dn_codes for e in experts])
    dn_s = np.stack([e.dn_scales for e in experts])
    dn_t = np.array([e.dn_ts for e in experts], dtype=F32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)  # noqa: E731
    w = B.ExpertWeights(t(gu_c), t(gu_s), t(gu_t), t(dn_c), t(dn_s), t(dn_t))
    if pack:
        B.moe_pack_experts(w)
    return w


def topk_margins(logits, k) -> np.ndarray:
    """k-th minus (k+1)-th largest float32 logit per token (inf when k == E)."""
    s = -np.sort(-np.asarray(logits, dtype=np.float64), axis=1)
    if s.shape[1] <= k:
        return np.full(s.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


def compare_topk(idx_gpu, idx_ref, logits_ref, k):
    """Set-wise top-k comparison; returns the tokens excused by the tie margin."""
    idx_gpu = np.asarray(idx_gpu)
    idx_ref = np.asarray(idx_ref)
    margins = topk_margins(logits_ref, k)
    bad = [t for t in range(idx_ref.shape[0]) if set(idx_gpu[t]) != set(idx_ref[t])]
    excused = [t for t in bad if margins[t] < TIE_MARGIN]
    unexcused = [t for t in bad if margins[t] >= TIE_MARGIN]
    assert not unexcused, f"top-k differs beyond the tie margin for tokens {unexcused[:10]}"
    return excused


def check_permutation_valid(idx, counts, offsets, sorted_assign, assign_pos, E):
    """Properties any correct stable counting sort of idx has (used when tie-excused tokens
    make the GPU's routing legitimately differ from the oracle's)."""
    flat = np.asarray(idx).reshape(-1).astype(np.int64)
    n = flat.size
    assert np.array_equal(np.asarray(counts), np.bincount(flat, minlength=E))
    assert np.array_equal(np.asarray(offsets), np.concatenate([[0], np.cumsum(counts)]))
    sa = np.asarray(sorted_assign)[:n]
    assert np.array_equal(np.sort(sa), np.arange(n))
    assert np.array_equal(np.asarray(assign_pos)[:n][sa], np.arange(n))
    for e in range(E):
        seg = sa[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


def route_buffers(T, k, E, d, I=16, device="cuda"):
    return dict(
        topk_idx=torch.empty(T, k, dtype=torch.int32, device=device),
        topk_w=torch.empty(T, k, dtype=torch.float32, device=device),
        counts=torch.empty(E, dtype=torch.int32, device=device),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
        sorted_assign=torch.empty(max(1, T * k), dtype=torch.int32, device=device),
        assign_pos=torch.empty(max(1, T * k), dtype=torch.int32, device=device),
        ws=torch.empty(max(256, B.moe_workspace_size(B.MOE_OP_LAYER, T, d, E, k, I)),
                       dtype=torch.uint8, device=device))
