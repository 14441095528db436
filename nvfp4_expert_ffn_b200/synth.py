"""Seeded synthetic inputs for the MoE layer: activations, router and expert weights.

This module only draws numbers. It holds none of the layer's arithmetic (no quantisation,
routing or FFN math), so that the CPU oracle and the CUDA path can both be fed from it
without sharing any code.

Generator: a counter-based hash (the splitmix64 output function applied to
``key + (i + 1) * 0x9E3779B97F4A7C15``), evaluated with integer tensor ops that give the
same bits on CPU and on CUDA. A normal deviate is approximated by the Irwin-Hall sum of the
four 16-bit lanes of one hash (mean 0, variance 1 after scaling), so no transcendental
function (whose last bits differ between libm and CUDA) is involved. Every float value is
produced by exactly one IEEE float32 multiply of an exact integer, so CPU and GPU agree
bit for bit.

Workload shapes follow the Basalt pages' MoE decode/prefill setting (page 2, "Experts can
move without becoming free": each token uses a subset of experts; page 3, "Expert tiers":
the most-routed experts are the hot ones). The pages give no dimensions; the sizes below
are the synthetic layer configurations this library is measured on.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _s64(v: int) -> int:
    """Two's-complement int64 view of an unsigned 64-bit integer."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _mix_py(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(*parts: int) -> int:
    """Fold integers (seed, config, layer, tensor id, expert ...) into one 64-bit key."""
    k = 0x5EED
    for p in parts:
        k = _mix_py(k ^ ((int(p) * _GOLDEN) & _MASK64))
    return k


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    # logical right shift on int64 tensors
    return (x >> s) & ((1 << (64 - s)) - 1)


def hash64(key: int, index: torch.Tensor) -> torch.Tensor:
    """splitmix64 output for counters ``index`` (int64 tensor) under ``key``."""
    z = index.to(torch.int64) + 1
    z = z * _s64(_GOLDEN) + _s64(key)
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


_IH4_SCALE = math.sqrt(3.0) / 131072.0  # (2*S - 4*65535) * this has unit variance


def normal_f32(key: int, n: int, std: float, device="cpu", offset: int = 0) -> torch.Tensor:
    """n approximately N(0, std^2) float32 values (Irwin-Hall of four 16-bit uniforms)."""
    idx = torch.arange(offset, offset + n, dtype=torch.int64, device=device)
    h = hash64(key, idx)
    s = (h & 0xFFFF) + (_lsr(h, 16) & 0xFFFF) + (_lsr(h, 32) & 0xFFFF) + _lsr(h, 48)
    zi = (2 * s - 4 * 65535).to(torch.float32)  # exact: |zi| <= 262140 < 2**24
    c = torch.tensor(np.float32(std * _IH4_SCALE), dtype=torch.float32, device=device)
    return zi * c


def f32_to_bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """Round float32 to bfloat16 (nearest, ties to even) and return the 16-bit patterns
    as int16 (same bits as uint16). Inputs here are finite."""
    b = x.contiguous().view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    b = b + 0x7FFF + ((b >> 16) & 1)
    return ((b >> 16) & 0xFFFF).to(torch.int32).to(torch.int16)


def bf16_bits_to_f32(bits: torch.Tensor) -> torch.Tensor:
    return (bits.to(torch.int32) << 16).view(torch.float32)


# ----------------------------------------------------------------------------------------
# workload configurations
# ----------------------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerShape:
    name: str
    cid: int               # integer id folded into the generator keys
    d: int                 # hidden size
    E: int                 # routed experts
    k: int                 # experts per token
    I: int                 # expert intermediate size
    shared: bool           # one always-on shared expert
    zipf_s: float          # router bias exponent (0 = none)
    router_std: float      # std of router weights
    weight_std: float = 0.02
    T_list: tuple = field(default=(16,))


CONFIGS = {
    # tiny parity layer
    "tiny": LayerShape("tiny", cid=1, d=256, E=8, k=2, I=128, shared=False, zipf_s=0.0,
                       router_std=0.02, T_list=(16,)),
    # decode layer, 1-8 tokens per call
    "decode": LayerShape("decode", cid=2, d=2048, E=512, k=10, I=512, shared=True, zipf_s=1.0,
                         router_std=0.02, T_list=(1, 4, 8)),
    # prefill layer, 16K tokens per call
    "prefill": LayerShape("prefill", cid=3, d=2048, E=512, k=10, I=512, shared=True, zipf_s=0.8,
                          router_std=0.02, T_list=(16384,)),
    # 48-layer decode stack, 8 tokens per step (hot set drifts every 64 steps)
    "stack48": LayerShape("stack48", cid=4, d=2048, E=512, k=10, I=512, shared=True, zipf_s=1.0,
                          router_std=0.02, T_list=(8,)),
    # wide experts, ragged prefill+decode mix batched in one call
    "wide": LayerShape("wide", cid=5, d=4096, E=256, k=8, I=2048, shared=True, zipf_s=0.0,
                       router_std=1.0 / 64.0, T_list=(512 + 2048 + 8192 + 16384 + 4,)),
}

# tensor ids inside one layer's key space
TID_X, TID_WR, TID_GATE, TID_UP, TID_DOWN, TID_SGATE, TID_SUP, TID_SDOWN, TID_PERM = range(9)


def make_x(seed: int, cfg: LayerShape, T: int, layer: int = 0, step: int = 0,
           device="cpu") -> torch.Tensor:
    """Activations ~N(0,1) as bf16 bit patterns (int16 [T][d])."""
    key = stream_key(seed, cfg.cid, layer, TID_X, step)
    return f32_to_bf16_bits(normal_f32(key, T * cfg.d, 1.0, device)).view(T, cfg.d)


def make_router(seed: int, cfg: LayerShape, layer: int = 0, epoch: int = 0, device="cpu"):
    """Router weights Wr [E][d] float32 and bias br [E] float32.

    With zipf_s > 0 the bias is -s*ln(rank_e) for a seeded permutation rank of 1..E, which
    makes expert popularity follow Zipf(s) over that permutation. ``epoch`` reseeds the
    permutation (used to let the hot set drift over time)."""
    key = stream_key(seed, cfg.cid, layer, TID_WR)
    Wr = normal_f32(key, cfg.E * cfg.d, cfg.router_std, device).view(cfg.E, cfg.d)
    if cfg.zipf_s > 0:
        # seeded permutation: order experts by a hash of their id (integer ops only)
        h = hash64(stream_key(seed, cfg.cid, layer, TID_PERM, epoch), torch.arange(cfg.E))
        perm = torch.argsort(h, stable=True).numpy()
        rank = np.empty(cfg.E, dtype=np.int64)
        rank[perm] = np.arange(1, cfg.E + 1)
        br = torch.from_numpy((-cfg.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32))
        br = br.to(device)
    else:
        br = torch.zeros(cfg.E, dtype=torch.float32, device=device)
    return Wr, br


def make_input_scales(cfg: LayerShape):
    """Static per-expert input scales (float32 [E + 1], the shared expert's last), standing
    in for calibrated ones: in_gu[e] = (1 + (e % 7) / 7) * 2*sqrt(3) / 2688 for the
    activations (2*sqrt(3) bounds |x| of the synthetic activations, so no block scale
    saturates) and in_dn[e] = (1 + (e % 5) / 5) / 64 for h. The factors vary by expert so that
    experts quantise the same token differently."""
    e = np.arange(cfg.E + 1)
    x_bound = np.float32(2.0 * np.sqrt(3.0))
    in_gu = ((1.0 + (e % 7) / 7.0) * (x_bound / np.float32(2688.0))).astype(np.float32)
    in_dn = ((1.0 + (e % 5) / 5.0) / 64.0).astype(np.float32)
    return torch.from_numpy(in_gu), torch.from_numpy(in_dn)


def make_expert_weights_bf16(seed: int, cfg: LayerShape, expert: int, layer: int = 0,
                             shared: bool = False, device="cpu"):
    """Unquantised weights of one expert as bf16 bit patterns (int16), the precision a
    checkpoint holds before NVFP4 quantisation: gate [I][d], up [I][d], down [d][I],
    each ~N(0, weight_std^2)."""
    tg, tu, td = (TID_SGATE, TID_SUP, TID_SDOWN) if shared else (TID_GATE, TID_UP, TID_DOWN)
    base = (seed, cfg.cid, layer)
    n = cfg.I * cfg.d
    mk = lambda tid: f32_to_bf16_bits(  # noqa: E731
        normal_f32(stream_key(*base, tid, expert), n, cfg.weight_std, device))
    return mk(tg).view(cfg.I, cfg.d), mk(tu).view(cfg.I, cfg.d), mk(td).view(cfg.d, cfg.I)


def normal_f32_rows(keys, n: int, std: float, device="cpu") -> torch.Tensor:
    """normal_f32(keys[r], n, std) for every key at once: a [len(keys)][n] float32 tensor,
    bit-identical row by row (the same integer steps, with the key broadcast per row)."""
    key = torch.tensor([_s64(k) for k in keys], dtype=torch.int64, device=device)[:, None]
    z = torch.arange(n, dtype=torch.int64, device=device)[None, :] + 1
    z = z * _s64(_GOLDEN) + key
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    h = z ^ _lsr(z, 31)
    s = (h & 0xFFFF) + (_lsr(h, 16) & 0xFFFF) + (_lsr(h, 32) & 0xFFFF) + _lsr(h, 48)
    zi = (2 * s - 4 * 65535).to(torch.float32)
    c = torch.tensor(np.float32(std * _IH4_SCALE), dtype=torch.float32, device=device)
    return zi * c


def make_experts_weights_bf16(seed: int, cfg: LayerShape, experts, layer: int = 0,
                              shared: bool = False, device="cpu"):
    """make_expert_weights_bf16 for several experts at once: gate [n][I][d], up [n][I][d],
    down [n][d][I] as bf16 bit patterns, row e equal to expert experts[e]'s draws."""
    tg, tu, td = (TID_SGATE, TID_SUP, TID_SDOWN) if shared else (TID_GATE, TID_UP, TID_DOWN)
    base = (seed, cfg.cid, layer)
    n = cfg.I * cfg.d
    ex = list(experts)
    mk = lambda tid: f32_to_bf16_bits(  # noqa: E731
        normal_f32_rows([stream_key(*base, tid, e) for e in ex], n, cfg.weight_std, device))
    return (mk(tg).view(len(ex), cfg.I, cfg.d), mk(tu).view(len(ex), cfg.I, cfg.d),
            mk(td).view(len(ex), cfg.d, cfg.I))


def make_expert_weights_f32(seed: int, cfg: LayerShape, expert: int, layer: int = 0,
                            shared: bool = False, device="cpu"):
    """The same weights widened (exactly) to float32."""
    return tuple(bf16_bits_to_f32(w) for w in
                 make_expert_weights_bf16(seed, cfg, expert, layer, shared, device))
