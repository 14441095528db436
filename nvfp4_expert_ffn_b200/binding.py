"""Thin Python binding of libmoe_nvfp4.so (argument marshalling only).

Every function here has the name of the C entry point it calls (include/moe_nvfp4.h) and
takes torch tensors that already live on the GPU; it passes their device pointers, sizes
and the current CUDA stream through ctypes and raises ``MoeError`` on a non-zero status.
No computation happens here: when the shared library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_NVFP4_LIB selects another build of the same library (e.g. the timeline-trace build)
LIB_PATH = os.environ.get("MOE_NVFP4_LIB") or os.path.join(_PKG, "lib", "libmoe_nvfp4.so")

MOE_OK = 0
MOE_FFN_ACCUMULATE, MOE_FFN_PER_ASSIGN = 0, 1
MOE_PATH_AUTO, MOE_PATH_DECODE, MOE_PATH_PREFILL, MOE_PATH_CUDA_CORE = 0, 1, 2, 3
MOE_OP_LAYER, MOE_OP_ROUTE, MOE_OP_QUANT, MOE_OP_FFN, MOE_OP_LAYER_DECODE = 0, 1, 2, 3, 4
MOE_OP_FFN_STATIC = 5
MOE_ERR_TIMEOUT, MOE_ERR_WORKSPACE = 4, 5
DEFAULT_WAIT_LIMIT_NS = 2_000_000_000

# (name, restype, argtypes) of every C export; tests check the header declares the same set
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
EXPORTS = {
    "nvfp4_quantize_act": (_I32, [_P, _I64, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_route": (_I32, [_P, _I32, _I32, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_permute": (_I32, [_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_route_noalloc": (_I32, [_P, _I32, _I32, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "moe_pack_experts": (_I32, [_P, _P, _P, _P, _P]),
    "moe_expert_ffn": (_I32, [_P, _P, _P, _I32, _P, _I32, _P, _P, _P, _I32, _I32, _P, _P, _P,
                              _SZ, _P]),
    "moe_expert_ffn_static": (_I32, [_P, _I32, _P, _P, _P, _I32, _P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "moe_combine": (_I32, [_I32, _I32, _I32, _I32, _P, _P, _P, _P, _I32, _P, _P]),
    "moe_expert_hist": (_I32, [_P, _I32, _P, _P, _I32, _P]),
    "moe_layer_decode": (_I32, [_P, _I32, _P, _P, _P, _P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                _P, _P, _I32, _P, _SZ, _P]),
    "moe_workspace_size": (_SZ, [_I32, _I64, _I32, _I32, _I32, _I32]),
    "moe_get_device_status": (_I32, [_P, _I32, ctypes.POINTER(_I32)]),
    "moe_set_wait_limit_ns": (_I32, [ctypes.c_uint64]),
    "moe_hot_tier_update": (_I32, [_P, _P, _I32, _P, _P, _P]),
    "moe_set_l2_persisting": (_I32, [_SZ, ctypes.POINTER(_SZ)]),
    "moe_status_string": (ctypes.c_char_p, [_I32]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_version": (_I32, []),
    "moe_launch_count": (ctypes.c_uint64, []),
}


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        super().__init__(f"{fn} failed with status {status}: {detail}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m nvfp4_expert_ffn_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != MOE_OK:
        L = lib()
        raise MoeError(fn, status, L.moe_last_error().decode() or
                       L.moe_status_string(status).decode())


# ------------------------------------------------------------------------- weights

class _WeightsC(ctypes.Structure):
    _fields_ = [("E", _I32), ("d", _I32), ("I", _I32),
                ("gu_codes", _P), ("gu_scales", _P), ("gu_ts", _P),
                ("dn_codes", _P), ("dn_scales", _P), ("dn_ts", _P),
                ("gu_sf_tiled", _P), ("dn_sf_tiled", _P),
                ("dec_pack", _P), ("hot_pack", _P), ("hot_slot", _P), ("n_hot", _I32)]


class _ExpertsC(ctypes.Structure):
    _fields_ = [("routed", _WeightsC), ("shared", _WeightsC), ("has_shared", _I32)]


@dataclass
class ExpertWeights:
    """NVFP4 weights of an expert group on the GPU (natural layout, see moe_nvfp4.h)."""
    gu_codes: Optional[torch.Tensor]   # uint8 [E][2I][d/2]
    gu_scales: Optional[torch.Tensor]  # uint8 [E][2I][d/16]
    gu_ts: torch.Tensor                # float32 [E][2]
    dn_codes: Optional[torch.Tensor]   # uint8 [E][d][I/2]
    dn_scales: Optional[torch.Tensor]  # uint8 [E][d][I/16]
    dn_ts: torch.Tensor                # float32 [E]
    gu_sf_tiled: Optional[torch.Tensor] = None
    dn_sf_tiled: Optional[torch.Tensor] = None
    dec_pack: Optional[torch.Tensor] = None
    dims: tuple = ()                   # (E, d, I), taken from gu_codes when not given
    hot_pack: Optional[torch.Tensor] = None   # uint8: n_hot experts' decode-pack units
    hot_slot: Optional[torch.Tensor] = None   # int32 [E]: slot in hot_pack or -1
    n_hot: int = 0

    def __post_init__(self):
        if not self.dims:
            E, twoI, dh = self.gu_codes.shape
            self.dims = (E, 2 * dh, twoI // 2)

    @property
    def E(self):
        return self.dims[0]

    @property
    def d(self):
        return self.dims[1]

    @property
    def I(self):
        return self.dims[2]

    def release_natural(self) -> None:
        """Drop the natural-layout arrays and the re-tiled scales, keeping the decode pack and
        the tensor scales: enough for moe_layer_decode and the DECODE path, with every
        weight byte held once."""
        if self.dec_pack is None:
            raise ValueError("release_natural needs the decode pack (moe_pack_experts)")
        self.gu_codes = self.gu_scales = self.dn_codes = self.dn_scales = None
        self.gu_sf_tiled = self.dn_sf_tiled = None

    def struct(self) -> _WeightsC:
        p = lambda t: None if t is None else _ptr(t).value  # noqa: E731
        return _WeightsC(self.E, self.d, self.I, p(self.gu_codes), p(self.gu_scales),
                         p(self.gu_ts), p(self.dn_codes), p(self.dn_scales), p(self.dn_ts),
                         p(self.gu_sf_tiled), p(self.dn_sf_tiled), p(self.dec_pack),
                         p(self.hot_pack), p(self.hot_slot), self.n_hot)


@dataclass
class Experts:
    routed: ExpertWeights
    shared: Optional[ExpertWeights] = None
    _c: Optional[_ExpertsC] = field(default=None, repr=False)

    def struct(self) -> _ExpertsC:
        sh = self.shared.struct() if self.shared is not None else _WeightsC()
        self._c = _ExpertsC(self.routed.struct(), sh, 1 if self.shared is not None else 0)
        return self._c


# ------------------------------------------------------------------------- calls

def moe_workspace_size(op: int, T: int, d: int, E: int, k: int, I: int) -> int:
    return int(lib().moe_workspace_size(op, T, d, E, k, I))


def nvfp4_quantize_act(x, codes, scales, ts_out, ts_in=None, ws=None, stream=None):
    rows, cols = x.shape
    _check("nvfp4_quantize_act", lib().nvfp4_quantize_act(
        _ptr(x), rows, cols, _ptr(ts_in), _ptr(codes), _ptr(scales), _ptr(ts_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_route(x, Wr, br, k, topk_idx, topk_w, counts, offsets, sorted_assign, assign_pos,
              ws, stream=None):
    T, d = x.shape
    E = Wr.shape[0]
    _check("moe_route", lib().moe_route(
        _ptr(x), T, d, _ptr(Wr), _ptr(br), E, k, _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
        _ptr(offsets), _ptr(sorted_assign), _ptr(assign_pos), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_layer_decode(x, ts_in, Wr, br, experts: "Experts", k, xq_codes, xq_scales, xq_ts, topk_idx,
                     topk_w, counts, offsets, sorted_assign, assign_pos, y_acc, y, rms_renorm, ws,
                     stream=None):
    """The whole layer for at most 8 tokens in one kernel (see include/moe_nvfp4.h); ws must
    be zero-filled before its first use."""
    T = x.shape[0]
    s = experts.struct()
    _check("moe_layer_decode", lib().moe_layer_decode(
        _ptr(x), T, _ptr(ts_in), _ptr(Wr), _ptr(br), ctypes.byref(s), k, _ptr(xq_codes),
        _ptr(xq_scales), _ptr(xq_ts), _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(offsets),
        _ptr(sorted_assign), _ptr(assign_pos), _ptr(y_acc), _ptr(y), 1 if rms_renorm else 0,
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_route_noalloc(x, Wr, br, k, topk_idx, topk_w, counts, offsets, sorted_assign, assign_pos,
                      stream=None):
    """moe_route without a workspace: the library uses its own fixed 256 KiB scratch array
    (for callers that cannot allocate device memory; see include/moe_nvfp4.h)."""
    T, d = x.shape
    E = Wr.shape[0]
    _check("moe_route_noalloc", lib().moe_route_noalloc(
        _ptr(x), T, d, _ptr(Wr), _ptr(br), E, k, _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
        _ptr(offsets), _ptr(sorted_assign), _ptr(assign_pos), _stream(stream)))


def moe_permute(topk_idx, E, counts, offsets, sorted_assign, assign_pos, ws, stream=None):
    T, k = topk_idx.shape
    _check("moe_permute", lib().moe_permute(
        _ptr(topk_idx), T, k, E, _ptr(counts), _ptr(offsets), _ptr(sorted_assign),
        _ptr(assign_pos), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_pack_experts(w: ExpertWeights, stream=None, decode_pack: bool = True):
    """Allocate and fill the derived layouts used by the tensor-core paths: re-tiled scales,
    and (decode_pack=True, d % 512 == 0) the decode pack: all weights again as the 18 KB blocks
    the decode kernel copies into shared memory."""
    if w.gu_sf_tiled is None:
        w.gu_sf_tiled = torch.empty_like(w.gu_scales)
    if w.dn_sf_tiled is None:
        w.dn_sf_tiled = torch.empty_like(w.dn_scales)
    if decode_pack and w.dec_pack is None and w.d % 512 == 0:
        w.dec_pack = torch.empty(dec_pack_bytes(w.E, w.d, w.I), dtype=torch.uint8,
                                 device=w.gu_codes.device)
    s = w.struct()
    _check("moe_pack_experts", lib().moe_pack_experts(
        ctypes.byref(s), _ptr(w.gu_sf_tiled), _ptr(w.dn_sf_tiled), _ptr(w.dec_pack),
        _stream(stream)))


def dec_pack_bytes(E: int, d: int, I: int) -> int:
    """Bytes of the decode pack of an expert group (d % 512 == 0, I % 64 == 0)."""
    return E * (I // 64) * (d // 256 + d // 512) * 18432


def moe_expert_ffn(xq_codes, xq_scales, xq_ts, experts: Experts, k, offsets, sorted_assign,
                   topk_w, mode, path, out, shared_out, ws, stream=None):
    T = xq_codes.shape[0]
    s = experts.struct()
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        _ptr(xq_codes), _ptr(xq_scales), _ptr(xq_ts), T, ctypes.byref(s), k, _ptr(offsets),
        _ptr(sorted_assign), _ptr(topk_w), mode, path, _ptr(out), _ptr(shared_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_expert_ffn_static(x, experts: Experts, in_scale_gu, in_scale_dn, k, offsets, sorted_assign,
                          topk_w, mode, out, shared_out, ws, stream=None):
    T = x.shape[0]
    s = experts.struct()
    _check("moe_expert_ffn_static", lib().moe_expert_ffn_static(
        _ptr(x), T, ctypes.byref(s), _ptr(in_scale_gu), _ptr(in_scale_dn), k, _ptr(offsets),
        _ptr(sorted_assign), _ptr(topk_w), mode, _ptr(out), _ptr(shared_out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_combine(T, d, k, mode, expert_out, shared_out, topk_w, assign_pos, rms_renorm, y,
                stream=None):
    _check("moe_combine", lib().moe_combine(
        T, d, k, mode, _ptr(expert_out), _ptr(shared_out), _ptr(topk_w), _ptr(assign_pos),
        1 if rms_renorm else 0, _ptr(y), _stream(stream)))


def moe_expert_hist(counts, cum, rank_out=None, reset=False, stream=None):
    _check("moe_expert_hist", lib().moe_expert_hist(
        _ptr(counts), counts.numel(), _ptr(cum), _ptr(rank_out), 1 if reset else 0,
        _stream(stream)))


def moe_launch_count() -> int:
    """Kernels this library has enqueued in this process (graph replays not counted)."""
    return int(lib().moe_launch_count())


def moe_get_device_status(clear=True, stream=None) -> int:
    out = _I32(0)
    _check("moe_get_device_status", lib().moe_get_device_status(_stream(stream),
                                                                 1 if clear else 0,
                                                                 ctypes.byref(out)))
    return out.value


def moe_hot_tier_update(w: ExpertWeights, rank, n_hot: int, stream=None) -> None:
    """Copy the units of experts rank[:n_hot] into w's hot tier (allocated here on first
    use, sized for n_hot) and point w at it; n_hot = 0 turns the tier off."""
    if n_hot > 0 and (w.hot_pack is None or w.hot_pack.numel() < dec_pack_bytes(n_hot, w.d, w.I)):
        w.hot_pack = torch.empty(dec_pack_bytes(n_hot, w.d, w.I), dtype=torch.uint8,
                                 device=w.dec_pack.device)
    if w.hot_slot is None:
        w.hot_slot = torch.empty(w.E, dtype=torch.int32, device=w.dec_pack.device)
    s = w.struct()
    _check("moe_hot_tier_update", lib().moe_hot_tier_update(
        ctypes.byref(s), _ptr(rank), n_hot, _ptr(w.hot_pack), _ptr(w.hot_slot), _stream(stream)))
    w.n_hot = n_hot


def moe_set_l2_persisting(nbytes: int) -> int:
    """Set this process's L2 set-aside for persisting lines (clamped to the device's
    maximum; 0 releases it); returns the size in effect."""
    out = _SZ(0)
    _check("moe_set_l2_persisting", lib().moe_set_l2_persisting(int(nbytes), ctypes.byref(out)))
    return int(out.value)


def moe_set_wait_limit_ns(ns: int) -> None:
    _check("moe_set_wait_limit_ns", lib().moe_set_wait_limit_ns(int(ns)))
