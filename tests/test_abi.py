"""The C ABI library: it loads, exports every function include/*.h declares, and rejects bad
arguments on the host before touching the GPU (CPU only)."""
import ctypes
import glob
import os
import re

import pytest

from nvfp4_expert_ffn_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M):
            name = m.group(1)
            if name not in ("defined",):
                names.add(name)
    return names


def test_library_loads_and_exports_every_declared_symbol():
    L = B.lib()
    declared = _declared()
    assert {"moe_route", "nvfp4_quantize_act", "moe_expert_ffn", "moe_combine",
            "moe_expert_hist"} <= declared
    for name in declared:
        assert hasattr(L, name), f"{name} declared but not exported"
    assert declared == set(B.EXPORTS), declared ^ set(B.EXPORTS)
    assert L.moe_version() >= 100


def _status(call):
    return int(call)


def test_host_validation_without_gpu():
    L = B.lib()
    INV, SHAPE, WS = 1, 2, 5
    # quantiser: cols not a multiple of 16 / negative rows
    assert L.nvfp4_quantize_act(None, 4, 24, None, None, None, None, None, 0, None) == SHAPE
    assert L.nvfp4_quantize_act(None, -1, 32, None, None, None, None, None, 0, None) == INV
    # misaligned pointer
    assert L.nvfp4_quantize_act(ctypes.c_void_p(0x1008), 4, 32, None, ctypes.c_void_p(0x2000),
                                ctypes.c_void_p(0x3000), None, None, 0, None) == INV
    # large input needs workspace
    assert L.nvfp4_quantize_act(ctypes.c_void_p(0x1000), 100000, 64, None, ctypes.c_void_p(0x2000),
                                ctypes.c_void_p(0x3000), None, None, 0, None) == WS
    p = ctypes.c_void_p(0x10000)
    # route: k out of range, E < k, d not /16
    assert L.moe_route(p, 4, 64, p, None, 8, 0, p, p, p, p, p, p, p, 1 << 20, None) == SHAPE
    assert L.moe_route(p, 4, 64, p, None, 4, 8, p, p, p, p, p, p, p, 1 << 20, None) == SHAPE
    assert L.moe_route(p, 4, 72, p, None, 8, 2, p, p, p, p, p, p, p, 1 << 20, None) == SHAPE
    assert L.moe_route(p, 4, 64, p, None, 2000, 2, p, p, p, p, p, p, p, 1 << 20, None) == SHAPE
    # route: workspace too small
    assert L.moe_route(p, 4, 64, p, None, 8, 2, p, p, p, p, p, p, p, 16, None) == WS
    # permute: null outputs
    assert L.moe_permute(p, 4, 2, 8, None, p, p, p, p, 1 << 20, None) == INV
    # ffn: null weights, bad mode
    assert L.moe_expert_ffn(p, p, p, 4, None, 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == INV
    # combine: bad d, bad mode
    assert L.moe_combine(4, 24, 2, 0, p, None, None, None, 0, p, None) == INV
    assert L.moe_combine(4, 32, 2, 7, p, None, None, None, 0, p, None) == INV
    # hist: E out of range
    assert L.moe_expert_hist(p, 0, p, None, 0, None) == SHAPE
    assert b"E must be" in L.moe_last_error()
    assert L.moe_status_string(5) == b"workspace too small, misaligned, or marked by a call that gave up"


def test_ffn_weight_validation():
    L = B.lib()
    p = ctypes.c_void_p(0x10000)
    w = B._WeightsC(8, 64, 32, p.value, p.value, p.value, p.value, p.value, p.value, None, None)
    bad = B._WeightsC(8, 64, 32, p.value, None, p.value, p.value, p.value, p.value, None, None)
    ex = B._ExpertsC(w, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 0, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 0, None) in (0, 3)
    ex = B._ExpertsC(bad, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == 1
    # shared expert with E != 1
    ex = B._ExpertsC(w, w, 1)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == 1
    # I not a multiple of 16
    w2 = B._WeightsC(8, 64, 40, p.value, p.value, p.value, p.value, p.value, p.value, None, None)
    ex = B._ExpertsC(w2, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == 2


def test_workspace_sizes_monotone():
    small = B.moe_workspace_size(B.MOE_OP_LAYER, 8, 2048, 512, 10, 512)
    big = B.moe_workspace_size(B.MOE_OP_LAYER, 16384, 2048, 512, 10, 512)
    assert 0 < small < big
    assert B.moe_workspace_size(B.MOE_OP_LAYER, 8, 2048, 512, 10, 512) >= \
        B.moe_workspace_size(B.MOE_OP_FFN, 8, 2048, 512, 10, 512)
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, -1, 2048, 512, 10, 512) == 0


def test_pack_and_layer_decode_validation():
    """Host-side checks of moe_pack_experts (the decode pack's shape rule) and of
    moe_layer_decode (alignment, the decode pack), which run before any device call."""
    L = B.lib()
    INV, SHAPE = 1, 2
    p = ctypes.c_void_p(0x10000)
    # d = 256 is packable for the tensor-core scales but not for the decode pack
    w = B._WeightsC(4, 256, 64, p.value, p.value, p.value, p.value, p.value, p.value)
    assert L.moe_pack_experts(ctypes.byref(w), p, p, p, None) == SHAPE
    assert L.moe_pack_experts(ctypes.byref(w), p, p, ctypes.c_void_p(0x10008), None) == INV
    assert L.moe_pack_experts(ctypes.byref(w), None, p, None, None) == INV
    # moe_layer_decode: weights without the decode pack, and a misaligned scale buffer
    w5 = B._WeightsC(16, 512, 64, p.value, p.value, p.value, p.value, p.value, p.value)
    ex = B._ExpertsC(w5, B._WeightsC(), 0)
    args = [p, 4, None, p, None, ctypes.byref(ex), 2, p, p, p, p, p, p, p, p, p, p, p, 0, p, 1 << 20, None]
    assert L.moe_layer_decode(*args) == SHAPE
    assert b"decode pack" in L.moe_last_error()
    args[8] = ctypes.c_void_p(0x10004)  # xq_scales
    assert L.moe_layer_decode(*args) == INV


def test_dec_pack_bytes_formula():
    """The binding's decode-pack size is the header's E*I*d*27/16 bytes (18 KB blocks)."""
    for E, d, I in [(1, 512, 64), (512, 2048, 512), (256, 4096, 2048), (8, 1024, 192)]:
        assert B.dec_pack_bytes(E, d, I) == E * I * d * 27 // 16


def test_route_workspace_has_no_permutation_scratch_up_to_4096_assignments():
    """The routing scratch is the T*E float32 logits (padded to 256 bytes); from 256 tokens
    on (tensor-core router) the bf16 split of the router matrix, E*2d*2 bytes; the per-chunk
    histograms of the multi-kernel permutation only above 4096 assignments."""
    E, d, k = 512, 2048, 10
    w2 = E * 2 * d * 2
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, 128, d, E, k, 512) == 128 * E * 4
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, 255, d, E, k, 512) == 255 * E * 4
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, 409, d, E, k, 512) == 409 * E * 4 + w2
    # 410 tokens x 10 = 4100 assignments: two chunks of histograms
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, 410, d, E, k, 512) == 410 * E * 4 + w2 + 2 * E * 4
    # E not a multiple of 128: the CUDA-core router, no split matrix
    assert B.moe_workspace_size(B.MOE_OP_ROUTE, 409, d, 500, k, 512) == (409 * 500 * 4 + 255) // 256 * 256


def test_wait_limit_rejects_out_of_range_without_gpu():
    """moe_set_wait_limit_ns checks its range on the host before any device call."""
    L = B.lib()
    assert L.moe_set_wait_limit_ns(999_999) == 1
    assert L.moe_set_wait_limit_ns(60_000_000_001) == 1
    assert b"wait limit" in L.moe_last_error()


def test_natural_weights_all_or_none():
    """A group may leave its natural-layout arrays NULL only all together and only when it has
    the decode pack; the checks run on the host before any device call."""
    L = B.lib()
    INV = 1
    p = ctypes.c_void_p(0x10000)
    # natural arrays NULL, no decode pack: nothing to read
    w = B._WeightsC(8, 512, 64, None, None, p.value, None, None, p.value, None, None, None)
    ex = B._ExpertsC(w, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == INV
    assert b"neither" in L.moe_last_error()
    # some natural arrays given, others NULL
    w = B._WeightsC(8, 512, 64, p.value, None, p.value, p.value, p.value, p.value, None, None, p.value)
    ex = B._ExpertsC(w, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == INV
    assert b"all be given or all NULL" in L.moe_last_error()
    # tensor scales are always needed
    w = B._WeightsC(8, 512, 64, None, None, None, None, None, p.value, None, None, p.value)
    ex = B._ExpertsC(w, B._WeightsC(), 0)
    assert L.moe_expert_ffn(p, p, p, 4, ctypes.byref(ex), 2, p, p, p, 0, 0, p, None, p, 1 << 20, None) == INV


def test_hot_tier_validation_without_gpu():
    """moe_hot_tier_update and moe_layer_decode check the hot tier's arguments on the host
    before any device call."""
    L = B.lib()
    INV, UNSUP = 1, 2
    p = ctypes.c_void_p(0x10000)
    w = B._WeightsC(8, 512, 64, p.value, p.value, p.value, p.value, p.value, p.value, None, None, p.value)
    # no decode pack
    w_nopack = B._WeightsC(8, 512, 64, p.value, p.value, p.value, p.value, p.value, p.value, None, None, None)
    assert L.moe_hot_tier_update(ctypes.byref(w_nopack), p, 2, p, p, None) == INV
    # n_hot out of range, missing buffers
    assert L.moe_hot_tier_update(ctypes.byref(w), p, -1, p, p, None) == INV
    assert L.moe_hot_tier_update(ctypes.byref(w), p, 9, p, p, None) == INV
    assert L.moe_hot_tier_update(ctypes.byref(w), p, 2, None, p, None) == INV
    assert L.moe_hot_tier_update(ctypes.byref(w), None, 2, p, p, None) == INV
    # shapes the tier does not take: E % 4 != 0, d % 512 != 0
    w6 = B._WeightsC(6, 512, 64, p.value, p.value, p.value, p.value, p.value, p.value, None, None, p.value)
    assert L.moe_hot_tier_update(ctypes.byref(w6), p, 2, p, p, None) == UNSUP
    w256 = B._WeightsC(8, 256, 64, p.value, p.value, p.value, p.value, p.value, p.value, None, None, p.value)
    assert L.moe_hot_tier_update(ctypes.byref(w256), p, 2, p, p, None) == UNSUP
    # misaligned hot_pack
    assert L.moe_hot_tier_update(ctypes.byref(w), p, 2, ctypes.c_void_p(0x10008), p, None) == INV
    # the layer call refuses a tier with n_hot > 0 but no buffers, or n_hot < 0
    for hot_pack, hot_slot, n_hot in ((None, p.value, 2), (p.value, None, 2), (p.value, p.value, -1)):
        wr = B._WeightsC(8, 512, 64, p.value, p.value, p.value, p.value, p.value, p.value, None, None, p.value,
                         hot_pack, hot_slot, n_hot)
        ex = B._ExpertsC(wr, B._WeightsC(), 0)
        args = [p, 4, None, p, None, ctypes.byref(ex), 2] + [p] * 11 + [0, p, 1 << 20, None]
        assert L.moe_layer_decode(*args) == INV, (hot_pack, hot_slot, n_hot)


def test_static_scales_validation_without_gpu():
    """moe_expert_ffn_static refuses shapes the m-tile kernel does not take, weights without
    their packed scales, and missing scale arrays, on the host."""
    L = B.lib()
    INV, UNSUP = 1, 2
    p = ctypes.c_void_p(0x10000)

    def call(E, d, I, packed=True, gu=p, dn=p, T=16):
        sf = p.value if packed else None
        w = B._WeightsC(E, d, I, p.value, p.value, p.value, p.value, p.value, p.value, sf, sf, None)
        ex = B._ExpertsC(w, B._WeightsC(), 0)
        return L.moe_expert_ffn_static(p, T, ctypes.byref(ex), gu, dn, 2, p, p, p, 0, p, None, p, 1 << 30, None)

    assert call(8, 4096, 512) == UNSUP      # d above the m-tile kernel's 2048
    assert call(8, 2048, 1024) == UNSUP     # I above 768
    assert call(8, 2048, 320) == UNSUP      # I % 256 != 0
    assert call(8, 2048, 512, packed=False) == UNSUP
    assert call(8, 2048, 512, gu=None) == INV
    assert call(8, 2048, 512, dn=None) == INV
    assert call(8, 2048, 512, T=-1) == INV
    assert call(8, 2048, 512, T=0) == 0     # nothing to do
