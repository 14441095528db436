"""The hot tier of the one-kernel decode layer: a compact copy of the most-routed experts'
decode-pack units that the kernel reads instead of the decode pack, with an L2 persisting
window over it ("Basalt" project page, section "Expert tiers": the busiest experts live in the
fastest memory, and the tiers follow the routing as it shifts).

Checked here: the update writes the slot map and copies exactly the ranked experts' units; the
layer's output and routing are unchanged by the tier; the kernel really reads the tier (a
changed copy changes the output of a token routed to that expert, and restoring it restores
the output); and the process's persisting set-aside can be set and released.
"""
import numpy as np
import pytest
import torch

from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import bits_to_f32

pytestmark = pytest.mark.gpu


def _layer(seed=3):
    cfg = synth.CONFIGS["decode"]
    routed = L.quantize_weights_gpu(seed, cfg)
    shared = L.quantize_weights_gpu(seed, cfg, shared=True)
    Wr, br = synth.make_router(seed, cfg)
    lay = L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), br.cuda(), cfg.k, 8, fused=True)
    assert lay.fused
    return cfg, lay


def _close(a_bits, b_bits, tol=1e-2):
    a, b = bits_to_f32(a_bits.cpu().numpy()), bits_to_f32(b_bits.cpu().numpy())
    return np.abs(a - b).max() <= tol * np.sqrt((b ** 2).mean())


def test_hot_tier_update_copies_ranked_units():
    cfg, lay = _layer()
    w = lay.experts.routed
    E = w.E
    unit = B.dec_pack_bytes(1, w.d, w.I)
    rank = torch.randperm(E, generator=torch.Generator().manual_seed(5)).to(torch.int32).cuda()
    n_hot = 6
    B.moe_hot_tier_update(w, rank, n_hot)
    torch.cuda.synchronize()
    slot = w.hot_slot.cpu().numpy()
    want = np.full(E, -1, dtype=np.int32)
    want[rank[:n_hot].cpu().numpy()] = np.arange(n_hot)
    assert np.array_equal(slot, want)
    pack = w.dec_pack.view(E, unit)
    hot = w.hot_pack[:n_hot * unit].view(n_hot, unit)
    for i, e in enumerate(rank[:n_hot].tolist()):
        assert torch.equal(hot[i], pack[e])
    # a smaller tier rewrites the map
    B.moe_hot_tier_update(w, rank, 2)
    torch.cuda.synchronize()
    want = np.full(E, -1, dtype=np.int32)
    want[rank[:2].cpu().numpy()] = np.arange(2)
    assert np.array_equal(w.hot_slot.cpu().numpy(), want)
    assert w.n_hot == 2


def test_layer_output_unchanged_and_tier_is_read():
    cfg, lay = _layer()
    w = lay.experts.routed
    unit = B.dec_pack_bytes(1, w.d, w.I)
    x = synth.make_x(4, cfg, 8, step=1).cuda()
    y0 = lay.forward(x).clone()
    idx0 = lay.topk_idx[:8].clone()
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0
    # the tier holds the experts token 0 chose, in the order chosen, then the rest by id
    chosen = idx0[0].tolist()
    rest = [e for e in range(w.E) if e not in chosen]
    rank = torch.tensor(chosen + rest, dtype=torch.int32, device="cuda")
    B.moe_set_l2_persisting(64 << 20)
    try:
        B.moe_hot_tier_update(w, rank, len(chosen))
        y1 = lay.forward(x).clone()
        torch.cuda.synchronize()
        assert B.moe_get_device_status() == 0
        assert torch.equal(lay.topk_idx[:8], idx0)
        assert _close(y1, y0)
        # change the copy of token 0's first expert: token 0's output moves, other tokens
        # that did not choose that expert stay as they were
        e0 = chosen[0]
        hot = w.hot_pack[:len(chosen) * unit].view(len(chosen), unit)
        saved = hot[0].clone()
        hot[0].zero_()
        y2 = lay.forward(x).clone()
        torch.cuda.synchronize()
        a2, a0 = bits_to_f32(y2.cpu().numpy()), bits_to_f32(y0.cpu().numpy())
        assert np.abs(a2[0] - a0[0]).max() > 1e-3 * np.sqrt((a0[0] ** 2).mean())
        for t in range(8):
            if e0 not in idx0[t].tolist():
                assert np.abs(a2[t] - a0[t]).max() <= 1e-2 * np.sqrt((a0[t] ** 2).mean())
        hot[0].copy_(saved)
        y3 = lay.forward(x).clone()
        torch.cuda.synchronize()
        assert _close(y3, y0)
        # tier off: the decode pack again
        B.moe_hot_tier_update(w, rank, 0)
        y4 = lay.forward(x).clone()
        torch.cuda.synchronize()
        assert _close(y4, y0)
        assert B.moe_get_device_status() == 0
    finally:
        B.moe_set_l2_persisting(0)


def test_l2_persisting_setaside_set_and_released():
    # the driver rounds the set-aside up to its own granularity
    got = B.moe_set_l2_persisting(8 << 20)
    assert got >= 8 << 20
    most = B.moe_set_l2_persisting(1 << 40)
    assert got <= most < (1 << 40)
    assert B.moe_set_l2_persisting(0) == 0
