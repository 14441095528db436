"""The 48-layer decode stack (8 tokens per step, per-token RMS renormalisation between layers,
each layer's router popularity re-drawn every 64 steps), every layer against the oracle, on
the two steps around the first drift boundary (steps 63 and 64).

The GPU holds only the decode pack of each of the 48 layers (release_natural: every weight
byte once, 43.6 GB). The oracle runs the stack as a chain of its own: layer l + 1 takes the
bf16 of the RMS-renormalised output of its own layer l. Each GPU layer is fed the oracle's
input of that layer, so a routing decision that flips near a tie in one layer does not carry
into the next one; the outputs, the quantised activations and the routing of every layer are
compared. The oracle's per-expert work runs on a pool of host processes.
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import nvfp4 as onv
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import assert_close_layer, bits_to_f32, compare_topk
from oracle_pool import OraclePool

pytestmark = pytest.mark.gpu

N_LAYERS = 48


def _oracle_layer(pool, cfg, layer, x_bits, Wr, br):
    xf = bits_to_f32(x_bits)
    xc, xs, xts = onv.quantize(xf)
    logits = omoe.router_logits(xf, Wr, br)
    idx = omoe.topk_fast(logits, cfg.k)
    w = omoe.routing_weights(logits, idx)
    counts = omoe.permute(idx, cfg.E)[0]
    x_hat = onv.dequantize(xc, xs, xts)
    T = x_bits.shape[0]
    tasks, where = [], {}
    for e in np.unique(idx):
        rows = np.argwhere(idx == e)
        where[int(e)] = rows
        tasks.append((int(e), False, x_hat[rows[:, 0]]))
    tasks.append((0, True, x_hat))
    outs = pool.expert_outputs(cfg.name, 0, layer, tasks)
    o = np.zeros((T, cfg.k, cfg.d))
    for e, rows in where.items():
        o[rows[:, 0], rows[:, 1]] = outs[(e, False)]
    y = omoe.combine(T, cfg.d, idx, w, o.reshape(-1, cfg.d), outs[(0, True)])
    return dict(y=omoe.rms_renorm(y), idx=idx, logits=logits, counts=counts, x_codes=xc, x_scales=xs)


def test_stack48_every_layer_across_a_drift_boundary():
    cfg = synth.CONFIGS["stack48"]
    layers, routers = [], []
    for li in range(N_LAYERS):
        routed = L.quantize_weights_gpu(0, cfg, layer=li, decode_only=True)
        shared = L.quantize_weights_gpu(0, cfg, layer=li, shared=True, decode_only=True)
        assert routed.gu_codes is None and routed.dec_pack is not None
        Wr, _ = synth.make_router(0, cfg, layer=li)
        brs = [synth.make_router(0, cfg, layer=li, epoch=ep)[1] for ep in (0, 1)]
        routers.append((Wr.numpy(), [b.numpy() for b in brs]))
        layers.append(L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), brs[0].cuda(), cfg.k, 8, fused=True))
        layers[-1].br_epochs = [b.cuda() for b in brs]
    assert all(lay.fused for lay in layers)
    excused_total, worst = 0, 0.0
    with OraclePool() as pool:
        for step in (63, 64):
            ep = step // 64
            x = synth.make_x(0, cfg, 8, step=step).numpy()
            for li, lay in enumerate(layers):
                Wr, brs = routers[li]
                ref = _oracle_layer(pool, cfg, li, x, Wr, brs[ep])
                lay.br = lay.br_epochs[ep]
                y = lay.forward(torch.from_numpy(x).cuda(), rms_renorm=True)
                torch.cuda.synchronize()
                assert B.moe_get_device_status() == 0
                assert np.array_equal(lay.xq_codes.cpu().numpy(), ref["x_codes"]), (step, li)
                assert np.array_equal(lay.xq_scales.cpu().numpy(), ref["x_scales"]), (step, li)
                excused = compare_topk(lay.topk_idx.cpu().numpy(), ref["idx"], ref["logits"], cfg.k)
                excused_total += len(excused)
                keep = [t for t in range(8) if t not in set(excused)]
                if not excused:
                    assert np.array_equal(lay.counts.cpu().numpy(), ref["counts"]), (step, li)
                rel, _ = assert_close_layer(bits_to_f32(y.cpu().numpy())[keep], ref["y"][keep], f"step {step} layer {li}")
                worst = max(worst, rel)
                # the oracle's own chain: bf16 of its renormalised output
                x = synth.f32_to_bf16_bits(torch.from_numpy(ref["y"].astype(np.float32))).numpy()
    print(f"stack48: 2 steps x {N_LAYERS} layers, worst rel-L2 {worst:.2e}, tie-excused tokens {excused_total}")
