"""Whole layer through the C ABI (MoeLayer.forward) vs the oracle's layer_forward, plus the
cumulative expert histogram."""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import (OracleWeights, assert_close_layer, bits_to_f32, check_permutation_valid,
                     compare_topk, oracle_expert_from_bf16, weights_to_gpu)

pytestmark = pytest.mark.gpu


def _layer(cfg_name, seed=0, T_max=64, fused=None):
    cfg = synth.CONFIGS[cfg_name]
    routed = L.quantize_weights_gpu(seed, cfg)
    shared = L.quantize_weights_gpu(seed, cfg, shared=True) if cfg.shared else None
    Wr, br = synth.make_router(seed, cfg)
    lay = L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), br.cuda(), cfg.k, T_max, fused=fused)
    return cfg, lay, Wr.numpy(), br.numpy()


@pytest.mark.parametrize("cfg_name,T,fused", [("tiny", 16, None), ("decode", 1, False), ("decode", 8, False),
                                              ("decode", 1, True), ("decode", 4, True), ("decode", 8, True)])
def test_layer_matches_oracle(cfg_name, T, fused):
    cfg, lay, Wr, br = _layer(cfg_name, fused=fused)
    if fused:
        assert lay.fused
    ow = OracleWeights(0, cfg)
    x = synth.make_x(0, cfg, T, step=3)
    y = lay.forward(x.cuda())
    torch.cuda.synchronize()
    ref = omoe.layer_forward(x.numpy(), Wr, br, cfg.k, ow, ow.shared if cfg.shared else None)
    excused = compare_topk(lay.topk_idx[:T].cpu().numpy(), ref["idx"], ref["logits"], cfg.k)
    keep = [t for t in range(T) if t not in set(excused)]
    assert_close_layer(bits_to_f32(y.cpu().numpy())[keep], ref["y"][keep], cfg_name)
    assert np.array_equal(lay.xq_codes[:T].cpu().numpy(), ref["x_codes"])
    assert np.array_equal(lay.xq_scales[:T].cpu().numpy(), ref["x_scales"])
    # whatever the tie excuses, the permutation is a stable counting sort of the GPU's own top-k
    check_permutation_valid(lay.topk_idx[:T].cpu().numpy(), lay.counts.cpu().numpy(),
                            lay.offsets.cpu().numpy(), lay.sorted_assign[:T * cfg.k].cpu().numpy(),
                            lay.assign_pos[:T * cfg.k].cpu().numpy(), cfg.E)
    if not excused:
        assert np.array_equal(lay.counts.cpu().numpy(), ref["counts"])
        assert np.array_equal(lay.offsets.cpu().numpy(), ref["offsets"])
        assert np.array_equal(lay.sorted_assign[:T * cfg.k].cpu().numpy(), ref["sorted_assign"])
        cum, rank = omoe.hist_update(ref["counts"])
        assert np.array_equal(lay.cum.cpu().numpy(), cum)
        assert np.array_equal(lay.rank.cpu().numpy(), rank)


def test_hist_over_calls():
    rng = np.random.default_rng(3)
    E = 512
    counts = [rng.integers(0, 50, E).astype(np.int32) for _ in range(5)]
    counts[2][:] = 7  # all tied
    cum_g = torch.zeros(E, dtype=torch.int64, device="cuda")
    rank_g = torch.empty(E, dtype=torch.int32, device="cuda")
    cum = None
    for i, c in enumerate(counts):
        reset = i == 3
        B.moe_expert_hist(torch.from_numpy(c).cuda(), cum_g, rank_g, reset=reset)
        cum, rank = omoe.hist_update(c, cum, reset=reset)
        torch.cuda.synchronize()
        assert np.array_equal(cum_g.cpu().numpy(), cum)
        assert np.array_equal(rank_g.cpu().numpy(), rank)


def test_stack_chaining_with_rms_renorm():
    """Two decode layers chained with per-token RMS renormalisation (decode-stack input)."""
    cfg = synth.CONFIGS["stack48"]
    T = 8
    layers, owl = [], []
    for li in range(2):
        routed = L.quantize_weights_gpu(0, cfg, layer=li)
        shared = L.quantize_weights_gpu(0, cfg, layer=li, shared=True)
        Wr, br = synth.make_router(0, cfg, layer=li)
        layers.append(L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), br.cuda(), cfg.k, T))
        owl.append((OracleWeights(0, cfg, li), Wr.numpy(), br.numpy()))
    x = synth.make_x(0, cfg, T)
    h = x.cuda()
    for lay in layers:
        h = lay.forward(h, rms_renorm=True).clone()
    torch.cuda.synchronize()
    xr = x.numpy()
    for ow, Wr, br in owl:
        ref = omoe.layer_forward(xr, Wr, br, cfg.k, ow, ow.shared)
        yr = omoe.rms_renorm(ref["y"])
        xr = synth.f32_to_bf16_bits(torch.from_numpy(yr.astype(np.float32))).numpy()
    # bf16 re-rounding between layers can flip an h code; compare loosely on the final layer
    assert_close_layer(bits_to_f32(h.cpu().numpy()), yr, "2-layer stack")


def test_graphed_layer_step_matches_forward():
    """GraphedMoeLayer.step (pinned host in/out around a captured forward) gives the same
    output as an eager forward on the same input, over several different inputs."""
    cfg, lay, Wr, br = _layer("decode", T_max=8)
    runner = lay.graphed(8)
    y_host = torch.empty(8, cfg.d, dtype=torch.int16).pin_memory()
    for step in range(3):
        x = synth.make_x(5, cfg, 8, step=step)
        runner.step(x.pin_memory(), y_host)
        runner.stream.synchronize()
        got = y_host.clone()
        want = lay.forward(x.cuda()).cpu()
        torch.cuda.synchronize()
        assert torch.equal(got, want) or np.allclose(
            bits_to_f32(got.numpy()), bits_to_f32(want.numpy()), rtol=1e-2, atol=1e-3)


def test_graphed_layer_slots_copy_in_and_out_inside_the_graph():
    """run(slot) replays one graph that copies pinned x_host[slot] in, runs the layer and
    copies y out: each slot's result equals an eager forward of the same input."""
    cfg, lay, Wr, br = _layer("decode", T_max=8)
    runner = lay.graphed(4, n_slots=3)
    xs = [synth.make_x(6, cfg, 4, step=s) for s in range(3)]
    for s in range(3):
        runner.x_host[s].copy_(xs[s])
    for s in (2, 0, 1):
        runner.run(s)
        runner.stream.synchronize()
        got = runner.y_host.clone()
        want = lay.forward(xs[s].cuda()).cpu()
        torch.cuda.synchronize()
        assert np.allclose(bits_to_f32(got.numpy()), bits_to_f32(want.numpy()), rtol=1e-2, atol=1e-3)


def barrier_generations(ws):
    """Generations completed on the one-kernel decode layer's barrier counter (the first
    64-bit word of its workspace; the grid has SMs - 1 CTAs), as a one-element list; None
    where the counter is not a whole number of generations."""
    grid = torch.cuda.get_device_properties(0).multi_processor_count - 1
    c = int(ws[:8].view(torch.int64).cpu()[0])
    return [c // grid if c % grid == 0 else None]


def test_fused_decode_layer_repeated_calls():
    """The one-kernel decode layer leaves its barrier counter aligned to the grid, gives the same
    result on repeated calls, and agrees with the five-call path on the same inputs."""
    cfg, lay, Wr, br = _layer("decode", T_max=8, fused=True)
    _, lay5, _, _ = _layer("decode", T_max=8, fused=False)
    outs = []
    for step in range(3):
        x = synth.make_x(7, cfg, 8, step=step).cuda()
        y = lay.forward(x).clone()
        y5 = lay5.forward(x).clone()
        torch.cuda.synchronize()
        assert B.moe_get_device_status() == 0
        # the barrier's arrival counter ends every call at a whole number of generations
        gens = barrier_generations(lay.ws_dec)
        assert gens[0] is not None and gens[0] > 0
        a, b5 = bits_to_f32(y.cpu().numpy()), bits_to_f32(y5.cpu().numpy())
        assert np.abs(a - b5).max() <= 2e-2 * np.sqrt((b5 ** 2).mean())
        assert np.array_equal(lay.topk_idx.cpu().numpy(), lay5.topk_idx.cpu().numpy())
        outs.append(y.cpu())
    x = synth.make_x(7, cfg, 8, step=0).cuda()
    y = lay.forward(x).clone()
    torch.cuda.synchronize()
    assert np.allclose(bits_to_f32(y.cpu().numpy()), bits_to_f32(outs[0].numpy()), rtol=1e-2, atol=1e-3)


def test_decode_layer_with_weights_held_once():
    """After release_natural() a group keeps only its decode pack and tensor scales (each
    weight byte once): the one-kernel decode layer gives the same result as before, and the
    paths that read the natural layout refuse instead of reading freed memory."""
    cfg, lay, Wr, br = _layer("decode", T_max=8, fused=True)
    x = synth.make_x(8, cfg, 8).cuda()
    y1 = lay.forward(x).clone()
    for g in (lay.experts.routed, lay.experts.shared):
        g.release_natural()
    torch.cuda.empty_cache()
    y2 = lay.forward(x).clone()
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0
    a, b = bits_to_f32(y2.cpu().numpy()), bits_to_f32(y1.cpu().numpy())
    assert np.abs(a - b).max() <= 1e-2 * np.sqrt((b ** 2).mean())
    with pytest.raises(B.MoeError):
        B.moe_expert_ffn(lay.xq_codes[:8], lay.xq_scales[:8], lay.xq_ts[:1], lay.experts, cfg.k, lay.offsets,
                         lay.sorted_assign[:8 * cfg.k], lay.topk_w[:8], B.MOE_FFN_ACCUMULATE, B.MOE_PATH_PREFILL,
                         lay.y_acc[:8], None, lay.ws)
