"""Checks of the seeded input generator (CPU only)."""
import numpy as np
import torch

from nvfp4_expert_ffn_b200 import synth


def test_deterministic_and_keyed():
    cfg = synth.CONFIGS["decode"]
    a = synth.make_x(0, cfg, 4)
    assert torch.equal(a, synth.make_x(0, cfg, 4))
    assert not torch.equal(a, synth.make_x(1, cfg, 4))
    assert not torch.equal(a, synth.make_x(0, cfg, 4, step=1))
    # a prefix of a longer draw equals the shorter draw (counter-based)
    key = synth.stream_key(3, 4)
    assert torch.equal(synth.normal_f32(key, 100, 1.0)[:50], synth.normal_f32(key, 50, 1.0))
    assert torch.equal(synth.normal_f32(key, 100, 1.0)[50:], synth.normal_f32(key, 50, 1.0, offset=50))


def test_moments():
    z = synth.normal_f32(synth.stream_key(9), 1 << 20, 0.02).double()
    assert abs(z.mean().item()) < 1e-4 and abs(z.std().item() - 0.02) < 2e-4
    assert z.abs().max().item() <= 0.02 * 3.47


def test_bf16_rounding_matches_torch():
    x = synth.normal_f32(synth.stream_key(5), 100000, 3.0) * 1.2345
    ours = synth.f32_to_bf16_bits(x)
    ref = x.to(torch.bfloat16).view(torch.int16)
    assert torch.equal(ours, ref)
    assert torch.equal(synth.bf16_bits_to_f32(ours), ref.view(torch.bfloat16).float())


def test_zipf_bias_is_log_rank_permutation():
    cfg = synth.CONFIGS["decode"]
    _, br = synth.make_router(0, cfg)
    ranks = np.rint(np.exp(-br.double().numpy() / cfg.zipf_s)).astype(int)
    assert sorted(ranks) == list(range(1, cfg.E + 1))
    _, br2 = synth.make_router(0, cfg, epoch=1)
    assert not torch.equal(br, br2)
    _, b0 = synth.make_router(0, synth.CONFIGS["wide"])
    assert not b0.any()


def test_batched_expert_draws_equal_single_draws():
    """The batched generator gives, row by row, the bits of the one-expert generator."""
    cfg = synth.CONFIGS["tiny"]
    g, u, dn = synth.make_experts_weights_bf16(3, cfg, [0, 5, 7], layer=2)
    for r, e in enumerate([0, 5, 7]):
        g1, u1, d1 = synth.make_expert_weights_bf16(3, cfg, e, layer=2)
        assert torch.equal(g[r], g1) and torch.equal(u[r], u1) and torch.equal(dn[r], d1)
    gs, us, ds = synth.make_experts_weights_bf16(3, cfg, [0], layer=2, shared=True)
    g1, u1, d1 = synth.make_expert_weights_bf16(3, cfg, 0, layer=2, shared=True)
    assert torch.equal(gs[0], g1) and torch.equal(ds[0], d1)
