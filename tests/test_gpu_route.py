"""moe_route / moe_permute on the GPU vs the oracle."""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import synth

from helpers import bits_to_f32, check_permutation_valid, compare_topk, route_buffers

pytestmark = pytest.mark.gpu


def _gpu_route(x, Wr, br, k):
    T, d = x.shape
    E = Wr.shape[0]
    b = route_buffers(T, k, E, d)
    B.moe_route(x.cuda(), Wr.cuda(), None if br is None else br.cuda(), k, b["topk_idx"],
                b["topk_w"], b["counts"], b["offsets"], b["sorted_assign"], b["assign_pos"], b["ws"])
    torch.cuda.synchronize()
    return {n: t.cpu().numpy() for n, t in b.items() if n != "ws"}


def _check_route(x, Wr, br, k):
    T, d = x.shape
    E = Wr.shape[0]
    g = _gpu_route(x, Wr, br, k)
    xf = bits_to_f32(x.numpy())
    logits = omoe.router_logits(xf, Wr.numpy(), None if br is None else br.numpy())
    idx = omoe.topk_fast(logits, k)
    w = omoe.routing_weights(logits, idx)
    excused = compare_topk(g["topk_idx"], idx, logits, k)
    ok = np.array([t not in set(excused) for t in range(T)], dtype=bool)
    # where the sets agree compare the weight of each expert (slot order inside the top-k is
    # descending logit; two chosen experts closer than the tie margin may swap slots)
    for t in np.flatnonzero(ok):
        og, orf = np.argsort(g["topk_idx"][t]), np.argsort(idx[t])
        assert np.array_equal(g["topk_idx"][t][og], idx[t][orf])
        np.testing.assert_allclose(g["topk_w"][t][og], w[t][orf], rtol=2e-6, atol=1e-7)
    lg_sel = np.take_along_axis(logits.astype(np.float64), g["topk_idx"].astype(np.int64), 1)
    assert np.all(np.diff(lg_sel[ok], axis=1) <= 1e-6), "GPU slots not in descending logit order"
    # the permutation must be a valid stable counting sort of the GPU's own top-k
    check_permutation_valid(g["topk_idx"], g["counts"], g["offsets"], g["sorted_assign"],
                            g["assign_pos"], E)
    if not excused:
        counts, offsets, sa, pos = omoe.permute(idx, E)
        assert np.array_equal(g["counts"], counts)
        assert np.array_equal(g["offsets"], offsets)
        # token ids per expert are unique; slot ids too unless near-tied slots swapped
        assert np.array_equal(g["sorted_assign"][:T * k] // k, sa // k)
        if np.array_equal(g["topk_idx"], idx):
            assert np.array_equal(g["sorted_assign"][:T * k], sa)
            assert np.array_equal(g["assign_pos"][:T * k], pos)
    return len(excused)


@pytest.mark.parametrize("cfg_name", ["prefill", "wide"])
def test_tensor_core_router_error_is_far_below_its_margin(cfg_name):
    """From 256 tokens on, moe_route takes approximate logits from a bf16-split tensor-core
    GEMM (left in the first T*E*4 bytes of the workspace) and recomputes exactly every expert
    within 2*delta (delta = 2e-3) of the k-th. That is exact as long as each approximate logit
    is within delta of the true one: check it is within delta/20 of the oracle's."""
    c = synth.CONFIGS[cfg_name]
    T = c.T_list[0]
    x = synth.make_x(0, c, T)
    Wr, br = synth.make_router(0, c)
    brg = br if c.zipf_s > 0 else None
    b = route_buffers(T, c.k, c.E, c.d)
    B.moe_route(x.cuda(), Wr.cuda(), None if brg is None else brg.cuda(), c.k, b["topk_idx"], b["topk_w"],
                b["counts"], b["offsets"], b["sorted_assign"], b["assign_pos"], b["ws"])
    torch.cuda.synchronize()
    approx = b["ws"][:T * c.E * 4].view(torch.float32).view(T, c.E).cpu().numpy().astype(np.float64)
    logits = omoe.router_logits(bits_to_f32(x.numpy()), Wr.numpy(), None if brg is None else brg.numpy())
    err = np.abs(approx - logits).max()
    print(f"{cfg_name}: max |approximate - oracle logit| = {err:.3e}")
    assert err < 2e-3 / 20


@pytest.mark.parametrize("cfg,T", [("tiny", 16), ("decode", 1), ("decode", 4), ("decode", 8),
                                   ("decode", 9), ("decode", 100), ("decode", 300), ("prefill", 16384),
                                   ("wide", 27140)])
def test_route_matches_oracle(cfg, T):
    c = synth.CONFIGS[cfg]
    x = synth.make_x(0, c, T)
    Wr, br = synth.make_router(0, c)
    n_exc = _check_route(x, Wr, br if c.zipf_s > 0 else None, c.k)
    print(f"{cfg} T={T}: {n_exc} tie-excused tokens")


def test_route_ties_go_to_lower_index():
    # identical router rows produce exactly tied logits: the lower ids must win
    c = synth.CONFIGS["tiny"]
    x = synth.make_x(1, c, 40)
    Wr, _ = synth.make_router(1, c)
    Wr[5] = Wr[2]
    Wr[7] = Wr[2]
    g = _gpu_route(x, Wr, None, 2)
    lg = omoe.router_logits(bits_to_f32(x.numpy()), Wr.numpy())
    assert np.array_equal(g["topk_idx"], omoe.topk(lg, 2))


def test_route_T0():
    c = synth.CONFIGS["decode"]
    Wr, br = synth.make_router(0, c)
    g = _gpu_route(torch.zeros(0, c.d, dtype=torch.int16), Wr, br, c.k)
    assert not g["counts"].any() and not g["offsets"].any()


@pytest.mark.parametrize("T,k,E,skew", [(1, 1, 8, 0), (16, 2, 8, 0), (409, 10, 512, 0),
                                        (410, 10, 512, 1), (16384, 10, 512, 0),
                                        (30000, 8, 1024, 1), (5000, 1, 3, 1), (0, 4, 16, 0)])
def test_permute_bit_exact(T, k, E, skew):
    rng = np.random.default_rng(T + 7 * E)
    if skew:  # heavy concentration on a few experts
        p = 1.0 / np.arange(1, E + 1) ** 1.5
        p /= p.sum()
    else:
        p = None
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32) \
        if T else np.zeros((0, k), np.int32)
    b = route_buffers(T, k, E, 16)
    B.moe_permute(torch.from_numpy(idx).cuda().view(T, k), E, b["counts"], b["offsets"],
                  b["sorted_assign"], b["assign_pos"], b["ws"])
    torch.cuda.synchronize()
    counts, offsets, sa, pos = omoe.permute(idx, E)
    assert np.array_equal(b["counts"].cpu().numpy(), counts)
    assert np.array_equal(b["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(b["sorted_assign"].cpu().numpy()[:T * k], sa)
    assert np.array_equal(b["assign_pos"].cpu().numpy()[:T * k], pos)
