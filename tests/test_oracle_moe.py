"""Pins for the oracle's routing, permutation, FFN, combine and histogram (CPU only)."""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe, nvfp4
from nvfp4_expert_ffn_b200 import synth

F32 = np.float32


# ------------------------------------------------------------------ router

def test_topk_matches_lexsort_prefix_and_breaks_ties_low_index():
    rng = np.random.default_rng(0)
    logits = rng.standard_normal((40, 64)).astype(F32)
    # plant exact ties around the k-th place
    logits[3, [5, 9, 30]] = 10.0
    logits[4, :] = 0.5
    idx = moe.topk(logits, 6)
    for t in range(40):
        order = np.lexsort((np.arange(64), -logits[t].astype(np.float64)))
        assert list(idx[t]) == list(order[:6])
    assert list(idx[3, :3]) == [5, 9, 30]
    assert list(idx[4]) == [0, 1, 2, 3, 4, 5]
    assert np.array_equal(moe.topk_fast(logits, 6), idx)


def test_routing_weights_are_restricted_renormalised_softmax():
    rng = np.random.default_rng(1)
    logits = (rng.standard_normal((32, 128)) * 3).astype(F32)
    idx = moe.topk(logits, 10)
    w = moe.routing_weights(logits, idx)
    p = scipy.special.softmax(logits.astype(np.float64), axis=1)
    ref = np.take_along_axis(p, idx, 1)
    ref = ref / ref.sum(1, keepdims=True)
    assert np.allclose(w, ref, rtol=2e-7, atol=0)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1) <= 10 * 2.0 ** -24)
    assert np.all(np.diff(w, axis=1) <= 0)  # descending logits -> descending weights


def test_router_logits_float64_then_float32_with_bias():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 64)).astype(F32)
    W = rng.standard_normal((7, 64)).astype(F32)
    b = rng.standard_normal(7).astype(F32)
    ref = (torch.from_numpy(x).double() @ torch.from_numpy(W).double().T
           + torch.from_numpy(b).double()).float().numpy()
    assert np.array_equal(moe.router_logits(x, W, b), ref)
    # a large bias on one expert makes it everyone's first choice, with weight 1 at k=1
    b2 = np.zeros(7, F32)
    b2[4] = 100.0
    lg = moe.router_logits(x, W, b2)
    idx = moe.topk(lg, 1)
    assert np.all(idx[:, 0] == 4)
    assert np.all(moe.routing_weights(lg, idx) == 1.0)


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("T,k,E", [(0, 2, 8), (1, 1, 4), (16, 2, 8), (37, 5, 64), (300, 10, 512)])
def test_permute_matches_stable_argsort_and_bincount(T, k, E):
    rng = np.random.default_rng(T * 131 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]) if T else \
        np.zeros((0, k), np.int64)
    counts, offsets, sa, pos = moe.permute(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(offsets[1:], np.cumsum(counts))
    assert np.array_equal(sa, np.argsort(flat, kind="stable"))
    assert np.array_equal(sa[pos], np.arange(T * k))
    for e in range(E):
        seg = sa[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)


# ------------------------------------------------------------------ expert FFN

def _small_expert(seed, d=64, I=32):
    rng = np.random.default_rng(seed)
    g = (rng.standard_normal((I, d)) * 0.05).astype(F32)
    u = (rng.standard_normal((I, d)) * 0.05).astype(F32)
    dn = (rng.standard_normal((d, I)) * 0.05).astype(F32)
    return moe.Expert.from_f32(g, u, dn)


def test_expert_ffn_matches_torch_float64_swiglu():
    ex = _small_expert(3)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((9, 64)).astype(F32)
    xc, xs, xts = nvfp4.quantize(x)
    xh = nvfp4.dequantize(xc, xs, xts)
    out = moe.expert_ffn(xh, ex)
    Wg, Wu, Wd = (torch.from_numpy(m) for m in ex.dense())
    xt = torch.from_numpy(xh)
    h = (torch.nn.functional.silu(xt @ Wg.T) * (xt @ Wu.T)).float().numpy()
    hc, hs, _ = nvfp4.quantize(h, ts=F32(1.0))
    ref = torch.from_numpy(nvfp4.dequantize(hc, hs, F32(1.0))) @ Wd.T
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-15)


def test_expert_ffn_linear_in_down_scale_and_zero_weights():
    ex = _small_expert(5)
    x = nvfp4.dequantize(*nvfp4.quantize(np.random.default_rng(6).standard_normal((4, 64))
                                         .astype(F32)))
    o1 = moe.expert_ffn(x, ex)
    ex2 = moe.Expert(ex.gu_codes, ex.gu_scales, ex.gate_ts, ex.up_ts, ex.dn_codes,
                     ex.dn_scales, ex.dn_ts * F32(2.0))
    assert np.array_equal(moe.expert_ffn(x, ex2), 2 * o1)
    z = moe.Expert(ex.gu_codes, ex.gu_scales, ex.gate_ts, ex.up_ts,
                   np.zeros_like(ex.dn_codes), ex.dn_scales, ex.dn_ts)
    assert not np.any(moe.expert_ffn(x, z))
    assert moe.expert_ffn(x[:0], ex).shape == (0, 64)


def test_swiglu_order_gate_rows_first():
    # swapping the gate and up halves changes the output (silu is not symmetric)
    ex = _small_expert(8)
    I = ex.I
    sw = moe.Expert(np.concatenate([ex.gu_codes[I:], ex.gu_codes[:I]]),
                    np.concatenate([ex.gu_scales[I:], ex.gu_scales[:I]]),
                    ex.up_ts, ex.gate_ts, ex.dn_codes, ex.dn_scales, ex.dn_ts)
    x = nvfp4.dequantize(*nvfp4.quantize(np.random.default_rng(9).standard_normal((4, 64))
                                         .astype(F32)))
    Wg, Wu, _ = ex.dense()
    g = x @ Wg.T
    assert np.allclose(moe.silu(g), g * scipy.special.expit(g), rtol=1e-14)
    assert not np.allclose(moe.expert_ffn(x, ex), moe.expert_ffn(x, sw))


# ------------------------------------------------------------------ whole layer

def _tiny_layer(seed=0, shared=False):
    cfg = synth.CONFIGS["tiny"]
    experts = []
    for e in range(cfg.E):
        g, u, dn = synth.make_expert_weights_f32(seed, cfg, e)
        experts.append(moe.Expert.from_f32(g.numpy(), u.numpy(), dn.numpy()))
    sh = None
    if shared:
        g, u, dn = synth.make_expert_weights_f32(seed, cfg, 0, shared=True)
        sh = moe.Expert.from_f32(g.numpy(), u.numpy(), dn.numpy())
    Wr, br = synth.make_router(seed, cfg)
    x = synth.make_x(seed, cfg, 16).numpy()
    return cfg, x, Wr.numpy(), br.numpy(), experts, sh


@pytest.mark.parametrize("shared", [False, True])
def test_layer_brute_force_dense_masked(shared):
    """Tiny layer, brute force: evaluate every expert on every token densely, then mask by
    a routing computed independently (scipy softmax over all experts, top-k by lexsort,
    renormalised) and sum; the oracle's gather/scatter path must agree."""
    cfg, x, Wr, br, experts, sh = _tiny_layer(0, shared)
    out = moe.layer_forward(x, Wr, br, cfg.k, experts, sh)
    xf = (x.astype(np.uint16).astype(np.uint32) << 16).view(F32)
    xh = nvfp4.dequantize(*nvfp4.quantize(xf))
    logits = (torch.from_numpy(xf).double() @ torch.from_numpy(Wr).double().T
              + torch.from_numpy(br).double()).float().numpy().astype(np.float64)
    p = scipy.special.softmax(logits, axis=1)
    y = np.zeros((16, cfg.d))
    for t in range(16):
        order = np.lexsort((np.arange(cfg.E), -logits[t]))[:cfg.k]
        wsum = p[t, order].sum()
        for e in order:
            y[t] += p[t, e] / wsum * moe.expert_ffn(xh[t:t + 1], experts[e])[0]
        if sh is not None:
            y[t] += moe.expert_ffn(xh[t:t + 1], sh)[0]
    rel = np.linalg.norm(out["y"] - y) / np.linalg.norm(y)
    assert rel < 1e-6
    assert out["counts"].sum() == 16 * cfg.k


def test_layer_one_hot_plus_shared_is_sum_of_two_dense_ffns():
    cfg, x, Wr, _, experts, sh = _tiny_layer(1, shared=True)
    br = np.zeros(cfg.E, F32)
    br[3] = 100.0
    out = moe.layer_forward(x, Wr, br, 1, experts, sh)
    assert np.all(out["idx"][:, 0] == 3) and np.all(out["w"] == 1.0)
    xf = (x.astype(np.uint16).astype(np.uint32) << 16).view(F32)
    xh = nvfp4.dequantize(*nvfp4.quantize(xf))
    ref = moe.expert_ffn(xh, experts[3]) + moe.expert_ffn(xh, sh)
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-14)


def test_layer_token_subset_matches_full():
    cfg, x, Wr, br, experts, sh = _tiny_layer(2, shared=True)
    full = moe.layer_forward(x, Wr, br, cfg.k, experts, sh)
    sub = moe.layer_forward(x, Wr, br, cfg.k, experts, sh, assign_subset=[1, 7, 15])
    assert np.array_equal(sub["y"][[1, 7, 15]], full["y"][[1, 7, 15]])
    assert np.isnan(sub["y"][0]).all()
    assert np.array_equal(sub["sorted_assign"], full["sorted_assign"])


def test_rms_renorm():
    y = np.array([[3.0, 4.0], [0.0, 0.0]])
    r = moe.rms_renorm(y)
    assert np.allclose(np.mean(r[0] ** 2), 1.0) and not r[1].any()


# ------------------------------------------------------------------ histogram

def test_hist_cumulates_and_ranks_hot_to_cold():
    c1 = np.array([0, 5, 2, 5, 1], np.int32)
    cum, rank = moe.hist_update(c1)
    assert list(cum) == [0, 5, 2, 5, 1]
    assert list(rank) == [1, 3, 2, 4, 0]  # ties 1/3 -> lower id first
    cum, rank = moe.hist_update(np.array([3, 0, 4, 0, 0], np.int32), cum)
    assert list(cum) == [3, 5, 6, 5, 1]
    assert list(rank) == list(np.lexsort((np.arange(5), -cum)))
    cum, _ = moe.hist_update(np.array([1, 1, 1, 1, 1]), cum, reset=True)
    assert list(cum) == [1, 1, 1, 1, 1]
