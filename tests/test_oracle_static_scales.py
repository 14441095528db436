"""Pins of the oracle's static per-expert input scales (reading R13; "Basalt" project page,
"All the numbers", list "Engines: commit, and what is not NVIDIA's weights": NVIDIA's NVFP4
experts carry an input_scale). Each check is something a misplaced or ignored scale fails:

* given the dynamic scale of the whole batch and 1.0 for h, the static path is the dynamic
  path exactly (its pinned pieces: the quantiser, the dequantiser, expert_ffn);
* scaling both static scales by a power of two, while every E4M3 block scale stays in the
  normal range, leaves every code, every block scale times its tensor scale, and so the
  output, exactly unchanged (E4M3 normals scale exactly by powers of two);
* with small activations (h of about 1e-4), a unit scale for h puts its E4M3 block scales
  below the normal range and loses precision, while a static scale sized to h keeps the
  output close to the float64 FFN on unquantised h (computed here with torch); likewise an
  activation scale far too small saturates x and moves the output far away.
"""
import numpy as np
import torch

from oracle import moe, nvfp4

F32 = np.float32


def _expert(rng, d, I, std=0.02):
    gate = rng.normal(0, std, (I, d)).astype(F32)
    up = rng.normal(0, std, (I, d)).astype(F32)
    down = rng.normal(0, std, (d, I)).astype(F32)
    return moe.Expert.from_f32(gate, up, down)


def test_static_equals_dynamic_with_the_dynamic_scale():
    rng = np.random.default_rng(11)
    d, I, n = 64, 32, 6
    ex = _expert(rng, d, I)
    x = rng.normal(0, 1, (n, d)).astype(F32)
    xc, xs, xts = nvfp4.quantize(x)
    want = moe.expert_ffn(nvfp4.dequantize(xc, xs, xts), ex)
    got = moe.expert_ffn_static(x, ex, xts, 1.0)
    assert np.array_equal(got, want)


def _h_block_amax(x_hat, ex):
    """max |h| of every 16-block of h = silu(g) * u, from torch float64 (precondition only)."""
    Wg, Wu, _ = (torch.from_numpy(m) for m in ex.dense())
    xt = torch.from_numpy(np.asarray(x_hat, dtype=np.float64))
    g, u = xt @ Wg.T, xt @ Wu.T
    h = torch.nn.functional.silu(g) * u
    return h.abs().reshape(h.shape[0], -1, 16).amax(dim=2).numpy()


def test_power_of_two_scales_leave_the_output_unchanged():
    rng = np.random.default_rng(12)
    d, I, n = 64, 32, 5
    ex = _expert(rng, d, I, std=0.2)
    x = rng.uniform(0.5, 2.0, (n, d)).astype(F32) * np.where(rng.random((n, d)) < 0.5, -1, 1).astype(F32)
    ts0 = F32(2.0 / (6 * 448))
    # precondition: every block scale of x and of h stays normal (>= 2^-6) and below 448 for
    # both choices of scales
    xb = np.abs(x).reshape(n, -1, 16).max(axis=2)
    hb = _h_block_amax(x, ex)
    for c in (1.0, 8.0):
        assert ((xb / 6 / (ts0 * c) >= 2 ** -6) & (xb / 6 / (ts0 * c) <= 448)).all()
        assert ((hb / 6 / c >= 2 ** -6 * 1.01) & (hb / 6 / c <= 448)).all()
    a = moe.expert_ffn_static(x, ex, ts0, 1.0)
    b = moe.expert_ffn_static(x, ex, F32(ts0 * 8), 8.0)
    assert np.array_equal(a, b)


def test_static_scales_are_applied():
    rng = np.random.default_rng(13)
    d, I, n = 128, 64, 4
    ex = _expert(rng, d, I, std=0.002)  # h of about 1e-4
    x = rng.normal(0, 1, (n, d)).astype(F32)
    xc, xs, xts = nvfp4.quantize(x)
    x_hat = nvfp4.dequantize(xc, xs, xts)
    # float64 reference on unquantised h (torch)
    Wg, Wu, Wd = (torch.from_numpy(m) for m in ex.dense())
    xt = torch.from_numpy(x_hat)
    ref = ((torch.nn.functional.silu(xt @ Wg.T) * (xt @ Wu.T)) @ Wd.T).numpy()
    amax_h = float(np.max(np.abs(_h_block_amax(x_hat, ex))))
    assert amax_h < 1e-2
    err = lambda o: float(np.sqrt(np.mean((o - ref) ** 2) / np.mean(ref ** 2)))  # noqa: E731
    unit = moe.expert_ffn_static(x, ex, xts, 1.0)
    sized = moe.expert_ffn_static(x, ex, xts, F32(amax_h / (6 * 448)))
    assert err(sized) < 0.1 and err(unit) > 10 * err(sized)
    # an activation scale 64x too small saturates most of x
    sat = moe.expert_ffn_static(x, ex, F32(xts / 64), F32(amax_h / (6 * 448)))
    assert err(sat) > 10 * err(sized)


def test_ffn_static_forward_matches_per_expert_sum():
    """The combine over experts: y[t] = sum_j w[t,j] o_e(x_t) + o_shared(x_t), with each
    expert's own scales; checked against an explicit loop over tokens."""
    rng = np.random.default_rng(14)
    d, I, E, k, T = 32, 16, 4, 2, 5
    experts = [_expert(rng, d, I) for _ in range(E)]
    shared = _expert(rng, d, I)
    xb = (rng.normal(0, 1, (T, d)).astype(F32).view(np.uint32) >> 16).astype(np.uint16)
    x = (xb.astype(np.uint32) << 16).view(F32)
    idx = np.array([[0, 1], [2, 3], [1, 0], [3, 2], [0, 3]])
    w = rng.random((T, k)).astype(F32)
    in_gu = (np.array([1, 2, 4, 8, 16], dtype=F32) * F32(1e-3))
    in_dn = np.array([1.0, 0.5, 0.25, 2.0, 1.0], dtype=F32) * F32(1e-3)
    y = moe.ffn_static_forward(xb, idx, w, experts, shared, in_gu, in_dn)
    for t in range(T):
        want = moe.expert_ffn_static(x[t:t + 1], shared, in_gu[E], in_dn[E])[0]
        for j in range(k):
            e = idx[t, j]
            want = want + np.float64(w[t, j]) * moe.expert_ffn_static(x[t:t + 1], experts[e], in_gu[e], in_dn[e])[0]
        assert np.allclose(y[t], want, rtol=1e-12, atol=1e-15)
    ysub = moe.ffn_static_forward(xb, idx, w, experts, shared, in_gu, in_dn, tokens=[1, 3])
    assert np.isnan(ysub[0]).all() and np.array_equal(ysub[[1, 3]], y[[1, 3]])
