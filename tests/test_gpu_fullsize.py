"""The whole five-call layer (MoeLayer.forward: quantise, route, expert FFN on the
tensor-core path, combine, histogram) at the full prefill sizes, against the oracle.

prefill: d=2048, 512 experts, top-10 + shared, I=512, T=16384, Zipf(0.8) routing.
wide:    d=4096, 256 experts, top-8 + shared, I=2048, T=27140, uniform routing.

Every token: the activation codes, scales and tensor scale bit-exact; the top-k set per
token (tokens whose k-th/(k+1)-th float32 logit margin is under 1e-6 are excused, and they
must be the ones tests/golden/near_ties.json lists); the routing weights; the permutation
and the per-call histogram bit-exact (or, if a token was excused, a valid stable counting
sort of the GPU's own top-k); the cumulative histogram and rank. A seeded subset of 2,048
tokens: the layer output against the oracle's float64 FFN and combine (rel-L2 <= 5e-3,
max-abs <= 2e-2 RMS), the oracle's per-expert work spread over host processes.

With MOE_PARITY_REPORT set to a file name, each case appends one JSON line (excused tokens,
errors) to that file.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import nvfp4 as onv
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import assert_close_layer, bits_to_f32, check_permutation_valid, compare_topk
from oracle_pool import expert_outputs

pytestmark = pytest.mark.gpu

SUBSET = 2048
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "near_ties.json")


def _golden_near_ties(cfg_name, T, step=0):
    for r in json.load(open(GOLDEN)):
        if r["config"] == cfg_name and r["T"] == T and r["step"] == step:
            return set(r["tokens"])
    raise KeyError((cfg_name, T, step))


def _report(rec):
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


@pytest.mark.parametrize("cfg_name", ["prefill", "wide"])
def test_five_call_layer_full_size(cfg_name):
    cfg = synth.CONFIGS[cfg_name]
    T, k, E, d = cfg.T_list[0], cfg.k, cfg.E, cfg.d
    routed = L.quantize_weights_gpu(0, cfg)
    shared = L.quantize_weights_gpu(0, cfg, shared=True)
    Wr, br = synth.make_router(0, cfg)
    use_br = cfg.zipf_s > 0
    lay = L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), br.cuda() if use_br else None, k, T, fused=False)
    x = synth.make_x(0, cfg, T)
    y = lay.forward(x.cuda())
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0
    g = {n: getattr(lay, n).cpu().numpy() for n in ("xq_codes", "xq_scales", "topk_idx", "topk_w", "counts",
                                                   "offsets", "sorted_assign", "assign_pos", "cum", "rank")}
    g["xq_ts"] = float(lay.xq_ts[0])
    yg = bits_to_f32(y.cpu().numpy())
    del routed, shared, lay
    torch.cuda.empty_cache()

    # every token: quantised activation, routing, permutation, histogram
    xf = bits_to_f32(x.numpy())
    xc, xs, xts = onv.quantize(xf)
    assert np.array_equal(g["xq_codes"], xc) and np.array_equal(g["xq_scales"], xs)
    assert g["xq_ts"] == float(xts)
    logits = omoe.router_logits(xf, Wr.numpy(), br.numpy() if use_br else None)
    idx = omoe.topk_fast(logits, k)
    w = omoe.routing_weights(logits, idx)
    excused = compare_topk(g["topk_idx"], idx, logits, k)
    assert set(excused) <= _golden_near_ties(cfg_name, T)
    ok = np.ones(T, bool)
    ok[excused] = False
    og, orf = np.argsort(g["topk_idx"][ok], 1), np.argsort(idx[ok], 1)
    np.testing.assert_allclose(np.take_along_axis(g["topk_w"][ok], og, 1), np.take_along_axis(w[ok], orf, 1),
                               rtol=2e-6, atol=1e-7)
    check_permutation_valid(g["topk_idx"], g["counts"], g["offsets"], g["sorted_assign"], g["assign_pos"], E)
    if not excused:
        counts, offsets, sa, pos = omoe.permute(idx, E)
        assert np.array_equal(g["counts"], counts) and np.array_equal(g["offsets"], offsets)
        assert np.array_equal(g["sorted_assign"][:T * k] // k, sa // k)
        if np.array_equal(g["topk_idx"], idx):
            assert np.array_equal(g["sorted_assign"][:T * k], sa)
            assert np.array_equal(g["assign_pos"][:T * k], pos)
    cum, rank = omoe.hist_update(g["counts"] if excused else omoe.permute(idx, E)[0])
    assert np.array_equal(g["cum"], cum) and np.array_equal(g["rank"], rank)

    # a seeded subset of tokens: the layer output against the oracle's FFN and combine
    rng = np.random.default_rng(2048)
    tokens = np.sort(rng.choice(np.flatnonzero(ok), min(SUBSET, int(ok.sum())), replace=False))
    x_hat = onv.dequantize(xc, xs, xts)
    sub_idx = idx[tokens]
    tasks = []
    where = {}
    for e in np.unique(sub_idx):
        rows = np.argwhere(sub_idx == e)  # (position in subset, slot)
        where[int(e)] = rows
        tasks.append((int(e), False, x_hat[tokens[rows[:, 0]]]))
    tasks.append((0, True, x_hat[tokens]))
    outs = expert_outputs(cfg_name, 0, 0, tasks)
    o_assign = np.zeros((tokens.size, k, d))
    for e, rows in where.items():
        o_assign[rows[:, 0], rows[:, 1]] = outs[(e, False)]
    y_ref = omoe.combine(tokens.size, d, sub_idx, w[tokens], o_assign.reshape(-1, d), outs[(0, True)])
    rel, mabs = assert_close_layer(yg[tokens], y_ref, f"{cfg_name} subset")
    _report({"test": "five_call_layer_full_size", "config": cfg_name, "T": T, "excused_tokens": len(excused),
             "golden_near_ties": len(_golden_near_ties(cfg_name, T)), "subset_tokens": int(tokens.size),
             "experts_checked": len(where) + 1, "rel_l2": rel, "max_abs_over_rms": mabs})
