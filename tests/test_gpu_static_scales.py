"""moe_expert_ffn_static (static per-expert input scales, reading R13) on the GPU against the
oracle, with the oracle's routing fed to the kernel.

* decode-shaped experts (d=2048, 512 experts, top-10 + shared, I=512) at T=300 (every expert's
  m-tiles ragged) and at the full prefill size T=16384, with each expert's own activation
  and h scales (synth.make_input_scales): rel-L2 and max-abs within the layer tolerance on a
  seeded token sample, in ACCUMULATE and PER_ASSIGN modes;
* given every expert the call's dynamic activation scale and h scale 1.0, the static kernel
  matches the ordinary PREFILL path of moe_expert_ffn on every token (both quantise the same
  rows to the same codes).
"""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import nvfp4 as onv
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import assert_close_layer, bits_to_f32
from oracle_pool import OraclePool

pytestmark = pytest.mark.gpu

CFG = "decode"


@pytest.fixture(scope="module")
def experts():
    cfg = synth.CONFIGS[CFG]
    return cfg, B.Experts(L.quantize_weights_gpu(0, cfg), L.quantize_weights_gpu(0, cfg, shared=True))


def _routing(cfg, T, step):
    x = synth.make_x(0, cfg, T, step=step)
    xf = bits_to_f32(x.numpy()).astype(np.float32)
    Wr, br = synth.make_router(0, cfg)
    logits = omoe.router_logits(xf, Wr.numpy(), br.numpy())
    idx = omoe.topk_fast(logits, cfg.k)
    w = omoe.routing_weights(logits, idx)
    counts, offsets, sa, pos = omoe.permute(idx, cfg.E)
    return x, xf, idx, w, offsets, sa, pos


def _run_static(cfg, ex, x, routing, in_gu, in_dn, mode):
    idx, w, offsets, sa, pos = routing
    T, k, d = x.shape[0], cfg.k, cfg.d
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    out = torch.empty((T if mode == 0 else T * k), d, dtype=torch.float32, device="cuda")
    sh = torch.empty(T, d, dtype=torch.float32, device="cuda") if mode == 1 else None
    ws = torch.empty(B.moe_workspace_size(B.MOE_OP_FFN_STATIC, T, d, cfg.E, k, cfg.I), dtype=torch.uint8,
                     device="cuda")
    B.moe_expert_ffn_static(x.cuda(), ex, in_gu.cuda(), in_dn.cuda(), k, cu(offsets), cu(sa), cu(w), mode, out,
                            sh, ws)
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0
    return out.cpu().numpy(), None if sh is None else sh.cpu().numpy()


def _oracle_y(cfg, xf, idx, w, tokens, in_gu, in_dn, pool):
    """y[t] = sum_j w o_e(x_t) + o_shared(x_t) for the sampled tokens, per expert on the pool."""
    k, E = cfg.k, cfg.E
    tasks, rows_of = [], {}
    for e in np.unique(idx[tokens]):
        rows = [(t, j) for t in tokens for j in range(k) if idx[t, j] == e]
        rows_of[int(e)] = rows
        tasks.append((int(e), False, xf[[t for t, _ in rows]], float(in_gu[e]), float(in_dn[e])))
    tasks.append((0, True, xf[tokens], float(in_gu[E]), float(in_dn[E])))
    outs = pool.expert_outputs_static(CFG, 0, 0, tasks)
    y = outs[(0, True)].copy()
    pos = {t: i for i, t in enumerate(tokens)}
    o_assign = {}
    for e, rows in rows_of.items():
        for (t, j), r in zip(rows, outs[(e, False)]):
            o_assign[(t, j)] = r
    for t in tokens:
        for j in range(k):
            y[pos[t]] += np.float64(w[t, j]) * o_assign[(t, j)]
    return y, o_assign, outs[(0, True)]


@pytest.mark.parametrize("T,n_sample", [(300, 300), (16384, 48)])
def test_static_scales_match_oracle(experts, T, n_sample):
    cfg, ex = experts
    x, xf, idx, w, offsets, sa, pos = _routing(cfg, T, step=2)
    in_gu, in_dn = synth.make_input_scales(cfg)
    rng = np.random.default_rng(T)
    tokens = np.arange(T) if n_sample >= T else np.unique(np.concatenate(
        [[0, T - 1], rng.choice(T, n_sample - 2, replace=False)]))
    with OraclePool() as pool:
        y_ref, o_ref, sh_ref = _oracle_y(cfg, xf, idx, w, tokens, in_gu.numpy(), in_dn.numpy(), pool)
    out, _ = _run_static(cfg, ex, x, (idx, w, offsets, sa, pos), in_gu, in_dn, B.MOE_FFN_ACCUMULATE)
    assert_close_layer(out[tokens], y_ref, f"static scales T={T}")
    if T <= 300:
        # per-assignment mode: o of every assignment in sorted order, the shared expert apart
        o, sh = _run_static(cfg, ex, x, (idx, w, offsets, sa, pos), in_gu, in_dn, B.MOE_FFN_PER_ASSIGN)
        k = cfg.k
        got = np.stack([o[pos[t * k + j]] for t in tokens for j in range(k)])
        want = np.stack([o_ref[(t, j)] for t in tokens for j in range(k)])
        assert_close_layer(got, want, "static scales, per assignment")
        assert_close_layer(sh[tokens], sh_ref, "static scales, shared expert")


def test_static_kernel_with_dynamic_scale_matches_prefill_path(experts):
    cfg, ex = experts
    T, k, d = 700, cfg.k, cfg.d
    x, xf, idx, w, offsets, sa, pos = _routing(cfg, T, step=3)
    xc, xs, xts = onv.quantize(xf)
    in_gu = torch.full((cfg.E + 1,), float(xts), dtype=torch.float32)
    in_dn = torch.ones(cfg.E + 1, dtype=torch.float32)
    y_static, _ = _run_static(cfg, ex, x, (idx, w, offsets, sa, pos), in_gu, in_dn, B.MOE_FFN_ACCUMULATE)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    out = torch.empty(T, d, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.moe_workspace_size(B.MOE_OP_FFN, T, d, cfg.E, k, cfg.I), dtype=torch.uint8, device="cuda")
    B.moe_expert_ffn(cu(xc), cu(xs), cu(np.array([xts], np.float32)), ex, k, cu(offsets), cu(sa), cu(w),
                     B.MOE_FFN_ACCUMULATE, B.MOE_PATH_PREFILL, out, None, ws)
    torch.cuda.synchronize()
    y_dyn = out.cpu().numpy()
    # same codes, same products: only the order of the float32 additions into y differs
    assert np.abs(y_static - y_dyn).max() <= 1e-5 * np.sqrt((y_dyn ** 2).mean())
