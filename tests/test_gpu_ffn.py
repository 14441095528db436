"""moe_expert_ffn and moe_combine on the GPU vs the oracle (routing given by the oracle)."""
import numpy as np
import pytest
import torch

from oracle import moe as omoe
from oracle import nvfp4 as onv
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import (OracleWeights, assert_close_layer, bits_to_f32, oracle_expert_from_bf16,
                     weights_to_gpu)

pytestmark = pytest.mark.gpu


def _oracle_route(xf, Wr, br, k, E):
    logits = omoe.router_logits(xf, Wr, br)
    idx = omoe.topk_fast(logits, k)
    w = omoe.routing_weights(logits, idx)
    counts, offsets, sa, pos = omoe.permute(idx, E)
    return idx, w, offsets, sa, pos


def _run_ffn(xq, routing, experts_gpu, k, mode, path, T, d):
    idx, w, offsets, sa, pos = routing
    xc, xs, xts = xq
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    E, I = experts_gpu.routed.E, experts_gpu.routed.I
    out = torch.empty((T if mode == 0 else T * k), d, dtype=torch.float32, device="cuda")
    sh = torch.empty(T, d, dtype=torch.float32, device="cuda") \
        if (mode == 1 and experts_gpu.shared is not None) else None
    ws = torch.empty(B.moe_workspace_size(B.MOE_OP_FFN, T, d, E, k, I), dtype=torch.uint8,
                     device="cuda")
    B.moe_expert_ffn(cu(xc), cu(xs), cu(np.array([xts], np.float32)), experts_gpu, k,
                     cu(offsets), cu(sa), cu(w), mode, path, out, sh, ws)
    y = torch.empty(T, d, dtype=torch.int16, device="cuda")
    B.moe_combine(T, d, k, mode, out, sh, cu(w), cu(pos), False, y)
    torch.cuda.synchronize()
    return out.cpu().numpy(), None if sh is None else sh.cpu().numpy(), y.cpu().numpy()


def _oracle_outputs(xq, routing, experts, shared, T, d, k, tokens=None):
    idx, w, offsets, sa, pos = routing
    xh = onv.dequantize(*xq)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    want = np.zeros(T, bool)
    want[tokens] = True
    o = np.full((T * k, d), np.nan)
    for e in np.unique(idx[tokens]):
        seg = sa[offsets[e]:offsets[e + 1]]
        seg = seg[want[seg // k]]
        o[seg] = omoe.expert_ffn(xh[seg // k], experts[int(e)])
    os_ = None
    if shared is not None:
        os_ = np.full((T, d), np.nan)
        os_[tokens] = omoe.expert_ffn(xh[tokens], shared)
    y = omoe.combine(len(tokens), d, idx[tokens], w[tokens],
                     np.concatenate([o[t * k:(t + 1) * k] for t in tokens]),
                     None if os_ is None else os_[tokens])
    return o, os_, y


def _tiny_case(seed, d, E, k, I, T, shared, zipf=0.0, pack=False):
    cfg = synth.LayerShape("t", cid=100 + seed, d=d, E=E, k=k, I=I, shared=shared, zipf_s=zipf,
                           router_std=0.02)
    experts = [oracle_expert_from_bf16(*synth.make_expert_weights_bf16(seed, cfg, e))
               for e in range(E)]
    sh = oracle_expert_from_bf16(*synth.make_expert_weights_bf16(seed, cfg, 0, shared=True)) \
        if shared else None
    x = synth.make_x(seed, cfg, T).numpy()
    Wr, br = synth.make_router(seed, cfg)
    xf = bits_to_f32(x)
    xq = onv.quantize(xf)
    routing = _oracle_route(xf, Wr.numpy(), br.numpy(), k, E)
    gpu = B.Experts(weights_to_gpu(experts, pack=pack), weights_to_gpu([sh], pack=pack) if shared else None)
    return experts, sh, xq, routing, gpu


@pytest.mark.parametrize("mode", [B.MOE_FFN_ACCUMULATE, B.MOE_FFN_PER_ASSIGN])
@pytest.mark.parametrize("d,E,k,I,T,shared", [
    (256, 8, 2, 128, 16, False),      # tiny layer
    (256, 8, 2, 128, 16, True),
    (128, 16, 3, 64, 1, True),        # single token
    (512, 32, 4, 96, 37, True),       # ragged: experts with 0..many tokens, I not /32
    (64, 64, 8, 32, 200, False),      # many tokens per expert (> token chunk)
    (2048, 16, 2, 512, 5, True),      # decode-like widths
    (48, 8, 2, 32, 9, True),          # d not a multiple of 32
])
def test_ffn_cuda_core_path_matches_oracle(mode, d, E, k, I, T, shared):
    experts, sh, xq, routing, gpu = _tiny_case(11, d, E, k, I, T, shared)
    o_g, os_g, y_g = _run_ffn(xq, routing, gpu, k, mode, B.MOE_PATH_CUDA_CORE, T, d)
    o_r, os_r, y_r = _oracle_outputs(xq, routing, experts, sh, T, d, k)
    idx, w, offsets, sa, pos = routing
    if mode == B.MOE_FFN_PER_ASSIGN:
        assert_close_layer(o_g, o_r[sa], "per-assignment o")
        if sh is not None:
            assert_close_layer(os_g, os_r, "shared o")
    else:
        assert_close_layer(o_g, y_r, "y_acc")
    assert_close_layer(bits_to_f32(y_g), y_r, "y bf16")


@pytest.mark.parametrize("mode", [B.MOE_FFN_ACCUMULATE, B.MOE_FFN_PER_ASSIGN])
@pytest.mark.parametrize("d,E,k,I,T,shared,zipf", [
    (256, 8, 2, 256, 16, False, 0.0),     # one k-stage per GEMM
    (512, 16, 4, 256, 1, True, 0.0),      # single token
    (512, 16, 4, 512, 37, True, 1.0),     # ragged, Zipf: experts with 0..many tokens
    (256, 4, 2, 256, 700, True, 0.0),     # several 128-row m-tiles per expert
    (2048, 32, 4, 512, 300, True, 0.8),   # decode/prefill widths
    (1024, 8, 1, 768, 129, False, 0.0),   # k=1, m-tile boundary +1, 3 k-stages of h
])
def test_ffn_tensor_core_path_matches_oracle(mode, d, E, k, I, T, shared, zipf):
    experts, sh, xq, routing, gpu = _tiny_case(12, d, E, k, I, T, shared, zipf=zipf, pack=True)
    o_g, os_g, y_g = _run_ffn(xq, routing, gpu, k, mode, B.MOE_PATH_PREFILL, T, d)
    o_r, os_r, y_r = _oracle_outputs(xq, routing, experts, sh, T, d, k)
    idx, w, offsets, sa, pos = routing
    if mode == B.MOE_FFN_PER_ASSIGN:
        assert_close_layer(o_g, o_r[sa], "per-assignment o")
        if sh is not None:
            assert_close_layer(os_g, os_r, "shared o")
    else:
        assert_close_layer(o_g, y_r, "y_acc")
    assert_close_layer(bits_to_f32(y_g), y_r, "y bf16")


@pytest.mark.parametrize("d,E,k,I,T,shared,zipf", [
    (512, 8, 2, 64, 1, False, 0.0),       # one token, one unit per expert, one down stage
    (512, 16, 4, 128, 3, True, 0.0),      # odd T, shared expert
    (1024, 32, 4, 192, 8, True, 1.0),     # full 8 tokens, Zipf: several tokens per expert
    (2048, 64, 8, 512, 5, True, 0.0),     # decode widths, T not a power of two
    (512, 4, 4, 256, 8, False, 0.0),      # every token uses every expert
    (4096, 8, 2, 64, 2, True, 0.0),       # wide d: 16 gate/up stages, 8 down stages
])
def test_ffn_decode_path_matches_oracle(d, E, k, I, T, shared, zipf):
    experts, sh, xq, routing, gpu = _tiny_case(13, d, E, k, I, T, shared, zipf=zipf, pack=True)
    o_g, _, y_g = _run_ffn(xq, routing, gpu, k, B.MOE_FFN_ACCUMULATE, B.MOE_PATH_DECODE, T, d)
    _, _, y_r = _oracle_outputs(xq, routing, experts, sh, T, d, k)
    assert_close_layer(o_g, y_r, "y_acc")
    assert_close_layer(bits_to_f32(y_g), y_r, "y bf16")


def test_ffn_decode_path_repeated_calls_and_unsupported():
    """The decode path leaves its workspace ready for the next call (same result twice), and
    rejects what it does not cover instead of falling back."""
    experts, sh, xq, routing, gpu = _tiny_case(14, 512, 16, 4, 128, 6, True, pack=True)
    _, _, y1 = _run_ffn(xq, routing, gpu, 4, B.MOE_FFN_ACCUMULATE, B.MOE_PATH_DECODE, 6, 512)
    _, _, y2 = _run_ffn(xq, routing, gpu, 4, B.MOE_FFN_ACCUMULATE, B.MOE_PATH_DECODE, 6, 512)
    assert np.allclose(bits_to_f32(y1), bits_to_f32(y2), rtol=1e-2, atol=1e-3)
    with pytest.raises(B.MoeError):
        _run_ffn(xq, routing, gpu, 4, B.MOE_FFN_PER_ASSIGN, B.MOE_PATH_DECODE, 6, 512)


@pytest.fixture(scope="module")
def decode_layer():
    cfg = synth.CONFIGS["decode"]
    routed = L.quantize_weights_gpu(0, cfg)
    shared = L.quantize_weights_gpu(0, cfg, shared=True)
    return cfg, B.Experts(routed, shared), OracleWeights(0, cfg)


@pytest.mark.parametrize("path", [B.MOE_PATH_DECODE, B.MOE_PATH_PREFILL, B.MOE_PATH_CUDA_CORE])
@pytest.mark.parametrize("T", [1, 4, 8])
def test_ffn_decode_config_full_size(decode_layer, T, path):
    cfg, gpu, ow = decode_layer
    x = synth.make_x(0, cfg, T).numpy()
    Wr, br = synth.make_router(0, cfg)
    xf = bits_to_f32(x)
    xq = onv.quantize(xf)
    routing = _oracle_route(xf, Wr.numpy(), br.numpy(), cfg.k, cfg.E)
    _, _, y_g = _run_ffn(xq, routing, gpu, cfg.k, B.MOE_FFN_ACCUMULATE, path, T, cfg.d)
    _, _, y_r = _oracle_outputs(xq, routing, ow, ow.shared, T, cfg.d, cfg.k)
    assert_close_layer(bits_to_f32(y_g), y_r, f"decode T={T}")
    # the GPU-quantised weights of the touched experts equal the oracle's
    for e in np.unique(routing[0])[:4]:
        assert np.array_equal(gpu.routed.gu_codes[int(e)].cpu().numpy(), ow[int(e)].gu_codes)
        assert np.array_equal(gpu.routed.dn_scales[int(e)].cpu().numpy(), ow[int(e)].dn_scales)


def test_combine_rms_renorm():
    T, d, k = 7, 64, 3
    rng = np.random.default_rng(5)
    y_acc = rng.standard_normal((T, d)).astype(np.float32)
    y_acc[3] = 0
    y = torch.empty(T, d, dtype=torch.int16, device="cuda")
    B.moe_combine(T, d, k, B.MOE_FFN_ACCUMULATE, torch.from_numpy(y_acc).cuda(), None, None, None,
                  True, y)
    torch.cuda.synchronize()
    ref = omoe.rms_renorm(y_acc)
    assert_close_layer(bits_to_f32(y.cpu().numpy()), ref, "rms renorm")
    assert not bits_to_f32(y.cpu().numpy())[3].any()


@pytest.mark.parametrize("cfg_name,n_sample", [("prefill", 8), ("wide", 3)])
def test_ffn_prefill_configs_sampled(cfg_name, n_sample):
    """Full-size prefill FFN on the tensor-core path; the oracle checks sampled tokens."""
    cfg = synth.CONFIGS[cfg_name]
    T = cfg.T_list[0]
    routed = L.quantize_weights_gpu(0, cfg)
    shared = L.quantize_weights_gpu(0, cfg, shared=True)
    gpu = B.Experts(routed, shared)
    ow = OracleWeights(0, cfg)
    x = synth.make_x(0, cfg, T).numpy()
    Wr, br = synth.make_router(0, cfg)
    xf = bits_to_f32(x)
    xq = onv.quantize(xf)
    routing = _oracle_route(xf, Wr.numpy(), br.numpy(), cfg.k, cfg.E)
    _, _, y_g = _run_ffn(xq, routing, gpu, cfg.k, B.MOE_FFN_ACCUMULATE, B.MOE_PATH_PREFILL, T, cfg.d)
    rng = np.random.default_rng(1)
    tokens = np.sort(rng.choice(T, n_sample, replace=False))
    _, _, y_r = _oracle_outputs(xq, routing, ow, ow.shared, T, cfg.d, cfg.k, tokens=tokens)
    assert_close_layer(bits_to_f32(y_g)[tokens], y_r, f"{cfg_name} sampled")
    # every output row is finite and not all zero
    yf = bits_to_f32(y_g)
    assert np.isfinite(yf).all() and (np.abs(yf).sum(1) > 0).all()


def _swizzle_rows(tile, piece_of):
    """Place 16-byte piece c of row r of a byte tile [rows][16 * n] at piece piece_of(r, c)."""
    rows, n = tile.shape[0], tile.shape[1] // 16
    t = tile.reshape(rows, n, 16)
    out = np.empty_like(t)
    r = np.arange(rows)[:, None]
    c = np.arange(n)[None, :]
    out[r, piece_of(r, c)] = t
    return out.reshape(-1)


def _scale_atom(rows4):
    """[128 rows][4 scale bytes] -> the 512-byte atom: row 32*r1 + r0, block b at r0*16 + r1*4 + b."""
    return rows4.reshape(4, 32, 4).transpose(1, 0, 2).reshape(512)


def test_pack_dec_layout():
    """The decode pack of moe_pack_experts holds, per unit (e, slice j) and 18432-byte block,
    exactly the bytes its header describes, rebuilt here from the natural layout: swizzled
    gate/up and down tiles and the scale atoms (integer, bit-exact)."""
    experts, sh, xq, routing, gpu = _tiny_case(15, 512, 4, 2, 192, 3, True, pack=True)
    for w in (gpu.routed, gpu.shared):
        E, d, I = w.E, w.d, w.I
        guc, gus = w.gu_codes.cpu().numpy(), w.gu_scales.cpu().numpy()
        dnc, dns = w.dn_codes.cpu().numpy(), w.dn_scales.cpu().numpy()
        blocks = []
        for e in range(E):
            for j in range(I // 64):
                rows = np.r_[64 * j:64 * j + 64, I + 64 * j:I + 64 * j + 64]
                for kb in range(d // 256):
                    tile = guc[e, rows, 128 * kb:128 * kb + 128]
                    blocks.append(_swizzle_rows(tile, lambda r, c: c ^ (r % 8)))
                    for a in range(4):
                        kc = 4 * kb + a
                        blocks.append(_scale_atom(gus[e, rows, 4 * kc:4 * kc + 4]))
                for q in range(d // 512):
                    for c in range(4 * q, 4 * q + 4):
                        tile = dnc[e, 128 * c:128 * c + 128, 32 * j:32 * j + 32]
                        blocks.append(_swizzle_rows(tile, lambda r, cc: cc ^ ((r // 4) % 2)))
                    for c in range(4 * q, 4 * q + 4):
                        blocks.append(_scale_atom(dns[e, 128 * c:128 * c + 128, 4 * j:4 * j + 4]))
        want = np.concatenate(blocks)
        got = w.dec_pack.cpu().numpy()
        assert got.size == B.dec_pack_bytes(E, d, I) == want.size
        assert np.array_equal(got, want)
