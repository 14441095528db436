"""nvfp4_quantize_act on the GPU vs the oracle quantiser: bit-exact codes, scales, ts."""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as onv
from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import synth

from helpers import bits_to_f32

pytestmark = pytest.mark.gpu


def _run(xbits: torch.Tensor, ts=None):
    rows, cols = xbits.shape
    x = xbits.cuda()
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device="cuda")
    ts_out = torch.empty(4, dtype=torch.float32, device="cuda")
    ws = torch.empty(B.moe_workspace_size(B.MOE_OP_QUANT, 1, 16, 1, 1, 16), dtype=torch.uint8,
                     device="cuda")
    ts_in = None if ts is None else torch.tensor([ts, 0, 0, 0], dtype=torch.float32, device="cuda")
    B.nvfp4_quantize_act(x, codes, scales, ts_out[:1], ts_in=None if ts_in is None else ts_in[:1],
                         ws=ws)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), np.float32(ts_out[0].item())


def _check(xbits, ts=None):
    c, s, t = _run(xbits, ts)
    rc, rs, rt = onv.quantize(bits_to_f32(xbits.numpy()), ts=None if ts is None else np.float32(ts))
    assert t == rt
    assert np.array_equal(s, rs), f"scale mismatch at {np.argwhere(s != rs)[:5]}"
    assert np.array_equal(c, rc), f"code mismatch at {np.argwhere(c != rc)[:5]}"


@pytest.mark.parametrize("cfg,T", [("tiny", 16), ("decode", 1), ("decode", 8), ("prefill", 16384),
                                   ("wide", 27140)])
def test_activation_quant_bit_exact(cfg, T):
    c = synth.CONFIGS[cfg]
    _check(synth.make_x(0, c, T))


@pytest.mark.parametrize("ts", [None, 1.0, 0.001, 0.37])
def test_adversarial_grid(ts):
    # E2M1 midpoints, E4M3 boundaries, zeros, -0, tiny and saturating values, all as bf16
    base = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 0.0, -0.0, 1e-30]
    vals = []
    for p in range(-12, 10):
        for v in base:
            vals += [v * 2.0 ** p, -v * 2.0 ** p]
    rng = np.random.default_rng(0)
    vals += list(rng.standard_normal(4096) * np.exp2(rng.integers(-20, 12, 4096)))
    x = torch.tensor(vals, dtype=torch.float32)
    n = (x.numel() // 256) * 256
    xb = synth.f32_to_bf16_bits(x[:n]).view(-1, 256)
    _check(xb, ts)
    # blocks whose amax sits on E4M3 rounding boundaries
    pos = onv.E4M3_TABLE[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2 * 6.0).astype(np.float32)
    blk = np.zeros((len(mids), 16), np.float32)
    blk[:, 0] = mids
    blk[:, 1:] = mids[:, None] * np.linspace(-1, 1, 15)[None, :]
    _check(synth.f32_to_bf16_bits(torch.from_numpy(blk)), ts if ts else 1.0)


def test_zero_rows_and_zero_tensor():
    c, s, t = _run(torch.zeros(0, 64, dtype=torch.int16))
    assert t == 1.0 and c.size == 0
    _check(torch.zeros(5, 64, dtype=torch.int16))
    _check(torch.zeros(5000, 64, dtype=torch.int16))  # multi-CTA path


def test_weight_matrix_quant_bit_exact():
    cfg = synth.CONFIGS["decode"]
    g, u, dn = synth.make_expert_weights_bf16(0, cfg, 7)
    for w in (g, u, dn):
        _check(w)


def test_deterministic():
    x = synth.make_x(3, synth.CONFIGS["prefill"], 4096)
    a = _run(x)
    b = _run(x)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))
