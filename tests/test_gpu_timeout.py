"""A bounded device-side wait that runs out, and recovery afterwards (the one-kernel decode
layer's grid barrier).

The wait limit is shortened to 5 ms and the workspace's hold word (byte 1536, which the
library never writes) is set, so CTA 0 holds back its barrier arrival and every other CTA
waits for an arrival that never comes: their waits give up, set the device status to
MOE_ERR_TIMEOUT and mark the workspace. Every access stays inside its buffers and every wait
is bounded, so the GPU context stays usable. The next call on the marked workspace does
nothing and reports MOE_ERR_WORKSPACE; after the caller zeroes the workspace the layer gives
its normal result again.
"""
import numpy as np
import pytest
import torch

from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import layer as L
from nvfp4_expert_ffn_b200 import synth

from helpers import bits_to_f32
from test_gpu_layer import barrier_generations

pytestmark = pytest.mark.gpu


def test_decode_layer_wait_runs_out_then_recovers():
    cfg = synth.CONFIGS["decode"]
    routed = L.quantize_weights_gpu(0, cfg)
    shared = L.quantize_weights_gpu(0, cfg, shared=True)
    Wr, br = synth.make_router(0, cfg)
    lay = L.MoeLayer(B.Experts(routed, shared), Wr.cuda(), br.cuda(), cfg.k, 8, fused=True)
    assert lay.fused
    x = synth.make_x(0, cfg, 8, step=9).cuda()
    y0 = lay.forward(x).clone()
    assert B.moe_get_device_status(clear=True) == 0
    hold = lay.ws_dec[1536:1540].view(torch.int32)
    assert None not in barrier_generations(lay.ws_dec)
    B.moe_set_wait_limit_ns(5_000_000)
    try:
        hold.fill_(1)  # CTA 0 does not arrive: the barrier never completes
        lay.forward(x)
        assert B.moe_get_device_status(clear=True) == B.MOE_ERR_TIMEOUT
        # the workspace is marked: the next call computes nothing and says so
        y_marked = lay.y[:8].clone()
        lay.y.fill_(0x7FC0)  # bf16 NaN bits: a call that wrote y would overwrite them
        lay.forward(x)
        assert B.moe_get_device_status(clear=True) == B.MOE_ERR_WORKSPACE
        assert bool((lay.y[:8] == 0x7FC0).all())
        del y_marked
        # recovery: the caller zeroes the workspace
        lay.ws_dec.zero_()
        y = lay.forward(x).clone()
        assert B.moe_get_device_status(clear=True) == 0
        a, b = bits_to_f32(y.cpu().numpy()), bits_to_f32(y0.cpu().numpy())
        assert np.abs(a - b).max() <= 1e-2 * np.sqrt((b ** 2).mean())
        gens = barrier_generations(lay.ws_dec)
        assert gens[0] is not None
    finally:
        B.moe_set_wait_limit_ns(B.DEFAULT_WAIT_LIMIT_NS)


def test_wait_limit_range_is_checked():
    with pytest.raises(B.MoeError):
        B.moe_set_wait_limit_ns(10)
    with pytest.raises(B.MoeError):
        B.moe_set_wait_limit_ns(10 ** 12)
    B.moe_set_wait_limit_ns(B.DEFAULT_WAIT_LIMIT_NS)
