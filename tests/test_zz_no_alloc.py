"""moe_route_noalloc: routing for callers that cannot give the library scratch memory.

Some callers cannot allocate device memory at all - a server that reserved every byte of
HBM at start-up, a C host with no device allocator, or code capturing a CUDA graph, where
cudaMalloc may not be called. For them the library keeps the router's scratch in a fixed
256 KiB array of its own. This test calls that entry point through the C ABI twice in a
row, on different inputs (so the second call finds the first call's leftovers in the
array), and checks each result against moe_route with a caller-provided workspace: the
same kernels run on the same inputs, so every output must match exactly.

The file is named so that pytest collects it last; it also passes when run on its own.
"""
import numpy as np
import pytest
import torch

from nvfp4_expert_ffn_b200 import binding as B
from nvfp4_expert_ffn_b200 import synth

pytestmark = pytest.mark.gpu

NAMES = ("topk_idx", "topk_w", "counts", "offsets", "sorted_assign", "assign_pos")


def _outputs(T, k, E):
    return dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device="cuda"),
                topk_w=torch.empty(T, k, dtype=torch.float32, device="cuda"),
                counts=torch.empty(E, dtype=torch.int32, device="cuda"),
                offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                sorted_assign=torch.empty(T * k, dtype=torch.int32, device="cuda"),
                assign_pos=torch.empty(T * k, dtype=torch.int32, device="cuda"))


def _with_workspace(x, Wr, br, k):
    T, d = x.shape
    E = Wr.shape[0]
    o = _outputs(T, k, E)
    ws = torch.empty(B.moe_workspace_size(B.MOE_OP_ROUTE, T, d, E, k, 16), dtype=torch.uint8,
                     device="cuda")
    B.moe_route(x, Wr, br, k, *(o[n] for n in NAMES), ws)
    return o


def _no_alloc(x, Wr, br, k):
    T, d = x.shape
    o = _outputs(T, k, Wr.shape[0])
    B.moe_route_noalloc(x, Wr, br, k, *(o[n] for n in NAMES))
    return o


def test_noalloc_route_matches_workspace_route_twice():
    cfg = synth.CONFIGS["decode"]
    Wr, br = synth.make_router(0, cfg)
    Wr, br = Wr.cuda(), br.cuda()
    cases = [synth.make_x(0, cfg, 8, step=1).cuda(),   # first call: 8 decode tokens
             synth.make_x(0, cfg, 64, step=2).cuda()]  # second call: 64 tokens (GEMM router)
    for x in cases:
        want = _with_workspace(x, Wr, br, cfg.k)
        got = _no_alloc(x, Wr, br, cfg.k)
        torch.cuda.synchronize()
        for n in NAMES:
            a, b = got[n].cpu().numpy(), want[n].cpu().numpy()
            if n == "topk_w":
                np.testing.assert_allclose(a, b, rtol=2e-6, atol=1e-7)
            else:
                assert np.array_equal(a, b), n


def test_noalloc_rejects_sizes_above_its_array():
    cfg = synth.CONFIGS["decode"]
    Wr, br = synth.make_router(0, cfg)
    x = synth.make_x(0, cfg, 1024).cuda()  # 1024 tokens x 512 experts of logits > 256 KiB
    o = _outputs(1024, cfg.k, cfg.E)
    with pytest.raises(B.MoeError) as err:
        B.moe_route_noalloc(x, Wr.cuda(), br.cuda(), cfg.k, *(o[n] for n in NAMES))
    assert err.value.status == 2 and "scratch" in str(err.value)


def test_noalloc_boundary_of_its_array():
    """128 tokens x 512 experts of float32 logits fill the 256 KiB array exactly (1280
    assignments need no permutation scratch): accepted and equal to moe_route. One more
    token needs more than the array holds and is rejected before anything is launched."""
    cfg = synth.CONFIGS["decode"]
    Wr, br = synth.make_router(0, cfg)
    Wr, br = Wr.cuda(), br.cuda()
    x = synth.make_x(0, cfg, 128, step=4).cuda()
    want = _with_workspace(x, Wr, br, cfg.k)
    got = _no_alloc(x, Wr, br, cfg.k)
    torch.cuda.synchronize()
    for n in NAMES:
        a, b = got[n].cpu().numpy(), want[n].cpu().numpy()
        if n == "topk_w":
            np.testing.assert_allclose(a, b, rtol=2e-6, atol=1e-7)
        else:
            assert np.array_equal(a, b), n
    x = synth.make_x(0, cfg, 129, step=5).cuda()
    o = _outputs(129, cfg.k, cfg.E)
    with pytest.raises(B.MoeError) as err:
        B.moe_route_noalloc(x, Wr, br, cfg.k, *(o[n] for n in NAMES))
    assert err.value.status == 2 and "scratch" in str(err.value)
