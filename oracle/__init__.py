"""CPU oracle for the NVFP4 mixture-of-experts layer forward.

TEST INFRASTRUCTURE ONLY. Only the test suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this package. The library's CUDA path never calls it, and it
shares no code with the CUDA sources.

What is computed comes from the Basalt pages:
  * "What Basalt changes in a Blackwell local inference stack", section "Experts can move
    without becoming free": a mixture-of-experts model selects a subset of experts for
    each token.
  * "Basalt" project page, section "Expert tiers": a token uses only a few experts, and the
    busiest (most routed) experts are kept in the fastest tier.
  * "Basalt" project page, "All the numbers" / "Engines: commit, and what is not NVIDIA's
    weights": routed experts are NVIDIA's NVFP4 ("bit-exact", with input_scale in the
    llama.cpp row).
The pages give no formula for NVFP4, the router or the FFN. Where they are silent this
oracle takes the plainest reading, listed in each function's docstring:
  R1 NVFP4 = E2M1 codes, one E4M3 scale per 16 consecutive elements of a row, one float32
     tensor scale per tensor; value = e2m1 * e4m3 * ts.
  R2 dynamic tensor scale ts = amax / (6 * 448); a given (static) scale is used as is.
  R3 all conversions round to nearest, ties to even, and saturate (E4M3 at 448, E2M1 at 6);
     a negative value that rounds to zero keeps its sign (code 0x8); a block whose E4M3
     scale rounds to zero stores scale 0 and sixteen +0 codes.
  R4 router: logits = x Wr^T + b; top-k by logit (ties to the lower expert index); weights
     softmax over all experts, renormalised over the chosen k.
  R5 expert FFN is SwiGLU, silu(gate) * up, with h re-quantised to NVFP4 (tensor scale 1.0)
     before the down projection; a shared expert, if present, is added with weight 1.
  R6 token permutation is a stable counting sort of the (token, slot) assignments by expert.
  R7 cumulative per-expert counts rank experts hot to cold (ties to the lower index).
  R13 static per-expert input scales (the input_scale of NVIDIA's experts): when given, an
     expert's token rows are quantised with its own static tensor scale in_gu[e] and its h
     with in_dn[e], instead of the per-call dynamic scale and 1.0.

Precision: float32 where the reading fixes float32 (quantiser steps, logits, routing
weights, h), float64 elsewhere (dot products, combine).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against closed forms,
library routines (torch float8 casts, numpy sorts, torch float64 matmul), brute force on
tiny inputs, and hand-computed examples under ``tests/golden/``. The pages print no worked
example or tensor, so nothing here is pinned to the pages' own numbers: parity with the
pages' own engine is unpinned.
"""
from . import nvfp4, moe  # noqa: F401
