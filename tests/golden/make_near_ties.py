"""Writes near_ties.json beside this file: for each routing input the GPU tests compare with
the oracle, the tokens whose k-th and (k+1)-th largest float32 oracle logits differ by less
than 1e-6. For those tokens either top-k set is correct within the float32 rounding of the
logits, so the tests excuse them (and only them) when the GPU's set differs; this file keeps
the count for each input on record.

    python tests/golden/make_near_ties.py

Uses only the oracle (router logits) and the seeded input generator; nothing here comes from
the CUDA path.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from nvfp4_expert_ffn_b200 import synth  # noqa: E402
from oracle import moe as omoe  # noqa: E402

TIE_MARGIN = 1e-6
# (configuration, tokens, x draw): the inputs of the routing, layer and full-size tests
CASES = [("tiny", 16, 0), ("decode", 1, 0), ("decode", 4, 0), ("decode", 8, 0), ("decode", 9, 0),
         ("decode", 100, 0), ("decode", 1, 3), ("decode", 4, 3), ("decode", 8, 3),
         ("prefill", 16384, 0), ("wide", 27140, 0)]


def near_ties(cfg_name: str, T: int, step: int, seed: int = 0):
    cfg = synth.CONFIGS[cfg_name]
    x = synth.make_x(seed, cfg, T, step=step)
    Wr, br = synth.make_router(seed, cfg)
    xf = synth.bf16_bits_to_f32(x).numpy()
    logits = omoe.router_logits(xf, Wr.numpy(), br.numpy() if cfg.zipf_s > 0 else None)
    s = -np.sort(-logits.astype(np.float64), axis=1)
    margin = s[:, cfg.k - 1] - s[:, cfg.k] if cfg.E > cfg.k else np.full(T, np.inf)
    tokens = np.flatnonzero(margin < TIE_MARGIN)
    return {"config": cfg_name, "T": T, "step": step, "seed": seed, "k": cfg.k, "E": cfg.E,
            "tie_margin": TIE_MARGIN, "count": int(tokens.size), "tokens": tokens.tolist(),
            "min_margin": float(margin.min())}


def main():
    out = [near_ties(*c) for c in CASES]
    with open(os.path.join(HERE, "near_ties.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    for r in out:
        print(r["config"], r["T"], r["step"], "near-tie tokens:", r["count"], "min margin %.3g" % r["min_margin"])


if __name__ == "__main__":
    main()
