"""Oracle-side expert weights of a synthetic layer (test infrastructure, like the rest of
this package).

The weights come from the seeded generator (bf16 draws, the precision a checkpoint holds)
and are quantised to NVFP4 by this package's own quantiser, one tensor scale per matrix
(gate, up, down), on first use: only the experts a check touches are ever built.
"""
from __future__ import annotations

import numpy as np

from nvfp4_expert_ffn_b200 import synth

from . import moe


def _bf16_to_f32(bits) -> np.ndarray:
    b = np.asarray(bits)
    return (b.astype(np.uint16).astype(np.uint32) << 16).view(np.float32)


def expert_from_bf16(g, u, dn) -> moe.Expert:
    """An oracle Expert from bf16 bit patterns (torch or numpy) of gate, up and down."""
    as_np = lambda t: t.cpu().numpy() if hasattr(t, "cpu") else np.asarray(t)  # noqa: E731
    return moe.Expert.from_f32(_bf16_to_f32(as_np(g)), _bf16_to_f32(as_np(u)), _bf16_to_f32(as_np(dn)))


def synth_expert(seed: int, cfg, e: int, layer: int = 0, shared: bool = False) -> moe.Expert:
    """Expert e (or the shared expert) of layer `layer` of a synthetic configuration."""
    return expert_from_bf16(*synth.make_expert_weights_bf16(seed, cfg, e, layer, shared=shared))


class OracleWeights:
    """Lazily quantised oracle experts of a synth layer (only the experts a check touches)."""

    def __init__(self, seed, cfg, layer=0):
        self.seed, self.cfg, self.layer = seed, cfg, layer
        self._cache = {}
        self._shared = None

    def __getitem__(self, e) -> moe.Expert:
        if e not in self._cache:
            self._cache[e] = synth_expert(self.seed, self.cfg, e, self.layer)
        return self._cache[e]

    @property
    def shared(self) -> moe.Expert:
        if self._shared is None:
            self._shared = synth_expert(self.seed, self.cfg, 0, self.layer, shared=True)
        return self._shared

    def __len__(self):
        return self.cfg.E
