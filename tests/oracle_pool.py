"""The oracle's expert FFN for many experts at once, spread over host processes.

At the full-size prefill workloads the oracle builds hundreds of experts (each: seeded bf16
weights, NVFP4 quantisation, then the float64 SwiGLU FFN of the rows routed to it), which
takes minutes in one process. Each task here is one expert: the worker draws and quantises
that expert's weights itself and returns oracle.moe.expert_ffn of the rows it is given, the
same calls oracle.moe.layer_forward makes per expert. The pool is started with `spawn`, so
it is safe to create after CUDA has been initialised in the parent.
"""
from __future__ import annotations

import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np


def _init_worker():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    import torch
    torch.set_num_threads(1)


def _expert_rows(cfg_name, seed, layer, e, shared, x_hat_rows):
    from nvfp4_expert_ffn_b200 import synth
    from oracle import moe as omoe
    from oracle.weights import synth_expert
    ex = synth_expert(seed, synth.CONFIGS[cfg_name], e, layer, shared=shared)
    return e, shared, omoe.expert_ffn(x_hat_rows, ex)


def _expert_rows_static(cfg_name, seed, layer, e, shared, x_rows, in_gu, in_dn):
    from nvfp4_expert_ffn_b200 import synth
    from oracle import moe as omoe
    from oracle.weights import synth_expert
    ex = synth_expert(seed, synth.CONFIGS[cfg_name], e, layer, shared=shared)
    return e, shared, omoe.expert_ffn_static(x_rows, ex, in_gu, in_dn)


class OraclePool:
    """A pool of host processes kept across many expert_outputs calls (use as a context
    manager)."""

    def __init__(self, workers=None):
        self.workers = workers or min(32, os.cpu_count() or 1)
        self.ex = cf.ProcessPoolExecutor(max_workers=self.workers, mp_context=mp.get_context("spawn"),
                                         initializer=_init_worker)

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.ex.shutdown()

    def expert_outputs(self, cfg_name, seed, layer, tasks):
        """tasks: list of (expert id, shared flag, x_hat rows float64 [n][d]). Returns a dict
        (expert id, shared) -> o rows float64 [n][d], in the order of the given rows."""
        futs = [self.ex.submit(_expert_rows, cfg_name, seed, layer, e, sh, np.ascontiguousarray(rows))
                for e, sh, rows in tasks]
        out = {}
        for f in cf.as_completed(futs):
            e, sh, o = f.result()
            out[(e, sh)] = o
        return out


    def expert_outputs_static(self, cfg_name, seed, layer, tasks):
        """As expert_outputs with static input scales: tasks are (expert id, shared flag,
        x rows float32 [n][d], in_gu, in_dn) and the rows are the unquantised activations."""
        futs = [self.ex.submit(_expert_rows_static, cfg_name, seed, layer, e, sh, np.ascontiguousarray(rows),
                               gu, dn)
                for e, sh, rows, gu, dn in tasks]
        out = {}
        for f in cf.as_completed(futs):
            e, sh, o = f.result()
            out[(e, sh)] = o
        return out


def expert_outputs(cfg_name, seed, layer, tasks, workers=None):
    """One-off OraclePool.expert_outputs."""
    with OraclePool(workers) as pool:
        return pool.expert_outputs(cfg_name, seed, layer, tasks)
