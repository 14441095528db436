"""Benchmark: NVFP4 MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--T 8] [--impl ours|reference]

One step = one full MoE layer forward (quantise x, route, expert FFN, combine, expert
histogram) of the decode layer d=2048, 512 experts, top-10 + 1 shared expert, I=512, on T
tokens (default 8). Each timed step runs on one of several distinct layer copies in turn
(several GB in total, far above the 126 MB L2), so every step streams its experts' weights
from HBM. Steps are replayed from CUDA graphs; timing uses CUDA events on the launching
stream, max over ranks. Prints one JSON line on rank 0.

--impl reference times the CPU oracle (oracle/, float64 numpy) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode T=1–8, prefill T=16K); % of HBM BW / FP4 MMA peak"
SEED = 0
N_LAYER_COPIES = 4  # overridden by --layers


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every few ms (reads only)."""

    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, windows):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        inside = [s for s in self.samples if any(a <= s[0] <= b for a, b in windows)]
        use = inside if inside else self.samples
        reasons = set()
        for _, _, rs in use:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in use]) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(use), "in_timed_region": bool(inside)}


# ---------------------------------------------------------------------------- GPU arm
def build_layers(T: int, device, n_layers: int, workload: str = "decode"):
    from nvfp4_expert_ffn_b200 import binding as B
    from nvfp4_expert_ffn_b200 import layer as L
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS[workload]
    layers = []
    for li in range(n_layers):
        routed = L.quantize_weights_gpu(SEED, cfg, layer=li, device=device)
        shared = L.quantize_weights_gpu(SEED, cfg, layer=li, shared=True, device=device)
        Wr, br = synth.make_router(SEED, cfg, layer=li)
        lay = L.MoeLayer(B.Experts(routed, shared), Wr.to(device), br.to(device), cfg.k, T,
                         device=device)
        lay.x_static = synth.make_x(SEED, cfg, T, layer=li).to(device)
        layers.append(lay)
    return cfg, layers


def layer_bytes(cfg, lay, T):
    """Algorithmic HBM bytes of one layer forward and of its FFN call."""
    U = int((lay.counts > 0).sum().item())
    per_expert = 3 * cfg.d * cfg.I * 0.5625
    ffn = (U + 1) * per_expert + T * cfg.d * (0.5625 + 4)          # weights + xq + y_acc
    total = ffn + cfg.E * cfg.d * 4 + cfg.E * 4 + T * cfg.d * 2 * 2  # + router + x + y
    return U, ffn, total


def run_gpu(args):
    from nvfp4_expert_ffn_b200 import binding as B
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    global N_LAYER_COPIES
    N_LAYER_COPIES = args.layers
    from nvfp4_expert_ffn_b200 import synth
    T = args.T if args.T else synth.CONFIGS[args.workload].T_list[-1]
    K, W = args.steps, args.warmup
    cfg, layers = build_layers(T, device, N_LAYER_COPIES, args.workload)
    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(local)
    sampler.start()

    # warm-up eagerly (first calls set kernel attributes), then capture one graph that runs
    # every layer copy once (N_LAYER_COPIES steps) and one with only their FFN calls
    with torch.cuda.stream(stream):
        for lay in layers:
            lay.forward(lay.x_static)
    torch.cuda.synchronize()
    bytes_info = [layer_bytes(cfg, lay, T) for lay in layers]
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        for lay in layers:
            lay.forward(lay.x_static)
    g_ffn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ffn, stream=stream):
        for lay in layers:
            B.moe_expert_ffn(lay.xq_codes[:T], lay.xq_scales[:T], lay.xq_ts[:1], lay.experts,
                             lay.k, lay.offsets, lay.sorted_assign[:T * lay.k], lay.topk_w[:T],
                             B.MOE_FFN_ACCUMULATE, lay.path, lay.y_acc[:T], None, lay.ws)
    reps = max(1, (K + N_LAYER_COPIES - 1) // N_LAYER_COPIES)
    K = reps * N_LAYER_COPIES
    wreps = max(1, (W + N_LAYER_COPIES - 1) // N_LAYER_COPIES)
    W = wreps * N_LAYER_COPIES

    def timed(graph, n):
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0h = time.time()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        t1h = time.time()
        ms = e0.elapsed_time(e1)
        if dist is not None:
            t = torch.tensor([ms], device=device)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms, (t0h, t1h)

    with torch.cuda.stream(stream):
        for _ in range(wreps):
            g_step.replay()
            g_ffn.replay()
    torch.cuda.synchronize()
    if args.eager:
        # profiling aid: the same steps launched directly (no graph), inside an NVTX range
        with torch.cuda.stream(stream):
            torch.cuda.nvtx.range_push("timed")
            for i in range(K):
                layers[i % N_LAYER_COPIES].forward(layers[i % N_LAYER_COPIES].x_static)
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed_graph")
    ms_total, win1 = timed(g_step, reps)
    ms_ffn, win2 = timed(g_ffn, reps)
    torch.cuda.nvtx.range_pop()

    # end to end through the public API: pinned host x -> device, forward, y -> pinned host
    xs_host = [lay.x_static.cpu().pin_memory() for lay in layers]
    y_host = torch.empty(T, cfg.d, dtype=torch.int16).pin_memory()
    x_dev = [torch.empty_like(lay.x_static) for lay in layers]
    e2e_steps = 0 if args.no_e2e else min(K, 2000)
    with torch.cuda.stream(stream):
        for i in range(min(W, 8)):
            li = i % N_LAYER_COPIES
            x_dev[li].copy_(xs_host[li], non_blocking=True)
            y_host.copy_(layers[li].forward(x_dev[li]), non_blocking=True)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0h = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            li = i % N_LAYER_COPIES
            x_dev[li].copy_(xs_host[li], non_blocking=True)
            y_host.copy_(layers[li].forward(x_dev[li]), non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    win3 = (t0h, time.time())
    ms_e2e = e0.elapsed_time(e1)
    if dist is not None:
        t = torch.tensor([ms_e2e], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_e2e = float(t.item())
    sampler.stop()

    ms_step = ms_total / K
    tokens_per_s = world * T * K / (ms_total / 1e3)
    e2e_tps = world * T * e2e_steps / (ms_e2e / 1e3) if e2e_steps else None
    hbm_peak, bf16_peak, peak_kind = _peaks()
    U_avg = float(np.mean([b[0] for b in bytes_info]))
    ffn_bytes = float(np.mean([b[1] for b in bytes_info]))
    ffn_ms = ms_ffn / K
    achieved = ffn_bytes / (ffn_ms * 1e-3) / 1e9
    ffn_flops = 2.0 * T * (cfg.k + 1) * 3 * cfg.d * cfg.I
    if args.workload == "decode":
        roof = {"kernel": "moe_expert_ffn (schedule + gather + tcgen05 FFN)", "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "peak_kind": peak_kind,
                "bytes_per_launch": int(ffn_bytes), "avg_launch_us": round(ffn_ms * 1e3, 3),
                "traffic": None}
    else:
        fp4_peak = bf16_peak * 4.0  # dense FP4 = 4 x dense bf16 (nominal ratio 9 / 2.25)
        tf = ffn_flops / (ffn_ms * 1e-3) / 1e12
        roof = {"kernel": "moe_expert_ffn (schedule + gather + tcgen05 FFN)", "bound": "tensor",
                "achieved": round(tf, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                "frac": round(tf / fp4_peak, 4),
                "peak_kind": f"{peak_kind} bf16 x 4 (nominal fp4/bf16 ratio)",
                "flops_per_launch": ffn_flops, "bytes_per_launch": int(ffn_bytes),
                "avg_launch_us": round(ffn_ms * 1e3, 3), "traffic": None}
    launches_per_step = 1 + 3 + 2 + 1 + 1  # quant, route(gemv,topk,perm), ffn(2), combine, hist
    out = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp32", "data": "synthetic",
        "config": {"workload": f"{args.workload} MoE layer: d={cfg.d}, {cfg.E} experts, "
                               f"top-{cfg.k} + {int(cfg.shared)} shared, I={cfg.I}, NVFP4 weights, "
                               f"T={T} tokens per step",
                   "T": T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                   "zipf_s": cfg.zipf_s, "parallelism": f"replicas x{world}",
                   "l2": f"{N_LAYER_COPIES} distinct layer copies "
                         f"({N_LAYER_COPIES * cfg.E * 3 * cfg.d * cfg.I * 0.5625 / 1e9:.1f} GB) "
                         f"rotated every step: inputs > L2",
                   "touched_experts_avg": U_avg},
        "roofline": roof,
        "e2e": {"value": None if e2e_tps is None else round(e2e_tps, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * 2,
                "steps": e2e_steps},
        "gpu_launches": launches_per_step * K,
        "clocks": sampler.summary([win1, win2, win3]),
    }
    if rank == 0 and not args.no_cpu_baseline and args.workload == "decode":
        out["cpu_baseline"] = cpu_baseline(T, args.cpu_steps)
    if dist is not None:
        del g_step, g_ffn
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


# ---------------------------------------------------------------------------- CPU oracle
def cpu_baseline(T: int, steps: int):
    """Time the float64 CPU oracle on `steps` decode layer forwards of T tokens (weights of
    the touched experts quantised before timing, like a resident model)."""
    from oracle import moe as omoe
    from nvfp4_expert_ffn_b200 import synth
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import OracleWeights
    cfg = synth.CONFIGS["decode"]
    ow = OracleWeights(SEED, cfg)
    Wr, br = synth.make_router(SEED, cfg)
    Wr, br = Wr.numpy(), br.numpy()
    xs = [synth.make_x(SEED, cfg, T, step=100 + s).numpy() for s in range(steps)]
    from oracle import nvfp4 as onv
    for x in xs:  # materialise the touched experts (model load, not timed)
        xf = (x.astype(np.uint16).astype(np.uint32) << 16).view(np.float32)
        idx = omoe.topk_fast(omoe.router_logits(xf, Wr, br), cfg.k)
        for e in np.unique(idx):
            ow[int(e)]
        ow.shared
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    t0 = time.perf_counter()
    for x in xs:
        omoe.layer_forward(x, Wr, br, cfg.k, ow, ow.shared)
    dt = time.perf_counter() - t0
    return {"value": round(T * steps / dt, 3), "unit": "tokens/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{steps} decode layer forwards of T={T} tokens (full layer, float64 numpy)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    T = args.T or 8
    K = max(1, min(args.steps, args.cpu_steps))
    W = max(0, min(args.warmup, 1))
    cb = cpu_baseline(T, K + W)
    out = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
           "n_gpus": 1, "steps": K, "warmup": W, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"decode MoE layer: d=2048, 512 experts, top-10 + 1 shared, "
                                  f"I=512, NVFP4 weights, T={T} tokens per step", "T": T},
           "cpu_baseline": cb,
           "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=40)
    ap.add_argument("--T", type=int, default=0, help="tokens per step (default: the workload's)")
    ap.add_argument("--workload", choices=["decode", "prefill", "wide"], default="decode")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-steps", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=4, help="distinct layer copies rotated")
    ap.add_argument("--eager", action="store_true",
                    help="also run K eager steps in an NVTX range 'timed' (for ncu)")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
