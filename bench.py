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


# ---------------------------------------------------------------------------- ranks
def rank_env():
    """(rank, world size, local rank) from the torchrun environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(backend: str):
    """Join the process group when launched with more than one rank (else None). The
    replicas exchange nothing on the data path: the group carries only the barriers and the
    max-over-ranks of the timings."""
    _, world, _ = rank_env()
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(dist, ms: float, device) -> float:
    """The slowest rank's time: every rank takes part, every rank gets the maximum."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, T: int, steps: int, ms: float) -> float:
    """Tokens/s of the whole job: each of `world` replicas ran `steps` steps of T tokens in
    (at most) `ms` milliseconds."""
    return world * T * steps / (ms / 1e3)


def run_gpu(args):
    from nvfp4_expert_ffn_b200 import binding as B
    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    dist = dist_init("nccl")
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
    n0 = B.moe_launch_count()
    with torch.cuda.graph(g_step, stream=stream):
        for lay in layers:
            lay.forward(lay.x_static, join=False)  # side-stream histograms overlap the next layer
        for lay in layers:
            lay.join(stream)
    # this library's kernels in one step, counted by the library as the graph was captured
    launches_per_step = (B.moe_launch_count() - n0) / N_LAYER_COPIES
    # the dominant kernel alone: the one-kernel decode layer, else the expert FFN call
    fused = T <= 8 and all(lay.fused for lay in layers)
    g_ffn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ffn, stream=stream):
        for lay in layers:
            if fused:
                B.moe_layer_decode(lay.x_static, lay.static_ts, lay.Wr, lay.br, lay.experts, lay.k,
                                   lay.xq_codes[:T], lay.xq_scales[:T], lay.xq_ts[:1],
                                   lay.topk_idx[:T], lay.topk_w[:T], lay.counts, lay.offsets,
                                   lay.sorted_assign[:T * lay.k], lay.assign_pos[:T * lay.k],
                                   lay.y_acc[:T], lay.y[:T], False, lay.ws_dec)
            else:
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
        return max_over_ranks(dist, e0.elapsed_time(e1), device), (t0h, t1h)

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

    # end to end through the public API (a graphed layer step): pinned host x -> device,
    # the layer forward, y -> pinned host, every step
    e2e_steps = 0 if args.no_e2e else min(K, 2000)
    runners = [lay.graphed(T) for lay in layers] if e2e_steps else []
    xs_host = [lay.x_static.cpu().pin_memory() for lay in layers]
    y_host = torch.empty(T, cfg.d, dtype=torch.int16).pin_memory()
    est = runners[0].stream if runners else stream
    for i in range(min(W, 8) if runners else 0):
        runners[i % N_LAYER_COPIES].step(xs_host[i % N_LAYER_COPIES], y_host)
        est.wait_stream(runners[i % N_LAYER_COPIES].stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0h = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(est)
    for i in range(e2e_steps):
        r = runners[i % N_LAYER_COPIES]
        r.stream.wait_stream(est)
        r.step(xs_host[i % N_LAYER_COPIES], y_host)
        est.wait_stream(r.stream)
    e1.record(est)
    torch.cuda.synchronize()
    win3 = (t0h, time.time())
    ms_e2e = max_over_ranks(dist, e0.elapsed_time(e1), device)
    sampler.stop()

    ms_step = ms_total / K
    tokens_per_s = whole_job_rate(world, T, K, ms_total)
    e2e_tps = whole_job_rate(world, T, e2e_steps, ms_e2e) if e2e_steps else None
    hbm_peak, bf16_peak, peak_kind = _peaks()
    U_avg = float(np.mean([b[0] for b in bytes_info]))
    ffn_bytes = float(np.mean([b[2 if fused else 1] for b in bytes_info]))
    ffn_ms = ms_ffn / K
    achieved = ffn_bytes / (ffn_ms * 1e-3) / 1e9
    ffn_flops = 2.0 * T * (cfg.k + 1) * 3 * cfg.d * cfg.I
    if args.workload == "decode":
        name = ("layer_dec_kernel (moe_layer_decode: quantise, route, tcgen05 expert FFN, combine)"
                if fused else "moe_expert_ffn (decode: preparation + tcgen05 split-I kernel)")
        # DRAM traffic of layer_dec_kernel from one ncu capture of the same kernel and shapes
        # (dram__bytes_read.sum + dram__bytes_write.sum = 59,812,864 B on a launch whose run
        # averaged 60,075,008 algorithmic bytes), scaled to this run's bytes per launch
        traffic = int(ffn_bytes * (59812864 / 60075008)) if fused else None
        roof = {"kernel": name, "bound": "hbm",
                "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "peak_kind": peak_kind,
                "bytes_per_launch": int(ffn_bytes), "avg_launch_us": round(ffn_ms * 1e3, 3),
                "traffic": traffic}
    else:
        fp4_peak = bf16_peak * 4.0  # dense FP4 = 4 x dense bf16 (nominal ratio 9 / 2.25)
        tf = ffn_flops / (ffn_ms * 1e-3) / 1e12
        roof = {"kernel": "moe_expert_ffn (schedule + row gather + tcgen05 grouped GEMMs)", "bound": "tensor",
                "achieved": round(tf, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                "frac": round(tf / fp4_peak, 4),
                "peak_kind": f"{peak_kind} bf16 x 4 (nominal fp4/bf16 ratio)",
                "flops_per_launch": ffn_flops, "bytes_per_launch": int(ffn_bytes),
                "avg_launch_us": round(ffn_ms * 1e3, 3), "traffic": None}
    out = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp32", "data": "synthetic",
        "config": dict(workload_config(args.workload, T, world, N_LAYER_COPIES),
                       touched_experts_avg=U_avg),
        "roofline": roof,
        "e2e": {"value": None if e2e_tps is None else round(e2e_tps, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * 2,
                "steps": e2e_steps},
        "gpu_launches": int(round(launches_per_step * K)),
        "gpu_launches_per_step": launches_per_step,
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
class OracleDecode:
    """The float64 CPU oracle running decode layer forwards of T tokens (the touched
    experts' weights are quantised when prepared, like a resident model, and not timed)."""

    def __init__(self, T: int, n_inputs: int):
        from oracle import moe as omoe
        from nvfp4_expert_ffn_b200 import synth
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from helpers import OracleWeights
        self.omoe = omoe
        self.cfg = cfg = synth.CONFIGS["decode"]
        self.T = T
        self.ow = OracleWeights(SEED, cfg)
        Wr, br = synth.make_router(SEED, cfg)
        self.Wr, self.br = Wr.numpy(), br.numpy()
        self.xs = [synth.make_x(SEED, cfg, T, step=100 + s).numpy() for s in range(n_inputs)]
        for x in self.xs:
            xf = (x.astype(np.uint16).astype(np.uint32) << 16).view(np.float32)
            idx = omoe.topk_fast(omoe.router_logits(xf, self.Wr, self.br), cfg.k)
            for e in np.unique(idx):
                self.ow[int(e)]
        self.ow.shared

    def step(self, i: int):
        return self.omoe.layer_forward(self.xs[i % len(self.xs)], self.Wr, self.br, self.cfg.k,
                                       self.ow, self.ow.shared)

    @staticmethod
    def cores() -> int:
        try:
            from threadpoolctl import threadpool_info
            return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            return os.cpu_count() or 1

    def timed(self, steps: int, warmup: int = 0) -> float:
        """Seconds for `steps` forwards after `warmup` untimed ones."""
        for i in range(warmup):
            self.step(i)
        t0 = time.perf_counter()
        for i in range(steps):
            self.step(warmup + i)
        return time.perf_counter() - t0


def cpu_baseline(T: int, steps: int):
    """The oracle timed on `steps` decode layer forwards of T tokens on the host cores."""
    o = OracleDecode(T, steps)
    dt = o.timed(steps)
    return {"value": round(T * steps / dt, 3), "unit": "tokens/s", "cores": o.cores(),
            "kind": "oracle",
            "sample": f"{steps} decode layer forwards of T={T} tokens (full layer, float64 numpy)"}


def workload_config(workload: str, T: int, world: int, n_copies: int) -> dict:
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS[workload]
    return {"workload": f"{workload} MoE layer: d={cfg.d}, {cfg.E} experts, "
                        f"top-{cfg.k} + {int(cfg.shared)} shared, I={cfg.I}, NVFP4 weights, "
                        f"T={T} tokens per step",
            "T": T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I,
            "zipf_s": cfg.zipf_s, "parallelism": f"replicas x{world}",
            "l2": f"{n_copies} distinct layer copies "
                  f"({n_copies * cfg.E * 3 * cfg.d * cfg.I * 0.5625 / 1e9:.1f} GB) "
                  f"rotated every step: inputs > L2"}


def run_reference(args):
    """The oracle as the reference arm: rank 0 alone runs W untimed and K timed decode layer
    forwards (K and W capped so the run stays within minutes); other ranks exit at once."""
    rank, world, _ = rank_env()
    if rank != 0:
        return None
    T = args.T or 8
    K = max(1, min(args.steps, args.cpu_steps))
    W = max(0, min(args.warmup, 1))
    o = OracleDecode(T, K + W)
    dt = o.timed(K, W)
    value = round(T * K / dt, 3)
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
           "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(dt * 1e3 / K, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": workload_config("decode", T, world, args.layers),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": o.cores(),
                            "kind": "oracle",
                            "sample": f"{K} decode layer forwards of T={T} tokens after {W} "
                                      f"warm-up (full layer, float64 numpy, rank 0 only)"},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))
    return out


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
