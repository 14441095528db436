"""Benchmark: NVFP4 MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--T 8] [--workload decode|prefill|wide]
                    [--impl ours|reference]

One step = one full MoE layer forward (quantise x, route, expert FFN with the shared expert,
combine, cumulative expert histogram). The headline workload is the decode layer: d=2048, 512
experts, top-10 + 1 shared expert, I=512, NVFP4 weights, T tokens (default 8). Step i runs on
layer copy i % L (L distinct copies, 8 by default: 7 GB of weights, far above the 126 MB L2)
with input draw (i // L) % 4 of that copy, so consecutive steps route to different experts of
different weight copies. Exactly K timed steps after W warm-up steps, replayed from CUDA graphs;
timing uses CUDA events on the launching stream, max over ranks. The same line carries decode
T=1 and T=4 and the prefill layer (same weights, Zipf(0.8) routing, T=16384) under
"extra_configs". Prints one JSON line on rank 0.

--impl reference times the CPU oracle (oracle/, float64 numpy) on the host cores on a bounded
sample of the same workload.
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
X_DRAWS = 4             # input draws per decode layer copy
# prefill layer copies: each has its own buffers and, end to end, its own stream, so one step's
# 64 MB host copies in and out overlap the neighbouring steps' compute
PREFILL_COPIES = 3
NOMINAL_HBM_GBS = 8000.0  # B200 spec-sheet HBM3e bandwidth, for context beside the measured peak
# DRAM bytes (read + write) per launch of the dominant kernels from ncu captures of the
# current kernels (profiles/); None when the kernel has changed since its capture
DECODE_TRAFFIC_RATIO = 0.899  # layer_dec_kernel: traffic / algorithmic bytes in the rotating loop
DECODE_TRAFFIC_SOURCE = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                         "--cache-control none (1 pass) on 16 launches inside the 8-copy rotating decode loop "
                         "(T=8): 51.27 MB per launch against 57.05 MB of algorithmic bytes; the ratio is "
                         "applied to this run's algorithmic bytes")
PREFILL_TRAFFIC_BYTES = 3_275_270_000  # tc_ffn_mt_kernel, T = 16384, one launch
PREFILL_TRAFFIC_SOURCE = ("ncu --set full (caches flushed before the passes) on one launch of tc_ffn_mt_kernel "
                          "at T=16384: 2.173 GB read + 1.103 GB written; about 2.1 GB of it is the float32 "
                          "output y (128 MB) leaving L2 between its 11 reductions per token")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm": float(j["hbm_gbs"]), "bf16": float(j["bf16_tflops"]),
                "bf16_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "kind": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "kind": "fallback"}


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every few ms (reads only)."""

    REASONS = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.002):
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


# ---------------------------------------------------------------------------- timing
class Timer:
    """Graphs of consecutive steps of a step function and their CUDA-event timing."""

    def __init__(self, stream, dist, device, sampler_windows):
        self.stream, self.dist, self.device = stream, dist, device
        self.windows = sampler_windows

    def capture(self, step_fn, m, finish=None):
        """One CUDA graph of steps 0..m-1 (then `finish`, e.g. joins of side streams);
        returns (graph, this library's launches per step counted at capture)."""
        from nvfp4_expert_ffn_b200 import binding as B
        g = torch.cuda.CUDAGraph()
        n0 = B.moe_launch_count()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(m):
                step_fn(i)
            if finish:
                finish()
        return g, (B.moe_launch_count() - n0) / max(m, 1)

    def plan(self, step_fn, n, cycle, finish=None):
        """Graphs that together run exactly n steps: a graph of min(n, cycle) steps replayed
        n // that times, then a graph of the remainder."""
        m = max(1, min(n, cycle))
        g, lps = self.capture(step_fn, m, finish)
        reps, rem = n // m, n % m
        g_rem = self.capture(step_fn, rem, finish)[0] if rem else None
        return (g, reps, g_rem), lps

    def replay(self, plan):
        g, reps, g_rem = plan
        for _ in range(reps):
            g.replay()
        if g_rem is not None:
            g_rem.replay()

    def time(self, plan):
        """ms for one replay of the plan, CUDA events on the launching stream, max over ranks."""
        if self.dist is not None:
            self.dist.barrier()
        torch.cuda.synchronize()
        t0h = time.time()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record(self.stream)
            self.replay(plan)
            e1.record(self.stream)
        torch.cuda.synchronize()
        self.windows.append((t0h, time.time()))
        return max_over_ranks(self.dist, e0.elapsed_time(e1), self.device)


# ---------------------------------------------------------------------------- workloads
def build_decode_copies(device, n_copies: int, T_max: int = 8):
    """n_copies distinct decode layers (own seeded weights and router each), with X_DRAWS
    input draws of T_max tokens per copy."""
    from nvfp4_expert_ffn_b200 import binding as B
    from nvfp4_expert_ffn_b200 import layer as L
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS["decode"]
    copies, xs = [], []
    ws_q = None
    for li in range(n_copies):
        if ws_q is None:
            ws_q = torch.empty(B.moe_workspace_size(B.MOE_OP_QUANT, 1, cfg.d, 1, 1, cfg.I), dtype=torch.uint8,
                               device=device)
        routed = L.quantize_weights_gpu(SEED, cfg, layer=li, device=device, ws=ws_q)
        shared = L.quantize_weights_gpu(SEED, cfg, layer=li, shared=True, device=device, ws=ws_q)
        Wr, br = synth.make_router(SEED, cfg, layer=li)
        copies.append(L.MoeLayer(B.Experts(routed, shared), Wr.to(device), br.to(device), cfg.k, T_max,
                                 device=device))
        xs.append([synth.make_x(SEED, cfg, T_max, layer=li, step=j).to(device) for j in range(X_DRAWS)])
    return cfg, copies, xs


def algorithmic_bytes(cfg, U: int, T: int) -> float:
    """HBM bytes one decode layer forward must move: the router matrix, the weights and scales
    of the U routed experts in use and the shared expert, x, its NVFP4 codes, y_acc and y."""
    per_expert = 3 * cfg.d * cfg.I * 0.5625
    return (cfg.E * cfg.d * 4 + cfg.E * 4 + (U + 1) * per_expert
            + T * cfg.d * (2 + 0.5625 + 4 + 2))


def hot_tier_on(layers, n_layers_sharing: int, stream):
    """Give every layer a hot tier of as many experts as this process's L2 set-aside holds
    for n_layers_sharing layers, ranked by each layer's routing so far. Returns the tier's
    description (n_hot 0 when the set-aside holds less than one expert per layer)."""
    from nvfp4_expert_ffn_b200 import binding as B
    lay0 = layers[0]
    setaside = B.moe_set_l2_persisting(1 << 40)
    per_expert = B.dec_pack_bytes(1, lay0.d, lay0.I)
    n_hot = int(round(setaside / (n_layers_sharing * per_expert)))
    with torch.cuda.stream(stream):
        for lay in layers:
            lay.update_hot_tier(n_hot, stream=stream)
    torch.cuda.synchronize()
    return {"n_hot_per_layer": n_hot, "l2_setaside_bytes": setaside, "expert_bytes": per_expert,
            "ranking": "each layer's cumulative routing counts (moe_expert_hist)"}


def hot_tier_off(layers, stream):
    from nvfp4_expert_ffn_b200 import binding as B
    with torch.cuda.stream(stream):
        for lay in layers:
            lay.update_hot_tier(0, stream=stream)
    torch.cuda.synchronize()
    B.moe_set_l2_persisting(0)


def time_e2e(timer, runners, steps, stream, slot_of):
    """Time `steps` graphed layer steps end to end (pinned host x -> device, the layer,
    y -> pinned host, every step). Step i replays runner i % len(runners) with input slot
    slot_of(i); each runner has its own stream, so the copies of one step overlap the
    compute of the steps before and after it, as consecutive requests would. Returns ms
    (max over ranks)."""
    n = len(runners)
    if timer.dist is not None:
        timer.dist.barrier()
    t0h = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for r in runners:
        r.stream.wait_event(e0)
    for i in range(steps):
        runners[i % n].run(slot_of(i))
    for r in runners:
        stream.wait_stream(r.stream)
    e1.record(stream)
    torch.cuda.synchronize()
    timer.windows.append((t0h, time.time()))
    return max_over_ranks(timer.dist, e0.elapsed_time(e1), timer.device)


def measure_decode(timer, cfg, copies, xs, T, K, W, e2e_steps, stream, world, peaks, hot=False):
    from nvfp4_expert_ffn_b200 import binding as B
    n = len(copies)
    cycle = n * X_DRAWS
    k = cfg.k
    fused = all(lay.fused for lay in copies)

    def x_of(i):
        return xs[i % n][(i // n) % X_DRAWS][:T]

    def step(i):
        copies[i % n].forward(x_of(i), join=False)  # each histogram overlaps the next step

    def finish():
        for lay in copies:
            lay.join(stream)

    def kernel(i):  # the dominant kernel alone: the one-kernel decode layer
        lay = copies[i % n]
        B.moe_layer_decode(x_of(i), lay.static_ts, lay.Wr, lay.br, lay.experts, k, lay.xq_codes[:T],
                           lay.xq_scales[:T], lay.xq_ts[:1], lay.topk_idx[:T], lay.topk_w[:T], lay.counts,
                           lay.offsets, lay.sorted_assign[:T * k], lay.assign_pos[:T * k], lay.y_acc[:T],
                           lay.y[:T], False, lay.ws_dec)

    # touched experts of every step of the cycle (eager, once)
    U = []
    with torch.cuda.stream(stream):
        for i in range(cycle):
            copies[i % n].forward(x_of(i))
            stream.synchronize()
            U.append(int((copies[i % n].counts > 0).sum().item()))
    Ui = [U[i % cycle] for i in range(K)]
    bytes_k = [algorithmic_bytes(cfg, u, T) for u in Ui]
    tier = hot_tier_on(copies, n, stream) if hot else None
    warm, _ = timer.plan(step, W, cycle, finish)
    main, lps = timer.plan(step, K, cycle, finish)
    kplan, _ = timer.plan(kernel, K, cycle) if fused else (None, 0)
    with torch.cuda.stream(stream):
        timer.replay(warm)
        if kplan:
            timer.replay(timer.plan(kernel, W, cycle)[0])
    torch.cuda.synchronize()
    ms = timer.time(main)
    ms_k = timer.time(kplan) if kplan else None
    out = {"value": round(whole_job_rate(world, T, K, ms), 1), "unit": "tokens/s",
           "ms_per_step": round(ms / K, 6), "T": T, "touched_experts_avg": round(float(np.mean(Ui)), 2),
           "gpu_launches": int(round(lps * K)), "gpu_launches_per_step": lps}
    if ms_k is not None:
        avg_b = float(np.mean(bytes_k))
        ach = avg_b / (ms_k / K * 1e-3) / 1e9
        out["roofline"] = {
            "kernel": "layer_dec_kernel (moe_layer_decode: quantise, route, tcgen05 expert FFN, combine)",
            "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm"], 4), "peak_kind": peaks["kind"] + " (HBM copy, burst)",
            "frac_vs_nominal_8tbs": round(ach / NOMINAL_HBM_GBS, 4),
            "bytes_per_launch": int(avg_b), "avg_launch_us": round(ms_k / K * 1e3, 3),
            # the ratio was captured at T = 8 without a hot tier; other token counts are not measured
            "traffic": (int(avg_b * DECODE_TRAFFIC_RATIO) if DECODE_TRAFFIC_RATIO is not None and T == 8 and not hot
                        else None),
            "traffic_source": DECODE_TRAFFIC_SOURCE if T == 8 and not hot else None}
    # end to end through the public API: each step is one replay of a graphed layer step that
    # copies the step's input from pinned host memory, runs the layer and copies y back
    if e2e_steps:
        runners = [lay.graphed(T, n_slots=X_DRAWS, stream=torch.cuda.Stream(stream.device)) for lay in copies]
        for c, r in enumerate(runners):
            for j in range(X_DRAWS):
                r.x_host[j].copy_(xs[c][j][:T].cpu())
        for i in range(min(W, cycle)):
            runners[i % n].run((i // n) % X_DRAWS)
        torch.cuda.synchronize()
        ms_e = time_e2e(timer, runners, e2e_steps, stream, lambda i: (i // n) % X_DRAWS)
        out["e2e"] = {"value": round(whole_job_rate(world, T, e2e_steps, ms_e), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * 2,
                      "steps": e2e_steps,
                      "api": "GraphedMoeLayer.run: pinned x -> device, layer, y -> pinned; one stream per layer "
                             "copy, so one step's copies overlap the neighbouring steps' compute"}
        del runners
    if tier is not None:
        out["hot_tier"] = tier
        hot_tier_off(copies, stream)
    return out


def build_prefill_layers(device, workload, decode_copies, n_copies: int, static_scales: bool = False):
    """Layers of the prefill workload. prefill: the decode copies' weights (the same layer)
    with the prefill router (Zipf(0.8) popularity); wide: its own seeded weights. With
    static_scales each layer quantises every expert's rows with the expert's own static
    input scales (synth.make_input_scales) instead of one per-call activation scale."""
    from nvfp4_expert_ffn_b200 import binding as B
    from nvfp4_expert_ffn_b200 import layer as L
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS[workload]
    T = cfg.T_list[0]
    layers, xs = [], []
    for li in range(n_copies):
        if workload == "prefill" and decode_copies:
            experts = decode_copies[li % len(decode_copies)].experts
        else:
            experts = B.Experts(L.quantize_weights_gpu(SEED, cfg, layer=li, device=device),
                                L.quantize_weights_gpu(SEED, cfg, layer=li, shared=True, device=device))
        Wr, br = synth.make_router(SEED, cfg, layer=li)
        scales = tuple(t.to(device) for t in synth.make_input_scales(cfg)) if static_scales else None
        layers.append(L.MoeLayer(experts, Wr.to(device), br.to(device) if cfg.zipf_s > 0 else None, cfg.k, T,
                                 device=device, fused=False, input_scales=scales))
        xs.append(synth.make_x(SEED, cfg, T, layer=li).to(device))
    return cfg, layers, xs


def measure_prefill(timer, cfg, layers, xs, K, W, e2e_steps, stream, world, peaks):
    from nvfp4_expert_ffn_b200 import binding as B
    n = len(layers)
    T, k = xs[0].shape[0], cfg.k

    def step(i):
        layers[i % n].forward(xs[i % n], join=False)

    def finish():
        for lay in layers:
            lay.join(stream)

    def ffn(i):  # the dominant call alone: the expert FFN (schedule, row gather, tcgen05 GEMMs)
        lay = layers[i % n]
        if lay.input_scales is not None:
            B.moe_expert_ffn_static(xs[i % n], lay.experts, lay.input_scales[0], lay.input_scales[1], k, lay.offsets,
                                    lay.sorted_assign[:T * k], lay.topk_w[:T], B.MOE_FFN_ACCUMULATE, lay.y_acc[:T],
                                    None, lay.ws)
        else:
            B.moe_expert_ffn(lay.xq_codes[:T], lay.xq_scales[:T], lay.xq_ts[:1], lay.experts, k, lay.offsets,
                             lay.sorted_assign[:T * k], lay.topk_w[:T], B.MOE_FFN_ACCUMULATE, lay.path,
                             lay.y_acc[:T], None, lay.ws)

    with torch.cuda.stream(stream):
        for i in range(n):
            step(i)
        finish()
    torch.cuda.synchronize()
    U = [int((lay.counts > 0).sum().item()) for lay in layers]
    warm, _ = timer.plan(step, W, n, finish)
    main, lps = timer.plan(step, K, n, finish)
    fplan, _ = timer.plan(ffn, K, n)
    with torch.cuda.stream(stream):
        timer.replay(warm)
    torch.cuda.synchronize()
    ms = timer.time(main)
    ms_f = timer.time(fplan)
    flops = 2.0 * T * (k + 1) * 3 * cfg.d * cfg.I
    fp4_peak = 4.0 * peaks["bf16"]
    tf = flops / (ms_f / K * 1e-3) / 1e12
    wbytes = (float(np.mean(U)) + 1) * 3 * cfg.d * cfg.I * 0.5625
    out = {"value": round(whole_job_rate(world, T, K, ms), 1), "unit": "tokens/s", "ms_per_step": round(ms / K, 6),
           "T": T, "touched_experts_avg": round(float(np.mean(U)), 2),
           "gpu_launches": int(round(lps * K)), "gpu_launches_per_step": lps,
           "roofline": {"kernel": ("moe_expert_ffn_static" if layers[0].input_scales is not None else "moe_expert_ffn")
                        + " (schedule, row gather, tcgen05 block-scaled grouped GEMMs)",
                        "bound": "tensor", "achieved": round(tf, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                        "frac": round(tf / fp4_peak, 4),
                        "peak_kind": f"{peaks['kind']} bf16 (burst) x 4, the nominal dense FP4 : bf16 ratio",
                        "flops_per_launch": flops, "weight_bytes_per_launch": int(wbytes),
                        "avg_launch_us": round(ms_f / K * 1e3, 3),
                        "traffic": (PREFILL_TRAFFIC_BYTES if PREFILL_TRAFFIC_BYTES is not None and cfg.name == "prefill"
                                    and layers[0].input_scales is None else None),
                        "traffic_source": (PREFILL_TRAFFIC_SOURCE if cfg.name == "prefill"
                                           and layers[0].input_scales is None else None)}}
    if e2e_steps:
        runners = [lay.graphed(T, n_slots=1, stream=torch.cuda.Stream(stream.device)) for lay in layers]
        for r, x in zip(runners, xs):
            r.x_host[0].copy_(x.cpu())
        for r in runners:
            r.run(0)
        torch.cuda.synchronize()
        ms_e = time_e2e(timer, runners, e2e_steps, stream, lambda i: 0)
        out["e2e"] = {"value": round(whole_job_rate(world, T, e2e_steps, ms_e), 1), "unit": "tokens/s",
                      "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * 2,
                      "steps": e2e_steps,
                      "api": "GraphedMoeLayer.run: pinned x -> device, layer, y -> pinned; one stream per layer "
                             "copy, so one step's copies overlap the neighbouring steps' compute"}
        del runners
    return out


def build_stack(device, n_layers: int = 48, epochs: int = 4, n_x: int = 64):
    """The decode stack: n_layers distinct decode layers (own weights, router and Zipf(1.0)
    popularity each; decode pack only, every weight byte held once), the router bias of every
    64-step epoch, and n_x input draws of 8 tokens."""
    from nvfp4_expert_ffn_b200 import binding as B
    from nvfp4_expert_ffn_b200 import layer as L
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS["stack48"]
    ws_q = torch.empty(B.moe_workspace_size(B.MOE_OP_QUANT, 1, cfg.d, 1, 1, cfg.I), dtype=torch.uint8, device=device)
    layers, biases = [], []
    for li in range(n_layers):
        routed = L.quantize_weights_gpu(SEED, cfg, layer=li, device=device, ws=ws_q, decode_only=True)
        shared = L.quantize_weights_gpu(SEED, cfg, layer=li, shared=True, device=device, ws=ws_q, decode_only=True)
        Wr, _ = synth.make_router(SEED, cfg, layer=li)
        biases.append([synth.make_router(SEED, cfg, layer=li, epoch=ep)[1].to(device) for ep in range(epochs)])
        layers.append(L.MoeLayer(B.Experts(routed, shared), Wr.to(device), biases[-1][0], cfg.k, 8, device=device,
                                 fused=True))
    xs = torch.stack([synth.make_x(SEED, cfg, 8, step=s) for s in range(n_x)]).to(device)
    return cfg, layers, biases, xs


def measure_stack(timer, cfg, layers, biases, xs, K, W, stream, world, peaks, hot=False):
    """Step = 8 tokens through every layer (RMS renormalisation between layers); step s uses
    input draw s % len(xs) and the router biases of epoch (s // 64) % epochs. With hot=True
    every layer keeps a hot tier in L2 that follows the drift: at the start of each epoch the
    layers' routing counts restart, and after its first 8 steps each layer's tier is refilled
    with its most-routed experts of those steps (inside the timed region)."""
    n_ep = len(biases[0])
    x_in = torch.empty_like(xs[0])
    tier = hot_tier_on(layers, len(layers), stream) if hot else None
    n_hot = tier["n_hot_per_layer"] if tier else 0
    graphs = []
    for ep in range(n_ep):
        for lay, b in zip(layers, biases):
            lay.br = b[ep]

        def step(i):
            h = x_in
            for lay in layers:
                h = lay.forward(h, rms_renorm=True, join=False)

        def finish():
            for lay in layers:
                lay.join(stream)

        with torch.cuda.stream(stream):
            step(0)
            finish()
        torch.cuda.synchronize()
        graphs.append(timer.capture(step, 1, finish))
    lps = graphs[0][1]

    def run(n, s0=0):
        for s in range(s0, s0 + n):
            if n_hot > 0 and s % 64 == 0:
                for lay in layers:
                    lay.cum.zero_()
            elif n_hot > 0 and s % 64 == 8:
                for lay in layers:
                    lay.update_hot_tier(n_hot, stream=stream)
            x_in.copy_(xs[s % len(xs)], non_blocking=True)
            graphs[(s // 64) % n_ep][0].replay()

    # touched experts per layer and step (for the bytes), on a sample of steps
    U = []
    with torch.cuda.stream(stream):
        for s in (0, 64, 128, 192):
            run(1, s)
            stream.synchronize()
            U.extend(int((lay.counts > 0).sum().item()) for lay in layers)
    with torch.cuda.stream(stream):
        run(W)
    torch.cuda.synchronize()
    if timer.dist is not None:
        timer.dist.barrier()
    t0h = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        run(K)
        e1.record(stream)
    torch.cuda.synchronize()
    timer.windows.append((t0h, time.time()))
    ms = max_over_ranks(timer.dist, e0.elapsed_time(e1), timer.device)
    per_layer_bytes = float(np.mean([algorithmic_bytes(cfg, u, 8) for u in U]))
    step_bytes = per_layer_bytes * len(layers)
    ach = step_bytes / (ms / K * 1e-3) / 1e9
    if tier is not None:
        hot_tier_off(layers, stream)
    return {"value": round(whole_job_rate(world, 8, K, ms), 1), "unit": "tokens/s", "ms_per_step": round(ms / K, 6),
            "hot_tier": tier,
            "steps": K, "T": 8, "layers": len(layers), "touched_experts_avg": round(float(np.mean(U)), 2),
            "gpu_launches": int(round(lps * K)), "gpu_launches_per_step": lps,
            "roofline": {"kernel": "whole step: 48 x (layer_dec_kernel + hist_kernel)", "bound": "hbm",
                         "achieved": round(ach, 1), "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": round(ach / peaks["hbm"], 4), "peak_kind": peaks["kind"] + " (HBM copy, burst)",
                         "frac_vs_nominal_8tbs": round(ach / NOMINAL_HBM_GBS, 4),
                         "bytes_per_step": int(step_bytes), "traffic": None},
            "workload": (f"48-layer decode stack: d={cfg.d}, {cfg.E} experts/layer, top-{cfg.k} + 1 shared, "
                         f"I={cfg.I}, 8 tokens per step, per-layer RMS renormalisation, Zipf(1.0) routing "
                         f"re-drawn every 64 steps, {len(layers)} x {cfg.E} experts resident "
                         f"({len(layers) * (cfg.E + 1) * 3 * cfg.d * cfg.I * 0.5625 / 1e9:.1f} GB, decode pack only)")}


def near_tie_record():
    """Tokens excused from the bit-exact top-k comparison in the parity tests (k-th/(k+1)-th
    oracle logit margin under 1e-6), per test input, from tests/golden/near_ties.json."""
    p = os.path.join(ROOT, "tests", "golden", "near_ties.json")
    if not os.path.exists(p):
        return None
    return {f"{r['config']}_T{r['T']}_draw{r['step']}": r["count"] for r in json.load(open(p))}


def run_gpu(args):
    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
    dist = dist_init("nccl")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from nvfp4_expert_ffn_b200 import synth
    K, W = args.steps, args.warmup
    peaks = _peaks()
    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(local)
    windows = []
    timer = Timer(stream, dist, device, windows)
    sampler.start()
    e2e_steps = 0 if args.no_e2e else K
    extra = {}
    copies = []
    if args.workload == "decode":
        T = args.T or 8
        cfg, copies, xs = build_decode_copies(device, args.layers)
        main = measure_decode(timer, cfg, copies, xs, T, K, W, e2e_steps, stream, world, peaks)
        workload = (f"decode MoE layer: d={cfg.d}, {cfg.E} experts, top-{cfg.k} + 1 shared, I={cfg.I}, "
                    f"NVFP4 weights, T={T} tokens per step")
        l2 = (f"{args.layers} distinct layer copies ({args.layers * cfg.E * 3 * cfg.d * cfg.I * 0.5625 / 1e9:.1f} GB"
              f" of expert weights) x {X_DRAWS} input draws, rotated every step: inputs > L2")
        if not args.no_extra:
            for Tx in (1, 4, 8):
                if Tx != T:
                    extra[f"decode_T{Tx}"] = measure_decode(timer, cfg, copies, xs, Tx, K, W, e2e_steps, stream,
                                                            world, peaks)
            if not args.no_hot:
                extra[f"decode_T{T}_hot_tier"] = measure_decode(timer, cfg, copies, xs, T, K, W, 0, stream, world,
                                                                peaks, hot=True)
            pcfg, players, pxs = build_prefill_layers(device, "prefill", copies, PREFILL_COPIES)
            extra["prefill_T16384"] = measure_prefill(timer, pcfg, players, pxs, K, W, e2e_steps, stream, world,
                                                      peaks)
            extra["prefill_T16384"]["workload"] = ("prefill MoE layer: the decode layer's weights, Zipf(0.8) "
                                                   f"routing, T=16384 tokens per step, {PREFILL_COPIES} layer copies")
            del players
            pcfg, players, pxs = build_prefill_layers(device, "prefill", copies, 2, static_scales=True)
            extra["prefill_T16384_static_scales"] = measure_prefill(timer, pcfg, players, pxs, K, W, 0, stream,
                                                                    world, peaks)
            extra["prefill_T16384_static_scales"]["workload"] = (
                "prefill_T16384 with static per-expert input scales: every expert quantises its own rows "
                "(moe_expert_ffn_static), no per-call activation quantisation")
            del players
            wcfg, players, pxs = build_prefill_layers(device, "wide", None, 2)
            extra[f"wide_T{pxs[0].shape[0]}"] = measure_prefill(timer, wcfg, players, pxs, K, W, e2e_steps, stream,
                                                                world, peaks)
            extra[f"wide_T{pxs[0].shape[0]}"]["workload"] = (
                f"wide chunked prefill MoE layer: d={wcfg.d}, {wcfg.E} experts, top-{wcfg.k} + 1 shared, "
                f"I={wcfg.I}, NVFP4 weights, T={pxs[0].shape[0]} tokens per step (512 + 2048 + 8192 + 16384 + 4), "
                "uniform routing, 2 layer copies")
            del players
            torch.cuda.empty_cache()
            if not args.no_stack:
                del copies, xs
                torch.cuda.empty_cache()
                copies = []
                scfg, slayers, sbiases, sxs = build_stack(device)
                extra["stack48"] = measure_stack(timer, scfg, slayers, sbiases, sxs, 256, max(W, 8), stream, world,
                                                 peaks)
                if not args.no_hot:
                    extra["stack48_hot_tier"] = measure_stack(timer, scfg, slayers, sbiases, sxs, 256, max(W, 8),
                                                              stream, world, peaks, hot=True)
                del slayers
    elif args.workload == "stack48":
        T = 8
        cfg, slayers, sbiases, sxs = build_stack(device)
        main = measure_stack(timer, cfg, slayers, sbiases, sxs, K, W, stream, world, peaks)
        workload = main["workload"]
        l2 = "48 layers x 513 experts resident (43.6 GB), far above L2"
    else:
        cfg, layers, xs = build_prefill_layers(device, args.workload, None, args.layers)
        T = xs[0].shape[0]
        main = measure_prefill(timer, cfg, layers, xs, K, W, e2e_steps, stream, world, peaks)
        workload = (f"{args.workload} MoE layer: d={cfg.d}, {cfg.E} experts, top-{cfg.k} + 1 shared, I={cfg.I}, "
                    f"NVFP4 weights, T={T} tokens per step")
        l2 = f"{args.layers} distinct layer copies rotated every step; each step touches > L2"
    sampler.stop()
    out = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 block scales), fp32 accumulate", "data": "synthetic",
        "config": {"workload": workload, "T": T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I,
                   "zipf_s": cfg.zipf_s, "parallelism": f"replicas x{world}", "l2": l2,
                   "touched_experts_avg": main["touched_experts_avg"]},
        "roofline": main.get("roofline"),
        "e2e": main.get("e2e"),
        "gpu_launches": main["gpu_launches"],
        "gpu_launches_per_step": main["gpu_launches_per_step"],
        "clocks": sampler.summary(windows),
    }
    if extra:
        out["extra_configs"] = extra
    ties = near_tie_record()
    if ties is not None:
        out["parity_near_tie_tokens"] = ties
    if rank == 0 and not args.no_cpu_baseline and args.workload == "decode":
        out["cpu_baseline"] = cpu_baseline(T, args.cpu_steps)
    if dist is not None:
        torch.cuda.synchronize()
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
        from oracle.weights import OracleWeights
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


def decode_config(T: int, world: int, n_copies: int) -> dict:
    from nvfp4_expert_ffn_b200 import synth
    cfg = synth.CONFIGS["decode"]
    return {"workload": f"decode MoE layer: d={cfg.d}, {cfg.E} experts, top-{cfg.k} + 1 shared, I={cfg.I}, "
                        f"NVFP4 weights, T={T} tokens per step",
            "T": T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I, "zipf_s": cfg.zipf_s,
            "parallelism": f"replicas x{world}",
            "l2": f"{n_copies} distinct layer copies x {X_DRAWS} input draws, rotated every step: inputs > L2"}


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
           "data": "synthetic", "config": decode_config(T, world, args.layers),
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--T", type=int, default=0, help="decode tokens per step (default 8)")
    ap.add_argument("--workload", choices=["decode", "prefill", "wide", "stack48"], default="decode")
    ap.add_argument("--no-hot", action="store_true", help="skip the hot-tier (L2 persisting) measurements")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-steps", type=int, default=16, help="oracle decode forwards timed (about 10 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="only the headline workload")
    ap.add_argument("--no-stack", action="store_true", help="leave out the 48-layer decode stack")
    ap.add_argument("--layers", type=int, default=8, help="distinct layer copies rotated")
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
