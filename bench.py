#!/usr/bin/env python
"""Benchmark of the AWQ per-layer scale search on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {awq,reference}]

One step = the whole hot path for one layer of the Llama-7B-shaped q_proj
workload (X [65536 x 4096] fp16 heavy-tailed, W [4096 x 4096], INT4 g128,
20 alphas + 20 clip ratios, packed): awq_act_stats -> awq_search_scale ->
awq_search_clip -> awq_quant_pack.  With N GPUs (torchrun, one process per
GPU) every rank runs the same step on its own layer (independent seeds): weak
scaling, no data-path collective.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the fp64 restatement of the method
the tests check the CUDA path against) on the host cores: each step is one
whole layer of the same workload (about 15-20 s on 16 cores).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "AWQ search ms/layer & candidate-GEMM TFLOP/s on 1 B200; % of TC/HBM roofline"
UNIT = "ms/layer"
WORKLOAD_INDEX = 1  # Llama-7B-shaped q_proj
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (dense fp16/bf16 tensor rate, HGX HBM3e bandwidth), reported beside
# the measured denominators
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "fp16_tflops": 2250.0}
KERNELS_PER_STEP = {  # kernels this library launches per step (memsets excluded)
    "act_stats": 2, "wmax": 1, "scale_grid": 1, "cand_quant": 1, "search_gemm": 1,
    "mse_argmin": 1, "gram_blocks": 2, "clip_eval": 1, "quant_pack": 1,
}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# search_gemm_kernel launch on this workload, from a one-pass ncu capture of
# the command below, together with the SHA-256 of the kernel's sources at
# capture time.  The figure is reported only while the sources still hash to
# that digest; after any change to them the line carries traffic = null until
# the kernel is captured again.
NCU_TRAFFIC = {
    "bytes": 15623107840 + 10422016,  # dram__bytes_read.sum + dram__bytes_write.sum
    "sources_sha256": "783bdf6248aceb0daeaef22bf3c1e10e9a61b126fa91114577c6692fc2dbc398",
    "command": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none "
                "-k regex:search_gemm -s 5 -c 1 python bench.py --steps 1 --warmup 5 "
                "--no-cpu-baseline --no-gram-form --no-cached-form --no-fused-form --no-w4a16 --no-workloads"),
}
TRAFFIC_SOURCES = ("post_weight_quantization_awq_b200/csrc/search_gemm.cu",
                   "post_weight_quantization_awq_b200/csrc/awq_device.cuh")
TILE_HEADER = "post_weight_quantization_awq_b200/csrc/awq_launch.h"


def traffic_sources_digest() -> str:
    """SHA-256 over the sources the scored-GEMM kernel is compiled from: its
    file, the device header, and the line of the launch header that fixes its
    tile shape."""
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, TILE_HEADER)) as f:
        tile = [ln for ln in f.read().splitlines() if "kGemmBM" in ln and "constexpr" in ln]
    h.update("\n".join(tile).encode())
    return h.hexdigest()


# Warp instructions of one cand_quant_kernel launch on this workload (it does
# not depend on the token count), from an ncu capture of the command below,
# with the SHA-256 of the kernel's sources at capture time; reported only
# while the sources still hash to it.  The kernel is bound by instruction
# issue, not by HBM: its roofline is the SMs' issue rate (4 warp
# instructions per SM and clock).
NCU_ISSUE = {
    "warp_instructions": 168989637,  # smsp__inst_executed.sum
    "sources_sha256": "7c86acea45a98a4da473c89f669b5dca4cb4af6d112b8a7fe22824866b6f013d",
    "command": ("ncu --metrics smsp__inst_executed.sum,gpu__time_duration.sum --clock-control none "
                "-k regex:cand_quant -c 1 python -m post_weight_quantization_awq_b200.run_case "
                "--op search --tokens 16384 --in 4096 --out 4096 --repeat 1"),
}
ISSUE_SOURCES = ("post_weight_quantization_awq_b200/csrc/quant_kernels.cu",
                 "post_weight_quantization_awq_b200/csrc/awq_device.cuh")


def issue_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in ISSUE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def cand_quant_issue(ms, sm_mhz, num_sms):
    """The candidate quantiser against the issue roofline: recorded warp
    instructions per launch / its in-step duration, against num_sms x 4 warp
    instructions per clock at the median SM clock sampled in the timed region."""
    n = NCU_ISSUE["warp_instructions"]
    if n is None or NCU_ISSUE["sources_sha256"] != issue_sources_digest():
        return {"bound": "alu", "warp_instructions": None,
                "note": "instruction count not captured for the current kernel sources"}
    if not ms or not sm_mhz:
        return {"bound": "alu", "warp_instructions": n, "note": "no in-step duration or clock"}
    achieved = n / (ms * 1e-3)
    peak = num_sms * 4 * sm_mhz * 1e6
    return {"bound": "alu", "warp_instructions": n, "achieved_winst_per_s": round(achieved / 1e9, 1),
            "peak_winst_per_s": round(peak / 1e9, 1), "unit": "G warp instructions/s",
            "frac": round(achieved / peak, 3), "sm_mhz": sm_mhz,
            "note": "peak = SMs x 4 issue slots x the median SM clock of the timed region; "
                    "instruction count: " + NCU_ISSUE["command"]}


def ncu_traffic():
    """(bytes per launch, note): the recorded capture if it describes the
    kernel as built now, else (None, why)."""
    if NCU_TRAFFIC["bytes"] is None:
        return None, "not captured for the current kernel"
    if NCU_TRAFFIC["sources_sha256"] != traffic_sources_digest():
        return None, "kernel sources changed since the capture"
    return NCU_TRAFFIC["bytes"], "ncu capture of the current kernel sources: " + NCU_TRAFFIC["command"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_description(wl, T, inn, out):
    return {
        "workload": f"{wl.name}: {wl.description}",
        "tokens": T, "in": inn, "out": out, "w_bit": wl.w_bit, "group_size": wl.group_size,
        "n_alpha": wl.n_alpha, "n_clip": wl.n_clip,
        "l2": "inputs larger than L2 (X is 512 MiB, candidate operand 640 MiB); no flush",
    }


# ---------------------------------------------------------------- distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str, world: int):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist) -> float:
    """Max of a per-rank float over all ranks (identity on one rank).  The
    scalar travels on the device the process group's backend uses."""
    if dist is None:
        return value
    import torch
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device != "cpu":
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


class CudaTimer:
    """CUDA events on the stream the work is launched on."""

    def __init__(self, torch, stream, device):
        self.torch, self.stream, self.device = torch, stream, device
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def sync(self):
        self.torch.cuda.synchronize(self.device)

    def start(self):
        self.e0.record(self.stream)

    def stop(self):
        self.e1.record(self.stream)

    def elapsed_ms(self):
        return self.e0.elapsed_time(self.e1)


def timed_steps(step, steps: int, dist, timer, barrier_device=None, before_stop=None) -> float:
    """Times exactly `steps` calls of `step` between a barrier + device sync on
    both sides; returns the max over ranks of ms per step.  `before_stop`
    makes the timed stream wait for work the steps left on other streams."""
    barrier(dist, barrier_device)
    timer.sync()
    timer.start()
    for _ in range(steps):
        step()
    if before_stop is not None:
        before_stop()
    timer.stop()
    timer.sync()
    barrier(dist, barrier_device)
    return max_over_ranks(timer.elapsed_ms() / steps, dist)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while the
    timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "", 1).isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [r for r in rows if pw and float(r[3]) > 0.5 * max(pw)] if pw else rows
        sm_load = [float(r[1]) for r in loaded if r[1].replace(".", "").isdigit()] or sm
        return {"sm_mhz": statistics.median(sm_load) if sm_load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------- oracle arm
def oracle_threads():
    """Threads the oracle's timed run uses: its matrix products run in the
    BLAS thread pool (numpy's), its elementwise steps on one thread."""
    try:
        import threadpoolctl
        n = max((i.get("num_threads", 0) for i in threadpoolctl.threadpool_info()
                 if i.get("user_api") == "blas"), default=0)
    except Exception:
        n = 0
    return n if n > 0 else os.cpu_count()


def oracle_layer_ms(X, W, wl, row_fraction: float = 1.0):
    """Times the CPU oracle on one layer of the workload: abar, X^T X, the
    alpha search, the block Grams, the clip search and the packing, in that
    order.  With row_fraction = 1 (the default) this is the whole layer, timed
    as it runs; with row_fraction < 1 the per-row phases run on
    round(row_fraction * out) rows and are scaled by 1/row_fraction (the
    row-independent phases are still timed in full).
    Returns (ms per layer, sample description)."""
    import numpy as np
    from oracle import awq_oracle as O
    Xn, Wn = X.numpy(), W.numpy()
    out = Wn.shape[0]
    rows = max(8, int(round(out * row_fraction)) // 8 * 8)
    Ws = Wn[:rows]
    t = {}
    t0 = time.perf_counter()
    abar = O.act_stats(Xn)
    t["act_stats"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    G = O.gram(Xn)
    t["gram"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    mse, best, s, _ = O.search_scale(Xn, Ws, abar, wl.w_bit, wl.group_size, wl.n_alpha, G=G)
    t["search"] = time.perf_counter() - t0
    clip_idx = None
    if wl.n_clip:
        t0 = time.perf_counter()
        Gk = O.block_grams(Xn, wl.group_size)
        t["block_grams"] = time.perf_counter() - t0
        t0 = time.perf_counter()
        clip_idx, _ = O.search_clip(Xn, Ws, s, wl.w_bit, wl.group_size, wl.n_clip, 0.5, Gk=Gk)
        t["clip"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.quant_pack(Ws, s, clip_idx, wl.w_bit, wl.group_size, max(wl.n_clip, 1), 0.5)
    t["pack"] = time.perf_counter() - t0
    scale = out / rows
    fixed = t["act_stats"] + t["gram"] + t.get("block_grams", 0.0)
    total = fixed + (t["search"] + t.get("clip", 0.0) + t["pack"]) * scale
    phases = json.dumps({k: round(v, 3) for k, v in t.items()})
    if rows == out:
        sample = (f"oracle (numpy fp64; matrix products on {oracle_threads()} BLAS threads, "
                  f"elementwise steps on one) on the whole layer, timed as it runs: "
                  f"X [{Xn.shape[0]} x {Xn.shape[1]}], all {out} output rows; phase seconds {phases}")
    else:
        sample = (f"oracle (numpy fp64, BLAS matmuls) on the full X [{Xn.shape[0]} x {Xn.shape[1]}] "
                  f"and {rows} of {out} output rows; abar, X^T X and the block Grams timed in full, "
                  f"the per-row phases (alpha search, clip search, packing) scaled by {scale:.0f}; "
                  f"phase seconds {phases}")
    return total * 1e3, sample


def run_reference(args):
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    from synthetic import WORKLOADS, workload_inputs
    wl = WORKLOADS[WORKLOAD_INDEX]
    d = workload_inputs(WORKLOAD_INDEX)
    _, X, W = d["groups"][0]
    vals, sample = [], ""
    for i in range(args.warmup + args.steps):
        ms, sample = oracle_layer_ms(X, W, wl, args.ref_row_fraction)
        if i >= args.warmup:
            vals.append(ms)
    value = statistics.mean(vals)
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(value, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded heavy-tailed X, N(0,0.02) W)",
        "config": workload_description(wl, X.shape[0], X.shape[1], W.shape[0]),
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- CUDA arm
def time_workloads(awq, torch, dev, dist, timer, local, args):
    """ms per layer of the Llama-7B-shaped MLP (gate|up jointly scaled, then
    down_proj on its SwiGLU input) and of the Llama-13B-shaped INT3 attention
    block (q|k|v jointly scaled, o_proj on its own input), each at 65536
    tokens: the groups' whole paths (act stats, alpha search, clip search
    where the workload has one, packing) run back to back as one step, with
    their candidate-GEMM flops."""
    from synthetic import WORKLOADS, workload_inputs
    res = {}
    for index in (2, 3):
        wl = WORKLOADS[index]
        groups = workload_inputs(index, device=str(dev))["groups"]
        cfg = awq.AwqConfig.make(w_bit=wl.w_bit, group_size=wl.group_size, n_alpha=wl.n_alpha,
                                 n_clip=wl.n_clip, clip_min=0.5)
        dev_groups = [(name, X.to(dev), W.to(dev)) for name, X, W in groups]
        need = max(awq.awq_workspace_size(X.shape[0], X.shape[1], W.shape[0], cfg)
                   for _, X, W in dev_groups)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)

        def step():
            for _, X, W in dev_groups:
                awq.quantize_layer(X, W, cfg, ws=ws)

        for _ in range(max(1, min(args.warmup, 3))):
            step()
        awq.awq_device_status(ws)
        steps = max(1, min(args.steps, 3))
        ms = timed_steps(step, steps, dist, timer, local)
        awq.awq_device_status(ws)
        flops = sum(2.0 * X.shape[0] * X.shape[1] * W.shape[0] * wl.n_alpha for _, X, W in dev_groups)
        res[wl.name] = {"ms_per_layer": round(ms, 3), "steps": steps,
                        "groups": {name: [int(X.shape[0]), int(X.shape[1]), int(W.shape[0])]
                                   for name, X, W in dev_groups},
                        "candidate_gemm_flops": flops,
                        "candidate_gemm_tflops_over_layer": round(flops / (ms * 1e-3) / 1e12, 1),
                        "note": wl.description}
        del dev_groups, groups, ws
        torch.cuda.empty_cache()
    # the 32-layer decoder: its first two layers, each timed with CUDA events
    # around the layer's quantisation (four groups, folds, clip, packing); the
    # fp16 forward that captures their inputs is input synthesis, untimed
    from post_weight_quantization_awq_b200 import decoder
    from synthetic import DecoderSpec, decoder_embeddings, decoder_layer_forward, decoder_layer_weights
    spec = DecoderSpec()
    cfg = awq.AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20, clip_min=0.5)
    x = decoder_embeddings(spec, device=dev)
    ws, times = None, []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.no_grad():
        for layer in range(2):
            w = decoder_layer_weights(spec, layer, device=dev)
            caps, x_next = decoder_layer_forward(x, w, spec)
            if ws is None:
                ws = decoder.workspace_for_layer(caps, w, cfg)
                decoder.quantize_layer_groups(caps, {k: v.clone() for k, v in w.items()}, cfg, ws)
            torch.cuda.synchronize(dev)
            e0.record()
            decoder.quantize_layer_groups(caps, w, cfg, ws)
            e1.record()
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
            x = x_next
    res["llama2_7b_decoder_layer"] = {
        "ms_per_layer": round(statistics.mean(times), 3), "layers_timed": len(times),
        "note": "layers 0 and 1 of the 32-layer decoder (128 x 512 calibration tokens, q|k|v, o, "
                "gate|up, down; INT4 g128, 20 alphas + 20 clip ratios, folds, packed); "
                "bench.py --workload decoder times all 32"}
    del x, ws, caps, w
    torch.cuda.empty_cache()
    return res


def run_awq(args):
    import torch
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the AWQ path has no CPU implementation)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl", world)
    import post_weight_quantization_awq_b200 as awq
    from synthetic import WORKLOADS, heavy_tailed_activations, gaussian_weight, OutlierSpec

    wl = WORKLOADS[WORKLOAD_INDEX]
    T, inn, out = wl.T, 4096, 4096
    # each rank quantises its own layer (weak scaling); rank 0 is the workload's seed
    seed = wl.seed + 1000 * rank
    X = heavy_tailed_activations(T, inn, OutlierSpec(0.01, 20.0, 50.0), seed)
    W = gaussian_weight(out, inn, seed)
    cfg = awq.AwqConfig.make(w_bit=wl.w_bit, group_size=wl.group_size, n_alpha=wl.n_alpha,
                             n_clip=wl.n_clip, clip_min=0.5)
    Xd, Wd = X.to(dev), W.to(dev)
    ws = awq.alloc_workspace(T, inn, out, cfg, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return awq.quantize_layer(Xd, Wd, cfg, ws=ws)

    # ---- device-timed region: inputs resident in HBM
    for _ in range(args.warmup):
        step()
    awq.awq_device_status(ws)
    torch.cuda.synchronize(dev)
    awq.profile_reset()
    awq.profile_enable(True)
    timer = CudaTimer(torch, stream, dev)
    with ClockSampler(local) as clk:
        ms_step = timed_steps(step, args.steps, dist, timer, local)
    awq.profile_enable(False)
    awq.awq_device_status(ws)
    kern = {}
    for name in KERNELS_PER_STEP:
        tot, n = awq.profile_read(name)
        kern[name] = (tot / n if n else None, n)
    awq.profile_reset()

    # ---- end to end through the public API: pinned host buffers in, results out.
    # Consecutive layers pipeline: a step's inputs go up on a copy stream into one
    # of two device buffers while the previous step computes, and its results go
    # down on another while the next one computes; every step still copies its
    # whole input up and its results down inside the timed region (which ends
    # with a device synchronisation).
    Xh, Wh = X.pin_memory(), W.pin_memory()
    Xe = [torch.empty_like(Xd), torch.empty_like(Xd)]
    We = [torch.empty_like(Wd), torch.empty_like(Wd)]
    copy_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)  # results go down while the next layer computes
    ready = [torch.cuda.Event(), torch.cuda.Event()]
    computed = torch.cuda.Event()
    done = [torch.cuda.Event(), torch.cuda.Event()]
    e2e_k = [0]
    e2e_first = [True]  # the first step of a region waits for everything before it
    g = wl.group_size
    host_out = {
        "qweight": torch.empty((inn, out // 8), dtype=torch.int32).pin_memory(),
        "qzeros": torch.empty((inn // g, out // 8), dtype=torch.int32).pin_memory(),
        "scales": torch.empty((inn // g, out), dtype=torch.float16).pin_memory(),
        "s_best": torch.empty(inn, dtype=torch.float32).pin_memory(),
        "mse": torch.empty(wl.n_alpha, dtype=torch.float64).pin_memory(),
        "best_idx": torch.empty(1, dtype=torch.int32).pin_memory(),
        "clip_idx": torch.empty((out, inn // g), dtype=torch.uint8).pin_memory(),
    }

    def e2e_step():
        b = e2e_k[0] % 2
        e2e_k[0] += 1
        cur = torch.cuda.current_stream(dev)
        if e2e_first[0]:  # not before the timed region starts
            copy_stream.wait_stream(cur)
            e2e_first[0] = False
        copy_stream.wait_event(done[b])  # buffer b's last reader (two steps back) is done
        with torch.cuda.stream(copy_stream):
            Xe[b].copy_(Xh, non_blocking=True)
            We[b].copy_(Wh, non_blocking=True)
            ready[b].record(copy_stream)
        cur.wait_event(ready[b])
        r = awq.quantize_layer(Xe[b], We[b], cfg, ws=ws)
        done[b].record(cur)
        computed.record(cur)
        d2h_stream.wait_event(computed)
        with torch.cuda.stream(d2h_stream):
            for k, h in host_out.items():
                t = getattr(r, k)
                t.record_stream(d2h_stream)  # not reused before its copy is done
                h.copy_(t, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        e2e_step()
    torch.cuda.synchronize(dev)
    e_steps = args.steps
    e2e_first[0] = True
    ms_e2e = timed_steps(e2e_step, e_steps, dist, timer, local,
                         before_stop=lambda: torch.cuda.current_stream(dev).wait_stream(d2h_stream))
    h2d = X.numel() * 2 + W.numel() * 2
    d2h = sum(h.numel() * h.element_size() for h in host_out.values())

    def time_form(search_form, names):
        """ms per step of the whole layer with another scoring form, and the
        average per-launch ms of the named kernels."""
        cfg_f = awq.AwqConfig.make(w_bit=wl.w_bit, group_size=wl.group_size, n_alpha=wl.n_alpha,
                                   n_clip=wl.n_clip, clip_min=0.5, search_form=search_form)
        ws_f = awq.alloc_workspace(T, inn, out, cfg_f, dev)

        def step_f():
            return awq.quantize_layer(Xd, Wd, cfg_f, ws=ws_f)

        for _ in range(args.warmup):
            step_f()
        awq.awq_device_status(ws_f)
        awq.profile_reset()
        awq.profile_enable(True)
        ms_f = timed_steps(step_f, args.steps, dist, timer, local)
        awq.profile_enable(False)
        awq.awq_device_status(ws_f)
        kf = {}
        for name in names:
            tot, n = awq.profile_read(name)
            kf[name] = tot / n if n else None
        awq.profile_reset()
        del ws_f
        return ms_f, kf

    # ---- the step after the search: the W4A16 GEMM on this layer's packed
    # output, fed the folded input X / s* (its own timing and flops)
    w4a16 = None
    if not args.no_w4a16:
        r = awq.quantize_layer(Xd, Wd, cfg, ws=ws)
        Xs = (Xd.float() / r.s_best[None, :]).half()
        Yq = torch.empty((T, out), dtype=torch.float16, device=dev)
        ws_q = torch.empty(awq.awq_w4a16_workspace_size(T, inn, out, cfg), dtype=torch.uint8, device=dev)

        def step_q():
            awq.awq_w4a16_gemm(Xs, r.qweight, r.qzeros, r.scales, cfg, Yq, ws_q)

        for _ in range(args.warmup):
            step_q()
        awq.awq_device_status(ws_q)
        ms_q = timed_steps(step_q, args.steps, dist, timer, local)
        awq.awq_device_status(ws_q)
        flops_q = 2.0 * T * inn * out
        # the same product with the weights dequantised tile by tile inside the GEMM
        ws_f = torch.empty(256, dtype=torch.uint8, device=dev)

        def step_f():
            awq.awq_w4a16_gemm(Xs, r.qweight, r.qzeros, r.scales, cfg, Yq, ws_f)

        for _ in range(args.warmup):
            step_f()
        awq.awq_device_status(ws_f)
        ms_f = timed_steps(step_f, args.steps, dist, timer, local)
        awq.awq_device_status(ws_f)
        w4a16 = {"ms": round(ms_q, 4), "tflops": round(flops_q / (ms_q * 1e-3) / 1e12, 1),
                 "flops": flops_q,
                 "note": "Y = X Wd^T with Wd = RN16((q - z) scale) from qweight/qzeros/scales, "
                         "T x in x out of the layer above: the weights dequantised once into the "
                         "workspace awq_w4a16_workspace_size asks for, then one fp16 GEMM",
                 "fused_dequant": {"ms": round(ms_f, 4),
                                   "tflops": round(flops_q / (ms_f * 1e-3) / 1e12, 1),
                                   "note": "the weights dequantised tile by tile inside the GEMM "
                                           "(256-byte workspace)"}}
        # decode-sized products (1, 8 and 16 tokens) through the workspace the
        # library asks for; the packed weights rotate over copies that
        # together exceed L2, so each step reads its weights from HBM
        wbytes = inn * out // 2 + (inn // g) * out * 2 + (inn // g) * out // 2  # codes, scales, zeros
        n_copy = max(2, -(-2 * 126 * 2 ** 20 // wbytes))
        copies = [(r.qweight.clone(), r.qzeros.clone(), r.scales.clone()) for _ in range(n_copy)]
        for td in (1, 8, 16):
            Xt = Xs[:td].contiguous()
            Yt = torch.empty((td, out), dtype=torch.float16, device=dev)
            ws_t = torch.empty(awq.awq_w4a16_workspace_size(td, inn, out, cfg), dtype=torch.uint8,
                               device=dev)
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                for c in copies[:3]:
                    awq.awq_w4a16_gemm(Xt, c[0], c[1], c[2], cfg, Yt, ws_t)
            torch.cuda.current_stream().wait_stream(side)
            awq.awq_device_status(ws_t)
            # one graph replay = one call per weight copy: a call costs a few
            # microseconds of device time, less than its host-side launch
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for c in copies:
                    awq.awq_w4a16_gemm(Xt, c[0], c[1], c[2], cfg, Yt, ws_t)
            for _ in range(args.warmup):
                graph.replay()
            ms_t = timed_steps(graph.replay, max(args.steps, 20), dist, timer, local) / n_copy
            awq.awq_device_status(ws_t)
            del graph
            xy = 2 * td * (inn + out)
            w4a16[f"decode_{td}_tokens"] = {
                "ms": round(ms_t, 5), "bytes": wbytes + xy,
                "gbs": round((wbytes + xy) / (ms_t * 1e-3) / 1e9, 1),
                "frac_hbm": round((wbytes + xy) / (ms_t * 1e-3) / 1e9 / float(load_peaks()[0]["hbm_gbs"]), 3),
                "form": "CUDA-core stream of the packed words" if td <= 8 else
                        "tcgen05 GEMM, K split over the SMs",
                "note": f"T = {td}: bound by reading the packed weights (codes, scales, zeros) "
                        f"once; device time per call from a CUDA graph of {n_copy} calls, one per "
                        "copy of the weights (together > L2), workspace awq_w4a16_workspace_size"}
            del Xt, Yt, ws_t
        del copies
        del Xs, Yq, ws_q, ws_f

    # ---- the literal fp16-output form on the same layer: Y = RN16(X W^T) once,
    # then every candidate's output scored against it in the GEMM's epilogue
    cached = None
    if not args.no_cached_form:
        ms_c, kc = time_form(awq.abi.SEARCH_CACHED_Y, ("ref_output", "search_gemm"))
        flops_c = 2.0 * T * inn * out * (wl.n_alpha + 1)
        gemm_c = (kc["ref_output"] or 0.0) + (kc["search_gemm"] or 0.0)
        cached = {"value": round(ms_c / world, 3), "unit": UNIT, "ms_per_step": round(ms_c, 3),
                  "kernels_ms": {k: round(v, 4) for k, v in kc.items() if v},
                  "algorithmic_flops_per_step": flops_c,
                  "gemm_tflops": round(flops_c / (gemm_c * 1e-3) / 1e12, 1) if gemm_c else None,
                  "note": "scores against the cached fp16 output RN16(X W^T) (one extra GEMM "
                          "with a store epilogue); candidates RN16(Qdeq/s)"}

    # ---- the fused form on the same layer: every candidate's B tile built
    # inside the scored GEMM from W (no candidate operand in HBM); the same
    # MSE bits as the direct form
    fused = None
    if not args.no_fused_form:
        ms_fu, kfu = time_form(awq.abi.SEARCH_FUSED, ("fused_params", "fused_gemm"))
        flops_fu = 2.0 * T * inn * out * wl.n_alpha
        cfg_fu = awq.AwqConfig.make(w_bit=wl.w_bit, group_size=wl.group_size, n_alpha=wl.n_alpha,
                                    n_clip=wl.n_clip, clip_min=0.5, search_form=awq.abi.SEARCH_FUSED)
        fused = {"value": round(ms_fu / world, 3), "unit": UNIT, "ms_per_step": round(ms_fu, 3),
                 "kernels_ms": {k: round(v, 4) for k, v in kfu.items() if v},
                 "algorithmic_flops_per_step": flops_fu,
                 "gemm_tflops": round(flops_fu / (kfu["fused_gemm"] * 1e-3) / 1e12, 1)
                 if kfu.get("fused_gemm") else None,
                 "workspace_bytes": awq.awq_workspace_size(T, inn, out, cfg_fu),
                 "note": "the candidates' B tiles converted from W in shared memory inside the "
                         "scored GEMM (per-group steps and zero points in the workspace), once "
                         "per 256-token tile; the same MSE bits as the direct form"}

    # ---- the same layer in the smallest workspace: the candidates built and
    # scored one at a time (the operand takes out x in fp16 instead of 20 times that)
    low_ws = None
    if not args.no_gram_form:
        nlow = awq.awq_workspace_size_min(T, inn, out, cfg)
        ws_low = torch.empty(nlow, dtype=torch.uint8, device=dev)

        def step_low():
            return awq.quantize_layer(Xd, Wd, cfg, ws=ws_low)

        for _ in range(args.warmup):
            step_low()
        awq.awq_device_status(ws_low)
        ms_low = timed_steps(step_low, max(1, min(args.steps, 5)), dist, timer, local)
        awq.awq_device_status(ws_low)
        low_ws = {"value": round(ms_low / world, 3), "unit": UNIT, "workspace_bytes": nlow,
                  "full_workspace_bytes": int(ws.numel()),
                  "note": "awq_workspace_size_min: the alpha search builds and scores one "
                          "candidate at a time; the same results bit for bit"}
        del ws_low

    # ---- the other workloads' layers (the MLP and the 13B INT3 attention
    # block), each group timed as quantize_layer runs it, with its own warm-up
    workloads = None
    if not args.no_workloads:
        workloads = time_workloads(awq, torch, dev, dist, timer, local, args)

    # ---- the Gram-form search on the same layer (same MSE, fewer flops), its
    # own timing and flop count; the headline value above is the direct form
    gram = None
    if not args.no_gram_form:
        ms_g, kg = time_form(awq.abi.SEARCH_GRAM, ("gram_full", "gram_score"))
        nb = (inn + 255) // 256  # G: the nb(nb+1)/2 upper 256x256 block pairs; scores: hi and lo
        out128 = (out + 127) // 128 * 128
        nt = inn // 128  # scores: the nt(nt+1)/2 upper 128-blocks of G~, hi and lo
        flops_g = (2.0 * T * 256 * 256 * (nb * (nb + 1) // 2)
                   + 2.0 * 2 * 128 * 128 * (nt * (nt + 1) // 2) * out128 * wl.n_alpha)
        gram = {"value": round(ms_g / world, 3), "unit": UNIT, "ms_per_step": round(ms_g, 3),
                "kernels_ms": {k: round(v, 4) for k, v in kg.items() if v},
                "executed_flops_per_step": flops_g,
                "note": "same MSE as the direct form (X^T X once, candidates scored against its "
                        "normalised fp16 hi+lo form); flops counted as executed, not the direct form's"}

    # ---- CPU baseline (rank 0 at N=1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms_cpu, sample = oracle_layer_ms(X, W, wl, args.ref_row_fraction)
        cpu = {"value": round(ms_cpu, 1), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
               "sample": sample}

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, src = load_peaks()
    flops = 2.0 * T * inn * out * wl.n_alpha
    gemm_ms = kern["search_gemm"][0]
    tflops = flops / (gemm_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"])
    launches = sum(KERNELS_PER_STEP.values()) * args.steps
    hbm = float(peaks["hbm_gbs"])
    per_kernel = {k: {"ms": round(v[0], 4) if v[0] is not None else None, "launches": v[1]}
                  for k, v in kern.items()}
    # algorithmic bytes of the HBM-bound kernels, per launch
    hbm_bytes = {"act_stats": T * inn * 2, "cand_quant": out * inn * 2 * (1 + wl.n_alpha),
                 "quant_pack": out * inn * 2 + out * inn // 2 + (inn // g) * out * 2.5}
    hbm_frac = {k: round(b / (kern[k][0] * 1e-3) / 1e9 / hbm, 3) for k, b in hbm_bytes.items()
                if kern[k][0]}
    value = ms_step / world  # whole job: world layers per step
    traffic = ncu_traffic()
    clocks = clk.summary()
    num_sms = torch.cuda.get_device_properties(local).multi_processor_count
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (seeded heavy-tailed X, N(0,0.02) W)",
        "config": workload_description(wl, T, inn, out),
        "candidate_gemm_tflops": round(tflops, 1),
        "roofline": {"kernel": "search_gemm", "bound": "tensor", "achieved": round(tflops, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(tflops / peak, 3),
                     "frac_of_burst_peak": round(tflops / float(peaks["bf16_tflops"]), 3),
                     "frac_of_nominal_peak": round(tflops / NOMINAL_PEAKS["fp16_tflops"], 3),
                     "traffic": traffic[0], "traffic_note": traffic[1],
                     "peak_source": f"{src} bf16 dense {'sustained' if 'bf16_tflops_sustained' in peaks else 'burst'} "
                                    "(fp16 has the same nominal rate)",
                     "algorithmic_flops_per_launch": flops},
        "hbm_kernels": {"peak_gbs": hbm, "frac": hbm_frac, "bytes_per_launch": hbm_bytes,
                        "frac_of_nominal": {k: round(v * hbm / NOMINAL_PEAKS["hbm_gbs"], 3)
                                            for k, v in hbm_frac.items()},
                        "cand_quant_issue": cand_quant_issue(kern["cand_quant"][0], clocks.get("sm_mhz"),
                                                             num_sms)},
        "kernels": per_kernel,
        "clocks": clocks,
        "e2e": {"value": round(ms_e2e / world, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e_steps,
                "note": "quantize_layer on inputs copied from pinned host memory every step and "
                        "results copied back every step; consecutive layers pipeline (a step's "
                        "upload runs on a copy stream, into one of two buffers, while the "
                        "previous layer computes, and its results go down on another stream "
                        "while the next one computes; the timed region waits for the last)"},
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "gram_form": gram,
        "cached_output_form": cached,
        "fused_form": fused,
        "w4a16_gemm": w4a16,
        "workloads": workloads,
        "smallest_workspace": low_ws,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_decoder(args):
    """Times the layer-by-layer AWQ of the 32-layer Llama-2-7B-architecture
    decoder (128 x 512 calibration tokens): per layer the four groups' alpha
    searches, the folds, the clip searches and the packing.  The fp16 forward
    that captures each layer's inputs is input synthesis and is not timed.
    --steps = layers quantised by the whole job (at most 32).  With N GPUs the
    layers split into N contiguous blocks (decoder.layer_block), one per rank,
    with no collective on the data path: each rank runs the untimed fp16
    forward up to its first layer, then quantises its block, each layer timed
    with CUDA events; the job's time is the max over ranks of the summed layer
    times (strong scaling: the layer count is fixed)."""
    import torch
    import post_weight_quantization_awq_b200 as awq
    from post_weight_quantization_awq_b200 import decoder
    from synthetic import DecoderSpec, decoder_embeddings, decoder_layer_forward, decoder_layer_weights
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl", world)
    spec = DecoderSpec()
    cfg = awq.AwqConfig.make(w_bit=4, n_alpha=20, n_clip=20, clip_min=0.5)
    layers = min(args.steps, spec.layers)
    block = decoder.layer_block(rank, world, layers)
    x = decoder_embeddings(spec, device=dev)
    with torch.no_grad():  # untimed: the fp16 forward up to this rank's first layer
        for layer in range(block.start):
            w = decoder_layer_weights(spec, layer, device=dev)
            _, x = decoder_layer_forward(x, w, spec)
    ws = None
    times, summaries = [], []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, local)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for layer in block:
            w = decoder_layer_weights(spec, layer, device=dev)
            caps, x_next = decoder_layer_forward(x, w, spec)
            if ws is None:
                ws = decoder.workspace_for_layer(caps, w, cfg)
                for _ in range(args.warmup):  # warm-up on copies of the first layer
                    decoder.quantize_layer_groups(caps, {k: v.clone() for k, v in w.items()}, cfg, ws)
            torch.cuda.synchronize(dev)
            e0.record()
            res = decoder.quantize_layer_groups(caps, w, cfg, ws)
            e1.record()
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
            summaries.append(decoder.layer_summary(layer, res))
            x = x_next
    barrier(dist, local)
    torch.cuda.synchronize(dev)
    rank_ms = sum(times)
    job_ms = max_over_ranks(rank_ms, dist)
    all_layers = decoder.gather_summaries(summaries, dist)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    flops_layer = 2.0 * spec.seq * spec.n_seq * cfg.n_alpha * spec.hidden * (
        3 * spec.hidden + spec.hidden + 2 * spec.ffn) + 2.0 * spec.seq * spec.n_seq * cfg.n_alpha * spec.ffn * spec.hidden
    value = job_ms / layers  # whole job: ms per layer
    print(json.dumps({
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": layers,
        "warmup": args.warmup, "ms_per_step": round(job_ms / max(1, len(block)), 3),
        "higher_is_better": False, "scaling": "strong" if world > 1 else "weak",
        "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (random-init decoder, random token ids, outlier embedding channels)",
        "config": {"workload": "llama2_7b_decoder_32_layers: hidden 4096, 32 heads, MLP 11008, "
                               "128 x 512 calibration tokens, four groups per layer (q|k|v, o, gate|up, "
                               "down), INT4 g128, 20 alphas + 20 clip ratios, folds, packed",
                   "layers": layers, "parallelism": f"layer blocks over {world} GPU(s)",
                   "forward_capture": "untimed",
                   "timing": "CUDA events around each layer's quantisation, summed per rank, "
                             "max over ranks"},
        "candidate_gemm_tflops": round(flops_layer * layers / (job_ms * 1e-3) / 1e12, 1),
        "rank0_ms_per_layer_min_max": [round(min(times), 3), round(max(times), 3)] if times else None,
        "clocks": clk.summary(),
        "layers_summary": [{"layer": d["layer"], **{g: d[g]["best_idx"] for g in ("qkv", "o", "gate_up", "down")}}
                           for d in all_layers],
    }), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("awq", "reference"), default="awq")
    ap.add_argument("--ref-row-fraction", type=float, default=1.0,
                    help="share of output rows the oracle runs on (1 = the whole layer; "
                         "below 1 the per-row phases are scaled up)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gram-form", action="store_true",
                    help="skip the extra measurement of the Gram-form search")
    ap.add_argument("--no-cached-form", action="store_true",
                    help="skip the extra measurement of the cached fp16-output form")
    ap.add_argument("--no-fused-form", action="store_true",
                    help="skip the extra measurement of the fused-candidate form")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the timing of the MLP and 13B-attention layers")
    ap.add_argument("--no-w4a16", action="store_true",
                    help="skip the measurement of the W4A16 GEMM on the packed output")
    ap.add_argument("--workload", choices=("q_proj", "decoder"), default="q_proj",
                    help="q_proj: the headline workload; decoder: the 32-layer decoder "
                         "(--steps = layers timed)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "decoder":
        return run_decoder(args)
    return run_awq(args)


if __name__ == "__main__":
    sys.exit(main())
