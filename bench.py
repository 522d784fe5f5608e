#!/usr/bin/env python
"""Benchmark of the routed-MoE layer stack over a shared LRU expert cache.

Headline workload (one step = one decode token through every MoE layer): the
DeepSeek-V4-Flash shapes, 8 MoE layers, 256 routed experts, hidden 4096, SwiGLU
intermediate 2048, top-6 sigmoid gating normalised over the selected experts,
plus one always-on shared expert; bf16 weights N(0, 0.02); the 103 GB expert pool
in pinned host memory; 512 HBM slots (25% of the routed experts) as one LRU shared
by the layers; hidden states from an AR(1) process x_t = 0.9 x_{t-1} + 0.436 eps_t
(routing locality), batch 1.  Synthetic data stands in for the agent workloads and
replayed traces of the FreeToken pages ("FreeToken linux", performance: DeepSeek-V4-
Flash decode on one RTX 5090).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--legs ...]

The one JSON line (rank 0) carries:
  - value: decode tokens/s of the headline workload, timed on the device with CUDA
    events (max over ranks), inputs resident in HBM;
  - e2e: the same tokens from the same cache state (the cache is emptied and the
    warm-up replayed), through pinned host buffers with the H2D of each token and the
    D2H of its layer outputs inside the timed region;
  - roofline: the dominant kernel (the decode gate/up expert GEMV, HBM-bound), from
    CUDA events around its launches in a stage-timed replay of the same tokens;
  - cache miss rate, H2D fill bandwidth against the measured host link, the
    cold-start figure of the warm-up steps, SM clocks sampled during the timed region,
    the CPU oracle timed on a bounded sample;
  - legs (N = 1 only): "int4-large-pool" decode at batch 1 (16 layers, H=7168, int4
    g128, 15% cached), and at batch 8 and 32 before and after the stated growth of the
    cache from 15% to 30%; "prefill" of the headline shapes (4096 tokens through the 8
    layers with whole-layer double buffering over PCIe, the same with every expert
    resident, a tensor-pipe sweep of one resident layer at 16k/32k/64k tokens, and one
    layer with NVFP4 weights, every expert resident, with its decode GEMVs at batch 1 and
    8 on the tensor cores and on the fp32 pipes); "shrink": decode
    tokens/s before and after shrinking the cache from 58% to 40% of the experts ("this
    tool runs datacenter AI on your PC", the cache shrink demo).
--impl reference times the CPU oracle alone on the headline workload.
N > 1 runs independent replicas (one stack per GPU, its own token chain, the
headline legs only): the path has no exchange step.
"""
import argparse
import concurrent.futures
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

HEADLINE = "dsv4flash-decode-bf16"
INT4 = "int4-large-pool"
PREFILL = "dsv4flash-prefill-bf16"
SHRINK = "decode-locality-bf16"
SHRINK_FROM, SHRINK_TO = 0.58, 0.40          # the pages' demo: 58% -> 40% of the model cached
SWEEP_TOKENS = (16384, 32768, 65536)
METRIC = "routed-MoE tokens/s (decode, prefill) and expert-weight HBM GB/s vs peak"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ALL_LEGS = ("int4", "prefill", "shrink")


def workload_desc(cfg, batch=1):
    return {
        "workload": "%s: %d MoE layers, E=%d, H=%d, I=%d, top-%d %s%s, %s weights, %d cache slots "
                    "(%.0f%% of experts), %s tokens, batch %d, decode" % (
                        cfg.name, cfg.L, cfg.E, cfg.H, cfg.I, cfg.k, cfg.gating,
                        " + 1 shared expert" if cfg.shared else "", cfg.wdtype, cfg.C,
                        100.0 * cfg.C / (cfg.L * cfg.E), "AR(1)" if cfg.process == "ar1" else "N(0,1)", batch),
        "layers": cfg.L, "experts": cfg.E, "hidden": cfg.H, "inter": cfg.I, "top_k": cfg.k,
        "shared_expert": bool(cfg.shared), "cache_slots": cfg.C, "batch": batch,
        "step": "one decode token through all layers",
        "l2": "not flushed: each step streams ~%d MB of expert weights, above the 126 MB L2"
              % round(cfg.L * ((cfg.k + cfg.shared) * cfg.blob_bytes + cfg.E * cfg.H * 4) / 1e6),
    }


def headline_config(world):
    return dict(workload_desc(synth.CONFIGS[HEADLINE]), parallelism="replicas x%d" % world)


# DRAM traffic per kernel from ncu captures: dram__bytes_read.sum + dram__bytes_write.sum of
# the kernel's launches divided by their algorithmic bytes.  A figure holds only while the
# kernel's sources hash to `sha256`; otherwise the line carries traffic null.
TRAFFIC = {
    "gemv_bf16": {"sources": ["moe_expert_offload_top_b200/csrc/decode_gemv.cuh",
                              "moe_expert_offload_top_b200/csrc/expert_decode.cu"],
                  "sha256": "9cd1211ebda91b779c1d2e915539c28360cdb91dcac741dc28e5b2f8e593c40d", "ratio": 1.00208,
                  "capture": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the 8 gate/up launches of "
                             "kernel_driver --workload dsv4flash-decode-bf16 --layers 1 --experts 16 --steps 8 "
                             "--perf (7 experts per launch, as here), 1.00208 of their algorithmic bytes; scaled "
                             "to the average launch here"},
    "gemv_int4": {"sources": ["moe_expert_offload_top_b200/csrc/decode_gemv.cuh",
                              "moe_expert_offload_top_b200/csrc/gemv_ring.cuh",
                              "moe_expert_offload_top_b200/csrc/gemv_int4_mma.cu"],
                  "sha256": "62989051d67e993764abb8f984f9a3d18c7df12b4686ef0e1949db6e16cd68ec", "ratio": 1.00158,
                  "capture": "ncu dram__bytes_read.sum + dram__bytes_write.sum of int4_prep_x_kernel + the gate/up "
                             "int4_i8_kernel of the 8 forwards of kernel_driver --workload int4-large-pool --layers 1 "
                             "--experts 64 --steps 8 --perf (8 experts per launch, as here), 1.00158 of their "
                             "algorithmic bytes; scaled to the average launch here"},
    "gemm": {"sources": ["moe_expert_offload_top_b200/csrc/grouped_gemm_sm100.cu"],
             "sha256": "0507ce91301990d38f67cede0ff1f116891de1794c23254f95a46243e0b318f6", "ratio": 1.03732,
             "capture": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the gate/up and down launches of "
                        "kernel_driver --workload dsv4flash-prefill-bf16 --layers 1 --experts 64 --tokens 8192 "
                        "--steps 2 --perf (768 pairs per expert, compute-bound like the sweep), 1.03732 of their "
                        "algorithmic bytes; scaled to the swept forward's bytes"},
}


def kernel_traffic(key, bytes_per_launch):
    t = TRAFFIC[key]
    h = hashlib.sha256()
    for rel in t["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if t["ratio"] is None or h.hexdigest() != t["sha256"]:
        return None, "no ncu capture of these kernel sources (sha256 %s)" % h.hexdigest()[:12]
    return t["ratio"] * bytes_per_launch, t["capture"]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def token_chain(cfg, chain, n):
    x = synth.ar1_chain(cfg.seed, chain, n, cfg.H)
    bits = synth.round_bf16(x)
    return (bits.astype(np.uint32) << 16).view(np.float32), bits


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                p = [v.strip() for v in ln.split(",")]
                if len(p) >= 7 and p[0].isdigit():
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [int(r[0]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": int(rows[0][1]), "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ distributed --

def dist_setup(n_gpus):
    """torchrun environment -> (rank, world, local_rank).  One process per GPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if os.environ.get("FT_BENCH_BACKEND", "nccl") == "nccl" else "gloo"
        if backend == "nccl":
            import torch
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def aggregate(tokens, seconds, device=None):
    """Whole-job throughput over replicas: total tokens of all ranks / the slowest
    rank's time.  Returns (total_tokens, max_seconds)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return tokens, seconds
    t = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    s = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    dist.all_reduce(s, op=dist.ReduceOp.MAX)
    return t.item(), s.item()


def host_memory_short(pool_bytes, replicas_on_node):
    """None when this node's available memory holds the replicas' pinned pools (with 10%
    to spare), else the reason.  Read before any rank allocates."""
    try:
        with open("/proc/meminfo") as f:
            avail = next(int(l.split()[1]) * 1024 for l in f if l.startswith("MemAvailable:"))
    except Exception:
        return None
    need = pool_bytes * replicas_on_node
    if need <= 0.9 * avail:
        return None
    return ("host memory: %d replicas on this node need %.0f GB of pinned expert pool, %.0f GB available"
            % (replicas_on_node, need / 1e9, avail / 1e9))


def agree_any(flag, device=None):
    """True on every rank if it is true on any rank (one collective, taken by all)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return flag
    t = torch.tensor([1.0 if flag else 0.0], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item() > 0


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


# ----------------------------------------------------------- CPU oracle leg --

def oracle_cores():
    try:
        import threadpoolctl
        return max([p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()] or [1])
    except Exception:
        return 1


def cpu_oracle_rate(cfg, vals, blob_of, budget_s=20.0, max_tokens=None, max_layers=None):
    """Decode tokens/s of the CPU oracle on a bounded sample of a decode workload: the
    tokens of `vals` ([n, H], batch 1) go through the layers in order (router, top-k,
    gates, LRU, expert FFN, combine) until the time budget is spent (checked after
    each layer) or max_tokens tokens / max_layers layers are done.  The rate counts
    finished layers: tokens/s = layers / seconds / L.  Returns (rate, layers, seconds)."""
    from oracle import lru as olru
    from oracle import moe
    routers = [synth.router_weights(cfg, l) for l in range(cfg.L)]
    shared = {l: synth.expert_blob(cfg, l, 0, shared=True) for l in range(cfg.L)} if cfg.shared else {}
    c = olru.SharedLru(cfg.C)
    layers = 0
    t0 = time.perf_counter()
    for s in range(len(vals)):
        x = vals[s:s + 1]
        for l in range(cfg.L):
            r = moe.route(x, routers[l], cfg.k, cfg.gating)
            c.access_set(s * cfg.L + l, l, moe.selected_set(r["ids"]))
            moe.experts_and_combine(x, r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H, cfg.I,
                                    lambda e, l=l: blob_of(l, e), shared.get(l))
            layers += 1
            if time.perf_counter() - t0 > budget_s or (max_layers and layers >= max_layers):
                break
        else:
            if max_tokens and s + 1 >= max_tokens:
                break
            continue
        break
    dt = time.perf_counter() - t0
    return layers / dt / cfg.L, layers, dt


def prebuilt_blobs(cfg, vals, n_layers_max):
    """The blobs the oracle will read for the first n_layers_max (token, layer) steps of
    vals, generated before any timing (on all host cores)."""
    from oracle import moe
    keys = set()
    done = 0
    for s in range(len(vals)):
        for l in range(cfg.L):
            if done >= n_layers_max:
                break
            r = moe.route(vals[s:s + 1], synth.router_weights(cfg, l), cfg.k, cfg.gating)
            keys.update((l, int(e)) for e in moe.selected_set(r["ids"]))
            done += 1
    keys = sorted(keys)
    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        blobs = dict(zip(keys, ex.map(lambda k: synth.expert_blob(cfg, k[0], k[1]), keys)))
    return blobs


# ------------------------------------------------------------ reference arm --

def run_reference(args):
    """The CPU oracle alone on the headline workload: its decode tokens/s over the
    timed chain, every blob it reads generated before the timing starts."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    cfg = synth.CONFIGS[HEADLINE]
    W, K = args.warmup, args.steps
    vals, _ = token_chain(cfg, 0, W + K)
    # a warm-up token (untimed), then the timed tokens until the budget is spent; one oracle
    # token takes seconds, so both are bounded
    n_warm = 1
    n_timed = max(1, min(K, args.reference_max_tokens))
    warm_vals, timed_vals = vals[W - n_warm:W], vals[W:W + n_timed]
    blobs = prebuilt_blobs(cfg, np.concatenate([warm_vals, timed_vals]), (n_warm + n_timed) * cfg.L)
    cpu_oracle_rate(cfg, warm_vals, lambda l, e: blobs[(l, e)], budget_s=60.0, max_tokens=n_warm)
    rate, layers, dt = cpu_oracle_rate(cfg, timed_vals, lambda l, e: blobs[(l, e)],
                                       budget_s=args.reference_budget_s, max_tokens=n_timed)
    cores = oracle_cores()
    sample = ("CPU oracle (float64 numpy), decode tokens %d.. of the timed chain: %d (token, layer) steps "
              "of %d layers in %.1f s (budget %.0f s), the blobs they read generated before timing"
              % (W, layers, cfg.L, dt, args.reference_budget_s))
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": K, "warmup": W, "ms_per_step": 1e3 / rate,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,0.02) weights, AR(1) hidden states)",
            "config": headline_config(world),
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- decode legs --

def timed_steps(stack, xs, out, stream, dev):
    """Runs the steps xs[i] ([B, H] on the device) on `stream`; CUDA-event seconds."""
    import torch
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for x in xs:
        stack.step(x, out, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) * 1e-3


def replay_warmup(stack, xs, out, stream, dev):
    """Empties the cache and replays the warm-up steps: the LRU is deterministic, so the
    cache then holds exactly what it held after the first warm-up."""
    import torch

    import moe_expert_offload_top_b200 as ft
    ft.ft_cache_clear(stack.h)
    for x in xs:
        stack.step(x, out, stream)
    torch.cuda.synchronize(dev)


def decode_legs(stack, cfg, W, K, chain, dev, clocks_index=None, sync_ranks=False):
    """Decode of W warm-up steps (from an empty cache) and K timed steps of one token,
    three times over the same tokens from the same cache state: device-timed (inputs in
    HBM, no instrumentation), stage-timed (CUDA events around every kernel), and end to
    end through pinned host buffers."""
    import torch

    import moe_expert_offload_top_b200 as ft
    batch = 1
    _, bits = token_chain(cfg, chain, W + K)
    bits = bits.reshape(W + K, 1, cfg.H)
    x_dev = torch.from_numpy(bits).view(torch.bfloat16).to(dev)
    out = torch.empty((cfg.L, batch, cfg.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    warm, timed = list(x_dev[:W]), list(x_dev[W:])

    ft.ft_cache_clear(stack.h)
    stack.reset_stats()
    cold_dt = timed_steps(stack, warm, out, stream, dev)
    cold_st = stack.stats()

    # ---- device-timed leg
    stack.reset_stats()
    ft.ft_moe_reset_perf(stack.h)
    clocks = ClockSampler(clocks_index) if clocks_index is not None else None
    if clocks:
        clocks.start()
    if sync_ranks:
        barrier(dev)
    dt = timed_steps(stack, timed, out, stream, dev)
    if sync_ranks:
        barrier(dev)
    clk = clocks.stop() if clocks else None
    perf_dev = ft.ft_moe_perf(stack.h)
    st = stack.stats()

    # ---- stage leg: the same tokens from the same cache state, CUDA events per kernel
    replay_warmup(stack, warm, out, stream, dev)
    ft.ft_moe_reset_perf(stack.h)
    ft.ft_moe_set_stage_timing(stack.h, 1)
    for x in timed:
        stack.step(x, out, stream)
    torch.cuda.synchronize(dev)
    perf = ft.ft_moe_perf(stack.h)
    ft.ft_moe_set_stage_timing(stack.h, 0)

    # ---- end-to-end leg: the same tokens from the same cache state, through pinned host
    # buffers: the H2D of each step's tokens and the D2H of its layer outputs, every step
    replay_warmup(stack, warm, out, stream, dev)
    stack.reset_stats()
    x_host = torch.from_numpy(bits[W:]).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((K, cfg.L, batch, cfg.H), dtype=torch.bfloat16).pin_memory()
    x_in = torch.empty((batch, cfg.H), dtype=torch.bfloat16, device=dev)
    if sync_ranks:
        barrier(dev)
    torch.cuda.synchronize(dev)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for s in range(K):
        x_in.copy_(x_host[s], non_blocking=True)
        stack.step(x_in, out, stream)
        out_host[s].copy_(out, non_blocking=True)
        stream.synchronize()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_dt = a0.elapsed_time(a1) * 1e-3
    st_e2e = stack.stats()
    return {"dt": dt, "cold_dt": cold_dt, "cold_st": cold_st, "st": st, "perf_dev": perf_dev, "perf": perf,
            "e2e_dt": e2e_dt, "st_e2e": st_e2e, "clocks": clk,
            "h2d_bytes_per_step": int(cfg.H * 2 * batch), "d2h_bytes_per_step": int(cfg.L * cfg.H * 2 * batch)}


def gemv_roofline(perf, peaks, peak_src, key, kernel_name):
    """Roofline of the decode gate/up GEMV (the dominant kernel) from stage-timed launches."""
    gu_s = perf["ffn_gate_up_ms"] * 1e-3
    gl = max(perf["ffn_gate_up_launches"], 1)
    achieved = perf["ffn_gate_up_bytes"] / gu_s / 1e9 if gu_s > 0 else None
    bpl = perf["ffn_gate_up_bytes"] / gl
    traffic, src = kernel_traffic(key, bpl)
    d_s = perf["ffn_down_ms"] * 1e-3
    down = perf["ffn_down_bytes"] / d_s / 1e9 if d_s > 0 else None
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"] if achieved else None, "traffic": traffic,
            "peak_source": peak_src + " hbm_gbs (copy bandwidth)", "kernel": kernel_name,
            "bytes_per_launch": bpl, "avg_launch_us": 1e6 * gu_s / gl,
            "launches_per_forward": gl / max(perf["timed_forwards"], 1), "traffic_source": src,
            "down_proj": {"achieved": down, "frac": down / peaks["hbm_gbs"] if down else None,
                          "bytes_per_launch": perf["ffn_down_bytes"] / gl, "avg_launch_us": 1e6 * d_s / gl}}


def cache_summary(st, link_h2d=None):
    gbs = st["h2d_bytes"] / st["h2d_seconds"] / 1e9 if st["h2d_seconds"] > 0 else None
    d = {"miss_rate": st["misses"] / max(st["routed"], 1), "routed": st["routed"], "misses": st["misses"],
         "h2d_bytes": st["h2d_bytes"], "h2d_gbs": gbs, "capacity": st["capacity"]}
    if link_h2d:
        d["h2d_frac_of_link"] = gbs / link_h2d if gbs else None
    return d


# ---------------------------------------------------------------- int4 leg --

def int4_leg(args, dev, peaks, peak_src, link_h2d):
    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack
    cfg = synth.CONFIGS[INT4]
    t0 = time.perf_counter()
    stack = GpuStack(cfg, device=dev)
    setup_s = time.perf_counter() - t0
    try:
        r = decode_legs(stack, cfg, args.warmup, args.int4_steps, 0, dev, clocks_index=dev.index)
        res = {"workload": workload_desc(cfg)["workload"], "value": args.int4_steps / r["dt"], "unit": "tokens/s",
               "steps": args.int4_steps, "warmup": args.warmup, "ms_per_step": 1e3 * r["dt"] / args.int4_steps,
               "e2e": {"value": args.int4_steps / r["e2e_dt"], "unit": "tokens/s",
                       "h2d_bytes_per_step": r["h2d_bytes_per_step"], "d2h_bytes_per_step": r["d2h_bytes_per_step"]},
               "gpu_launches": int(r["perf_dev"]["kernel_launches"]), "clocks": r["clocks"],
               "roofline": gemv_roofline(r["perf"], peaks, peak_src, "gemv_int4",
                                         "int4_prep_x_kernel + int4_i8_kernel<0> (int4 g128 expert gate/up + SwiGLU, "
                                         "int8 mma.sync m16n8k32, decode)"),
               "cache": cache_summary(r["st"], link_h2d),
               "cold_start": {"value": args.warmup / r["cold_dt"], "unit": "tokens/s",
                              "miss_rate": r["cold_st"]["misses"] / max(r["cold_st"]["routed"], 1)},
               "stages_us_per_forward": stage_us(r["perf"]), "pool_setup_s": setup_s,
               "note": "fixed capacity (no resize inside the timed steps)"}
        if args.int4_batch_steps > 0:
            res["batches"] = int4_batches(args, stack, cfg, dev)
        if not args.no_cpu_baseline:
            vals, _ = token_chain(cfg, 0, args.warmup + 1)
            rate, layers, cdt = cpu_oracle_rate(cfg, vals[args.warmup:], stack.pool_blob,
                                                budget_s=args.cpu_budget_s, max_layers=cfg.L)
            res["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                                   "sample": "decode token %d of the timed chain through %d of its %d layers "
                                             "(float64 numpy oracle, %.1f s), scaled to the whole stack"
                                             % (args.warmup, layers, cfg.L, cdt)}
    finally:
        stack.close()
    return res


def int4_batches(args, stack, cfg, dev):
    """The int4-large-pool workload at decode batch 8 and 32 (independent AR(1) chains), with
    the stated mid-run cache resize: steps at 15% of the experts, then at 30% after growing
    the cache at a safe point.  Device-timed with CUDA events, a few steps per point (a step
    at batch 32 reads several hundred experts over PCIe)."""
    import torch

    import moe_expert_offload_top_b200 as ft
    stream = torch.cuda.current_stream(dev)
    res = {}
    K, W = args.int4_batch_steps, 2
    for B in (8, 32):
        vals, bits = synth.tokens(cfg, B)
        x = torch.from_numpy(bits[:W + 2 * K]).view(torch.bfloat16).to(dev)
        out = torch.empty((cfg.L, B, cfg.H), dtype=torch.bfloat16, device=dev)
        stack.resize(cfg.C)
        ft.ft_cache_clear(stack.h)
        timed_steps(stack, list(x[:W]), out, stream, dev)
        pts = {}
        for label, lo in (("slots_15pct", W), ("slots_30pct", W + K)):
            if label == "slots_30pct":
                stack.resize(cfg.resize_to)
            stack.reset_stats()
            dt = timed_steps(stack, list(x[lo:lo + K]), out, stream, dev)
            st = stack.stats()
            pts[label] = {"cache_slots": stack.C, "tokens_per_s": B * K / dt, "ms_per_step": 1e3 * dt / K,
                          "miss_rate": st["misses"] / max(st["routed"], 1),
                          "h2d_gbs": st["h2d_bytes"] / st["h2d_seconds"] / 1e9 if st["h2d_seconds"] > 0 else None}
        res["batch_%d" % B] = dict(steps=K, warmup=W, **pts)
    stack.resize(cfg.C)
    return res


def stage_us(perf):
    fwd = max(perf["timed_forwards"], 1)
    return {k: 1e3 * perf[k + "_ms"] / fwd for k in ("router", "permute", "ffn_gate_up", "ffn_down", "combine")}


# ------------------------------------------------------------- prefill leg --

def prefill_leg(args, stack, dev, peaks, peak_src):
    """Prefill of the headline shapes on the headline stack (same weights): 4096 N(0,1)
    tokens through the 8 layers in prefill mode, with 512 slots (whole-layer double
    buffering over PCIe) and with every expert resident (2048 slots); then one resident
    layer at growing token counts, where the grouped GEMMs become compute-bound."""
    import torch

    import moe_expert_offload_top_b200 as ft
    cfg = synth.CONFIGS[PREFILL]
    T = cfg.tokens
    Tmax = max(SWEEP_TOKENS) if args.sweep else T
    stream = torch.cuda.current_stream(dev)
    xall = synth.normal_f32(cfg.seed, synth.T_TOKENS, 0, 0, Tmax * cfg.H, 1.0).reshape(Tmax, cfg.H)
    x_dev = torch.from_numpy(synth.round_bf16(xall)).view(torch.bfloat16).to(dev)
    del xall
    out = torch.empty((cfg.L, T, cfg.H), dtype=torch.bfloat16, device=dev)
    out_sweep = torch.empty((Tmax, cfg.H), dtype=torch.bfloat16, device=dev) if args.sweep else None
    ft.ft_moe_set_mode(stack.h, 1)
    ft.ft_moe_reserve(stack.h, Tmax)
    res = {"workload": "%s: %d layers, E=%d, H=%d, I=%d, top-%d %s + shared expert, bf16, %d N(0,1) tokens, "
                       "prefill" % (cfg.name, cfg.L, cfg.E, cfg.H, cfg.I, cfg.k, cfg.gating, T)}

    def gemm_figures(perf):
        gemm_s = (perf["ffn_gate_up_ms"] + perf["ffn_down_ms"]) * 1e-3
        byts = perf["ffn_gate_up_bytes"] + perf["ffn_down_bytes"]
        tf = perf["ffn_flops"] / gemm_s / 1e12 if gemm_s > 0 else None
        gbs = byts / gemm_s / 1e9 if gemm_s > 0 else None
        return {"kernel": "grouped_gemm_kernel<0>+<1> (tcgen05 kind::f16, TMEM, TMA)",
                "ms_per_forward": 1e3 * gemm_s / max(perf["timed_forwards"], 1), "tflops": tf, "gbs": gbs,
                "tensor_frac_sustained": tf / peaks["bf16_tflops_sustained"] if tf else None,
                "tensor_frac_burst": tf / peaks["bf16_tflops"] if tf else None,
                "hbm_frac": gbs / peaks["hbm_gbs"] if gbs else None,
                "intensity_flop_per_byte": perf["ffn_flops"] / byts if byts > 0 else None,
                "flops_per_forward": perf["ffn_flops"] / max(perf["timed_forwards"], 1),
                "bytes_per_forward": byts / max(perf["timed_forwards"], 1)}

    def run(x, layers, passes, out_of):
        for l in layers:                                  # warm-up pass
            stack.forward(l, x, out_of(l))
        ft.ft_moe_sync(stack.h)
        stack.reset_stats()
        dt = 0.0
        for _ in range(passes):
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for l in layers:
                stack.forward(l, x, out_of(l))
            e1.record(stream)
            torch.cuda.synchronize(dev)
            dt += e0.elapsed_time(e1) * 1e-3
        ft.ft_moe_sync(stack.h)
        st = stack.stats()
        # one more pass, stage-timed, for the GEMM figures
        ft.ft_moe_reset_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 1)
        for l in layers:
            stack.forward(l, x, out_of(l))
        torch.cuda.synchronize(dev)
        perf = ft.ft_moe_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 0)
        return dt, st, perf

    xs = x_dev[:T]
    for label, slots in (("offload", cfg.C), ("resident", cfg.L * cfg.E)):
        stack.resize(slots)
        ft.ft_cache_clear(stack.h)
        dt, st, perf = run(xs, range(cfg.L), args.prefill_passes, lambda l: out[l])
        res[label] = {"cache_slots": slots, "passes": args.prefill_passes,
                      "tokens_per_s": T * args.prefill_passes / dt,
                      "ms_per_layer": 1e3 * dt / (args.prefill_passes * cfg.L),
                      "routed_misses": st["misses"], "prefetch_misses": st["prefetch_misses"],
                      "h2d_gbs": st["h2d_bytes"] / st["h2d_seconds"] / 1e9 if st["h2d_seconds"] > 0 else None,
                      "grouped_gemm": gemm_figures(perf), "stages_ms_per_layer": {
                          k: v / 1e3 for k, v in stage_us(perf).items()}}
    if args.sweep:
        sweep = []
        for Ts in SWEEP_TOKENS:
            dt, st, perf = run(x_dev[:Ts], [0], args.prefill_passes, lambda l, Ts=Ts: out_sweep[:Ts])
            sweep.append({"tokens": Ts, "layer_ms": 1e3 * dt / args.prefill_passes,
                          "grouped_gemm": gemm_figures(perf)})
        res["sweep_one_resident_layer"] = sweep
        top = max(sweep, key=lambda s: s["grouped_gemm"]["tflops"] or 0)["grouped_gemm"]
        traffic, src = kernel_traffic("gemm", top["bytes_per_forward"])
        res["roofline"] = {"bound": "tensor", "achieved": top["tflops"], "peak": peaks["bf16_tflops_sustained"],
                           "unit": "TFLOP/s", "frac": top["tensor_frac_sustained"], "traffic": traffic,
                           "traffic_source": src,
                           "peak_source": peak_src + " bf16_tflops_sustained (cuBLAS bf16, seconds-long loop)",
                           "kernel": top["kernel"], "at_tokens": max(sweep, key=lambda s: s["grouped_gemm"]["tflops"]
                                                                      or 0)["tokens"]}
    if args.nvfp4:
        res["nvfp4_resident"] = nvfp4_prefill(args, dev, peaks, x_dev[:T], res["resident"]["ms_per_layer"],
                                              gemm_figures)
    if not args.no_cpu_baseline:
        # the oracle on the first layer of the prompt (every expert of the layer is read)
        from oracle import moe
        vals = (synth.round_bf16(synth.normal_f32(cfg.seed, synth.T_TOKENS, 0, 0, T * cfg.H, 1.0))
                .astype(np.uint32) << 16).view(np.float32).reshape(T, cfg.H)
        t0 = time.perf_counter()
        moe.moe_layer(vals, synth.router_weights(cfg, 0), cfg.k, cfg.gating, cfg.wdtype, cfg.H, cfg.I,
                      lambda e: stack.pool_blob(0, e), stack.shared_blobs[0])
        cdt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": T / (cdt * cfg.L), "unit": "tokens/s", "cores": oracle_cores(),
                               "kind": "oracle", "sample": "the %d-token prompt through layer 0 of %d (float64 "
                                                           "numpy oracle, %.1f s), scaled to the whole stack"
                                                           % (T, cfg.L, cdt)}
    return res


def nvfp4_prefill(args, dev, peaks, x, bf16_ms_per_layer, gemm_figures):
    """The prefill shapes with NVFP4 expert weights (e2m1 codes, an e4m3 scale per 16
    elements, an fp32 scale per matrix; "FreeToken linux", performance: the NVFP4 4-bit
    release), every expert resident: the GEMMs expand each weight tile to bf16 in shared
    memory.  One layer (its 256 experts: generating NVFP4 blobs is slow on the host)."""
    import dataclasses

    import torch

    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack
    base = synth.CONFIGS[PREFILL]
    cfg = dataclasses.replace(base, name="dsv4flash-prefill-nvfp4", wdtype="nvfp4", L=1, C=base.E)
    T = x.shape[0]
    t0 = time.perf_counter()
    stack = GpuStack(cfg, device=dev, max_tokens=T)
    setup_s = time.perf_counter() - t0
    stream = torch.cuda.current_stream(dev)
    out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    try:
        stack.forward(0, x, out, stream)              # warm-up (and the one-time prefetch of layer 0)
        ft.ft_moe_sync(stack.h)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.prefill_passes):
            stack.forward(0, x, out, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        dt = e0.elapsed_time(e1) * 1e-3 / args.prefill_passes
        ft.ft_moe_reset_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 1)
        stack.forward(0, x, out, stream)
        torch.cuda.synchronize(dev)
        perf = ft.ft_moe_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 0)
        decode = nvfp4_decode_gemv(stack, x, dev, peaks)
    finally:
        stack.close()
    return {"workload": "%s: 1 layer, E=%d, H=%d, I=%d, top-%d %s + shared expert, NVFP4 weights, %d N(0,1) "
                        "tokens, prefill, every expert resident" % (cfg.name, cfg.E, cfg.H, cfg.I, cfg.k, cfg.gating, T),
            "ms_per_layer": 1e3 * dt, "tokens_per_s_per_layer": T / dt,
            "vs_bf16_resident_ms_per_layer": 1e3 * dt / bf16_ms_per_layer,
            "grouped_gemm": dict(gemm_figures(perf), kernel="grouped_gemm_kernel<0,1>+<1,1> (NVFP4 tiles expanded "
                                                           "to bf16 in shared memory, tcgen05 kind::f16)"),
            "stages_ms_per_layer": {k2: v / 1e3 for k2, v in stage_us(perf).items()}, "pool_setup_s": setup_s,
            "decode_gemv": decode}


def nvfp4_decode_gemv(stack, x, dev, peaks, steps=16):
    """Decode on the same resident NVFP4 layer (every expert in its slot, so no fills): the
    expert GEMVs per launch, stage-timed, on the f16 tensor cores and on the fp32 pipes, at
    batch 1 and 8; the tokens are rows of the prefill prompt."""
    import torch

    import moe_expert_offload_top_b200 as ft
    ft.ft_moe_set_mode(stack.h, 0)
    stream = torch.cuda.current_stream(dev)
    res = {"peak_gbs": peaks["hbm_gbs"]}
    for batch in (1, 8):
        out = torch.empty((1, batch, stack.cfg.H), dtype=torch.bfloat16, device=dev)
        row = {}
        for name, on in (("tensor_cores", 1), ("fp32_pipes", 0)):
            ft.ft_moe_set_int4_tensor_cores(stack.h, on)
            for s in range(3):
                stack.forward(0, x[s * batch:(s + 1) * batch], out[0], stream)
            ft.ft_moe_sync(stack.h)
            torch.cuda.synchronize(dev)
            ft.ft_moe_reset_perf(stack.h)
            ft.ft_moe_set_stage_timing(stack.h, 1)
            for s in range(3, 3 + steps):
                stack.forward(0, x[s * batch:(s + 1) * batch], out[0], stream)
            torch.cuda.synchronize(dev)
            p = ft.ft_moe_perf(stack.h)
            ft.ft_moe_set_stage_timing(stack.h, 0)
            n = max(p["ffn_gate_up_launches"], 1)
            gu = p["ffn_gate_up_bytes"] / (p["ffn_gate_up_ms"] * 1e-3) / 1e9
            dn = p["ffn_down_bytes"] / (p["ffn_down_ms"] * 1e-3) / 1e9
            row[name] = {"gate_up_us": 1e3 * p["ffn_gate_up_ms"] / n, "gate_up_gbs": gu,
                         "gate_up_frac": gu / peaks["hbm_gbs"], "down_us": 1e3 * p["ffn_down_ms"] / n,
                         "down_gbs": dn, "down_frac": dn / peaks["hbm_gbs"],
                         "gate_up_bytes_per_launch": p["ffn_gate_up_bytes"] / n, "launches": n}
        res["batch_%d" % batch] = row
    ft.ft_moe_set_int4_tensor_cores(stack.h, 1)
    return res


# -------------------------------------------------------------- shrink leg --

def shrink_leg(args, dev):
    """Decode tokens/s on the decode-locality workload with 58% of the experts cached, then
    after an elastic shrink to 40% at a safe point (no restart; the survivors keep their
    recency), over the next steps of the same token chain."""
    import torch

    from moe_expert_offload_top_b200.workload import GpuStack
    cfg = synth.CONFIGS[SHRINK]
    c_from = int(SHRINK_FROM * cfg.L * cfg.E)
    c_to = int(SHRINK_TO * cfg.L * cfg.E)
    K, W = args.shrink_steps, args.warmup
    _, bits = token_chain(cfg, 0, W + 3 * K)
    x_dev = torch.from_numpy(bits).view(torch.bfloat16).to(dev).view(W + 3 * K, 1, cfg.H)
    out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    stack = GpuStack(cfg, capacity=c_from, device=dev)
    try:
        timed_steps(stack, list(x_dev[:W]), out, stream, dev)
        legs = {}
        for label, lo, hi in (("before", W, W + K), ("after", W + K, W + 2 * K), ("settled", W + 2 * K, W + 3 * K)):
            if label == "after":
                t0 = time.perf_counter()
                stack.resize(c_to)
                resize_ms = 1e3 * (time.perf_counter() - t0)
            stack.reset_stats()
            dt = timed_steps(stack, list(x_dev[lo:hi]), out, stream, dev)
            st = stack.stats()
            legs[label] = {"cache_slots": stack.C, "tokens_per_s": K / dt, "miss_rate": st["misses"] / max(st["routed"], 1)}
    finally:
        stack.close()
    return {"workload": "%s, batch 1, AR(1) tokens; cache %d -> %d slots (%.0f%% -> %.0f%% of the experts)"
                        % (cfg.name, c_from, c_to, 100 * SHRINK_FROM, 100 * SHRINK_TO),
            "steps": K, **legs, "resize_ms": resize_ms,
            "speed_change_after": legs["after"]["tokens_per_s"] / legs["before"]["tokens_per_s"] - 1,
            "speed_change_settled": legs["settled"]["tokens_per_s"] / legs["before"]["tokens_per_s"] - 1}


# ----------------------------------------------------------------- our arm --

def run_ours(args):
    import torch

    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[HEADLINE]
    W, K = args.warmup, args.steps
    legs = set(ALL_LEGS if args.legs == "all" else [s for s in args.legs.split(",") if s])
    peaks, peak_src = measured_peaks()
    short = host_memory_short(cfg.L * cfg.E * cfg.blob_bytes, int(os.environ.get("LOCAL_WORLD_SIZE", "1")))
    if agree_any(short is not None, dev):
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": world,
                              "config": headline_config(world),
                              "error": short or "another rank's node is short of host memory"}), flush=True)
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
        return 1
    link_h2d, link_d2h = ft.ft_probe_host_link(256 << 20, 5)
    t0 = time.perf_counter()
    stack = GpuStack(cfg, device=dev)
    setup_s = time.perf_counter() - t0
    try:
        r = decode_legs(stack, cfg, W, K, rank, dev, clocks_index=local, sync_ranks=True)
        tokens, t_max = aggregate(K, r["dt"], dev)
        e2e_tokens, e2e_max = aggregate(K, r["e2e_dt"], dev)
        line = None
        if rank == 0:
            perf = r["perf"]
            line = {
                "metric": METRIC, "value": tokens / t_max, "unit": "tokens/s", "n_gpus": world,
                "steps": K, "warmup": W, "ms_per_step": 1e3 * t_max / K, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,0.02) weights, AR(1) hidden states)",
                "config": headline_config(world),
                "roofline": gemv_roofline(perf, peaks, peak_src, "gemv_bf16",
                                          "grouped_gemv_kernel (expert gate/up + SwiGLU, decode)"),
                "e2e": {"value": e2e_tokens / e2e_max, "unit": "tokens/s",
                        "h2d_bytes_per_step": r["h2d_bytes_per_step"], "d2h_bytes_per_step": r["d2h_bytes_per_step"],
                        "miss_rate": r["st_e2e"]["misses"] / max(r["st_e2e"]["routed"], 1),
                        "same_tokens_and_cache_state_as_value": True},
                "gpu_launches": int(r["perf_dev"]["kernel_launches"]),
                "cold_start": {"value": W / r["cold_dt"] if r["cold_dt"] > 0 else None, "unit": "tokens/s",
                               "steps": W, "from": "empty cache (the warm-up steps)",
                               "miss_rate": r["cold_st"]["misses"] / max(r["cold_st"]["routed"], 1)},
                "clocks": r["clocks"],
                "cache": dict(cache_summary(r["st"], link_h2d), link_h2d_gbs_measured=link_h2d,
                              link_d2h_gbs_measured=link_d2h),
                "stages_us_per_forward": stage_us(perf),
                "host_wait_us_per_forward": 1e3 * perf["host_wait_ms"] / max(perf["forwards"], 1),
                "host_issue_us_per_forward": 1e3 * r["perf_dev"]["host_issue_ms"] / max(r["perf_dev"]["forwards"], 1),
                "pool_setup_s": setup_s,
            }
            if world == 1 and not args.no_cpu_baseline:
                vals, _ = token_chain(cfg, 0, W + K)
                rate, layers, cdt = cpu_oracle_rate(cfg, vals[W:], stack.pool_blob, budget_s=args.cpu_budget_s,
                                                    max_tokens=K)
                line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
                                        "sample": "decode tokens %d.. of the timed chain: %d (token, layer) steps of "
                                                  "%d layers (float64 numpy oracle, %.1f s)" % (W, layers, cfg.L, cdt)}
            if world == 1:
                line["legs"] = {}
                if "prefill" in legs:
                    line["legs"]["prefill"] = prefill_leg(args, stack, dev, peaks, peak_src)
        stack.close()
        stack = None
        if rank == 0 and world == 1:
            if "int4" in legs:
                line["legs"]["int4-large-pool"] = int4_leg(args, dev, peaks, peak_src, link_h2d)
            if "shrink" in legs:
                line["legs"]["shrink"] = shrink_leg(args, dev)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if stack is not None:
            stack.close()
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=160)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--legs", default="all", help="comma list of %s, or all (N = 1 only)" % ",".join(ALL_LEGS))
    ap.add_argument("--int4-steps", type=int, default=96)
    ap.add_argument("--int4-batch-steps", type=int, default=4, help="steps per point at batch 8 and 32 (0: skip)")
    ap.add_argument("--shrink-steps", type=int, default=256)
    ap.add_argument("--prefill-passes", type=int, default=2)
    ap.add_argument("--no-sweep", dest="sweep", action="store_false", help="skip the prefill token sweep")
    ap.add_argument("--no-nvfp4", dest="nvfp4", action="store_false", help="skip the NVFP4 prefill layer")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--reference-budget-s", type=float, default=90.0)
    ap.add_argument("--reference-max-tokens", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
