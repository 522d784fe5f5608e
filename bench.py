#!/usr/bin/env python
"""Benchmark of the routed-MoE layer stack over a shared LRU expert cache.

Workload (one step = one decode token through every MoE layer): 4 MoE layers,
128 experts, hidden 2048, SwiGLU intermediate 768, top-8 softmax gating,
bf16 weights N(0, 0.02); the expert pool in pinned host memory; 204 HBM slots
(40% of all experts) as one LRU shared by the layers; hidden states from an
AR(1) process x_t = 0.9 x_{t-1} + 0.436 eps_t (routing locality), batch 1.
Synthetic data stands in for the agent workloads and replayed traces of the
FreeToken pages.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--prefill]

Reports (one JSON line, rank 0): decode tokens/s timed on the device with
CUDA events (max over ranks), an end-to-end figure through host buffers, the
roofline of the dominant kernel (the decode gate/up expert GEMV, HBM-bound) from
live CUDA events, cache miss rate and H2D fill bandwidth, the cold-start figure
of the warm-up steps, SM clocks sampled during the timed region, and the CPU
oracle timed on a bounded sample.  --prefill adds the 4096-token prefill of the
DeepSeek-V4-Flash-shaped stack (8 layers, 256 experts), offloaded and resident.
--impl reference times the CPU oracle alone on the same workload.
N > 1 runs independent replicas (one stack per GPU, its own token chain):
the path has no exchange step.
"""
import argparse
import datetime
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

WORKLOAD = "decode-locality-bf16"
METRIC = "routed-MoE tokens/s (decode, prefill) and expert-weight HBM GB/s vs peak"
FALLBACK_HBM_GBS = 6650.0


def workload_desc(cfg):
    return {
        "workload": "%s: %d MoE layers, E=%d, H=%d, I=%d, top-%d %s, %s weights, %d cache slots "
                    "(%.0f%% of experts), %s tokens, batch %d, decode" % (
                        cfg.name, cfg.L, cfg.E, cfg.H, cfg.I, cfg.k, cfg.gating, cfg.wdtype, cfg.C,
                        100.0 * cfg.C / (cfg.L * cfg.E), "AR(1)" if cfg.process == "ar1" else "N(0,1)",
                        cfg.batches[0]),
        "layers": cfg.L, "experts": cfg.E, "hidden": cfg.H, "inter": cfg.I, "top_k": cfg.k,
        "cache_slots": cfg.C, "batch": cfg.batches[0], "step": "one decode token through all layers",
        "l2": "not flushed: each step streams ~%d MB of expert weights, above the 126 MB L2"
              % round(cfg.L * (cfg.k * cfg.blob_bytes + cfg.E * cfg.H * 4) / 1e6),
    }


# DRAM traffic of the dominant kernel (the decode gate/up GEMV) from one ncu capture of
# this workload: dram__bytes_read.sum + dram__bytes_write.sum of its launches divided by
# their algorithmic bytes.  Valid only while the kernel's sources hash to `sha256`;
# otherwise the JSON line carries traffic null.
GEMV_TRAFFIC = {"sources": ["moe_expert_offload_top_b200/csrc/decode_gemv.cuh",
                            "moe_expert_offload_top_b200/csrc/expert_decode.cu"],
                "sha256": "d962fe1108896e0aa147d3154d919a575024eaa9dd0a685f792b9d7bcac0da8e",
                "ratio": 0.99954,
                "capture": "ncu dram__bytes_read.sum + dram__bytes_write.sum of 12 gate/up launches (1 to 8 "
                           "experts) of this workload, 0.99954 of their algorithmic bytes; scaled to the "
                           "average launch here"}


def kernel_traffic(bytes_per_launch):
    import hashlib
    h = hashlib.sha256()
    for rel in GEMV_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if GEMV_TRAFFIC["ratio"] is None or h.hexdigest() != GEMV_TRAFFIC["sha256"]:
        return None, h.hexdigest()
    return GEMV_TRAFFIC["ratio"] * bytes_per_launch, h.hexdigest()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


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


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1])])
        else:
            dist.barrier()


# ----------------------------------------------------------- CPU oracle leg --

def cpu_oracle_rate(cfg, vals, budget_s=20.0, blob_of=None, max_tokens=None):
    """Decode tokens/s of the CPU oracle on a bounded sample of the same workload:
    tokens of the chain are pushed through every layer (router, top-k, gates, LRU,
    expert FFN, combine) until the time budget is spent.  Returns (rate, tokens, cores)."""
    from oracle import lru as olru
    from oracle import moe
    try:
        import threadpoolctl
        cores = max([p.get("num_threads", 1) for p in threadpoolctl.threadpool_info()] or [1])
    except Exception:
        cores = 1
    cache = {}

    def blob(l, e):
        if blob_of is not None:
            return blob_of(l, e)
        if (l, e) not in cache:
            cache[(l, e)] = synth.expert_blob(cfg, l, e)
        return cache[(l, e)]

    routers = [synth.router_weights(cfg, l) for l in range(cfg.L)]
    c = olru.SharedLru(cfg.C)
    done = 0
    t0 = time.perf_counter()
    for s in range(len(vals)):
        x = vals[s:s + 1]
        for l in range(cfg.L):
            r = moe.route(x, routers[l], cfg.k, cfg.gating)
            c.access_set(s * cfg.L + l, l, moe.selected_set(r["ids"]))
            moe.experts_and_combine(x, r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H, cfg.I,
                                    lambda e, l=l: blob(l, e))
        done += 1
        if time.perf_counter() - t0 > budget_s or (max_tokens and done >= max_tokens):
            break
    dt = time.perf_counter() - t0
    return done / dt, done, cores, dt


# ------------------------------------------------------------ reference arm --

def run_reference(args):
    rank, world, local = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    if rank != 0:
        return 0
    cfg = synth.CONFIGS[WORKLOAD]
    vals, _ = token_chain(cfg, 0, args.warmup + args.steps)
    # warm-up steps untimed, then the timed steps, bounded to a few minutes in all
    cpu_oracle_rate(cfg, vals[:args.warmup], budget_s=30.0, max_tokens=args.warmup)
    rate, n, cores, dt = cpu_oracle_rate(cfg, vals[args.warmup:], budget_s=args.reference_budget_s,
                                         max_tokens=args.steps)
    sample = ("CPU oracle (float64 numpy), %d of the %d timed decode tokens through all %d layers "
              "(stopped after %.0f s)" % (n, args.steps, cfg.L, args.reference_budget_s))
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": n, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(n, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_desc(cfg),
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ prefill leg --

def run_prefill_leg(args, dev):
    """Prefill of the DeepSeek-V4-Flash-shaped stack (8 layers, 256 experts, top-6
    sigmoid + shared expert, bf16): N(0,1) tokens through every layer in prefill
    mode.  Two caches: 512 slots (25%%, whole-layer double buffering over PCIe) and
    every expert resident (2048 slots), which isolates the tcgen05 grouped GEMMs."""
    import dataclasses

    import torch

    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack

    base = synth.CONFIGS["dsv4flash-prefill-bf16"]
    T = args.prefill_tokens or base.tokens
    cfg = dataclasses.replace(base, tokens=T, batches=(T,))
    stack = GpuStack(cfg, device=dev, max_tokens=T)
    vals, x = stack.tokens(T)
    out = torch.empty((cfg.L, T, cfg.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    res = {"workload": "%s: %d layers, E=%d, H=%d, I=%d, top-%d %s + shared expert, bf16, %d tokens, prefill"
                       % (cfg.name, cfg.L, cfg.E, cfg.H, cfg.I, cfg.k, cfg.gating, T)}
    for label, slots, passes in (("offload", base.C, args.prefill_passes), ("resident", cfg.L * cfg.E,
                                                                             args.prefill_passes)):
        if slots != stack.C:
            stack.resize(slots)
        stack.step(x[0], out, stream)                       # warm-up pass
        ft.ft_moe_sync(stack.h)
        stack.reset_stats()
        ft.ft_moe_reset_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(passes):
            stack.step(x[0], out, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ft.ft_moe_sync(stack.h)
        dt = e0.elapsed_time(e1) * 1e-3
        perf = ft.ft_moe_perf(stack.h)
        ft.ft_moe_set_stage_timing(stack.h, 0)
        st = stack.stats()
        gemm_s = (perf["ffn_gate_up_ms"] + perf["ffn_down_ms"]) * 1e-3
        tf = perf["ffn_flops"] / gemm_s / 1e12 if gemm_s > 0 else None
        gbs = (perf["ffn_gate_up_bytes"] + perf["ffn_down_bytes"]) / gemm_s / 1e9 if gemm_s > 0 else None
        res[label] = {
            "cache_slots": slots, "passes": passes, "tokens_per_s": T * passes / dt,
            "ms_per_layer": 1e3 * dt / (passes * cfg.L),
            "routed_misses": st["misses"], "prefetch_misses": st["prefetch_misses"],
            "h2d_gbs": st["h2d_bytes"] / st["h2d_seconds"] / 1e9 if st["h2d_seconds"] > 0 else None,
            "grouped_gemm": {
                "kernel": "grouped_gemm_kernel<0>+<1> (tcgen05 kind::f16, TMEM, TMA)",
                "ms_per_layer": 1e3 * gemm_s / max(perf["timed_forwards"], 1),
                "tflops": tf, "gbs": gbs,
                "tensor_frac_of_dense_peak": tf / peaks["bf16_tflops_sustained"] if tf and "bf16_tflops_sustained" in peaks else None,
                "hbm_frac": gbs / peaks["hbm_gbs"] if gbs and "hbm_gbs" in peaks else None,
                "intensity_flop_per_byte": perf["ffn_flops"] / (perf["ffn_gate_up_bytes"] + perf["ffn_down_bytes"])
                if perf["ffn_gate_up_bytes"] > 0 else None,
            },
            "stages_ms_per_layer": {k2: perf[k2 + "_ms"] / max(perf["timed_forwards"], 1) for k2 in
                                    ("router", "permute", "ffn_gate_up", "ffn_down", "combine")},
        }
    stack.close()
    return res


# ----------------------------------------------------------------- our arm --

def run_ours(args):
    import torch

    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[WORKLOAD]
    W, K = args.warmup, args.steps
    vals, bits = token_chain(cfg, rank, W + 3 * K)      # device leg, stage leg, e2e leg
    stack = GpuStack(cfg, device=dev)
    x_dev = torch.from_numpy(bits).view(torch.bfloat16).to(dev).view(W + 3 * K, 1, cfg.H)
    out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    link_h2d, link_d2h = ft.ft_probe_host_link(256 << 20, 5)
    # warm-up steps from an empty cache, timed as the cold-start figure
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    c0.record(stream)
    for s in range(W):
        stack.step(x_dev[s], out, stream)
    c1.record(stream)
    torch.cuda.synchronize(dev)
    cold_dt = c0.elapsed_time(c1) * 1e-3
    cold_st = stack.stats()

    # ---- device-timed leg: inputs resident in HBM, no instrumentation
    stack.reset_stats()
    ft.ft_moe_reset_perf(stack.h)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(W, W + K):
        stack.step(x_dev[s], out, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clk = clocks.stop()
    dt = e0.elapsed_time(e1) * 1e-3
    perf_dev = ft.ft_moe_perf(stack.h)      # the uninstrumented leg's counters
    launches = perf_dev["kernel_launches"]
    st = stack.stats()
    tokens, t_max = aggregate(K * cfg.batches[0], dt, dev)

    # ---- stage leg: the same number of steps (the chain continued) with CUDA events
    # around every stage on the forward's stream; gives each kernel's device time
    ft.ft_moe_reset_perf(stack.h)
    ft.ft_moe_set_stage_timing(stack.h, 1)
    for s in range(W + K, W + 2 * K):
        stack.step(x_dev[s], out, stream)
    torch.cuda.synchronize(dev)
    perf = ft.ft_moe_perf(stack.h)
    ft.ft_moe_set_stage_timing(stack.h, 0)

    # ---- end-to-end leg through host buffers (pinned): H2D of the step's token and
    # D2H of the step's layer outputs inside the timed region, read back every step
    x_host = torch.from_numpy(bits[W + 2 * K:W + 3 * K]).view(torch.bfloat16).view(K, 1, cfg.H).pin_memory()
    out_host = torch.empty((K, cfg.L, 1, cfg.H), dtype=torch.bfloat16).pin_memory()
    x_in = torch.empty((1, cfg.H), dtype=torch.bfloat16, device=dev)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
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
    e2e_tokens, e2e_max = aggregate(K * cfg.batches[0], e2e_dt, dev)

    if rank == 0:
        peak, peak_src = measured_peaks()
        fwd = max(perf["timed_forwards"], 1)
        fl = perf["ffn_fused_launches"]
        if fl > 0:
            # the fused decode FFN (gate/up + SwiGLU + down + combine in one launch)
            f_s = perf["ffn_fused_ms"] * 1e-3
            achieved = perf["ffn_fused_bytes"] / f_s / 1e9 if f_s > 0 else None
            roof = {"kernel": "ffn_decode_fused_kernel (expert gate/up + SwiGLU + down + combine, decode)",
                    "bytes_per_launch": perf["ffn_fused_bytes"] / fl, "avg_launch_us": 1e6 * f_s / fl,
                    "launches_per_forward": fl / fwd}
        else:
            gu_s = perf["ffn_gate_up_ms"] * 1e-3
            gl = max(perf["ffn_gate_up_launches"], 1)
            achieved = perf["ffn_gate_up_bytes"] / gu_s / 1e9 if gu_s > 0 else None
            traffic, src_hash = kernel_traffic(perf["ffn_gate_up_bytes"] / gl)
            roof = {"kernel": "grouped_gemv_kernel (expert gate/up + SwiGLU, decode)",
                    "bytes_per_launch": perf["ffn_gate_up_bytes"] / gl, "avg_launch_us": 1e6 * gu_s / gl,
                    "launches_per_forward": gl / fwd, "traffic": traffic,
                    "traffic_source": GEMV_TRAFFIC["capture"] if traffic is not None else
                    "no ncu capture of these kernel sources (sha256 %s)" % src_hash[:12],
                    "down_proj_gbs": perf["ffn_down_bytes"] / (perf["ffn_down_ms"] * 1e-3) / 1e9
                    if perf["ffn_down_ms"] > 0 else None}
        line = {
            "metric": METRIC, "value": tokens / t_max, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": 1e3 * t_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,0.02) weights, AR(1) hidden states)",
            "config": dict(workload_desc(cfg), parallelism="replicas x%d" % world),
            "roofline": dict({"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                              "frac": achieved / peak if achieved else None, "peak_source": peak_src,
                              "traffic": None}, **roof),
            "e2e": {"value": e2e_tokens / e2e_max, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(cfg.H * 2 * cfg.batches[0]),
                    "d2h_bytes_per_step": int(cfg.L * cfg.H * 2 * cfg.batches[0])},
            "gpu_launches": int(launches),
            "cold_start": {"value": W * cfg.batches[0] / cold_dt if cold_dt > 0 else None, "unit": "tokens/s",
                           "steps": W, "from": "empty cache (the warm-up steps)",
                           "miss_rate": cold_st["misses"] / max(cold_st["routed"], 1)},
            "clocks": clk,
            "cache": {"miss_rate": st["misses"] / max(st["routed"], 1), "routed": st["routed"],
                      "misses": st["misses"], "h2d_bytes": st["h2d_bytes"],
                      "h2d_gbs": st["h2d_bytes"] / st["h2d_seconds"] / 1e9 if st["h2d_seconds"] > 0 else None,
                      "link_h2d_gbs_measured": link_h2d, "link_d2h_gbs_measured": link_d2h,
                      "h2d_frac_of_link": (st["h2d_bytes"] / st["h2d_seconds"] / 1e9) / link_h2d
                      if st["h2d_seconds"] > 0 and link_h2d else None},
            "stages_us_per_forward": {k2: 1e3 * perf[k2 + "_ms"] / fwd for k2 in
                                      ("router", "permute", "ffn_gate_up", "ffn_down", "combine", "ffn_fused")},
            "host_wait_us_per_forward": 1e3 * perf["host_wait_ms"] / max(perf["forwards"], 1),
            "host_issue_us_per_forward": 1e3 * perf_dev["host_issue_ms"] / max(perf_dev["forwards"], 1),
        }
        if world == 1 and args.prefill:
            line["prefill"] = run_prefill_leg(args, dev)
        if world == 1 and not args.no_cpu_baseline:
            rate, n, cores, cdt = cpu_oracle_rate(cfg, vals[W:W + K], budget_s=args.cpu_budget_s,
                                                  blob_of=stack.pool_blob)
            line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                    "sample": "%d decode tokens of the timed chain through all %d layers "
                                              "(float64 numpy oracle, %.1f s)" % (n, cfg.L, cdt)}
        print(json.dumps(line), flush=True)
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
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", action="store_true",
                    help="add the prefill leg (N=1 only; pins a 103 GB host pool)")
    ap.add_argument("--prefill-tokens", type=int, default=None)
    ap.add_argument("--prefill-passes", type=int, default=2)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
