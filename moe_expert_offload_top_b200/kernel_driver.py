"""Runs a named workload at reduced size through the C ABI, for kernel profiling.

    python -m moe_expert_offload_top_b200.kernel_driver --workload NAME
        [--layers L] [--experts E] [--slots C] [--steps S] [--batch B] [--tokens T] [--wdtype W] [--perf]
        [--fp32-pipes]

The workload keeps its shapes (hidden, intermediate, top-k, gating, weight format,
shared expert) and token process; --layers / --experts shrink the pool so that a
profiler's capture stays small (a few GB on the device), and --slots defaults to every
expert resident, so the launches are the kernels alone.  Decode workloads run S steps of
B tokens; prefill workloads run S forwards of T tokens through every layer.  Prints one
line with the steps run and the cache counters (with --perf, stage timing is on and the
line adds each FFN launch's algorithmic bytes and flops, averaged over the launches, for
setting a profiler's DRAM counters against).
"""
import argparse
import dataclasses
import json
import sys

import torch

import moe_expert_offload_top_b200 as ft
import synth
from moe_expert_offload_top_b200.workload import GpuStack


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", required=True, choices=sorted(synth.CONFIGS))
    ap.add_argument("--layers", type=int, default=1)
    ap.add_argument("--experts", type=int, default=None)
    ap.add_argument("--slots", type=int, default=None, help="cache slots (default: every expert resident)")
    ap.add_argument("--steps", type=int, default=12)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--tokens", type=int, default=None, help="prefill: tokens per forward")
    ap.add_argument("--wdtype", default=None, choices=["f32", "bf16", "int4", "nvfp4"],
                    help="another weight format for the workload's shapes")
    ap.add_argument("--perf", action="store_true",
                    help="stage timing on: also print the algorithmic bytes and flops per FFN launch")
    ap.add_argument("--fp32-pipes", action="store_true",
                    help="decode GEMV on the fp32 pipes instead of the tensor cores (int4, NVFP4, bf16)")
    a = ap.parse_args(argv)
    base = synth.CONFIGS[a.workload]
    E = a.experts or base.E
    k = min(base.k, E)
    prefill = base.mode == "prefill"
    T = (a.tokens or base.tokens) if prefill else a.batch
    n_tok = T * a.steps if prefill else max(base.tokens, T * a.steps)
    cfg = dataclasses.replace(base, L=a.layers, E=E, k=k, C=a.slots or a.layers * E, tokens=n_tok,
                              batches=(T,), resize_to=None, wdtype=a.wdtype or base.wdtype)
    with GpuStack(cfg, max_tokens=T) as st:
        vals, x = st.tokens(T)
        out = torch.empty((cfg.L, T, cfg.H), dtype=st.xdt, device=st.device)
        if a.fp32_pipes:
            ft.ft_moe_set_int4_tensor_cores(st.h, 0)
        if a.perf:
            ft.ft_moe_set_stage_timing(st.h, 1)
        for s in range(a.steps):
            st.step(x[s % x.shape[0]], out)
        torch.cuda.synchronize()
        line = {"workload": cfg.name, "layers": cfg.L, "experts": cfg.E, "slots": cfg.C, "steps": a.steps,
                "tokens_per_step": T, "cache": st.stats()}
        if a.perf:
            p = ft.ft_moe_perf(st.h)
            n = max(p["ffn_gate_up_launches"], 1)
            line["per_launch"] = {"gate_up_bytes": p["ffn_gate_up_bytes"] / n, "down_bytes": p["ffn_down_bytes"] / n,
                                  "flops": p["ffn_flops"] / n, "gate_up_us": 1e3 * p["ffn_gate_up_ms"] / n,
                                  "down_us": 1e3 * p["ffn_down_ms"] / n, "launches": n}
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
