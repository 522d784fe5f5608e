"""Drives a whole workload - steps x layers - through the oracle's layer and cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).

READINGS (the pages describe a full model; this project's unit is the routed
MoE layer stack):
  * every layer of the stack receives the same hidden state of the step (no
    residual, no norm); each layer has its own router and experts;
  * a decode step is one batch of tokens (one token per chain) through all
    layers; the LRU sees the layers in order 0..L-1 within a step;
  * prefill: before layer 0 the whole of layer 0 is prefetched, and after the
    routed accesses of layer l the whole of layer l+1 is prefetched (FreeToken
    linux, "FreeToken's MoE memory handling": whole-layer double buffering);
  * a grow (resize_to) happens at the step boundary half-way through the run.
"""
from typing import Callable, Dict, Iterable, Optional

import numpy as np

from . import moe
from .lru import PREFETCH, ROUTED, SharedLru


def run_workload(*, L: int, E: int, H: int, I: int, k: int, gating: str, wdtype: str,
                 capacity: int, x_steps: np.ndarray, router_of: Callable[[int], np.ndarray],
                 blob_of: Callable[[int, int], np.ndarray],
                 shared_of: Optional[Callable[[int], np.ndarray]] = None,
                 prefill: bool = False, resize_to: Optional[int] = None,
                 ffn_steps: Optional[Iterable[int]] = None, through_slots: bool = False) -> Dict:
    """x_steps: [steps, B, H].  ffn_steps: steps whose layer outputs are computed
    (None = all).  through_slots: read expert bytes from a simulated slot arena
    filled on each miss instead of from the pool (same result by construction of
    the method - a check that the trace's slots hold the right experts).

    Returns dict(ids [steps,L,B,k], gates, gap, zsel (the selected logits, in id order),
    trace, stats, out {(s,l): [B,H]}).
    """
    steps, B, _ = x_steps.shape
    lru = SharedLru(capacity)
    want = set(range(steps)) if ffn_steps is None else set(ffn_steps)
    ids_all = np.zeros((steps, L, B, k), dtype=np.int32)
    g_all = np.zeros((steps, L, B, k))
    gap_all = np.zeros((steps, L, B))
    zsel_all = np.zeros((steps, L, B, k))
    outs = {}
    routers = {l: router_of(l) for l in range(L)}
    arena = {}

    def fill(recs):
        if through_slots:
            for r in recs:
                if not r.hit:
                    arena[r.slot] = np.array(blob_of(r.layer, r.expert), copy=True)

    for s in range(steps):
        if resize_to is not None and s == steps // 2:
            moves = lru.resize(resize_to)
            if through_slots:
                for old, new in moves:
                    arena[new] = arena.pop(old)
        x = x_steps[s]
        for l in range(L):
            call = s * L + l
            r = moe.route(x, routers[l], k, gating)
            ids_all[s, l], g_all[s, l], gap_all[s, l] = r["ids"], r["gates"], r["gap"]
            zsel_all[s, l] = np.take_along_axis(r["z"], r["ids"].astype(np.int64), axis=1)
            if prefill and l == 0:
                fill(lru.access_set(call, 0, range(E), PREFETCH))
            fill(lru.access_set(call, l, moe.selected_set(r["ids"]), ROUTED))
            if prefill and l + 1 < L:
                fill(lru.access_set(call, l + 1, range(E), PREFETCH))
            if s in want:
                if through_slots:
                    get = lambda e, l=l: arena[lru.slot_of(l, e)]
                else:
                    get = lambda e, l=l: blob_of(l, e)
                sh = shared_of(l) if shared_of is not None else None
                outs[(s, l)] = moe.experts_and_combine(x, r["ids"], r["gates"], E, wdtype, H, I,
                                                       get, sh)
    return {"ids": ids_all, "gates": g_all, "gap": gap_all, "zsel": zsel_all, "trace": lru.trace,
            "stats": lru.stats, "out": outs, "lru": lru}
