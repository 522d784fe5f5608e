"""Helpers of the GPU parity tests (comparison bounds and oracle drivers)."""
import numpy as np

import synth
from oracle import moe
from oracle.run import run_workload

# Floating-point bounds.  bf16 / int4 paths: relative L2 <= 5e-3 and max-abs <= 2e-2 * rms
# (the stated parity bound).  fp32 path: the kernels compute in fp32 throughout; the
# difference to the float64 oracle is summation-order rounding, far below 1e-5.
BOUNDS = {"bf16": (5e-3, 2e-2), "int4": (5e-3, 2e-2), "nvfp4": (5e-3, 2e-2), "f32": (1e-5, 1e-4)}
TIE_GAP = 1e-5   # logit gap below which either top-k choice is correct


def bf16_half_ulp(v):
    """Half the spacing of bf16 values at |v| (the largest rounding error of storing v as
    bf16, round to nearest): |v| in [2^e, 2^(e+1)) has 8 significant bits, ulp 2^(e-7)."""
    m, e = np.frexp(np.abs(np.asarray(v, dtype=np.float64)))   # |v| = m 2^e, m in [0.5, 1)
    return np.where(m == 0, 0.0, np.ldexp(1.0, (e - 9).astype(np.int64)))


def assert_close(got, ref, wdtype, what="", stored_bf16=False):
    """The stated parity bound: relative L2 <= rl2 and max-abs <= rmax * rms(ref).

    stored_bf16: got holds bf16 outputs of the library.  Storing a value as bf16 rounds it by
    up to half an ulp of itself, on top of any error of the computation; the max-abs bound is
    applied to the computation, so each element is allowed its own half ulp in addition.
    (Without it, even the exact result rounded to bf16 fails the bound on outputs beyond about
    five times rms(out), which full-layer comparisons of millions of outputs contain.)"""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rl2, rmax = BOUNDS[wdtype]
    rms = np.sqrt(np.mean(ref * ref))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= rl2, "%s: relative L2 %.3g > %.3g" % (what, rel, rl2)
    if got.size:
        err = np.abs(got - ref)
        allow = rmax * rms + (bf16_half_ulp(np.maximum(np.abs(got), np.abs(ref))) if stored_bf16 else 0.0)
        i = int(np.argmax(err - allow))
        assert err.flat[i] <= np.broadcast_to(allow, err.shape).flat[i], \
            "%s: max-abs %.3g > %.3g (%.3g * rms %.3g%s) at %.4g vs %.4g" % (
                what, err.flat[i], np.broadcast_to(allow, err.shape).flat[i], rmax, rms,
                " + half an ulp of the stored bf16" if stored_bf16 else "", got.flat[i], ref.flat[i])
    return rel


def first_divergence(gpu_ids, ref_ids, gap, zsel=None):
    """Index of the first token whose selected set differs.

    Two readings of "a tie" are accepted, both at logit gaps below TIE_GAP: a
    different set where the oracle's k-th / (k+1)-th gap is that small, and the same
    set listed in another order where the swapped logits (zsel: the oracle's logits
    of its own selection, in its order) are that close.  Any other difference fails.
    Returns None when every token agrees (up to such reorderings)."""
    g = np.asarray(gpu_ids).reshape(-1, gpu_ids.shape[-1])
    r = np.asarray(ref_ids).reshape(-1, ref_ids.shape[-1])
    gp = np.asarray(gap).reshape(-1)
    zs = None if zsel is None else np.asarray(zsel, dtype=np.float64).reshape(-1, r.shape[1])
    for i in range(len(r)):
        if np.array_equal(g[i], r[i]):
            continue
        if zs is not None and np.array_equal(np.sort(g[i]), np.sort(r[i])):
            zmap = dict(zip(r[i].tolist(), zs[i].tolist()))
            zg = np.array([zmap[e] for e in g[i].tolist()])
            assert np.max(np.abs(zg - zs[i])) < TIE_GAP, "token %d: order %s vs oracle %s" % (
                i, g[i].tolist(), r[i].tolist())
            continue
        assert len(set(g[i].tolist())) == len(g[i]), "token %d: repeated ids %s" % (i, g[i].tolist())
        assert gp[i] < TIE_GAP, "token %d: ids %s vs oracle %s with logit gap %.3g" % (
            i, g[i].tolist(), r[i].tolist(), gp[i])
        if zs is not None:
            # the experts left out must sit at the oracle's cut (its k-th logit): a tie
            # moves only those
            zmap = dict(zip(r[i].tolist(), zs[i].tolist()))
            cut = float(np.min(zs[i]))
            dropped = [e for e in r[i].tolist() if e not in set(g[i].tolist())]
            assert all(zmap[e] - cut < TIE_GAP for e in dropped), \
                "token %d: ids %s vs oracle %s drop an expert above the cut" % (i, g[i].tolist(), r[i].tolist())
        return i
    return None


def same_selection(gpu_ids, ref_ids):
    """Per token: the same set of experts (order free)."""
    return np.all(np.sort(gpu_ids, axis=-1) == np.sort(ref_ids, axis=-1), axis=-1)


def trace_tuples(ref_trace):
    return [(a.call, a.layer, a.expert, a.kind, int(a.hit), a.slot, a.ev_layer, a.ev_expert)
            for a in ref_trace]


def oracle_run(cfg, stack, vals, capacity=None, ffn_steps=None, resize_to=None, prefill=None):
    return run_workload(L=cfg.L, E=cfg.E, H=cfg.H, I=cfg.I, k=cfg.k, gating=cfg.gating,
                        wdtype=cfg.wdtype, capacity=capacity or cfg.C, x_steps=vals,
                        router_of=lambda l: synth.router_weights(cfg, l),
                        blob_of=lambda l, e: stack.pool_blob(l, e),
                        shared_of=(lambda l: stack.shared_blobs[l]) if cfg.shared else None,
                        prefill=cfg.mode == "prefill" if prefill is None else prefill,
                        resize_to=resize_to, ffn_steps=ffn_steps)


def run_and_check(cfg, batch, sample_steps, sample_tokens=None, gemm_threshold=None, capacity=None,
                  resize_at=None, resize_to=None, n_steps=None, stack=None, sample_layers=None,
                  full_layers=(), workers=None):
    """Runs a workload through the C ABI (GpuStack) and checks it against the oracle.

    Routing and the cache trace are compared on every step (bit-exact up to near-ties,
    see first_divergence).  Outputs are compared at the steps in sample_steps: on the
    tokens sample_tokens (all when None) of the layers sample_layers (all when None),
    and on every token of the layers in full_layers.  The oracle's per-(step, layer)
    evaluations run in a thread pool (numpy releases the GIL in its array loops).
    A shared `stack` starts from an empty cache of `capacity` slots."""
    import concurrent.futures
    import contextlib
    import os

    import torch

    import moe_expert_offload_top_b200 as ft
    from moe_expert_offload_top_b200.workload import GpuStack
    from oracle import lru as olru

    ctx = contextlib.nullcontext(stack) if stack is not None else GpuStack(cfg, capacity=capacity)
    with ctx as st:
        if stack is not None:
            ft.ft_moe_set_mode(st.h, cfg.mode == "prefill")
            ft.ft_cache_resize(st.h, capacity or cfg.C)
            st.C = capacity or cfg.C
            ft.ft_cache_clear(st.h)
            ft.ft_cache_set_trace(st.h, 0)
            ft.ft_cache_set_trace(st.h, 1)
            st.reset_stats()
        if gemm_threshold is not None:
            ft.ft_moe_set_gemm_threshold(st.h, gemm_threshold)
        from moe_expert_offload_top_b200.workload import _to_device_tokens
        vals, bits = synth.tokens(cfg, batch)       # cfg's token process (a shared stack may have another)
        x = _to_device_tokens(cfg, vals, bits, st.device)
        steps = n_steps or vals.shape[0]
        out = torch.empty((cfg.L, batch, cfg.H), dtype=st.xdt, device=st.device)
        gpu_ids = np.zeros((steps, cfg.L, batch, cfg.k), dtype=np.int32)
        outs = {}
        for s in range(steps):
            if resize_at is not None and s == resize_at:
                st.resize(resize_to)
            for l in range(cfg.L):
                st.forward(l, x[s], out[l])
                gpu_ids[s, l] = st.last_routing(batch)[0]
            if s in sample_steps:
                outs[s] = out.float().cpu().numpy().copy()
        ft.ft_moe_sync(st.h)
        trace = st.trace()
        if stack is not None and trace:
            # a shared stack keeps counting forward calls across runs (the cache clear keeps
            # the handle's counters): number this run's calls from 0, as the oracle does
            base = trace[0][0]
            trace = [(t[0] - base,) + tuple(t[1:]) for t in trace]
        stats = st.stats()
        # oracle: routing and cache trace of every step
        routers = [synth.router_weights(cfg, l) for l in range(cfg.L)]
        ref_lru = olru.SharedLru(capacity or cfg.C)
        ref_ids = np.zeros_like(gpu_ids)
        gaps = np.zeros((steps, cfg.L, batch))
        zsel = np.zeros(gpu_ids.shape)
        for s in range(steps):
            if resize_at is not None and s == resize_at:
                ref_lru.resize(resize_to)
            for l in range(cfg.L):
                r = moe.route(vals[s], routers[l], cfg.k, cfg.gating)
                ref_ids[s, l], gaps[s, l] = r["ids"], r["gap"]
                zsel[s, l] = np.take_along_axis(r["z"], r["ids"].astype(np.int64), axis=1)
                call = s * cfg.L + l
                if cfg.mode == "prefill" and l == 0:
                    ref_lru.access_set(call, 0, range(cfg.E), olru.PREFETCH)
                ref_lru.access_set(call, l, moe.selected_set(r["ids"]))
                if cfg.mode == "prefill" and l + 1 < cfg.L:
                    ref_lru.access_set(call, l + 1, range(cfg.E), olru.PREFETCH)
        div = first_divergence(gpu_ids, ref_ids, gaps, zsel)
        want = trace_tuples(ref_lru.trace)
        if div is None:
            assert [tuple(t) for t in trace] == want
        else:
            last = div // (cfg.L * batch)
            n = sum(1 for a in ref_lru.trace if a.call < last * cfg.L)
            assert [tuple(t) for t in trace[:n]] == want[:n]
        # oracle: outputs of the sampled (step, layer, tokens)
        jobs = []
        for s in sample_steps:
            layers = set(range(cfg.L) if sample_layers is None else sample_layers) | set(full_layers)
            for l in sorted(layers):
                if not np.all(same_selection(gpu_ids[s, l], ref_ids[s, l])):
                    continue      # a near-tie flip (checked above): another valid selection
                toks = list(range(batch)) if (sample_tokens is None or l in full_layers) else list(sample_tokens)
                jobs.append((s, l, toks))

        def oracle_out(job):
            s, l, toks = job
            r = moe.route(vals[s][toks], routers[l], cfg.k, cfg.gating)
            return moe.experts_and_combine(vals[s][toks], r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H, cfg.I,
                                           lambda e, l=l: st.pool_blob(l, e),
                                           st.shared_blobs[l] if cfg.shared else None)

        nw = workers or min(8, os.cpu_count() or 1, max(len(jobs), 1))
        with concurrent.futures.ThreadPoolExecutor(max_workers=nw) as ex:
            for (s, l, toks), ref in zip(jobs, ex.map(oracle_out, jobs)):
                assert_close(outs[s][l][toks], ref, cfg.wdtype, "step %d layer %d (%d tokens)" % (s, l, len(toks)),
                             stored_bf16=cfg.x_dtype == "bf16")
        return {**stats, "compared": [(s, l, len(t)) for s, l, t in jobs]}
