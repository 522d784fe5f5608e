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


def assert_close(got, ref, wdtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rl2, rmax = BOUNDS[wdtype]
    rms = np.sqrt(np.mean(ref * ref))
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.max(np.abs(got - ref)) if got.size else 0.0
    assert rel <= rl2, "%s: relative L2 %.3g > %.3g" % (what, rel, rl2)
    assert mx <= rmax * rms, "%s: max-abs %.3g > %.3g * rms %.3g" % (what, mx, rmax, rms)
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
