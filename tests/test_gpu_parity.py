"""GPU parity: every step of the hot path, and whole forwards through the C ABI,
against the CPU oracle on the same seeded inputs."""
import dataclasses

import numpy as np
import pytest
import torch

import moe_expert_offload_top_b200 as ft
import synth
from moe_expert_offload_top_b200.workload import GpuStack
from oracle import moe
from gpu_util import (TIE_GAP, assert_close, first_divergence, oracle_run, trace_tuples)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16_dev(vals_f32):
    bits = synth.round_bf16(vals_f32)
    return torch.from_numpy(bits).view(torch.bfloat16).to(DEV), (bits.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------ step level --

@pytest.mark.parametrize("T,H,E,k,gating,xbf16", [
    (1, 256, 16, 2, "softmax", False), (7, 2048, 128, 8, "softmax", True),
    (33, 4096, 256, 6, "sigmoid", True), (130, 7168, 256, 8, "sigmoid", True),
    (5, 64, 8, 8, "softmax", False), (0, 256, 16, 2, "softmax", True),
])
def test_router_topk_parity(T, H, E, k, gating, xbf16):
    x = synth.normal_f32(3, 8, 0, 0, max(T, 1) * H).reshape(max(T, 1), H)[:T]
    w = synth.normal_f32(3, 4, 0, 0, E * H, 0.02).reshape(E, H)
    if xbf16:
        xd, xv = _bf16_dev(x)
    else:
        xd, xv = torch.from_numpy(np.ascontiguousarray(x)).to(DEV), x
    wd = torch.from_numpy(w).to(DEV)
    z = torch.full((max(T, 1), E), float("nan"), device=DEV)
    ids = torch.full((max(T, 1), k), -7, dtype=torch.int32, device=DEV)
    g = torch.full((max(T, 1), k), float("nan"), device=DEV)
    ft.ft_router_topk(xd, xbf16, wd, T, H, E, k, gating, z, ids, g)
    torch.cuda.synchronize()
    if T == 0:
        assert int(ids[0, 0]) == -7
        return
    zr = moe.router_logits(xv, w)
    assert np.max(np.abs(z.cpu().numpy() - zr)) <= 2e-6 * max(1.0, np.abs(zr).max())
    ir, gap = moe.topk(zr, k)
    gi = ids.cpu().numpy()
    assert first_divergence(gi, ir, gap) is None or np.min(gap) < TIE_GAP
    ok = np.all(gi == ir, axis=1)
    gr = moe.gates(np.take_along_axis(zr, ir.astype(np.int64), axis=1), gating)
    assert np.max(np.abs(g.cpu().numpy()[ok] - gr[ok])) <= 2e-6


@pytest.mark.parametrize("T,H,E,xbf16", [(4096, 4096, 256, True), (150, 7168, 200, True), (97, 512, 64, False)])
def test_tiled_router_fast_path_and_one_step_kernel(T, H, E, xbf16):
    # Above 64 tokens the logits come from the tiled router.  On 16-byte aligned x it streams K
    # steps through a cp.async ring: bf16 x on the tf32 tensor cores (the weight split into tf32
    # hi + lo), fp32 x on the fp32 pipes.  An x one element off that alignment takes the
    # one-step kernel on the fp32 pipes.  All sum a partial per 32 elements of H into each logit
    # in H order; the fp32-pipe kernels agree bit for bit, and every path meets the oracle's
    # bound (2e-6 of the largest |z|).
    x = synth.normal_f32(11, 8, 0, 0, T * H).reshape(T, H)
    w = synth.normal_f32(11, 4, 0, 0, E * H, 0.02).reshape(E, H)
    if xbf16:
        xd, xv = _bf16_dev(x)
    else:
        xd, xv = torch.from_numpy(np.ascontiguousarray(x)).to(DEV), x
    pad = torch.empty(T * H + 8, dtype=xd.dtype, device=DEV)
    xm = pad[1:1 + T * H].view(T, H)   # 2 or 4 bytes past a 16-byte boundary
    xm.copy_(xd)
    assert xd.data_ptr() % 16 == 0 and xm.data_ptr() % 16 != 0
    wd = torch.from_numpy(w).to(DEV)
    za = torch.full((T, E), float("nan"), device=DEV)
    zb = torch.full((T, E), float("nan"), device=DEV)
    ids = torch.empty((T, 4), dtype=torch.int32, device=DEV)
    g = torch.empty((T, 4), device=DEV)
    ft.ft_router_topk(xd, xbf16, wd, T, H, E, 4, "sigmoid", za, ids, g)
    ft.ft_router_topk(xm, xbf16, wd, T, H, E, 4, "sigmoid", zb, ids, g)
    torch.cuda.synchronize()
    a, b = za.cpu().numpy(), zb.cpu().numpy()
    if not xbf16:
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    rows = np.random.default_rng(T).choice(T, min(T, 64), replace=False)   # the oracle on a sample
    zr = moe.router_logits(xv[rows], w)
    bound = 2e-6 * max(1.0, np.abs(zr).max())
    assert np.max(np.abs(a[rows] - zr)) <= bound
    assert np.max(np.abs(b[rows] - zr)) <= bound
    assert np.all(np.isfinite(a)) and np.max(np.abs(a - b)) <= 2 * bound


@pytest.mark.parametrize("T,H,E,k,gating,xbf16", [
    (1, 256, 16, 2, "softmax", False), (1, 2048, 128, 8, "softmax", True), (1, 4096, 256, 6, "sigmoid", True),
    (8, 7168, 256, 8, "sigmoid", True), (32, 7168, 256, 8, "sigmoid", True), (64, 512, 256, 16, "softmax", True),
    (3, 64, 8, 8, "softmax", False), (48, 256, 16, 2, "sigmoid", True), (64, 256, 16, 16, "sigmoid", True),
])
def test_fused_decode_routing_parity(T, H, E, k, gating, xbf16):
    x = synth.normal_f32(5, 8, 0, 0, T * H).reshape(T, H)
    w = synth.normal_f32(5, 4, 0, 0, E * H, 0.02).reshape(E, H)
    xd, xv = _bf16_dev(x) if xbf16 else (torch.from_numpy(np.ascontiguousarray(x)).to(DEV), x)
    wd = torch.from_numpy(w).to(DEV)
    z = torch.empty((T, E), device=DEV)
    ids = torch.full((T, k), -1, dtype=torch.int32, device=DEV)
    g = torch.empty((T, k), device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offs = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ticket = torch.zeros(1, dtype=torch.int32, device=DEV)
    for rep in range(2):                      # the ticket is left at 0 for the next call
        ft.ft_route_decode(xd, xbf16, wd, T, H, E, k, gating, z, ids, g, counts, offs, perm, inv, ticket)
    torch.cuda.synchronize()
    assert int(ticket.item()) == 0
    zr = moe.router_logits(xv, w)
    ir, gap = moe.topk(zr, k)
    gi = ids.cpu().numpy()
    div = first_divergence(gi, ir, gap)
    ok = np.all(gi == ir, axis=1)
    gr = moe.gates(np.take_along_axis(zr, ir.astype(np.int64), axis=1), gating)
    assert np.max(np.abs(g.cpu().numpy()[ok] - gr[ok])) <= 2e-6
    pp, iv = perm.cpu().numpy(), inv.cpu().numpy()
    if div is None:                             # same selection: the oracle's permutation, bit for bit
        c, o, p = moe.permute(ir, E)
        assert np.array_equal(counts.cpu().numpy(), c) and np.array_equal(offs.cpu().numpy(), o)
        assert np.array_equal(pp, p) and np.array_equal(iv, np.argsort(p))
    else:                                       # a near-tie flip: check the sort's properties
        flat = gi.reshape(-1)
        assert sorted(pp.tolist()) == list(range(T * k)) and np.array_equal(pp[iv], np.arange(T * k))
        keys = flat[pp] * (T * k) + pp
        assert np.all(np.diff(keys) > 0)


def test_fused_decode_routing_after_wider_call():
    # a 256-expert call leaves every row of the kernel's per-warp counts dirty in
    # shared memory; a following 16-expert call with many tokens must not read them
    def run(T, H, E, k):
        x = synth.normal_f32(T + E, 8, 0, 0, T * H).reshape(T, H)
        w = synth.normal_f32(T + E, 4, 0, 0, E * H, 0.3).reshape(E, H)
        xd, xv = _bf16_dev(x)
        bufs = [torch.empty((T, E), device=DEV), torch.empty((T, k), dtype=torch.int32, device=DEV),
                torch.empty((T, k), device=DEV), torch.empty(E, dtype=torch.int32, device=DEV),
                torch.empty(E + 1, dtype=torch.int32, device=DEV), torch.empty(T * k, dtype=torch.int32, device=DEV),
                torch.empty(T * k, dtype=torch.int32, device=DEV)]
        ticket = torch.zeros(1, dtype=torch.int32, device=DEV)
        ft.ft_route_decode(xd, True, torch.from_numpy(w).to(DEV), T, H, E, k, "softmax", *bufs, ticket)
        torch.cuda.synchronize()
        ir, gap = moe.topk(moe.router_logits(xv, w), k)
        if first_divergence(bufs[1].cpu().numpy(), ir, gap) is None:
            c, o, p = moe.permute(ir, E)
            assert np.array_equal(bufs[4].cpu().numpy(), o)
            assert np.array_equal(bufs[5].cpu().numpy(), p) and np.array_equal(bufs[6].cpu().numpy(), np.argsort(p))
    for rep in range(4):
        run(64, 512, 256, 16)
        run(48, 256, 16, 2)
        run(64, 256, 8, 4)


@pytest.mark.parametrize("T,k,E", [(1, 2, 16), (7, 8, 128), (33, 6, 256), (300, 8, 256), (4096, 6, 256),
                                   (5, 16, 16), (0, 2, 16), (128, 8, 16), (129, 8, 16), (3000, 5, 7)])
def test_permute_parity(T, k, E):
    # up to 1024 pairs: one CTA; more: one CTA per chunk of 1024 (128 x 8 is exactly one chunk,
    # 129 x 8 leaves 8 pairs in a second one; few experts put many equal keys in every warp)
    rng = np.random.default_rng(T * 31 + k)
    ids = np.array([rng.choice(E, k, replace=False) for _ in range(T)], dtype=np.int32).reshape(T, k)
    if T > 20:
        ids[: T // 3] = ids[0]            # a hot set: many pairs on few experts
    idd = torch.from_numpy(ids).to(DEV) if T else torch.zeros(1, dtype=torch.int32, device=DEV)
    counts = torch.full((E,), -1, dtype=torch.int32, device=DEV)
    offs = torch.full((E + 1,), -1, dtype=torch.int32, device=DEV)
    perm = torch.full((max(T * k, 1),), -1, dtype=torch.int32, device=DEV)
    inv = torch.full((max(T * k, 1),), -1, dtype=torch.int32, device=DEV)
    ft.ft_permute(idd, T, k, E, counts, offs, perm, inv)
    torch.cuda.synchronize()
    c, o, p = moe.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offs.cpu().numpy(), o)
    if T:
        assert np.array_equal(perm.cpu().numpy(), p)
        assert np.array_equal(inv.cpu().numpy(), np.argsort(p))


@pytest.mark.parametrize("wd,H,I,T,E,k,shared", [
    ("f32", 256, 128, 1, 16, 2, False), ("f32", 256, 128, 20, 4, 2, True),
    ("bf16", 2048, 768, 1, 128, 8, False), ("bf16", 2048, 768, 3, 16, 8, True),
    ("bf16", 1024, 512, 37, 6, 3, True), ("int4", 1024, 512, 1, 16, 4, False),
    ("int4", 7168, 2048, 2, 8, 8, False), ("int4", 1024, 256, 19, 5, 2, True),
    # int4: 9 groups of 128 on the gate/up reduction axis split 2/2/2/3 over the 4 warps; 5
    # token columns per pass (4 ring stages)
    ("int4", 1152, 384, 5, 6, 3, True),
    ("nvfp4", 2048, 768, 1, 16, 8, False), ("nvfp4", 1024, 512, 3, 8, 4, True), ("nvfp4", 256, 96, 12, 4, 2, True),
    # NVFP4 on the tensor cores: more pairs per expert than one pass of 8 columns (the shared
    # expert's 19); 9 groups split 2/2/2/3 over the gate/up warps with 5 columns per pass
    ("nvfp4", 1024, 256, 19, 5, 2, True), ("nvfp4", 1152, 384, 5, 6, 3, True),
])
def test_expert_ffn_and_combine_parity(wd, H, I, T, E, k, shared):
    cfg = synth.MoeConfig("t", 1, E, H, I, k, "sigmoid", wd, shared, E, T, (T,), "iid", "decode")
    rng = np.random.default_rng(H + T)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    gates /= gates.sum(axis=1, keepdims=True)
    x = synth.normal_f32(9, 8, 0, 0, T * H).reshape(T, H)
    if wd == "f32":
        xd, xv = torch.from_numpy(x).to(DEV), x
    else:
        xd, xv = _bf16_dev(x)
    blobs = {e: synth.expert_blob(cfg, 0, e) for e in range(E)}
    sh = synth.expert_blob(cfg, 0, 0, shared=True) if shared else None
    S = sorted(set(ids.reshape(-1).tolist()))
    dblobs = [torch.from_numpy(blobs[e]).to(DEV) for e in S]
    experts = list(S)
    if shared:
        dblobs.append(torch.from_numpy(sh).to(DEV))
        experts.append(-1)
    idd = torch.from_numpy(ids).to(DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offs = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    ft.ft_permute(idd, T, k, E, counts, offs, perm, inv)
    hbuf = torch.zeros((T * k + T, I), device=DEV)
    ybuf = torch.zeros((T * k + T, H), device=DEV)
    maxp = int(np.bincount(ids.reshape(-1), minlength=E).max())
    ft.ft_expert_ffn_decode(xd, T, H, I, k, wd, dblobs, experts, maxp, offs, perm, hbuf, ybuf)
    out = torch.empty((T, H), dtype=torch.float32 if wd == "f32" else torch.bfloat16, device=DEV)
    gd = torch.from_numpy(gates).to(DEV)
    ft.ft_combine(ybuf, gd, inv, T, H, k, shared, wd != "f32", out)
    torch.cuda.synchronize()
    # per-pair expert outputs against the oracle's FFN
    _, _, p = moe.permute(ids, E)
    y = ybuf.cpu().numpy()
    for e in S:
        wg, wu, wdn = moe.expert_weights(blobs[e], wd, H, I)
        for q in np.nonzero(ids.reshape(-1)[p] == e)[0]:
            pair = p[q]
            ref = moe.swiglu_ffn(xv[pair // k][None], wg, wu, wdn)[0]
            assert_close(y[q], ref, wd, "y pair %d expert %d" % (pair, e))
    ref_out = moe.experts_and_combine(xv, ids, gates.astype(np.float64), E, wd, H, I, lambda e: blobs[e], sh)
    assert_close(out.float().cpu().numpy(), ref_out, wd, "combined out", stored_bf16=wd != "f32")


# ------------------------------------------------------------- forwards --

def _run_gpu(stack, x, steps, sample=None, stream=None, routing=True, resize_at=None, resize_to=None):
    cfg = stack.cfg
    B = x.shape[1]
    out = torch.empty((cfg.L, B, cfg.H), dtype=stack.xdt, device=DEV)
    outs, ids = {}, np.zeros((steps, cfg.L, B, cfg.k), dtype=np.int32)
    sample = set(range(steps)) if sample is None else set(sample)
    for s in range(steps):
        if resize_at is not None and s == resize_at:
            stack.resize(resize_to)
        for l in range(cfg.L):
            stack.forward(l, x[s], out[l], stream)
            if routing:
                ids[s, l] = stack.last_routing(B)[0]
        if s in sample:
            outs[s] = out.float().cpu().numpy().copy()
    torch.cuda.synchronize()
    return outs, ids


def _check_run(cfg, stack, vals, outs, ids, ref, steps):
    div = first_divergence(ids, ref["ids"][:steps], ref["gap"][:steps], ref.get("zsel"))
    last = steps if div is None else div // (cfg.L * vals.shape[1])
    tr = stack.trace()
    want = trace_tuples(ref["trace"])
    if div is None:
        assert [tuple(t) for t in tr] == want
    else:   # a near-tie flipped a choice: the trace must agree up to that step
        n = sum(1 for a in ref["trace"] if a.call < last * cfg.L)
        assert [tuple(t) for t in tr[:n]] == want[:n]
    for s, o in outs.items():
        if s >= last:
            continue
        for l in range(cfg.L):
            assert_close(o[l], ref["out"][(s, l)], cfg.wdtype, "step %d layer %d" % (s, l),
                         stored_bf16=cfg.x_dtype == "bf16")


def test_config1_tiny_forward_parity():
    cfg = synth.CONFIGS["tiny-fp32"]
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        outs, ids = _run_gpu(st, x, cfg.tokens)
        ref = oracle_run(cfg, st, vals)
        _check_run(cfg, st, vals, outs, ids, ref, cfg.tokens)
        s = st.stats()
        assert (s["routed"], s["hits"], s["misses"]) == (ref["stats"].routed, ref["stats"].hits, ref["stats"].misses)
        assert s["h2d_bytes"] == ref["stats"].fills * cfg.blob_bytes


def test_config2_decode_locality_full_size_parity():
    cfg = synth.CONFIGS["decode-locality-bf16"]
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        steps = cfg.tokens
        sample = list(range(0, steps, 37)) + [steps - 1]
        outs, ids = _run_gpu(st, x, steps, sample=sample)
        ref = oracle_run(cfg, st, vals, ffn_steps=sample)
        _check_run(cfg, st, vals, outs, ids, ref, steps)
        s = st.stats()
        assert s["misses"] == ref["stats"].misses and s["hits"] == ref["stats"].hits
        assert 0 < s["misses"] < s["routed"]


def test_capacity_changes_speed_not_result():
    # FreeToken RTX 5090, dynamic reconfiguration: the output does not depend on the
    # cache size; with every expert resident (`fused`) it is the same again.
    base = synth.CONFIGS["decode-locality-bf16"]
    cfg = dataclasses.replace(base, tokens=24)
    results = []
    for C in (cfg.k, cfg.L * cfg.E // 3, cfg.L * cfg.E):
        with GpuStack(cfg, capacity=C) as st:
            vals, x = st.tokens(1)
            outs, ids = _run_gpu(st, x, cfg.tokens, routing=False)
            results.append((outs, st.stats()))
    for s in results[0][0]:
        for other in results[1:]:
            assert np.array_equal(results[0][0][s], other[0][s])
    assert results[0][1]["misses"] > results[1][1]["misses"] >= results[2][1]["misses"]
    assert results[0][1]["evictions"] > results[1][1]["evictions"] > 0
    assert results[2][1]["evictions"] == 0


def test_evict_every_step_war_hazard():
    # capacity = k: nearly every step overwrites slots read by the previous step's kernels
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=40, C=8)
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        outs, ids = _run_gpu(st, x, cfg.tokens)
        ref = oracle_run(cfg, st, vals)
        _check_run(cfg, st, vals, outs, ids, ref, cfg.tokens)
        assert st.stats()["evictions"] > 100


def test_capacity_error_changes_nothing():
    cfg = dataclasses.replace(synth.CONFIGS["tiny-fp32"], C=1)
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((1, cfg.H), dtype=torch.float32, device=DEV)
        with pytest.raises(ft.FtError) as ei:
            st.forward(0, x[0], out)
        assert ei.value.code == ft.FT_ERR_CAPACITY
        assert st.trace() == [] and st.stats()["routed"] == 0


def test_resize_grow_and_shrink_mid_run():
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], tokens=60)
    with GpuStack(cfg, capacity=40) as st:
        vals, x = st.tokens(1)
        out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=DEV)
        got = {}
        for s in range(cfg.tokens):
            if s == 20:
                st.resize(90)
            if s == 40:
                st.resize(17)
            st.step(x[s], out)
            got[s] = out.float().cpu().numpy().copy()
        from oracle import lru as olru
        ref_l = olru.SharedLru(40)
        for s in range(cfg.tokens):
            if s == 20:
                ref_l.resize(90)
            if s == 40:
                ref_l.resize(17)
            for l in range(cfg.L):
                r = moe.route(vals[s], synth.router_weights(cfg, l), cfg.k, cfg.gating)
                ref_l.access_set(s * cfg.L + l, l, moe.selected_set(r["ids"]))
                if s % 10 == 9:
                    o = moe.experts_and_combine(vals[s], r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H,
                                                cfg.I, lambda e, l=l: st.pool_blob(l, e))
                    assert_close(got[s][l], o, cfg.wdtype, "step %d layer %d" % (s, l), stored_bf16=cfg.x_dtype == "bf16")
        assert [tuple(t) for t in st.trace()] == trace_tuples(ref_l.trace)
        assert st.stats()["capacity"] == 17


def test_prefill_policy_small():
    cfg = synth.MoeConfig("t", L=3, E=16, H=256, I=128, k=2, gating="sigmoid", wdtype="bf16", shared=True,
                          C=32, tokens=48, batches=(48,), process="iid", mode="prefill")
    with GpuStack(cfg) as st:
        vals, x = st.tokens(48)
        outs, ids = _run_gpu(st, x, 1)
        ref = oracle_run(cfg, st, vals)
        _check_run(cfg, st, vals, outs, ids, ref, 1)
        s = st.stats()
        assert s["misses"] == 0 and s["prefetch_misses"] == 3 * 16


def test_nvfp4_stack_decode_forward_parity():
    cfg = synth.MoeConfig("nvfp4-small", L=2, E=32, H=1024, I=512, k=4, gating="softmax", wdtype="nvfp4",
                          shared=False, C=24, tokens=16, batches=(1,), process="ar1", mode="decode")
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        outs, ids = _run_gpu(st, x, cfg.tokens)
        ref = oracle_run(cfg, st, vals)
        _check_run(cfg, st, vals, outs, ids, ref, cfg.tokens)


def test_forwards_on_alternating_streams():
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=16, C=20)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=DEV)
        got = {}
        for s in range(cfg.tokens):
            for l in range(cfg.L):
                st.forward(l, x[s], out[l], s1 if (s + l) % 2 else s2)
            torch.cuda.synchronize()
            got[s] = out.float().cpu().numpy().copy()
        ref = oracle_run(cfg, st, vals)
        for s in range(cfg.tokens):
            for l in range(cfg.L):
                assert_close(got[s][l], ref["out"][(s, l)], "bf16", "step %d layer %d" % (s, l), stored_bf16=True)


def test_empty_forward_changes_nothing():
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=1, tokens=4, C=16)
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.zeros((1, cfg.H), dtype=torch.bfloat16, device=DEV)
        st.forward(0, x[0][:0], out[:0])                       # zero tokens: a no-op
        torch.cuda.synchronize()
        assert st.trace() == [] and st.stats()["routed"] == 0
        assert float(out.abs().sum()) == 0.0


def test_every_expert_selected():
    # k = E: every expert of the layer is selected for every token (top-k is a sort)
    cfg = synth.MoeConfig("k-eq-e", L=2, E=8, H=256, I=128, k=8, gating="softmax", wdtype="bf16",
                          shared=False, C=16, tokens=6, batches=(1,), process="ar1", mode="decode")
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        outs, ids = _run_gpu(st, x, cfg.tokens)
        ref = oracle_run(cfg, st, vals)
        _check_run(cfg, st, vals, outs, ids, ref, cfg.tokens)
        assert st.stats()["misses"] == 16                      # only the first step's compulsory misses
