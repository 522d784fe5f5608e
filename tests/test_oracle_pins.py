"""Pins the CPU oracle to facts other than itself: hand-worked examples
(tests/golden), library routines, closed forms, brute force on tiny inputs,
and the invariants the FreeToken pages fix (capacity changes speed, not the
result; the all-resident `fused` result equals the cached one; gates sum to 1).
"""
import os

import numpy as np
import pytest
import scipy.special

import synth
from oracle import lru as olru
from oracle import moe
from oracle.run import run_workload
from naive_lru import NaiveLru

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------- formats ----

def _golden_lines(name):
    with open(os.path.join(GOLD, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln.split()


def test_bf16_widening_golden():
    n = 0
    for f in _golden_lines("int4_bf16_formats.txt"):
        if f[0] == "bf16":
            bits = np.array([int(f[1], 16)], dtype=np.uint16)
            assert moe.widen_bf16(bits)[0] == float(f[2])
            n += 1
    assert n >= 6


def test_int4_nibbles_golden():
    n = 0
    for f in _golden_lines("int4_bf16_formats.txt"):
        if f[0] == "int4":
            b = np.array([[int(f[1], 16)]], dtype=np.uint8)
            assert moe.decode_int4(b).tolist() == [[int(f[2]), int(f[3])]]
            n += 1
    assert n >= 5


def test_int4_roundtrip_within_half_step():
    # quantise (data fixture) then dequantise (oracle): every element within s/2
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    w[3, :128] = 0.0                                  # an all-zero group -> s = 0, q = 0
    w[5, 7] = 0.5                                     # an outlier group
    q, s = synth.quantise_int4(w)
    deq = moe.dequant_int4(q, s)
    sc = np.repeat(moe.widen_bf16(s), 128, axis=1)
    err = np.abs(deq - w.astype(np.float64))
    assert np.all(err <= sc / 2 * (1 + 1e-6) + 1e-30)
    assert np.all(deq[3, :128] == 0.0)
    # the largest element of each group maps to +-7 or +-6 steps (s = bf16(max/7))
    qi = moe.decode_int4(q)
    assert np.abs(qi).max() == 7 and qi.min() >= -8


def test_expert_blob_layout_matches_draws():
    # bf16 and f32 blobs hold exactly the draws, rounded; int4 blobs within s/2
    for wd, H, I in (("f32", 32, 16), ("bf16", 64, 32), ("int4", 256, 128)):
        cfg = synth.MoeConfig("t", 1, 2, H, I, 1, "softmax", wd, False, 1, 1, (1,), "iid", "decode")
        blob = synth.expert_blob(cfg, 0, 1)
        assert blob.nbytes == cfg.blob_bytes
        wg, wu, wd_ = moe.expert_weights(blob, wd, H, I)
        fg, fu, fd = synth.expert_weights_f32(cfg, 0, 1)
        for a, b in ((wg, fg), (wu, fu), (wd_, fd)):
            if wd == "f32":
                assert np.array_equal(a, b.astype(np.float64))
            elif wd == "bf16":
                assert np.max(np.abs(a - b) / np.abs(b).clip(1e-30)) <= 2.0 ** -8
            else:
                assert np.max(np.abs(a - b)) <= np.abs(b).max() / 7 * 0.51 + 1e-9


# ------------------------------------------------------------- routing ----

def test_topk_matches_stable_argsort_and_breaks_ties_low():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((50, 16)).astype(np.float32)
    z[0, :] = 0.5                                     # all equal -> 0, 1, 2, ...
    z[1, [3, 9, 12]] = 7.0                            # tie at the top
    z[2, [4, 6]] = -9.0
    z[2, :] = np.where(np.arange(16) < 14, -9.0, z[2, :])  # many ties at the cut
    for k in (1, 2, 5, 16):
        ids, gap = moe.topk(z, k)
        ref = np.argsort(-z, axis=1, kind="stable")[:, :k]
        assert np.array_equal(ids, ref)
    ids, _ = moe.topk(z, 3)
    assert ids[0].tolist() == [0, 1, 2] and ids[1].tolist() == [3, 9, 12]
    # the near-tie gap: k-th largest minus (k+1)-th largest logit, from a library sort;
    # zero on a tie at the cut, infinite when every expert is selected
    srt = -np.sort(-z.astype(np.float64), axis=1)
    for k in (1, 3, 14, 15, 16):
        _, gap = moe.topk(z, k)
        want = srt[:, k - 1] - srt[:, k] if k < 16 else np.full(z.shape[0], np.inf)
        assert np.array_equal(gap, want)
    assert moe.topk(z, 3)[1][0] == 0.0 and moe.topk(z, 13)[1][2] == 0.0


def test_router_logits_rank1_closed_form_and_einsum():
    rng = np.random.default_rng(3)
    a = rng.standard_normal(12)
    b = rng.standard_normal(40)
    W = np.outer(a, b).astype(np.float32)             # W_r[e, h] = a_e b_h
    x = rng.standard_normal((5, 40)).astype(np.float32)
    z = moe.router_logits(x, W)
    closed = np.outer(x.astype(np.float64) @ b, a)    # z[t,e] = a_e (b . x_t)
    assert np.allclose(z, closed, rtol=1e-6, atol=1e-6)
    z2 = np.einsum("th,eh->te", x.astype(np.float64), W.astype(np.float64)).astype(np.float32)
    assert np.max(np.abs(z.view(np.int32) - z2.view(np.int32))) <= 1   # within one fp32 ulp
    assert z.dtype == np.float32


def test_gates_library_forms():
    rng = np.random.default_rng(4)
    z = rng.standard_normal((20, 32)).astype(np.float32) * 3
    for k in (1, 2, 6, 32):
        ids, _ = moe.topk(z, k)
        zs = np.take_along_axis(z, ids.astype(np.int64), axis=1)
        gs = moe.gates(zs, "softmax")
        full = scipy.special.softmax(z.astype(np.float64), axis=1)
        ref = np.take_along_axis(full, ids.astype(np.int64), axis=1)
        ref /= ref.sum(axis=1, keepdims=True)
        assert np.allclose(gs, ref, rtol=1e-12, atol=1e-15)
        gg = moe.gates(zs, "sigmoid")
        sref = scipy.special.expit(zs.astype(np.float64))
        assert np.allclose(gg, sref / sref.sum(axis=1, keepdims=True), rtol=1e-12)
        assert np.allclose(gs.sum(axis=1), 1.0, atol=1e-12)
        assert np.allclose(gg.sum(axis=1), 1.0, atol=1e-12)
        if k == 1:
            assert np.all(gs == 1.0) and np.all(gg == 1.0)
    # k = E: the renormalised softmax is the full softmax
    ids, _ = moe.topk(z, 32)
    zs = np.take_along_axis(z, ids.astype(np.int64), axis=1)
    assert np.allclose(moe.gates(zs, "softmax"),
                       np.take_along_axis(scipy.special.softmax(z.astype(np.float64), axis=1),
                                          ids.astype(np.int64), axis=1), rtol=1e-12)


def test_permute_matches_stable_sort_and_bincount():
    rng = np.random.default_rng(5)
    for T, k, E in ((1, 2, 16), (7, 3, 8), (33, 8, 128), (64, 6, 256)):
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
        counts, offsets, perm = moe.permute(ids, E)
        assert np.array_equal(counts, np.bincount(ids.reshape(-1), minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(perm, np.argsort(ids.reshape(-1), kind="stable"))


# ---------------------------------------------------------- expert FFN ----

def test_swiglu_rank1_closed_form():
    rng = np.random.default_rng(6)
    H, I = 24, 10
    ag, bg, au, bu = rng.standard_normal(I), rng.standard_normal(H), rng.standard_normal(I), rng.standard_normal(H)
    ad, bd = rng.standard_normal(H), rng.standard_normal(I)
    Wg, Wu, Wd = np.outer(ag, bg), np.outer(au, bu), np.outer(ad, bd)
    x = rng.standard_normal((3, H))
    y = moe.swiglu_ffn(x, Wg, Wu, Wd)
    for t in range(3):
        u = ag * (bg @ x[t])
        v = au * (bu @ x[t])
        h = u * scipy.special.expit(u) * v
        assert np.allclose(y[t], ad * (bd @ h), rtol=1e-10, atol=1e-12)


def test_moe_hand_example_golden():
    vals = {f[0]: f[1:] for f in _golden_lines("moe_hand_example.txt") if f[0] != "expert"}
    experts = [f[1:] for f in _golden_lines("moe_hand_example.txt") if f[0] == "expert"]
    x = np.array([[float(v) for v in vals["x"]]])
    Wr = np.array([float(v) for v in vals["router"]]).reshape(3, 2).astype(np.float32)
    blobs = {}
    for f in experts:
        e = int(f[0])
        w = np.array([float(v) for v in f[1:]], dtype=np.float32)   # gate[1x2] up[1x2] down[2x1]
        blobs[e] = w.view(np.uint8)
    r = moe.moe_layer(x, Wr, 2, "softmax", "f32", 2, 1, lambda e: blobs[e])
    assert r["ids"][0].tolist() == [int(v) for v in vals["ids"]]
    assert np.allclose(r["gates"][0], [float(v) for v in vals["gates"]], rtol=1e-14)
    assert np.allclose(r["out"][0], [float(v) for v in vals["out"]], rtol=1e-13)


def _dense_brute_force(x, Wr, k, gating, weights):
    """All E experts on every token, a dense gate vector zero off the top-k."""
    T, H = x.shape
    E = Wr.shape[0]
    out = np.zeros((T, H))
    for t in range(T):
        z = [float(np.float32(sum(float(x[t, h]) * float(Wr[e, h]) for h in range(H)))) for e in range(E)]
        rank = [sum(1 for f in range(E) if z[f] > z[e] or (z[f] == z[e] and f < e)) for e in range(E)]
        mask = [1.0 if rank[e] < k else 0.0 for e in range(E)]
        if gating == "softmax":
            m = max(z[e] for e in range(E) if mask[e])
            w = [mask[e] * np.exp(z[e] - m) for e in range(E)]
        else:
            w = [mask[e] / (1 + np.exp(-z[e])) for e in range(E)]
        w = np.array(w) / sum(w)
        for e in range(E):
            Wg, Wu, Wd = weights[e]
            hvec = np.array([(lambda u, v: u / (1 + np.exp(-u)) * v)(
                sum(Wg[i, c] * x[t, c] for c in range(H)), sum(Wu[i, c] * x[t, c] for c in range(H)))
                for i in range(Wg.shape[0])])
            ye = np.array([sum(Wd[r, i] * hvec[i] for i in range(Wg.shape[0])) for r in range(H)])
            out[t] += w[e] * ye
    return out


@pytest.mark.parametrize("E,H,I,k,gating,wd", [
    (6, 8, 4, 2, "softmax", "f32"),
    (5, 6, 3, 1, "sigmoid", "f32"),
    (8, 8, 6, 3, "sigmoid", "bf16"),
    (4, 6, 2, 4, "softmax", "bf16"),
    (4, 128, 128, 2, "sigmoid", "int4"),
    (4, 64, 32, 2, "softmax", "nvfp4"),
])
def test_sparse_layer_equals_dense_brute_force(E, H, I, k, gating, wd):
    cfg = synth.MoeConfig("t", 1, E, H, I, k, gating, wd, False, E, 5, (5,), "iid", "decode")
    x = synth.normal_f32(11, 8, 0, 0, 5 * H).reshape(5, H).astype(np.float64)
    Wr = synth.normal_f32(11, 4, 0, 0, E * H, 0.3).reshape(E, H)
    blobs = [synth.expert_blob(cfg, 0, e) for e in range(E)]
    weights = []
    for e in range(E):
        fg, fu, fd = synth.expert_weights_f32(cfg, 0, e)
        if wd == "bf16":
            widen = lambda a: (synth.round_bf16(a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            fg, fu, fd = widen(fg), widen(fu), widen(fd)
        elif wd in ("int4", "nvfp4"):
            fg, fu, fd = moe.expert_weights(blobs[e], wd, H, I)   # dequant pinned separately
        weights.append((np.asarray(fg, np.float64), np.asarray(fu, np.float64), np.asarray(fd, np.float64)))
    if wd in ("int4", "nvfp4"):
        x = x[:2]
    r = moe.moe_layer(x, Wr, k, gating, wd, H, I, lambda e: blobs[e])
    ref = _dense_brute_force(x, Wr, k, gating, weights)
    assert np.allclose(r["out"], ref, rtol=1e-9, atol=1e-12)
    assert np.allclose(r["gates"].sum(axis=1), 1.0, atol=1e-12)


# ----------------------------------------------------------------- LRU ----

def test_lru_hand_worked_golden():
    c = None
    exp = []
    got = []
    for f in _golden_lines("lru_hand_4slot.txt"):
        if f[0] == "capacity":
            c = olru.SharedLru(int(f[1]))
        elif f[0] == "step":
            got.extend(c.access_set(int(f[1]), int(f[2]), [int(v) for v in f[3:]]))
        elif f[0] in ("hit", "miss"):
            exp.append((f[0] == "hit",) + tuple(int(v) for v in f[1:]))
        elif f[0] == "capacity_error":
            before = (dict(c.order), list(c.order))
            with pytest.raises(olru.CapacityError):
                c.access_set(int(f[1]), int(f[2]), [int(v) for v in f[3:]])
            assert (dict(c.order), list(c.order)) == before
        elif f[0] == "resize":
            moves = c.resize(int(f[1]))
            want = [tuple(int(v) for v in m.split("->")) for m in f[2:]]
            assert moves == want
        elif f[0] == "stats":
            st = c.stats
            assert (st.routed, st.hits, st.misses, st.evictions) == tuple(int(v) for v in f[1:])
    assert [(a.hit, a.layer, a.expert, a.slot, a.ev_layer, a.ev_expert) for a in got] == exp


def _random_steps(rng, n, L, E, smax):
    for call in range(n):
        l = call % L
        m = int(rng.integers(1, smax + 1))
        yield call, l, rng.choice(E, m, replace=False)


@pytest.mark.parametrize("C,L,E,smax", [(1, 1, 4, 1), (4, 1, 16, 2), (7, 3, 10, 5), (20, 4, 32, 8), (64, 2, 64, 40)])
def test_lru_equals_naive_lru(C, L, E, smax):
    rng = np.random.default_rng(C * 100 + E)
    a, b = olru.SharedLru(C), NaiveLru(C)
    for call, l, S in _random_steps(rng, 400, L, E, min(smax, C)):
        a.access_set(call, l, S)
        b.access_set(call, l, S)
        # exact invariants after every step: the step's experts are resident, size <= C
        assert all((l, int(e)) in a.order for e in S)
        assert len(a.order) <= C and len(set(a.order.values())) == len(a.order)
    assert [tuple(x.__dict__.values()) for x in a.trace] == b.trace
    st = a.stats
    assert st.hits + st.misses == st.routed == len(a.trace)


def test_lru_compulsory_misses_only_when_everything_fits():
    rng = np.random.default_rng(7)
    L, E = 3, 12
    c = olru.SharedLru(L * E)
    keys = set()
    for call, l, S in _random_steps(rng, 300, L, E, 5):
        c.access_set(call, l, S)
        keys.update((l, int(e)) for e in S)
    assert c.stats.misses == len(keys) and c.stats.evictions == 0


def test_lru_shrink_keeps_recency_and_packs_slots():
    rng = np.random.default_rng(8)
    c = olru.SharedLru(40)
    for call, l, S in _random_steps(rng, 200, 2, 30, 6):
        c.access_set(call, l, S)
    before = list(c.order.keys())
    c.resize(17)
    assert list(c.order.keys()) == before[-17:]
    assert all(s < 17 for s in c.order.values()) and len(set(c.order.values())) == 17
    c.resize(25)
    assert sorted(c.free) == list(range(17, 25))


# ---------------------------------------------------------- invariants ----

def _tiny_run(cfg, capacity, through_slots, steps=6):
    x, _ = synth.tokens(cfg, cfg.batches[0])
    x = x[:steps]
    blobs = {(l, e): synth.expert_blob(cfg, l, e) for l in range(cfg.L) for e in range(cfg.E)}
    return run_workload(L=cfg.L, E=cfg.E, H=cfg.H, I=cfg.I, k=cfg.k, gating=cfg.gating,
                        wdtype=cfg.wdtype, capacity=capacity, x_steps=x,
                        router_of=lambda l: synth.router_weights(cfg, l),
                        blob_of=lambda l, e: blobs[(l, e)], through_slots=through_slots)


def test_capacity_independence_and_fused_equivalence():
    cfg = synth.MoeConfig("t", L=3, E=12, H=32, I=16, k=3, gating="sigmoid", wdtype="bf16",
                          shared=False, C=4, tokens=12, batches=(2,), process="ar1", mode="decode")
    runs = [_tiny_run(cfg, C, True) for C in (cfg.k * 2, cfg.L * cfg.E // 3, cfg.L * cfg.E)]
    direct = _tiny_run(cfg, cfg.L * cfg.E, False)       # `fused`: every expert read in place
    for r in runs:
        assert np.array_equal(r["ids"], direct["ids"])
        for key in direct["out"]:
            assert np.array_equal(r["out"][key], direct["out"][key])
    assert runs[0]["stats"].misses > runs[-1]["stats"].misses


def test_results_unchanged_by_a_resize_through_the_slots():
    # a grow and a shrink half-way (FreeToken RTX 5090, dynamic reconfiguration: the
    # cache size changes speed, not the result); experts are read from the slot arena,
    # so a shrink's slot moves must carry the bytes along
    # one token per step and 2 of 8 experts per layer: the survivors a shrink moves are
    # read again before they are evicted
    cfg = synth.MoeConfig("t", L=2, E=8, H=32, I=16, k=2, gating="softmax", wdtype="bf16",
                          shared=False, C=4, tokens=16, batches=(1,), process="ar1", mode="decode")
    x, _ = synth.tokens(cfg, 1)
    x = x[:12]
    blobs = {(l, e): synth.expert_blob(cfg, l, e) for l in range(cfg.L) for e in range(cfg.E)}
    kw = dict(L=cfg.L, E=cfg.E, H=cfg.H, I=cfg.I, k=cfg.k, gating=cfg.gating, wdtype=cfg.wdtype,
              x_steps=x, router_of=lambda l: synth.router_weights(cfg, l), blob_of=lambda l, e: blobs[(l, e)])
    direct = run_workload(capacity=cfg.L * cfg.E, through_slots=False, **kw)
    for c0, c1 in ((20, 4), (4, 20)):
        r = run_workload(capacity=c0, resize_to=c1, through_slots=True, **kw)
        assert np.array_equal(r["ids"], direct["ids"])
        for key in direct["out"]:
            assert np.array_equal(r["out"][key], direct["out"][key]), (c0, c1, key)
        assert r["lru"].capacity == c1


def test_config1_oracle_runs_and_gates_sum_to_one():
    cfg = synth.CONFIGS["tiny-fp32"]
    r = _tiny_run(cfg, cfg.C, True, steps=8)
    assert r["ids"].shape == (8, 1, 1, 2)
    assert np.allclose(r["gates"].sum(axis=-1), 1.0, atol=1e-12)
    assert r["stats"].routed == 16


def test_prefill_double_buffer_evicts_exactly_the_previous_layer():
    cfg = synth.MoeConfig("t", L=4, E=8, H=16, I=8, k=2, gating="sigmoid", wdtype="bf16",
                          shared=False, C=16, tokens=24, batches=(24,), process="iid", mode="prefill")
    x, _ = synth.tokens(cfg, 24)
    blobs = {(l, e): synth.expert_blob(cfg, l, e) for l in range(cfg.L) for e in range(cfg.E)}
    r = run_workload(L=4, E=8, H=16, I=8, k=2, gating="sigmoid", wdtype="bf16", capacity=16,
                     x_steps=x, router_of=lambda l: synth.router_weights(cfg, l),
                     blob_of=lambda l, e: blobs[(l, e)], prefill=True, through_slots=True)
    st = r["stats"]
    assert st.misses == 0 and st.hits == st.routed            # every routed access was prefetched
    assert st.prefetch == 4 * 8 and st.prefetch_misses == 4 * 8
    for a in r["trace"]:
        if a.kind == olru.PREFETCH and a.ev_layer >= 0:
            assert a.ev_layer == a.layer - 2                   # victims: the layer before last


def test_prefill_double_buffer_hand_worked_golden():
    # routers built so that one-hot tokens make the file's selections (top-1, 2 tokens
    # per step: token 0 picks the first listed expert, token 1 the last)
    L, E, H, steps = 3, 3, 4, 2
    sel, want, stats = {}, [], None
    for f in _golden_lines("prefill_double_buffer_hand.txt"):
        if f[0] == "select":
            sel[(int(f[1]), int(f[2]))] = [int(v) for v in f[3:]]
        elif f[0] == "stats":
            stats = tuple(int(v) for v in f[1:])
        else:
            want.append((int(f[0]), int(f[1]), int(f[2]), olru.PREFETCH if f[3] == "P" else olru.ROUTED,
                         f[4] == "hit", int(f[5]), int(f[6]), int(f[7])))
    W = np.zeros((L, E, H), dtype=np.float32)
    for (s_, l), es in sel.items():
        W[l, es[0], 2 * s_] = 1.0
        W[l, es[-1], 2 * s_ + 1] = 1.0
    x = np.zeros((steps, 2, H))
    for s_ in range(steps):
        x[s_, 0, 2 * s_] = x[s_, 1, 2 * s_ + 1] = 1.0
    r = run_workload(L=L, E=E, H=H, I=8, k=1, gating="softmax", wdtype="f32", capacity=2 * E,
                     x_steps=x, router_of=lambda l: W[l], blob_of=lambda l, e: None,
                     prefill=True, ffn_steps=[])
    for (s_, l), es in sel.items():
        assert sorted(set(r["ids"][s_, l].reshape(-1).tolist())) == es
    got = [(a.call, a.layer, a.expert, a.kind, a.hit, a.slot, a.ev_layer, a.ev_expert) for a in r["trace"]]
    assert got == want
    st = r["stats"]
    assert (st.routed, st.hits, st.misses, st.prefetch, st.prefetch_hits, st.prefetch_misses,
            st.evictions) == stats


def test_ar1_tokens_have_locality():
    x = synth.ar1_chain(0, 0, 4000, 64).astype(np.float64)
    assert abs(x.var() - 1.0) < 0.1
    rho = np.mean(np.sum(x[1:] * x[:-1], axis=1) / np.sum(x[:-1] * x[:-1], axis=1))
    assert abs(rho - 0.9) < 0.02


def test_shared_expert_adds_with_weight_one():
    cfg = synth.MoeConfig("t", 1, 6, 16, 8, 2, "sigmoid", "bf16", True, 6, 3, (3,), "iid", "decode")
    x = synth.normal_f32(5, 8, 0, 0, 3 * 16).reshape(3, 16)
    Wr = synth.router_weights(cfg, 0)
    blobs = [synth.expert_blob(cfg, 0, e) for e in range(6)]
    sh = synth.expert_blob(cfg, 0, 0, shared=True)
    with_sh = moe.moe_layer(x, Wr, 2, "sigmoid", "bf16", 16, 8, lambda e: blobs[e], sh)["out"]
    without = moe.moe_layer(x, Wr, 2, "sigmoid", "bf16", 16, 8, lambda e: blobs[e])["out"]
    widen = lambda a: (synth.round_bf16(a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    fg, fu, fd = (widen(a) for a in synth.expert_weights_f32(cfg, 0, 0, shared=True))
    xs = x.astype(np.float64)
    u, v = xs @ fg.T, xs @ fu.T
    shared_direct = (u * scipy.special.expit(u) * v) @ fd.T
    assert np.allclose(with_sh - without, shared_direct, rtol=1e-10, atol=1e-14)
    assert not np.array_equal(sh, blobs[0])


def test_fp4_fp8_decoders_golden():
    n4 = n8 = 0
    for f in _golden_lines("int4_bf16_formats.txt"):
        if f[0] == "e2m1":
            v = moe.decode_e2m1(np.array([int(f[1])]))[0]
            assert v == float(f[2]) and np.signbit(v) == f[2].startswith("-")
            n4 += 1
        elif f[0] == "e4m3":
            assert moe.decode_e4m3(np.array([int(f[1], 16)]))[0] == float(f[2])
            n8 += 1
    assert n4 == 16 and n8 >= 8
    assert np.isnan(moe.decode_e4m3(np.array([0x7F]))[0])


def test_nvfp4_roundtrip_is_nearest_grid_point():
    # brute force: every dequantised element is the grid value e2m1 * (block scale) nearest
    # to the draw (saturating at 6 * scale), the block scale is the e4m3 value nearest to
    # max|w| / 6 / g
    rng = np.random.default_rng(12)
    w = (rng.standard_normal((8, 64)) * 0.02).astype(np.float32)
    w[2, :16] = 0.0
    g = float(np.float32(np.abs(w).max() / (448 * 6)))
    q, s = synth.quantise_nvfp4(w, g)
    deq = moe.dequant_nvfp4(q, s, g)
    grid = moe.decode_e2m1(np.arange(16))
    e4 = moe.decode_e4m3(np.arange(0x7F))
    for r in range(8):
        for b in range(4):
            blk = w[r, 16 * b:16 * b + 16].astype(np.float64)
            want_s = e4[np.argmin(np.abs(e4 - np.float32(np.abs(blk).max() / 6.0 / np.float32(g))))]
            sc = moe.decode_e4m3(s[r, b:b + 1])[0]
            assert sc == want_s
            step = sc * g
            for j in range(16):
                if step == 0:
                    assert deq[r, 16 * b + j] == 0.0
                    continue
                dist = np.abs(blk[j] / np.float32(step) - grid)
                assert abs(deq[r, 16 * b + j] / step - grid[np.argmin(dist)]) < 1e-12 or \
                    abs(dist[np.argmin(dist)] - np.sort(dist)[1]) < 1e-6     # a tie: either neighbour


def test_nvfp4_blob_layout_matches_draws():
    cfg = synth.MoeConfig("t", 1, 2, 64, 32, 1, "softmax", "nvfp4", False, 1, 1, (1,), "iid", "decode")
    blob = synth.expert_blob(cfg, 0, 1)
    assert blob.nbytes == cfg.blob_bytes
    wg, wu, wd = moe.expert_weights(blob, "nvfp4", 64, 32)
    fg, fu, fd = synth.expert_weights_f32(cfg, 0, 1)
    for a, b in ((wg, fg), (wu, fu), (wd, fd)):
        assert a.shape == b.shape
        # within half the largest grid step (2 * block scale * g) of the draw
        assert np.max(np.abs(a - b)) <= np.abs(b).max() / 6 * 1.1
        assert np.corrcoef(a.reshape(-1), b.reshape(-1))[0, 1] > 0.98
