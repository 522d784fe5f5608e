"""CPU checks of the C ABI: the library loads, exports every function the
header declares, rejects bad arguments without a GPU, and its own slot table
(run host-only through ft_cache_simulate) matches the oracle's LRU."""
import os
import re
import subprocess

import numpy as np
import pytest

import moe_expert_offload_top_b200 as ft
from oracle import lru as olru

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLD = os.path.join(ROOT, "tests", "golden")


def _declared():
    names = []
    with open(os.path.join(ROOT, "include", "ftmoe.h")) as f:
        for ln in f:
            m = re.match(r"^FT_API\s+[\w\s\*]+?\b(ft_\w+)\(", ln)
            if m:
                names.append(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    decl = _declared()
    assert len(decl) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", ft.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in decl if n not in exported]
    assert not missing, missing
    assert set(decl) == set(ft.EXPORTED)
    assert ft.ft_version().startswith("ftmoe")


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", ft.LIB_PATH], capture_output=True, text=True).stdout
    arches = set(re.findall(r"sm_(\d+a?)", out))
    assert arches == {"100a"}, arches


def test_invalid_arguments_are_rejected_without_a_gpu():
    with pytest.raises(ft.FtError):
        ft.ft_moe_create(0, 1, 8, 8, "bf16", 1)
    with pytest.raises(ft.FtError):
        ft.ft_moe_create(300, 1, 8, 8, "bf16", 1)             # > FT_MAX_EXPERTS
    with pytest.raises(ft.FtError):
        ft.ft_moe_create(16, 2, 200, 128, "int4", 4)          # int4 needs multiples of 128
    assert "invalid" in ft.ft_last_error(None) or "int4" in ft.ft_last_error(None)
    with pytest.raises(ft.FtError):
        ft.ft_router_topk(0, 1, 0, 1, 8, 300, 2, 0, 0, 0, 0)
    with pytest.raises(ft.FtError):
        ft.ft_cache_simulate(1, 4, 2, [7, 1])                 # unknown op


def _golden_script():
    ops, expect, cap0 = [], [], None
    with open(os.path.join(GOLD, "lru_hand_4slot.txt")) as f:
        for ln in f:
            t = ln.split()
            if not t or t[0].startswith("#"):
                continue
            if t[0] == "capacity":
                cap0 = int(t[1])
            elif t[0] == "step":
                es = [int(v) for v in t[3:]]
                ops += [0, int(t[1]), int(t[2]), 0, len(es)] + es
            elif t[0] == "capacity_error":
                es = [int(v) for v in t[3:]]
                ops += [0, int(t[1]), int(t[2]), 0, len(es)] + es
            elif t[0] == "resize":
                ops += [1, int(t[1])]
            elif t[0] in ("hit", "miss"):
                expect.append((int(t[0] == "hit"),) + tuple(int(v) for v in t[1:]))
            elif t[0] == "stats":
                stats = tuple(int(v) for v in t[1:])
    return cap0, ops, expect, stats


def test_library_lru_matches_hand_worked_golden():
    cap, ops, expect, stats = _golden_script()
    trace, st, nerr = ft.ft_cache_simulate(2, 16, cap, ops)
    assert nerr == 1
    got = [(a[4], a[1], a[2], a[5], a[6], a[7]) for a in trace]
    assert got == expect
    assert (st["routed"], st["hits"], st["misses"], st["evictions"]) == stats


@pytest.mark.parametrize("C,L,E,smax,resizes", [
    (1, 1, 4, 1, ()), (4, 1, 16, 2, ()), (7, 3, 10, 5, (12, 5)), (20, 4, 32, 8, (40, 9, 33)),
    (64, 2, 64, 40, (100, 64)), (204, 4, 128, 8, ()),
])
def test_library_lru_matches_oracle_on_random_scripts(C, L, E, smax, resizes):
    rng = np.random.default_rng(C + 7 * E)
    ref = olru.SharedLru(C)
    ops = []
    cap = C
    todo = list(resizes)
    n_steps = 600
    for call in range(n_steps):
        if todo and call % (n_steps // (len(resizes) + 1)) == 0 and call > 0:
            cap = todo.pop(0)
            ops += [1, cap]
            ref.resize(cap)
        l = call % L
        kind = int(rng.random() < 0.2)
        m = int(rng.integers(1, min(smax, cap) + 1))
        es = sorted(rng.choice(E, m, replace=False).tolist())
        ops += [0, call, l, kind, m] + es
        ref.access_set(call, l, es, kind)
    trace, st, nerr = ft.ft_cache_simulate(L, E, C, ops)
    want = [(a.call, a.layer, a.expert, a.kind, int(a.hit), a.slot, a.ev_layer, a.ev_expert) for a in ref.trace]
    assert nerr == 0
    assert trace == want
    s = ref.stats
    assert (st["routed"], st["hits"], st["misses"], st["prefetch"], st["prefetch_hits"],
            st["prefetch_misses"], st["evictions"]) == (s.routed, s.hits, s.misses, s.prefetch,
                                                        s.prefetch_hits, s.prefetch_misses, s.evictions)
    assert st["resident"] == len(ref.order) and st["capacity"] == cap


def test_static_policy_hand_worked():
    # 2 layers x 4 experts, capacity 3: keys (0,0) (0,1) (0,2) are resident for good.
    ops = [0, 0, 0, 0, 2, 1, 3,      # layer 0: expert 1 hit (slot 1), expert 3 miss
           0, 1, 1, 0, 2, 0, 2,      # layer 1: both miss (keys 4, 6)
           1, 5,                     # resize: keys 0..4 resident
           0, 2, 1, 0, 2, 0, 3]      # layer 1: expert 0 (key 4) hit, expert 3 (key 7) miss
    trace, st, nerr = ft.ft_cache_simulate_policy(ft.FT_POLICY_STATIC, 2, 4, 3, ops)
    assert [(a[1], a[2], a[4], a[5]) for a in trace] == [
        (0, 1, 1, 1), (0, 3, 0, -1), (1, 0, 0, -1), (1, 2, 0, -1), (1, 0, 1, 4), (1, 3, 0, -1)]
    assert (st["routed"], st["hits"], st["misses"], st["evictions"]) == (6, 2, 4, 0)
    lru = ft.ft_cache_simulate_policy(ft.FT_POLICY_LRU, 2, 4, 3, ops)
    assert lru == ft.ft_cache_simulate(2, 4, 3, ops)


def test_lru_beats_static_split_on_locality_traces():
    # Trend of the pages (FreeToken linux, performance: 16% vs 62% of expert reads
    # missed): on the AR(1) decode workload the shared LRU misses far less than a
    # static split of the same capacity.  A trend, not a pin.
    import synth
    from oracle import moe
    cfg = synth.CONFIGS["decode-locality-bf16"]
    vals, _ = synth.tokens(cfg, 1)
    routers = [synth.router_weights(cfg, l) for l in range(cfg.L)]
    ops = []
    for s in range(256):
        for l in range(cfg.L):
            S = moe.selected_set(moe.topk(moe.router_logits(vals[s], routers[l]), cfg.k)[0]).tolist()
            ops += [0, s * cfg.L + l, l, 0, len(S)] + S
    rates = {}
    for pol in (ft.FT_POLICY_LRU, ft.FT_POLICY_STATIC):
        _, st, _ = ft.ft_cache_simulate_policy(pol, cfg.L, cfg.E, cfg.C, ops)
        rates[pol] = st["misses"] / st["routed"]
    assert rates[ft.FT_POLICY_LRU] < 0.5 * rates[ft.FT_POLICY_STATIC]
    assert 0.3 < rates[ft.FT_POLICY_STATIC] < 0.9


def test_bandwidth_profile_host_part(tmp_path):
    # the host half of the bandwidth profile runs without a GPU and writes its file
    from moe_expert_offload_top_b200 import bwprofile
    out = tmp_path / "bw.json"
    assert bwprofile.main(["--host-only", "--out", str(out), "--bytes", str(1 << 22), "--iters", "2"]) == 0
    import json
    prof = json.loads(out.read_text())
    assert prof["host_memcpy_gbs_1_thread"] > 0 and prof["host_memcpy_gbs_all_threads"] > 0
    assert "h2d_gbs" not in prof
    with pytest.raises(ft.FtError):
        ft.ft_probe_host_memory(16, 1, 1)          # below the minimum size


def test_calls_fail_cleanly_without_a_device():
    # with no GPU the library refuses with a message instead of crashing; invalid
    # arguments are refused first in any case
    import torch
    with pytest.raises(ft.FtError) as ei:
        ft.ft_moe_create(16, 20, 256, 128, "f32", 4)          # top_k > num_experts
    assert "invalid argument" in str(ei.value)
    with pytest.raises(ft.FtError):
        ft.ft_moe_create(16, 2, 100, 128, "int4", 4)          # int4 needs multiples of 128
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(ft.FtError) as ei:
        ft.ft_moe_create(16, 2, 256, 128, "f32", 4)
    assert "allocation" in str(ei.value) or "CUDA" in str(ei.value)


def test_import_fails_loudly_without_the_library(tmp_path):
    # the package's Python files without libftmoe.so: no fallback, the import raises
    import shutil
    import sys
    src = os.path.dirname(ft.__file__)
    dst = tmp_path / "moe_expert_offload_top_b200"
    dst.mkdir()
    for name in os.listdir(src):
        if name.endswith(".py"):
            shutil.copy(os.path.join(src, name), dst / name)
    r = subprocess.run([sys.executable, "-c", "import moe_expert_offload_top_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "ImportError" in r.stderr and "not built" in r.stderr
