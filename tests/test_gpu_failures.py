"""Failure handling, with every failure made on the host or by a bounded wait that
runs out (no GPU fault): a slot fill that fails, a routing wait that times out,
a device wait on a barrier nothing arrives on, a step larger than the cache."""
import dataclasses

import numpy as np
import pytest
import torch

import moe_expert_offload_top_b200 as ft
import synth
from moe_expert_offload_top_b200.workload import GpuStack
from gpu_util import assert_close, oracle_run

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg():
    return dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=12, C=24)


def test_failed_fill_rolls_back_and_next_forward_recovers():
    cfg = _cfg()
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=DEV)
        got = {}
        st.step(x[0], out)                      # 16 misses: cache warm-up
        ft.ft_moe_debug_inject(st.h, ft.FT_INJECT_COPY_FAIL, 1)
        with pytest.raises(ft.FtError) as ei:   # the first fill of the next miss fails
            st.step(x[5], out)
        assert ei.value.code == ft.FT_ERR_CUDA and "slot fill" in str(ei.value)
        tr = st.trace()
        failed = [a for a in tr if a[0] == tr[-1][0] and not a[4]]
        assert failed and all(ft.ft_cache_slot_of(st.h, a[1], a[2]) == -1 for a in failed)
        torch.cuda.synchronize()
        # the run continues from a consistent cache and gives the oracle's outputs
        for s in range(1, cfg.tokens):
            st.step(x[s], out)
            got[s] = out.float().cpu().numpy().copy()
        ft.ft_moe_sync(st.h)
        for s in range(1, cfg.tokens):
            for l in range(cfg.L):
                from oracle import moe
                r = moe.route(vals[s], synth.router_weights(cfg, l), cfg.k, cfg.gating)
                ref = moe.experts_and_combine(vals[s], r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H, cfg.I,
                                              lambda e, l=l: st.pool_blob(l, e))
                assert_close(got[s][l], ref, "bf16", "step %d layer %d" % (s, l), stored_bf16=True)


def test_routing_timeout_changes_nothing():
    cfg = _cfg()
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=DEV)
        st.step(x[0], out)
        before = (st.trace(), st.stats()["routed"])
        ft.ft_moe_debug_inject(st.h, ft.FT_INJECT_ROUTE_TIMEOUT, 1)
        with pytest.raises(ft.FtError) as ei:
            st.forward(0, x[1], out[0])
        assert ei.value.code == ft.FT_ERR_TIMEOUT
        assert (st.trace(), st.stats()["routed"]) == before
        st.step(x[1], out)                       # works again
        ft.ft_moe_sync(st.h)
        assert st.stats()["routed"] > before[1]


def test_device_wait_gives_up_and_context_survives():
    rc = ft.ft_debug_device_wait_selftest(10000)     # 10 ms on a barrier nobody arrives on
    assert rc == ft.FT_ERR_DEVICE_CHECK
    a = torch.ones(1024, device=DEV)
    assert float((a * 2).sum()) == 2048.0             # the context still runs work
    cfg = synth.CONFIGS["tiny-fp32"]
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((1, 1, cfg.H), dtype=torch.float32, device=DEV)
        st.step(x[0], out)
        ft.ft_moe_sync(st.h)


def test_step_larger_than_cache_is_rejected_first():
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=1, tokens=4, C=5)   # k = 8 > 5 slots
    with GpuStack(cfg) as st:
        vals, x = st.tokens(1)
        out = torch.empty((1, cfg.H), dtype=torch.bfloat16, device=DEV)
        with pytest.raises(ft.FtError) as ei:
            st.forward(0, x[0], out)
        assert ei.value.code == ft.FT_ERR_CAPACITY
        assert st.trace() == [] and st.stats()["resident"] == 0


def test_fused_ffn_wait_gives_up_and_is_reported():
    """A fused decode FFN launch whose down items wait for a count nothing reaches: each
    wait gives up after 1 ms, the kernel completes, the error word is reported at the next
    synchronisation, and the following forwards are correct again."""
    cfg = _cfg()
    with GpuStack(cfg) as st:
        ft.ft_moe_set_fused_ffn(st.h, 1)
        vals, x = st.tokens(1)
        out = torch.empty((cfg.L, 1, cfg.H), dtype=torch.bfloat16, device=DEV)
        st.step(x[0], out)
        ft.ft_moe_sync(st.h)
        ft.ft_moe_debug_inject(st.h, ft.FT_INJECT_FUSED_WAIT, 1)
        st.forward(0, x[1], out[0])              # the kernel's waits run out; the call returns
        with pytest.raises(ft.FtError) as ei:
            ft.ft_moe_sync(st.h)
        assert ei.value.code == ft.FT_ERR_DEVICE_CHECK and "111" in str(ei.value)
        a = torch.ones(1024, device=DEV)
        assert float((a * 2).sum()) == 2048.0    # the context still runs work
        got = {}
        for s in range(2, 6):
            st.step(x[s], out)
            got[s] = out.float().cpu().numpy().copy()
        ft.ft_moe_sync(st.h)
        from oracle import moe
        for s in range(2, 6):
            for l in range(cfg.L):
                r = moe.route(vals[s], synth.router_weights(cfg, l), cfg.k, cfg.gating)
                ref = moe.experts_and_combine(vals[s], r["ids"], r["gates"], cfg.E, cfg.wdtype, cfg.H, cfg.I,
                                              lambda e, l=l: st.pool_blob(l, e))
                assert_close(got[s][l], ref, "bf16", "step %d layer %d" % (s, l), stored_bf16=True)
