"""The fused decode FFN (gate/up + SwiGLU, down and combine in one launch, resident
experts launched before the wait for this call's misses) against the per-pass kernels
and the oracle: the same inputs through two stacks, one per launch shape, give the
same trace and bit-identical outputs, and the oracle's outputs within the bound."""
import dataclasses

import numpy as np
import pytest
import torch

import moe_expert_offload_top_b200 as ft
import synth
from moe_expert_offload_top_b200.workload import GpuStack
from gpu_util import assert_close, first_divergence, oracle_run

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(cfg, fused, batch=1, steps=None, gemm_threshold=None, stage_timing=False, oracle=False,
         int4_tensor=True):
    steps = cfg.tokens // batch if steps is None else steps
    with GpuStack(cfg) as st:
        ft.ft_moe_set_fused_ffn(st.h, int(fused))
        ft.ft_moe_set_int4_tensor_cores(st.h, int(int4_tensor))
        if gemm_threshold is not None:
            ft.ft_moe_set_gemm_threshold(st.h, gemm_threshold)
        if stage_timing:
            ft.ft_moe_set_stage_timing(st.h, 1)
        vals, x = st.tokens(batch)
        out = torch.empty((cfg.L, batch, cfg.H), dtype=st.xdt, device=DEV)
        outs, ids = [], np.zeros((steps, cfg.L, batch, cfg.k), dtype=np.int32)
        for s in range(steps):
            for l in range(cfg.L):
                st.forward(l, x[s], out[l])
                ids[s, l] = st.last_routing(batch)[0]
            outs.append(out.float().cpu().numpy().copy())
        torch.cuda.synchronize()
        res = {"outs": outs, "ids": ids, "trace": st.trace(), "stats": st.stats(), "vals": vals,
               "perf": ft.ft_moe_perf(st.h)}
        if oracle:
            res["ref"] = oracle_run(cfg, st, vals[:steps])
    return res


CASES = {
    # name: (config, batch)
    "bf16-misses": (dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=24, C=40), 1),
    "bf16-batch8": (dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=48, C=160), 8),
    "bf16-shared": (synth.MoeConfig("shared-small", L=2, E=32, H=1024, I=512, k=6, gating="sigmoid",
                                    wdtype="bf16", shared=True, C=20, tokens=12, batches=(1,),
                                    process="ar1", mode="decode"), 1),
    "f32-tiny": (synth.CONFIGS["tiny-fp32"], 1),
    "int4": (synth.MoeConfig("int4-small", L=2, E=32, H=1024, I=512, k=8, gating="sigmoid", wdtype="int4",
                             shared=False, C=24, tokens=12, batches=(1,), process="ar1", mode="decode"), 1),
    "nvfp4": (synth.MoeConfig("nvfp4-small", L=2, E=32, H=1024, I=512, k=4, gating="softmax", wdtype="nvfp4",
                              shared=False, C=16, tokens=12, batches=(1,), process="ar1", mode="decode"), 1),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_matches_per_pass_bitwise_and_oracle(name):
    cfg, batch = CASES[name]
    if batch > 1:
        cfg = dataclasses.replace(cfg, batches=(batch,))
    a = _run(cfg, fused=True, batch=batch, oracle=True)
    b = _run(cfg, fused=False, batch=batch, int4_tensor=False)   # the same per-row arithmetic
    assert np.array_equal(a["ids"], b["ids"])
    assert a["trace"] == b["trace"]
    assert a["stats"]["misses"] > 0
    for s, (oa, ob) in enumerate(zip(a["outs"], b["outs"])):
        assert np.array_equal(oa, ob), "step %d: fused and per-pass outputs differ" % s
    ref = a["ref"]
    steps = len(a["outs"])
    div = first_divergence(a["ids"], ref["ids"][:steps], ref["gap"][:steps], ref.get("zsel"))
    last = steps if div is None else div // (cfg.L * batch)
    for s in range(last):
        for l in range(cfg.L):
            assert_close(a["outs"][s][l], ref["out"][(s, l)], cfg.wdtype, "%s step %d layer %d" % (name, s, l),
                         stored_bf16=cfg.x_dtype == "bf16")


def test_many_tokens_gemv_path_fused():
    # 80 tokens at once on the GEMV path (the tcgen05 GEMMs switched off): three-launch
    # routing, then the fused FFN with up to 8 pairs per weight pass
    cfg = synth.MoeConfig("wide-gemv", L=1, E=16, H=1024, I=512, k=4, gating="softmax", wdtype="bf16",
                          shared=True, C=16, tokens=160, batches=(80,), process="iid", mode="decode")
    a = _run(cfg, fused=True, batch=80, gemm_threshold=1 << 30, oracle=True)
    b = _run(cfg, fused=False, batch=80, gemm_threshold=1 << 30, int4_tensor=False)   # the same per-row arithmetic
    for oa, ob in zip(a["outs"], b["outs"]):
        assert np.array_equal(oa, ob)
    ref = a["ref"]
    div = first_divergence(a["ids"], ref["ids"], ref["gap"], ref.get("zsel"))
    last = 2 if div is None else div // 80
    for s in range(last):
        assert_close(a["outs"][s][0], ref["out"][(s, 0)], "bf16", "step %d" % s, stored_bf16=True)


def test_resident_experts_run_before_the_fill_wait():
    # fused launch shape: forwards with both resident and copied experts run two fused
    # launches (the resident experts, then the copied ones with the combine)
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=24, C=40)
    fwd = cfg.L * cfg.tokens
    a = _run(cfg, fused=True)
    p = a["perf"]
    assert p["forwards"] == fwd
    assert 2 * fwd < p["kernel_launches"] < 3 * fwd       # routing + 1, + 1 where split
    # stage timing runs every forward unsplit, so its events time whole-list launches
    b = _run(cfg, fused=True, stage_timing=True)
    q = b["perf"]
    assert q["timed_forwards"] == fwd and q["ffn_fused_launches"] == fwd
    assert q["ffn_fused_ms"] > 0 and q["ffn_fused_bytes"] > 0
    assert q["ffn_gate_up_ms"] == 0 and q["combine_ms"] == 0
    for oa, ob in zip(a["outs"], b["outs"]):
        assert np.array_equal(oa, ob)


@pytest.mark.parametrize("tensor,batch,per_pass", [(True, 1, 2), (True, 8, 3), (False, 8, 2)])
def test_per_pass_kernels_split_around_the_fill_wait(tensor, batch, per_pass):
    # the default launch shape: forwards with both resident and copied experts run two FFN
    # passes (gate/up + down; on the bf16 tensor cores from 2 tokens on, with the h split
    # between them), the others one, then the combine
    cfg = dataclasses.replace(synth.CONFIGS["decode-locality-bf16"], L=2, tokens=24 * batch, C=40 if batch == 1 else 160,
                              batches=(batch,))
    fwd = cfg.L * (cfg.tokens // batch)
    a = _run(cfg, fused=False, batch=batch, int4_tensor=tensor)
    p = a["perf"]
    assert p["forwards"] == fwd and p["ffn_fused_launches"] == 0
    one = 1 + per_pass + 1                                # routing, one pass, combine
    assert one * fwd < p["kernel_launches"] < (one + per_pass) * fwd     # + one pass where split
    b = _run(cfg, fused=False, batch=batch, stage_timing=True, int4_tensor=tensor)
    q = b["perf"]
    assert q["kernel_launches"] == one * fwd and q["ffn_gate_up_launches"] == fwd
    assert q["ffn_gate_up_ms"] > 0 and q["ffn_down_ms"] > 0 and q["combine_ms"] > 0
    for oa, ob in zip(a["outs"], b["outs"]):
        assert np.array_equal(oa, ob)


@pytest.mark.parametrize("wdtype,batch", [("int4", 1), ("int4", 8), ("nvfp4", 1), ("nvfp4", 8), ("bf16", 8)])
def test_int4_tensor_core_gemv_against_cuda_cores_and_oracle(wdtype, batch):
    # the decode GEMV on mma.sync (int4: int8 products; NVFP4: f16 products; bf16 from 2 tokens:
    # bf16 products, h as hi + lo) and on the fp32 pipes: the same routing and cache trace,
    # outputs that differ only by summation order (and the h operand's rounding), both within
    # the oracle's bound
    cfg = synth.MoeConfig("%s-tc" % wdtype, L=2, E=32, H=1024, I=512, k=8, gating="sigmoid", wdtype=wdtype,
                          shared=True, C=64, tokens=16 * batch, batches=(batch,), process="ar1", mode="decode")
    a = _run(cfg, fused=False, batch=batch, oracle=True, int4_tensor=True)
    b = _run(cfg, fused=False, batch=batch, int4_tensor=False)
    assert np.array_equal(a["ids"], b["ids"]) and a["trace"] == b["trace"]
    for oa, ob in zip(a["outs"], b["outs"]):
        # outputs are bf16: fp32 results that differ in the last bits flip a few roundings
        rel = np.linalg.norm(oa - ob) / np.linalg.norm(ob)
        assert rel < 2e-3, rel
    ref = a["ref"]
    steps = len(a["outs"])
    div = first_divergence(a["ids"], ref["ids"][:steps], ref["gap"][:steps], ref.get("zsel"))
    last = steps if div is None else div // (cfg.L * batch)
    for s in range(last):
        for l in range(cfg.L):
            assert_close(a["outs"][s][l], ref["out"][(s, l)], wdtype, "step %d layer %d" % (s, l), stored_bf16=True)
