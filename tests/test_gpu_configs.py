"""GPU parity of the prefill (tcgen05 grouped GEMM) path and of the three large
workloads at their full sizes: DeepSeek-V4-Flash-shaped decode (8 layers, 256
experts, shared expert, 25% cache), the same shapes in prefill with whole-layer
double buffering (4096 tokens).  Outputs are compared on sampled steps and
tokens (every token of a layer where stated); routing and the cache trace on
every step.  The int4 large pool has its own module, so that its 93 GB pool is
pinned only after this module's 103 GB pool is freed."""
import numpy as np
import pytest

import synth
from moe_expert_offload_top_b200.workload import GpuStack
from gpu_util import run_and_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gemm_threshold", [0, 1 << 30])
def test_prefill_gemm_and_gemv_paths_match_oracle(gemm_threshold):
    cfg = synth.MoeConfig("prefill-small", L=2, E=16, H=512, I=256, k=4, gating="sigmoid", wdtype="bf16",
                          shared=True, C=32, tokens=700, batches=(700,), process="iid", mode="prefill")
    st = run_and_check(cfg, 700, sample_steps=[0], gemm_threshold=gemm_threshold)
    assert st["misses"] == 0 and st["prefetch_misses"] == 2 * 16


@pytest.mark.parametrize("gemm_threshold", [0, 1 << 30])
def test_nvfp4_prefill_fused_gemm_and_gemv_paths_match_oracle(gemm_threshold):
    # NVFP4 stacks in prefill: the GEMMs expand each weight tile to bf16 (exact) in shared
    # memory, and their epilogue applies each matrix's fp32 scale; or the GEMV path
    cfg = synth.MoeConfig("prefill-nvfp4", L=2, E=16, H=512, I=256, k=4, gating="sigmoid", wdtype="nvfp4",
                          shared=True, C=32, tokens=700, batches=(700,), process="iid", mode="prefill")
    st = run_and_check(cfg, 700, sample_steps=[0], gemm_threshold=gemm_threshold)
    assert st["misses"] == 0 and st["prefetch_misses"] == 2 * 16


def test_nvfp4_fused_gemm_uneven_groups():
    # NVFP4 on the GEMM path needs H and I multiples of 256 (block scales in 16-byte boxes)
    cfg = synth.MoeConfig("skew-nvfp4", L=1, E=8, H=768, I=512, k=2, gating="softmax", wdtype="nvfp4",
                          shared=False, C=8, tokens=400, batches=(400,), process="ar1", mode="decode")
    run_and_check(cfg, 400, sample_steps=[0], gemm_threshold=0)


def test_gemm_path_uneven_groups_and_many_tiles():
    # one hot expert with > 2 M-tiles, others tiny; H, I at the multiples the tiles need
    cfg = synth.MoeConfig("skew", L=1, E=8, H=768, I=384, k=2, gating="softmax", wdtype="bf16",
                          shared=False, C=8, tokens=400, batches=(400,), process="ar1", mode="decode")
    run_and_check(cfg, 400, sample_steps=[0], gemm_threshold=0)


@pytest.fixture(scope="module")
def dsv4_stack():
    # the decode and prefill workloads of the DeepSeek-V4-Flash shapes share their weights
    # (same seed, layers, experts, shapes): one 103 GB pinned pool serves both tests
    st = GpuStack(synth.CONFIGS["dsv4flash-decode-bf16"])
    yield st
    st.close()


@pytest.mark.slow
def test_config3_dsv4flash_decode_full_size(dsv4_stack):
    cfg = synth.CONFIGS["dsv4flash-decode-bf16"]
    st = run_and_check(cfg, 1, sample_steps=[5, 255, 511, 767, 1023], stack=dsv4_stack)
    assert 0 < st["misses"] < st["routed"]


@pytest.mark.slow
def test_config4_prefill_double_buffer_full_size(dsv4_stack):
    # every token of the last layer (the persistent tcgen05 tile loop runs many tiles per
    # CTA at these sizes), plus three sampled tokens of every other layer
    cfg = synth.CONFIGS["dsv4flash-prefill-bf16"]
    rng = np.random.default_rng(4)
    toks = sorted(rng.choice(4096, 3, replace=False).tolist())
    st = run_and_check(cfg, 4096, sample_steps=[0], sample_tokens=toks, stack=dsv4_stack,
                       full_layers=(cfg.L - 1,))
    assert st["misses"] == 0 and st["prefetch_misses"] == cfg.L * cfg.E
    assert (0, cfg.L - 1, 4096) in st["compared"]
