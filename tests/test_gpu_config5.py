"""GPU parity of the int4 large-pool workload at full size: 16 MoE layers, 256
experts, H=7168, I=2048, top-8 sigmoid, int4 g128 weights, 15% of the experts
cached, the cache grown to 30% halfway, at decode batch 1, 8 and 32.  Routing and
the cache trace are compared on every step; outputs on every token of two
sampled steps (one before and one after the resize), first and last layer."""
import pytest

import synth
from moe_expert_offload_top_b200.workload import GpuStack
from gpu_util import run_and_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def config5_stack():
    # the 93 GB int4 pool is generated and pinned once for the three batch sizes
    st = GpuStack(synth.CONFIGS["int4-large-pool"])
    yield st
    st.close()


@pytest.mark.slow
@pytest.mark.parametrize("batch", [1, 8, 32])
def test_config5_int4_large_pool_with_resize(batch, config5_stack):
    cfg = synth.CONFIGS["int4-large-pool"]
    steps = cfg.tokens // batch
    # every token of the sampled steps, on the first and the last layer
    st = run_and_check(cfg, batch, sample_steps=[1, steps - 1],
                       resize_at=steps // 2, resize_to=cfg.resize_to, stack=config5_stack,
                       sample_layers=[0, cfg.L - 1])
    assert st["capacity"] == cfg.resize_to
