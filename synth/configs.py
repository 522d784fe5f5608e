"""Workload recipes for the routed-MoE layer over a shared LRU expert cache.

Each recipe names the shapes, gating, weight format, cache capacity and token
process of one synthetic workload.  Sources: the FreeToken pages describe the
method (routed experts in host memory, GPU slots as a shared LRU cache, e.g.
"6 of 256 routed experts" in FreeToken-linux, "MoE memory handling"); the
shapes, gating and int4 format are the five stated workloads of this project.
The pages use real checkpoints and agent workloads; seeded N(0, 0.02) weights
and N(0,1) or AR(1) hidden states stand in for them.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class MoeConfig:
    name: str
    L: int            # MoE layers in the stack
    E: int            # routed experts per layer
    H: int            # hidden size
    I: int            # SwiGLU intermediate size
    k: int            # top-k
    gating: str       # "softmax" (renormalised over the k selected) or "sigmoid" (normalised over the k)
    wdtype: str       # "f32", "bf16", "int4" (g128, bf16 scales) or "nvfp4" (e2m1, e4m3 per 16, fp32 global)
    shared: bool      # one always-on shared expert per layer, gate weight 1
    C: int            # cache slots (shared across all layers)
    tokens: int       # tokens in the whole run
    batches: Tuple[int, ...]   # decode batch sizes (one run per batch size); prefill: (tokens,)
    process: str      # "iid" N(0,1) tokens or "ar1" x_t = 0.9 x_{t-1} + 0.436 eps_t
    mode: str         # "decode" or "prefill"
    resize_to: Optional[int] = None   # slots after the first half of the run (grow)
    seed: int = 0
    sigma: float = 0.02

    @property
    def x_dtype(self) -> str:
        return "f32" if self.wdtype == "f32" else "bf16"

    @property
    def blob_bytes(self) -> int:
        n = 3 * self.H * self.I
        if self.wdtype == "f32":
            return 4 * n
        if self.wdtype == "bf16":
            return 2 * n
        if self.wdtype == "nvfp4":
            return n // 2 + n // 16 + 16
        return n // 2 + 2 * (n // 128)

    @property
    def pool_bytes(self) -> int:
        return self.L * self.E * self.blob_bytes


def _slots(frac: float, L: int, E: int) -> int:
    # C = floor(frac * L * E): the workloads state the cache as a fraction of all experts.
    return int(frac * L * E + 1e-9)


AR_PHI = 0.9
AR_SIG = 0.436

# The stated workloads, by name.
CONFIGS = {
    "tiny-fp32": MoeConfig("tiny-fp32", L=1, E=16, H=256, I=128, k=2, gating="softmax", wdtype="f32",
                 shared=False, C=4, tokens=8, batches=(1,), process="iid", mode="decode"),
    "decode-locality-bf16": MoeConfig("decode-locality-bf16", L=4, E=128, H=2048, I=768, k=8, gating="softmax",
                 wdtype="bf16", shared=False, C=_slots(0.40, 4, 128), tokens=512, batches=(1,),
                 process="ar1", mode="decode"),
    "dsv4flash-decode-bf16": MoeConfig("dsv4flash-decode-bf16", L=8, E=256, H=4096, I=2048, k=6, gating="sigmoid",
                 wdtype="bf16", shared=True, C=_slots(0.25, 8, 256), tokens=1024, batches=(1,),
                 process="ar1", mode="decode"),
    "dsv4flash-prefill-bf16": MoeConfig("dsv4flash-prefill-bf16", L=8, E=256, H=4096, I=2048, k=6, gating="sigmoid",
                 wdtype="bf16", shared=True, C=_slots(0.25, 8, 256), tokens=4096, batches=(4096,),
                 process="iid", mode="prefill"),
    "int4-large-pool": MoeConfig("int4-large-pool", L=16, E=256, H=7168, I=2048, k=8, gating="sigmoid",
                 wdtype="int4", shared=False, C=_slots(0.15, 16, 256), tokens=2048, batches=(1, 8, 32),
                 process="ar1", mode="decode", resize_to=_slots(0.30, 16, 256)),
}
