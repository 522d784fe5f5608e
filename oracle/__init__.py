"""CPU oracle for the routed-MoE layer over a shared LRU expert cache.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the hot path computes, in float64 (router logits are
rounded once to float32, the precision in which top-k is decided).  Only the
test suite, the smoke check and the benchmark's CPU-baseline leg may import
it; the product library never does, and it imports nothing from the product.

Sources (FreeToken pages, cited by page title and section):
  * "FreeToken linux" - "FreeToken's MoE memory handling": the router
    activates a few experts per token (6 of 256 routed experts in
    DeepSeek-V4-Flash); the full routed-expert pool lives in host memory; GPU
    expert slots form one LRU cache shared by every MoE layer; a missed expert
    is sent over PCIe and kept for reuse; prefill double-buffers whole layers.
  * "FreeToken RTX 5090" - memory hierarchy / dynamic reconfiguration: host
    memory stays the reference store, so the cache capacity changes speed, not
    the result; resizing happens at scheduler safe points.
  * "FreeToken gguf" - MoE backends: `offload` keeps experts in host RAM with
    an LRU of GPU slots; `fused` keeps every expert on the GPU.
The pages give no formula.  Gating (softmax / sigmoid over the selected k),
SwiGLU, and the int4 group-128 format are the stated workloads of this
project; every reading taken where the pages are silent is marked READING in
the function that takes it.

Modules:
  moe  - router logits, top-k, gates, permutation, blob decoding, SwiGLU FFN,
         weighted combine, one MoE layer.
  lru  - the shared LRU slot table (hit/miss/slot/eviction trace, prefetch,
         resize, statistics).
  run  - drives a whole workload (steps x layers) through moe + lru.
Parity unpinned: nothing in the oracle reproduces the pages' own measured miss
rates or tokens/s (real checkpoints and traces are not available).
"""
from . import lru, moe, run  # noqa: F401
