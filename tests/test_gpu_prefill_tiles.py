"""GPU parity of the tcgen05 grouped GEMMs where every CTA of the persistent grid
runs several tiles: the second TMEM accumulator, the accumulator barriers' phase
flips and the pipeline's stage reuse across tiles are all exercised.

64 experts, H=1024, I=512, top-6 sigmoid plus a shared expert, 2048 tokens: the
gate/up and down GEMMs each have about 700 tiles for the 148 CTAs.  Checked
through the C ABI on every y row of the step-level entry (ft_expert_ffn_prefill)
and on every token of the forward (ft_moe_forward in prefill mode), for bf16 and
NVFP4 weights."""
import numpy as np
import pytest
import torch

import moe_expert_offload_top_b200 as ft
import synth
from oracle import moe
from gpu_util import assert_close, run_and_check

pytestmark = pytest.mark.gpu
DEV = "cuda"
E, K, H, I, T = 64, 6, 1024, 512, 2048
BM, BN = 128, 256   # the GEMM tile: 128 pair rows x 256 accumulator columns


def _cfg(L=1, wdtype="bf16"):
    return synth.MoeConfig("prefill-tiles", L=L, E=E, H=H, I=I, k=K, gating="sigmoid", wdtype=wdtype,
                           shared=True, C=L * E, tokens=T, batches=(T,), process="iid", mode="prefill")


def _tiles(counts, n_tiles):
    return sum((int(c) + BM - 1) // BM for c in counts if c > 0) * n_tiles


def test_step_level_prefill_gemms_every_y_row():
    cfg = _cfg()
    vals, bits = synth.tokens(cfg, T)
    x_f = vals[0]
    r = moe.route(x_f, synth.router_weights(cfg, 0), K, cfg.gating)
    counts, offsets, perm = moe.permute(r["ids"], E)
    S = [e for e in range(E) if counts[e] > 0]
    rows_per_group = [counts[e] for e in S] + [T]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # several tiles per CTA in both GEMMs
    assert _tiles(rows_per_group, I // (BN // 2)) > 3 * sms and _tiles(rows_per_group, H // BN) > 3 * sms

    blobs = [synth.expert_blob(cfg, 0, e) for e in range(E)] + [synth.expert_blob(cfg, 0, 0, shared=True)]
    # the weight array in slot order: slot s holds blob s; experts are placed in reverse order of
    # their index so that slot and expert differ
    slot_of = {e: E - 1 - e for e in range(E)}
    slot_of[-1] = E
    arena = np.empty((E + 1, cfg.blob_bytes), dtype=np.uint8)
    for e in range(E):
        arena[slot_of[e]] = blobs[e]
    arena[E] = blobs[E]
    w_dev = torch.from_numpy(arena).to(DEV)

    x_dev = torch.from_numpy(bits[0]).view(torch.bfloat16).to(DEV)
    ids_dev = torch.from_numpy(r["ids"]).to(DEV)
    cnt_dev = torch.empty(E, dtype=torch.int32, device=DEV)
    off_dev = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm_dev = torch.empty(T * K, dtype=torch.int32, device=DEV)
    inv_dev = torch.empty(T * K, dtype=torch.int32, device=DEV)
    ft.ft_permute(ids_dev, T, K, E, cnt_dev, off_dev, perm_dev, inv_dev)
    rows = T * K + T
    a_rows = torch.empty((rows, H), dtype=torch.bfloat16, device=DEV)
    h = torch.empty((rows, I), dtype=torch.bfloat16, device=DEV)
    y = torch.full((rows, H), float("nan"), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    experts = S + [-1]
    ft.ft_expert_ffn_prefill(x_dev, T, H, I, K, w_dev, E + 1, experts, [slot_of[e] for e in experts], off_dev,
                             perm_dev, a_rows, h, y, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(perm_dev.cpu().numpy(), perm)     # the permutation the rows follow
    y_got = y.cpu().numpy()
    assert np.all(np.isfinite(y_got))

    y_ref = np.empty((rows, H))
    for e in S:
        q = np.arange(offsets[e], offsets[e + 1])
        tok = perm[q] // K
        y_ref[q] = moe.swiglu_ffn(x_f[tok], *moe.expert_weights(blobs[e], "bf16", H, I))
    y_ref[T * K:] = moe.swiglu_ffn(x_f, *moe.expert_weights(blobs[E], "bf16", H, I))
    for e in S:   # per expert group: every M-tile, including the ragged last one
        q = slice(offsets[e], offsets[e + 1])
        assert_close(y_got[q], y_ref[q], "bf16", "expert %d y rows" % e)
    assert_close(y_got[T * K:], y_ref[T * K:], "bf16", "shared expert y rows")

    # the combined output of these rows against the oracle's layer
    g_dev = torch.from_numpy(r["gates"].astype(np.float32)).to(DEV)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    ft.ft_combine(y, g_dev, inv_dev, T, H, K, True, True, out)
    ref = moe.experts_and_combine(x_f, r["ids"], r["gates"], E, "bf16", H, I, lambda e: blobs[e], blobs[E])
    assert_close(out.float().cpu().numpy(), ref, "bf16", "combined output", stored_bf16=True)


@pytest.mark.parametrize("wdtype", ["bf16", "nvfp4"])
def test_prefill_forward_many_tiles_per_cta_every_token(wdtype):
    # nvfp4: each CTA expands its weight tiles in shared memory, and its block-scale ring
    # (two slots of 4 stages) turns over across the tiles it runs
    cfg = _cfg(L=2, wdtype=wdtype)
    st = run_and_check(cfg, T, sample_steps=[0], gemm_threshold=0)
    assert st["misses"] == 0 and st["prefetch_misses"] == 2 * E
    assert (0, 0, T) in st["compared"] and (0, 1, T) in st["compared"]
