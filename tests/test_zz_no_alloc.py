"""ft_expert_ffn_decode_noalloc: the decode expert FFN + combine for callers that
may not allocate device memory (their intermediate rows live in the library's
static device array).  Checked through the C ABI against the allocating entry
points (ft_expert_ffn_decode with caller scratch, then ft_combine) on two calls
in a row, for bf16, int4 and NVFP4 weights: both run the same kernels on the same
inputs, so the outputs must agree bit for bit.  Also checked: its size limit
and its check of the shared-expert entry."""
import numpy as np
import pytest
import torch

import moe_expert_offload_top_b200 as ft
import synth
from gpu_util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
E, K, H, I, T = 16, 8, 2048, 768, 3


def _inputs(seed, wdtype="bf16"):
    cfg = synth.MoeConfig("t", 1, E, H, I, K, "sigmoid", wdtype, True, E, T, (T,), "iid", "decode")
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    gates = rng.random((T, K)).astype(np.float32)
    gates /= gates.sum(axis=1, keepdims=True)
    x = synth.round_bf16(synth.normal_f32(seed, 8, 0, 0, T * H).reshape(T, H))
    S = sorted(set(ids.reshape(-1).tolist()))
    blobs = [torch.from_numpy(synth.expert_blob(cfg, 0, e)).to(DEV) for e in S]
    blobs.append(torch.from_numpy(synth.expert_blob(cfg, 0, 0, shared=True)).to(DEV))
    experts = S + [-1]
    idd = torch.from_numpy(ids).to(DEV)
    offs = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * K, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * K, dtype=torch.int32, device=DEV)
    ft.ft_permute(idd, T, K, E, counts, offs, perm, inv)
    maxp = int(np.bincount(ids.reshape(-1), minlength=E).max())
    return dict(wdtype=wdtype, x=torch.from_numpy(x).view(torch.bfloat16).to(DEV), blobs=blobs, experts=experts,
                maxp=maxp, offs=offs, perm=perm, inv=inv, gates=torch.from_numpy(gates).to(DEV))


def _with_caller_scratch(a):
    h = torch.empty((T * K + T, I), device=DEV)
    y = torch.empty((T * K + T, H), device=DEV)
    ft.ft_expert_ffn_decode(a["x"], T, H, I, K, a["wdtype"], a["blobs"], a["experts"], a["maxp"], a["offs"],
                            a["perm"], h, y)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    ft.ft_combine(y, a["gates"], a["inv"], T, H, K, True, True, out)
    return out


def _no_alloc(a):
    out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=DEV)
    ft.ft_expert_ffn_decode_noalloc(a["x"], T, H, I, K, a["wdtype"], a["blobs"], a["experts"], a["maxp"], a["offs"],
                                    a["perm"], a["gates"], a["inv"], True, out)
    return out


@pytest.mark.parametrize("wdtype", ["bf16", "int4", "nvfp4"])
def test_no_alloc_entry_matches_the_allocating_path_twice(wdtype):
    first, second = _inputs(21, wdtype), _inputs(22, wdtype)
    for a in (first, second):          # two calls in a row share the static scratch
        got = _no_alloc(a)
        torch.cuda.synchronize()
        ref = _with_caller_scratch(a)
        torch.cuda.synchronize()
        assert np.all(np.isfinite(got.float().cpu().numpy()))
        # the same kernels on the same inputs: identical bits
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), "no-alloc output differs from caller scratch"
        assert_close(got.float().cpu().numpy(), ref.float().cpu().numpy(), wdtype, "no-alloc vs caller scratch")


def test_no_alloc_entry_rejects_sizes_beyond_its_scratch():
    a = _inputs(23)
    big_T = ft.FT_NOALLOC_SCRATCH_FLOATS // ((K + 1) * (I + H)) + 1
    out = torch.empty((1, H), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ft.FtError) as ei:
        ft.ft_expert_ffn_decode_noalloc(a["x"], big_T, H, I, K, "bf16", a["blobs"], a["experts"], a["maxp"],
                                        a["offs"], a["perm"], a["gates"], a["inv"], True, out)
    assert ei.value.code == ft.FT_ERR_INVALID
    assert "exceeds the static scratch" in str(ei.value)


def test_no_alloc_entry_checks_the_shared_entry():
    a = _inputs(24)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ft.FtError) as ei:      # has_shared without a -1 entry
        ft.ft_expert_ffn_decode_noalloc(a["x"], T, H, I, K, "bf16", a["blobs"][:-1], a["experts"][:-1], a["maxp"],
                                        a["offs"], a["perm"], a["gates"], a["inv"], True, out)
    assert ei.value.code == ft.FT_ERR_INVALID
