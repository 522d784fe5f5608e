"""The oracle's pins catch plausible mistakes: each case plants one mistake in the CPU
oracle (a swapped operand, a wrong index, sign, bias or order, a dropped term), runs
every pin of `test_oracle_pins.py` against the planted oracle, and requires at least
one pin to fail.  Mistakes are planted only in the oracle, on the CPU, through
monkeypatch; nothing here touches the CUDA path."""
import heapq
from collections import OrderedDict

import numpy as np
import pytest

import synth
import test_oracle_pins as pins
from oracle import lru as olru
from oracle import moe
from oracle import run as orun

_o = {n: getattr(moe, n) for n in (
    "widen_bf16", "decode_int4", "dequant_int4", "decode_e2m1", "decode_e4m3", "dequant_nvfp4",
    "expert_weights", "router_logits", "topk", "gates", "permute", "silu", "swiglu_ffn",
    "selected_set", "experts_and_combine")}


# ----------------------------------------------------------- the pin suite ----

def _pin_cases():
    """Every pin as (id, zero-argument callable), parametrized pins expanded."""
    out = []
    for name in sorted(n for n in dir(pins) if n.startswith("test_")):
        fn = getattr(pins, name)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            out.append((name, fn))
            continue
        assert len(marks) == 1
        argnames, argvalues = marks[0].args[0], marks[0].args[1]
        names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
        for vals in argvalues:
            vals = vals.values if hasattr(vals, "values") else vals
            vals = vals if len(names) > 1 else (vals,)
            out.append(("%s%s" % (name, list(vals)), lambda fn=fn, kw=dict(zip(names, vals)): fn(**kw)))
    return out


def _failing_pins(stop_at_first=True):
    failed = []
    for pid, call in _pin_cases():
        try:
            call()
        except Exception as exc:                    # an assertion, or the planted oracle breaking
            failed.append((pid, type(exc).__name__))
            if stop_at_first:
                break
    return failed


# ----------------------------------------------------------------- mutants ----

def _swap_pairs(a):
    b = a.copy()
    b[:, 0::2], b[:, 1::2] = a[:, 1::2], a[:, 0::2]
    return b


def _swap_nibbles(p):
    p = np.asarray(p, dtype=np.uint8)
    return ((p & 0x0F) << 4) | (p >> 4)


def _int4_tiled_scales(packed, scale_bits):
    q = moe.decode_int4(packed).astype(np.float64)
    s = moe.widen_bf16(scale_bits)
    return q * np.tile(s, (1, 128))                 # group c % G instead of c // 128


def _e2m1_subnormal_as_integer(codes):
    c = np.asarray(codes, dtype=np.int64)
    v = _o["decode_e2m1"](c)
    return np.where(((c >> 1) & 3) == 0, 2.0 * v, v)


def _down_read_transposed(blob, wdtype, H, I):
    wg, wu, wd = _o["expert_weights"](blob, wdtype, H, I)
    return wg, wu, wd.reshape(-1).reshape(I, H).T


def _topk_by(key):
    def topk(z, k):
        z = np.asarray(z, dtype=np.float32)
        T, E = z.shape
        ids = np.empty((T, k), dtype=np.int32)
        gap = np.full(T, np.inf)
        for t in range(T):
            order = sorted(range(E), key=lambda e: key(float(z[t, e]), e))
            ids[t] = order[:k]
            if k < E:
                gap[t] = float(z[t, order[k - 1]]) - float(z[t, order[k]])
        return ids, gap
    return topk


def _topk_ids_ascending(z, k):
    ids, gap = _o["topk"](z, k)
    return np.sort(ids, axis=1), gap


def _topk_gap_one_deeper(z, k):
    ids, _ = _o["topk"](z, k)
    if k + 1 < np.asarray(z).shape[1]:
        _, gap = _o["topk"](z, k + 1)
    else:
        gap = np.full(np.asarray(z).shape[0], np.inf)
    return ids, gap


def _gates_softmax_negated(z_sel, gating):
    return _o["gates"](-np.asarray(z_sel) if gating == "softmax" else z_sel, gating)


def _gates_sigmoid_unnormalised(z_sel, gating):
    if gating == "sigmoid":
        return 1.0 / (1.0 + np.exp(-np.asarray(z_sel, dtype=np.float64)))
    return _o["gates"](z_sel, gating)


def _permute_tokens_descending(ids, E):
    counts, offsets, perm = _o["permute"](ids, E)
    perm = perm.copy()
    for e in range(E):
        perm[offsets[e]:offsets[e + 1]] = perm[offsets[e]:offsets[e + 1]][::-1]
    return counts, offsets, perm


def _permute_inclusive_offsets(ids, E):
    counts, offsets, perm = _o["permute"](ids, E)
    return counts, np.concatenate([offsets[1:], offsets[-1:]]), perm


def _int4_gate_up_scales_swapped(blob, wdtype, H, I):
    if wdtype != "int4":
        return _o["expert_weights"](blob, wdtype, H, I)
    blob = np.asarray(blob, dtype=np.uint8).reshape(-1)
    m, g = H * I, H * I // 128
    q, s = blob[:3 * m // 2], blob[3 * m // 2:].view(np.uint16)
    return (moe.dequant_int4(q[:m // 2].reshape(I, H // 2), s[g:2 * g].reshape(I, H // 128)),
            moe.dequant_int4(q[m // 2:m].reshape(I, H // 2), s[:g].reshape(I, H // 128)),
            moe.dequant_int4(q[m:3 * m // 2].reshape(H, I // 2), s[2 * g:3 * g].reshape(H, I // 128)))


def _nvfp4_swap_regions(first, size):
    def expert_weights(blob, wdtype, H, I):
        if wdtype != "nvfp4":
            return _o["expert_weights"](blob, wdtype, H, I)
        b = np.array(blob, dtype=np.uint8).reshape(-1)
        o, n = first(H * I), size(H * I)
        a, c = b[o:o + n].copy(), b[o + n:o + 2 * n].copy()
        b[o:o + n], b[o + n:o + 2 * n] = c, a
        return _o["expert_weights"](b, wdtype, H, I)
    return expert_weights


def _router_rounded_to_bf16(x, w):
    z = _o["router_logits"](x, w)
    return (synth.round_bf16(z).astype(np.uint32) << 16).view(np.float32)


def _shared_expert_halved(x, ids, g, E, wd, H, I, blob_of, shared_blob=None):
    out = _o["experts_and_combine"](x, ids, g, E, wd, H, I, blob_of, None)
    if shared_blob is not None:
        wg, wu, wdn = moe.expert_weights(shared_blob, wd, H, I)
        out = out + 0.5 * moe.swiglu_ffn(np.asarray(x, np.float64), wg, wu, wdn)
    return out


class _GrowAddsNoFreeSlot:
    heapify = staticmethod(heapq.heapify)
    heappop = staticmethod(heapq.heappop)
    heappush = staticmethod(lambda a, v: None)


class _EvictMru(OrderedDict):
    def popitem(self, last=True):
        return super().popitem(last=True)


class _NoRefresh(OrderedDict):
    def move_to_end(self, key, last=True):
        pass


class _HighestFreeSlot:
    heapify = staticmethod(lambda a: a.sort())
    heappush = staticmethod(lambda a, v: (a.append(v), a.sort()))
    heappop = staticmethod(lambda a: a.pop())


class _NoLayer0Prefetch(olru.SharedLru):
    def access_set(self, call, layer, experts, kind=olru.ROUTED):
        if kind == olru.PREFETCH and layer == 0:
            return []
        return super().access_set(call, layer, experts, kind)


class _PrefetchCountedAsRouted(olru.SharedLru):
    def access_set(self, call, layer, experts, kind=olru.ROUTED):
        return super().access_set(call, layer, experts, olru.ROUTED)


class _ShrinkMovesNotReported(olru.SharedLru):
    def resize(self, new_capacity):
        super().resize(new_capacity)
        return []


MUTANTS = {
    # name: [(module, attribute, replacement)]
    "bf16 widened with a 15-bit shift": [
        (moe, "widen_bf16", lambda b: (np.asarray(b, np.uint16).astype(np.uint32) << 15)
         .view(np.float32).astype(np.float64))],
    "int4 nibbles in swapped order": [(moe, "decode_int4", lambda p: _swap_pairs(_o["decode_int4"](p)))],
    "int4 without sign extension": [
        (moe, "decode_int4", lambda p: np.where(_o["decode_int4"](p) < 0, _o["decode_int4"](p) + 16,
                                                _o["decode_int4"](p)))],
    "int4 scale groups tiled instead of repeated": [(moe, "dequant_int4", _int4_tiled_scales)],
    "e2m1 subnormal read as an integer": [(moe, "decode_e2m1", _e2m1_subnormal_as_integer)],
    "e4m3 exponent bias 8": [(moe, "decode_e4m3", lambda c: _o["decode_e4m3"](c) / 2.0)],
    "nvfp4 nibbles in swapped order": [
        (moe, "dequant_nvfp4", lambda p, s, g: _o["dequant_nvfp4"](_swap_nibbles(p), s, g))],
    "nvfp4 tensor scale dropped": [(moe, "dequant_nvfp4", lambda p, s, g: _o["dequant_nvfp4"](p, s, 1.0))],
    "int4 gate and up scale arrays swapped": [(moe, "expert_weights", _int4_gate_up_scales_swapped)],
    "nvfp4 gate and up tensor scales swapped": [
        (moe, "expert_weights", _nvfp4_swap_regions(lambda m: 3 * m // 2 + 3 * m // 16, lambda m: 4))],
    "nvfp4 gate and up block-scale arrays swapped": [
        (moe, "expert_weights", _nvfp4_swap_regions(lambda m: 3 * m // 2, lambda m: m // 16))],
    "router logits rounded to bf16": [(moe, "router_logits", _router_rounded_to_bf16)],
    "shared expert at weight 1/2": [(moe, "experts_and_combine", _shared_expert_halved)],
    "grow adds no free slot": [(olru, "heapq", _GrowAddsNoFreeSlot)],
    "gate and up swapped in the blob": [
        (moe, "expert_weights", lambda b, w, H, I: (lambda r: (r[1], r[0], r[2]))(_o["expert_weights"](b, w, H, I)))],
    "down matrix read transposed": [(moe, "expert_weights", _down_read_transposed)],
    "router rows in reversed expert order": [
        (moe, "router_logits", lambda x, w: _o["router_logits"](x, np.asarray(w)[::-1]))],
    "router logits left in float64": [
        (moe, "router_logits", lambda x, w: np.asarray(x, np.float64) @ np.asarray(w, np.float64).T)],
    "top-k ties to the higher index": [(moe, "topk", _topk_by(lambda v, e: (-v, -e)))],
    "top-k of the smallest logits": [(moe, "topk", _topk_by(lambda v, e: (v, e)))],
    "top-k ids in ascending id order": [(moe, "topk", _topk_ids_ascending)],
    "near-tie gap halved": [(moe, "topk", lambda z, k: (lambda r: (r[0], r[1] / 2))(_o["topk"](z, k)))],
    "near-tie gap one place too deep": [(moe, "topk", _topk_gap_one_deeper)],
    "softmax of the negated logits": [(moe, "gates", _gates_softmax_negated)],
    "sigmoid gates not renormalised": [(moe, "gates", _gates_sigmoid_unnormalised)],
    "permutation with tokens descending": [(moe, "permute", _permute_tokens_descending)],
    "permutation offsets inclusive": [(moe, "permute", _permute_inclusive_offsets)],
    "silu with the wrong sign": [(moe, "silu", lambda a: a / (1.0 + np.exp(a)))],
    "silu on the up projection": [(moe, "swiglu_ffn", lambda a, g, u, d: _o["swiglu_ffn"](a, u, g, d))],
    "combine with the gate of the wrong slot": [
        (moe, "experts_and_combine", lambda x, ids, g, *a, **kw: _o["experts_and_combine"](
            x, ids, np.asarray(g)[:, ::-1], *a, **kw))],
    "shared expert dropped": [
        (moe, "experts_and_combine", lambda x, ids, g, E, wd, H, I, blob_of, shared_blob=None:
         _o["experts_and_combine"](x, ids, g, E, wd, H, I, blob_of, None))],
    "only each token's first choice made resident": [
        (moe, "selected_set", lambda ids: _o["selected_set"](np.asarray(ids)[:, :1]))],
    "shrink moves not carried to the slot arena": [(orun, "SharedLru", _ShrinkMovesNotReported)],
    "prefill skips the prefetch of layer 0": [(orun, "SharedLru", _NoLayer0Prefetch)],
    "prefill prefetches counted as routed accesses": [(orun, "SharedLru", _PrefetchCountedAsRouted)],
    "LRU evicts the most recently used": [(olru, "OrderedDict", _EvictMru)],
    "LRU hits not refreshed": [(olru, "OrderedDict", _NoRefresh)],
    "misses take the highest free slot": [(olru, "heapq", _HighestFreeSlot)],
    "experts of a step in descending order": [(olru, "sorted", lambda it: sorted(it, reverse=True))],
    "shrink moves survivors least recent first": [(olru, "reversed", lambda seq: iter(seq))],
}


def test_unplanted_oracle_passes_every_pin():
    assert _failing_pins(stop_at_first=False) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    for module, attr, repl in MUTANTS[name]:
        monkeypatch.setattr(module, attr, repl, raising=False)
    assert _failing_pins(), "no pin fails with the planted mistake: %s" % name
