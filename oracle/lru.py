"""The shared LRU expert-slot cache, restated as a plain simulator.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Method: GPU expert slots form one cache under an LRU policy shared by every
MoE layer, so recently chosen experts stay for later tokens; a missed expert is
copied over PCIe into a slot and kept for reuse (FreeToken linux, "FreeToken's
MoE memory handling"; FreeToken gguf, the `offload` backend).  Prefill streams
the next layer's experts while the current layer runs (FreeToken linux, same
section; FreeToken RTX 5090, prefill/decode).  The cache can be resized at a
safe point without a restart (FreeToken RTX 5090, dynamic reconfiguration).

READINGS (the pages give no order of operations):
  * key = (layer, expert); one access per distinct expert chosen in a step.
  * Within one (step, layer): first every selected expert that is resident, in
    ascending expert order, is a hit and moves to most-recently-used; then
    every selected expert that is not resident, in ascending order, is a miss:
    it takes the lowest-numbered free slot, or else evicts the least recently
    used entry and reuses its slot, and is inserted as most-recently-used.
  * Capacity below the number of distinct experts a step needs is an error,
    raised before any state changes.
  * Prefetch accesses follow the same rule with kind "prefetch".
  * Grow: entries keep slot and recency, new slots are free.  Shrink: evict
    from the LRU end down to the new capacity, then move survivors that sit in
    slots >= new capacity into the lowest free slots below it, taking survivors
    in most- to least-recently-used order; recency is kept.
"""
import heapq
from collections import OrderedDict
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

ROUTED, PREFETCH = 0, 1


class CapacityError(Exception):
    pass


@dataclass(frozen=True)
class Access:
    call: int       # forward-call index (one per layer per step)
    layer: int
    expert: int
    kind: int       # ROUTED or PREFETCH
    hit: bool
    slot: int
    ev_layer: int   # evicted key, (-1, -1) if a free slot was taken
    ev_expert: int


@dataclass
class Stats:
    routed: int = 0
    hits: int = 0
    misses: int = 0
    evictions: int = 0
    prefetch: int = 0
    prefetch_hits: int = 0
    prefetch_misses: int = 0
    fills: int = 0          # slot fills from host memory (routed + prefetch misses)


class SharedLru:
    def __init__(self, capacity: int):
        if capacity < 1:
            raise ValueError("capacity must be >= 1")
        self.capacity = capacity
        self.order: "OrderedDict[Tuple[int,int], int]" = OrderedDict()   # LRU first ... MRU last
        self.free: List[int] = list(range(capacity))
        heapq.heapify(self.free)
        self.trace: List[Access] = []
        self.stats = Stats()

    def slot_of(self, layer: int, expert: int) -> Optional[int]:
        return self.order.get((layer, expert))

    def resident(self):
        return dict(self.order)

    def access_set(self, call: int, layer: int, experts, kind: int = ROUTED) -> List[Access]:
        """Accesses for the distinct experts `experts` of one layer in one step."""
        S = sorted(set(int(e) for e in experts))
        if len(S) > self.capacity:
            raise CapacityError("step needs %d slots, cache has %d" % (len(S), self.capacity))
        recs = []
        hit_set = [e for e in S if (layer, e) in self.order]
        miss_set = [e for e in S if (layer, e) not in self.order]
        for e in hit_set:                             # phase 1: hits, ascending
            key = (layer, e)
            self.order.move_to_end(key)
            recs.append(Access(call, layer, e, kind, True, self.order[key], -1, -1))
        for e in miss_set:                            # phase 2: misses, ascending
            key = (layer, e)
            if self.free:
                slot = heapq.heappop(self.free)
                ev = (-1, -1)
            else:
                ev, slot = self.order.popitem(last=False)
                self.stats.evictions += 1
            self.order[key] = slot
            recs.append(Access(call, layer, e, kind, False, slot, ev[0], ev[1]))
        for r in recs:
            if kind == ROUTED:
                self.stats.routed += 1
                self.stats.hits += r.hit
                self.stats.misses += not r.hit
            else:
                self.stats.prefetch += 1
                self.stats.prefetch_hits += r.hit
                self.stats.prefetch_misses += not r.hit
            self.stats.fills += not r.hit
        self.trace.extend(recs)
        return recs

    def resize(self, new_capacity: int):
        """Returns the list of (old_slot, new_slot) moves a shrink needs (empty for a grow)."""
        if new_capacity < 1:
            raise ValueError("capacity must be >= 1")
        moves = []
        if new_capacity >= self.capacity:
            for s in range(self.capacity, new_capacity):
                heapq.heappush(self.free, s)
        else:
            while len(self.order) > new_capacity:
                self.order.popitem(last=False)
                self.stats.evictions += 1
            used = set(self.order.values())
            free_low = sorted(s for s in range(new_capacity) if s not in used)
            for key in reversed(list(self.order.keys())):      # MRU -> LRU
                s = self.order[key]
                if s >= new_capacity:
                    ns = free_low.pop(0)
                    moves.append((s, ns))
                    self.order[key] = ns
            used = set(self.order.values())
            self.free = [s for s in range(new_capacity) if s not in used]
            heapq.heapify(self.free)
        self.capacity = new_capacity
        return moves
