"""A second, deliberately different statement of the shared-LRU rule, used only
to pin the oracle's simulator: per-entry timestamps and a linear scan for the
least recently used entry and for the lowest free slot (no ordered dict, no heap)."""


class NaiveLru:
    def __init__(self, capacity):
        self.capacity = capacity
        self.slot = {}     # key -> slot
        self.stamp = {}    # key -> last-use clock
        self.clock = 0
        self.trace = []

    def _touch(self, key):
        self.clock += 1
        self.stamp[key] = self.clock

    def access_set(self, call, layer, experts, kind=0):
        S = sorted(set(int(e) for e in experts))
        if len(S) > self.capacity:
            raise RuntimeError("capacity")
        resident_now = [e for e in S if (layer, e) in self.slot]
        for e in resident_now:
            self._touch((layer, e))
            self.trace.append((call, layer, e, kind, True, self.slot[(layer, e)], -1, -1))
        for e in S:
            if e in resident_now:
                continue
            used = set(self.slot.values())
            free = [s for s in range(self.capacity) if s not in used]
            if free:
                s, ev = free[0], (-1, -1)
            else:
                ev = min(self.stamp, key=lambda kk: self.stamp[kk])
                s = self.slot.pop(ev)
                del self.stamp[ev]
            self.slot[(layer, e)] = s
            self._touch((layer, e))
            self.trace.append((call, layer, e, kind, False, s, ev[0], ev[1]))
