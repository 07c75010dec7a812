"""CPU simulation of the device LRU expert cache (test infrastructure only).

Source: winzheng.com "FreeToken ... 753B local inference MoE", section
"FreeToken's Three-Layer Mechanism" (a global LRU expert cache reuses
high-frequency experts, with weight movement overlapped with compute); the
aimodeling.com English page, section "Three Engineering Cores" (the same LRU
cache plus double-buffered streaming). The pages name the policy only ("LRU");
the rules below are the reading taken here, written so that the hit/miss trace
and the final table are fully determined:

* S slots, all free at start. A miss takes the lowest-index free slot.
* With no free slot, a miss evicts the least recently referenced slot that is
  not protected. Protected: slots referenced by the current call or by the call
  just before it (that call's GEMM or copies may still be in flight).
* A call (resolve or prefetch) handles its expert ids in ascending order, each
  id once. Every referenced slot becomes the most recently used.
* Hits and misses are counted on resolve calls only; every load (miss or
  prefetch) counts its bytes.
* If every occupied slot is protected and none is free the call fails with
  CACHE_FULL and leaves the table as it was before the call.

Independent of the device code: this keeps explicit integer stamps and scans
for the minimum, where the kernel keeps an intrusive linked list.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Tuple


class CacheFull(Exception):
    pass


class LruSim:
    def __init__(self, n_slots: int, n_layers: int, n_experts: int, expert_bytes: int):
        self.S, self.L, self.E = n_slots, n_layers, n_experts
        self.expert_bytes = expert_bytes
        self.owner: List[Optional[Tuple[int, int]]] = [None] * n_slots
        self.stamp: List[int] = [-1] * n_slots         # time of last reference
        self.ref_call: List[int] = [-(10**9)] * n_slots  # index of the last call that referenced it
        self.slot_of: Dict[Tuple[int, int], int] = {}
        self.clock = 0
        self.calls = 0
        self.hits = self.misses = self.loads = 0
        self.bytes_h2d = 0

    def _call(self, layer: int, ids: Iterable[int], count: bool) -> List[Tuple[int, int]]:
        ids = sorted(set(int(i) for i in ids))
        c = self.calls
        snapshot = (list(self.owner), list(self.stamp), list(self.ref_call), dict(self.slot_of), self.clock)
        loads: List[Tuple[int, int]] = []
        hits = misses = 0
        for e in ids:
            key = (layer, e)
            s = self.slot_of.get(key)
            if s is not None:
                hits += 1
            else:
                misses += 1
                free = [i for i in range(self.S) if self.owner[i] is None]
                if free:
                    s = free[0]
                else:
                    cand = [i for i in range(self.S) if self.ref_call[i] < c - 1]
                    if not cand:
                        (self.owner, self.stamp, self.ref_call, self.slot_of, self.clock) = snapshot
                        raise CacheFull(f"no evictable slot for layer {layer} expert {e}")
                    s = min(cand, key=lambda i: (self.stamp[i], i))
                    del self.slot_of[self.owner[s]]
                self.owner[s] = key
                self.slot_of[key] = s
                loads.append((e, s))
            self.clock += 1
            self.stamp[s] = self.clock
            self.ref_call[s] = c
        self.calls += 1
        if count:
            self.hits += hits
            self.misses += misses
        self.loads += len(loads)
        self.bytes_h2d += len(loads) * self.expert_bytes
        return loads

    def resolve(self, layer: int, ids: Iterable[int]) -> List[Tuple[int, int]]:
        """Map the experts a layer needs to slots; returns the (expert, slot) loads."""
        return self._call(layer, ids, True)

    def prefetch(self, layer: int, ids: Iterable[int]) -> List[Tuple[int, int]]:
        return self._call(layer, ids, False)

    def evict(self, layer: int = -1, ids: Optional[Iterable[int]] = None) -> None:
        """Free slots: all (layer=-1), one layer's (ids=None) or the listed experts of a layer."""
        for s in range(self.S):
            o = self.owner[s]
            if o is None:
                continue
            if layer >= 0 and o[0] != layer:
                continue
            if ids is not None and o[1] not in set(ids):
                continue
            del self.slot_of[o]
            self.owner[s] = None
            self.stamp[s] = -1
            self.ref_call[s] = -(10**9)

    def table(self) -> List[int]:
        """slot_of as a dense [L*E] list (-1 = not resident)."""
        out = [-1] * (self.L * self.E)
        for (l, e), s in self.slot_of.items():
            out[l * self.E + e] = s
        return out
