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
* Prediction of a layer's next call (aimodeling.com English page, "Three
  Engineering Cores": full-layer double-buffered streaming; winzheng.com,
  "FreeToken's Three-Layer Mechanism": transfers sized to the bandwidth
  measured): the experts its last resolve used, ranked by the pairs each
  received, more first, ties to the lower id (counts above 2^20 - 1 rank as
  equal). A prefetch of depth d takes the first d of them; a full-layer
  prefetch takes every expert of the layer.
* Resize to S' slots (aimodeling.com, "Three Engineering Cores": elastic memory
  without weight reloads): growing adds free slots. Shrinking keeps the
  min(occupied, S') most recently referenced experts and drops the others;
  kept experts in slots >= S' then move, least recent first, each to the
  lowest free slot below S', keeping their recency and call index.

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
        self.moves = 0
        self.last_counts: Dict[int, Dict[int, int]] = {}   # layer -> {expert: pairs} at its last resolve

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
        """Map the experts a layer needs to slots; returns the (expert, slot) loads.

        ``ids`` may repeat an expert once per pair routed to it: the number of
        repeats is the pair count that ranks the layer's next prediction."""
        ids = [int(i) for i in ids]
        loads = self._call(layer, ids, True)
        counts: Dict[int, int] = {}
        for e in ids:
            counts[e] = counts.get(e, 0) + 1
        self.last_counts[layer] = counts
        return loads

    def predict(self, layer: int, depth: int = -1, full: bool = False) -> List[int]:
        """Experts a prefetch of ``layer`` loads: all E when ``full``, else the
        first ``depth`` of the layer's prediction in rank order (depth < 0: all)."""
        if full:
            return list(range(self.E))
        counts = self.last_counts.get(layer, {})
        ranked = sorted(counts, key=lambda e: (-min(counts[e], (1 << 20) - 1), e))
        return sorted(ranked if depth < 0 else ranked[:depth])

    def resize(self, n_slots: int) -> List[Tuple[int, int]]:
        """Change the pool to ``n_slots`` slots; returns the (from, to) slot moves."""
        S = self.S
        if n_slots >= S:
            self.owner += [None] * (n_slots - S)
            self.stamp += [-1] * (n_slots - S)
            self.ref_call += [-(10**9)] * (n_slots - S)
            self.S = n_slots
            return []
        occ = sorted((i for i in range(S) if self.owner[i] is not None), key=lambda i: self.stamp[i])
        keep = occ[len(occ) - min(len(occ), n_slots):]
        for i in occ[: len(occ) - len(keep)]:
            del self.slot_of[self.owner[i]]
            self.owner[i] = None
            self.stamp[i] = -1
            self.ref_call[i] = -(10**9)
        moves = []
        for i in keep:   # least recent first
            if i < n_slots:
                continue
            f = min(j for j in range(n_slots) if self.owner[j] is None)
            self.owner[f], self.stamp[f], self.ref_call[f] = self.owner[i], self.stamp[i], self.ref_call[i]
            self.slot_of[self.owner[f]] = f
            self.owner[i], self.stamp[i], self.ref_call[i] = None, -1, -(10**9)
            moves.append((i, f))
        del self.owner[n_slots:], self.stamp[n_slots:], self.ref_call[n_slots:]
        self.S = n_slots
        self.moves += len(moves)
        return moves

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
