"""Expert-cache residency: the LRU slot bookkeeping and the miss split.

Pages: a global LRU expert cache in VRAM follows router demand (freetoken.wiki
"FreeToken 753b model", mechanism table "Global LRU expert cache";
explainx.ai hardware guide, "Decode: ..."); a missed expert is either copied
over PCIe into the cache and kept, or computed on the CPU; q* is the number of
experts to fill (futuresignalnews.com, mechanism 1); the first request is
served from a cold cache (futuresignalnews.com, mechanism 3).

Readings (the pages give no eviction details):
  * a step's distinct experts U_t are handled in ascending id; hits refresh
    their timestamp; each filled miss takes the lowest free slot, else the
    slot with the oldest timestamp whose expert is not in the step's protected
    set, ties to the lowest slot; no victim -> capacity error;
  * the split: of the step's misses, the round(q * m) with the most routed
    tokens are filled (ties to the lower id), the rest are host-computed;
  * the q* policy balances fill time and host time:
    q* = m * bw_pcie / (bw_pcie + bw_host), rounded, clamped to [0, m];
  * one cache shared by L layers (the pages' global LRU: cache decisions are
    shared across MoE layers, freetoken.wiki mechanism table) is this same
    cache over keys l*E + e, with a clock that advances per layer and step;
  * a resize to n slots at a safe point (futuresignalnews.com, mechanism 3:
    the cache is rebuilt under a new VRAM budget without reloading the host
    pool) keeps the min(residents, n) residents with the latest last use
    (ties: lower slot first), in their old slot order in slots 0, 1, ...,
    with their last-use times; the rest are evicted.

Pins (tests/test_oracle_lru.py): hand-worked traces (one layer; two layers
sharing three slots; shrinking and growing resizes); invariants (hits +
misses = sum |U_t|, residency <= slots, with slots >= E the misses equal the
distinct experts seen, a resize keeps exactly the most recent residents); the
pages' bandwidths for q*.
"""
from __future__ import annotations

import math


class CapacityError(RuntimeError):
    pass


class LRUCache:
    def __init__(self, n_slots: int, n_experts: int):
        self.n_slots = n_slots
        self.expert_of_slot = [-1] * n_slots
        self.last_used = [-1] * n_slots
        self.slot_of_expert = [-1] * n_experts

    def resident(self, e: int) -> bool:
        return self.slot_of_expert[e] >= 0

    def step(self, t: int, to_gpu, protect=None):
        """Make every expert of `to_gpu` resident for step t.
        Returns (hits, fills) with fills = [(expert, slot, evicted_expert or -1)]."""
        want = sorted(set(int(e) for e in to_gpu))
        prot = set(want) if protect is None else set(int(e) for e in protect) | set(want)
        hits, fills = [], []
        for e in want:
            if self.resident(e):
                self.last_used[self.slot_of_expert[e]] = t
                hits.append(e)
        for e in want:
            if self.resident(e):
                continue
            free = [s for s in range(self.n_slots) if self.expert_of_slot[s] < 0]
            if free:
                s = free[0]
            else:
                cand = [s for s in range(self.n_slots) if self.expert_of_slot[s] not in prot]
                if not cand:
                    raise CapacityError(f"step {t}: no evictable slot")
                s = min(cand, key=lambda q: (self.last_used[q], q))
            old = self.expert_of_slot[s]
            if old >= 0:
                self.slot_of_expert[old] = -1
            self.expert_of_slot[s] = e
            self.slot_of_expert[e] = s
            self.last_used[s] = t
            fills.append((e, s, old))
        return hits, fills


    def resize(self, n: int):
        """Rebuild the cache with n slots (see the module header).  Returns
        [(key, old slot)] of the kept residents in their new slot order."""
        res = [s for s in range(self.n_slots) if self.expert_of_slot[s] >= 0]
        res.sort(key=lambda s: (-self.last_used[s], s))
        keep = sorted(res[:n])
        for s in res[n:]:
            self.slot_of_expert[self.expert_of_slot[s]] = -1
        eos, lu = [-1] * n, [-1] * n
        for j, s in enumerate(keep):
            eos[j], lu[j] = self.expert_of_slot[s], self.last_used[s]
            self.slot_of_expert[eos[j]] = j
        self.n_slots, self.expert_of_slot, self.last_used = n, eos, lu
        return [(eos[j], s) for j, s in enumerate(keep)]


def split_misses(misses, tokens_per_expert, q: float):
    """Choose which misses to fill: the round(q*m) misses with the most routed
    tokens, ties to the lower id.  Returns (filled, host) as sorted lists."""
    m = len(misses)
    n_fill = int(math.floor(q * m + 0.5))
    ranked = sorted(misses, key=lambda e: (-tokens_per_expert[e], e))
    filled = sorted(ranked[:n_fill])
    host = sorted(ranked[n_fill:])
    return filled, host


def q_star(m: int, bw_pcie: float, bw_host: float) -> int:
    """Number of misses to fill so that fill time and host-compute time balance:
    q * B / bw_pcie = (m - q) * B / bw_host."""
    q = m * bw_pcie / (bw_pcie + bw_host)
    return max(0, min(m, int(math.floor(q + 0.5))))
