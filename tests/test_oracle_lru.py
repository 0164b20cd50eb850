"""Pins of oracle.lru: hand-worked trace, invariants, the pages' figures."""
import json
import os

import numpy as np
import pytest

from oracle import lru as L


def test_hand_worked_trace():
    c = L.LRUCache(n_slots=2, n_experts=6)
    # t0: {3,1}: cold cache, misses ascending -> 1 in slot 0, 3 in slot 1
    assert c.step(0, [3, 1]) == ([], [(1, 0, -1), (3, 1, -1)])
    # t1: {3}: hit
    assert c.step(1, [3]) == ([3], [])
    # t2: {5,3}: 3 hit; 5 misses, victim = oldest not in step = slot 0 (expert 1)
    assert c.step(2, [5, 3]) == ([3], [(5, 0, 1)])
    # t3: {0,2}: both slots stamped 2 -> ties to lowest slot first
    assert c.step(3, [2, 0]) == ([], [(0, 0, 5), (2, 1, 3)])
    # t4: {0} hit, {4} protected set includes 0 -> evict slot 1 (expert 2)
    assert c.step(4, [4, 0]) == ([0], [(4, 1, 2)])
    assert c.slot_of_expert == [0, -1, -1, -1, 1, -1]


def test_capacity_error_when_step_needs_more_slots():
    c = L.LRUCache(n_slots=2, n_experts=5)
    with pytest.raises(L.CapacityError):
        c.step(0, [0, 1, 2])


def test_invariants_random_trace():
    rng = np.random.default_rng(0)
    E, S = 32, 8
    c = L.LRUCache(S, E)
    hits = misses = total = 0
    for t in range(200):
        u = rng.choice(E, rng.integers(1, S + 1), replace=False)
        h, f = c.step(t, u)
        hits += len(h)
        misses += len(f)
        total += len(set(u.tolist()))
        assert sum(1 for e in c.expert_of_slot if e >= 0) <= S
        for s, e in enumerate(c.expert_of_slot):
            if e >= 0:
                assert c.slot_of_expert[e] == s
        assert all(c.resident(int(e)) for e in u)
    assert hits + misses == total


def test_enough_slots_misses_equal_distinct():
    rng = np.random.default_rng(1)
    E = 20
    c = L.LRUCache(E, E)
    seen = set()
    misses = 0
    for t in range(100):
        u = rng.choice(E, 4, replace=False)
        misses += len(c.step(t, u)[1])
        seen |= set(u.tolist())
    assert misses == len(seen)


def test_split_misses_ranking():
    tok = {3: 2, 5: 4, 7: 2, 9: 1}
    filled, host = L.split_misses([3, 5, 7, 9], tok, 0.5)
    assert filled == [3, 5] and host == [7, 9]
    assert L.split_misses([3, 5, 7, 9], tok, 0.0) == ([], [3, 5, 7, 9])
    assert L.split_misses([3, 5, 7, 9], tok, 1.0) == ([3, 5, 7, 9], [])


def test_q_star_with_pages_bandwidths(golden_dir):
    fig = json.load(open(os.path.join(golden_dir, "pages_figures.json")))["glm_workstation_bandwidth"]
    frac = fig["pcie_gbs"] / (fig["pcie_gbs"] + fig["host_gbs"])
    assert abs(frac - 0.2244) < 1e-4
    assert L.q_star(10, fig["pcie_gbs"], fig["host_gbs"]) == 2
    assert L.q_star(40, fig["pcie_gbs"], fig["host_gbs"]) == 9
    assert L.q_star(0, 1, 1) == 0


def test_pages_arithmetic_closes(golden_dir):
    fig = json.load(open(os.path.join(golden_dir, "pages_figures.json")))
    p = fig["rtx5090_prefill"]
    t = p["pool_gb"] / p["link_gbs"]
    assert p["chunk_seconds"][0] - 0.01 <= t <= p["chunk_seconds"][1] + 0.01
    r = fig["deepseek_v4_flash_routing"]
    assert r["top_k"] / r["experts"] < r["active_params_b"] / r["total_params_b"] * 1.01


def test_two_layers_share_three_slots_hand_worked():
    """One cache over keys l*E + e (E = 4), clock = step * 2 + layer."""
    c = L.LRUCache(n_slots=3, n_experts=8)
    assert c.step(0, [0, 1]) == ([], [(0, 0, -1), (1, 1, -1)])          # step 0, layer 0
    assert c.step(1, [4 + 2]) == ([], [(6, 2, -1)])                      # step 0, layer 1
    # step 1, layer 0: key 1 hit; key 3 evicts the oldest unprotected: key 0 (slot 0)
    assert c.step(2, [1, 3]) == ([1], [(3, 0, 0)])
    # step 1, layer 1: key 6 hit; key 4 ties between slots 0 and 1 (time 2): slot 0
    assert c.step(3, [6, 4]) == ([6], [(4, 0, 3)])
    # step 2, layer 0: key 3 again: the oldest is slot 1 (key 1, time 2)
    assert c.step(4, [3]) == ([], [(3, 1, 1)])
    assert c.expert_of_slot == [4, 3, 6] and c.last_used == [3, 4, 3]


def test_resize_hand_worked():
    c = L.LRUCache(n_slots=4, n_experts=10)
    c.step(0, [2])
    c.step(1, [5, 2])          # slot 0: 2 (t1), slot 1: 5 (t1)
    c.step(2, [7])             # slot 2: 7 (t2)
    c.step(3, [9, 5])          # slot 3: 9 (t3), 5 refreshed (t3)
    assert c.expert_of_slot == [2, 5, 7, 9] and c.last_used == [1, 3, 2, 3]
    # shrink to 2: the latest are slot 1 (t3) and slot 3 (t3); they move to 0, 1
    assert c.resize(2) == [(5, 1), (9, 3)]
    assert c.expert_of_slot == [5, 9] and c.last_used == [3, 3]
    assert c.slot_of_expert[2] == -1 and c.slot_of_expert[7] == -1 and c.slot_of_expert[9] == 1
    # grow to 3: everything kept; the next miss takes the free slot 2
    assert c.resize(3) == [(5, 0), (9, 1)]
    assert c.step(4, [1]) == ([], [(1, 2, -1)])
    # shrink below a tie: slots 0 and 1 both t3, slot 2 t4 -> keep slots 0 and 2
    assert c.resize(2) == [(5, 0), (1, 2)]
    assert c.expert_of_slot == [5, 1]


def test_resize_keeps_exactly_the_most_recent():
    rng = np.random.default_rng(3)
    c = L.LRUCache(16, 64)
    for t in range(60):
        c.step(t, rng.choice(64, 5, replace=False))
    for n in (16, 9, 3, 12, 1):
        before = {e: lu for e, lu in zip(c.expert_of_slot, c.last_used) if e >= 0}
        kept = c.resize(n)
        order = sorted(before, key=lambda e: -before[e])
        cutoff = before[order[min(n, len(order)) - 1]]
        assert all(before[e] >= cutoff for e, _ in kept)
        assert len(kept) == min(n, len(before))
        assert [e for e, _ in kept] == [e for e in c.expert_of_slot if e >= 0]
        for s, e in enumerate(c.expert_of_slot):
            assert e < 0 or c.slot_of_expert[e] == s
        assert sum(1 for v in c.slot_of_expert if v >= 0) == len(kept)
