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
