"""Pins for the oracle's expert-cache model (CPU only): the textbook behaviour of an LRU
cache, checked on patterns whose outcome is known without running it."""
import numpy as np
import pytest

import oracle


def test_cyclic_working_set_that_fits_hits_after_the_first_pass():
    E, S = 32, 8
    steps = [[i % 8] for i in range(40)]  # 8 distinct experts, one per step
    out, _ = oracle.lru_cache_steps(steps, E, S)
    misses = [len(m) for _, m, _ in out]
    assert sum(misses[:8]) == 8 and sum(misses[8:]) == 0


def test_cyclic_working_set_one_larger_than_the_cache_always_misses():
    E, S = 32, 8
    steps = [[i % 9] for i in range(45)]  # classic LRU thrash
    out, _ = oracle.lru_cache_steps(steps, E, S)
    assert all(len(m) == 1 for _, m, _ in out)


def test_victim_is_least_recently_used_and_empty_slots_go_first():
    E, S = 16, 3
    out, (slot_of, expert_of, last_use) = oracle.lru_cache_steps(
        [[0], [1], [2], [0], [3]], E, S)
    assert [f for _, _, f in out[:3]] == [[(0, 0)], [(1, 1)], [(2, 2)]]  # empty slots in order
    assert out[3] == ([0], [], [])                      # a hit
    assert out[4][2] == [(3, 1)]                        # 1 is now the least recently used
    assert slot_of[1] == -1 and slot_of[3] == 1 and expert_of == [0, 3, 2]
    assert last_use == [4, 5, 3]


def test_experts_of_the_current_step_are_never_evicted():
    E, S = 16, 4
    out, _ = oracle.lru_cache_steps([[0, 1], [2, 3], [0, 4, 5, 6]], E, S)
    fills = out[2][2]
    assert out[2][0] == [0]                              # expert 0 hits
    assert sorted(e for e, _ in fills) == [4, 5, 6]
    slots = [s for _, s in fills]
    assert len(set(slots)) == 3 and 0 not in slots       # slot 0 holds expert 0


def test_invariants_on_random_zipf_traffic():
    rng = np.random.default_rng(3)
    E, S, k = 64, 12, 4
    p = 1.0 / np.arange(1, E + 1)
    p /= p.sum()
    steps = [rng.choice(E, k, replace=False, p=p) for _ in range(300)]
    out, (slot_of, expert_of, _) = oracle.lru_cache_steps(steps, E, S)
    for (hits, misses, fills), sel in zip(out, steps):
        assert sorted(hits + misses) == sorted(set(sel.tolist()))
        assert [e for e, _ in fills] == misses
    for s, e in enumerate(expert_of):
        if e >= 0:
            assert slot_of[e] == s
    assert sum(1 for v in slot_of if v >= 0) == sum(1 for e in expert_of if e >= 0) <= S


def test_too_few_slots_is_an_error():
    with pytest.raises(ValueError):
        oracle.lru_cache_steps([[0, 1, 2]], 8, 2)
