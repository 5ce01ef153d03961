"""Pins for the user-id map model (hand example + invariants)."""

import numpy as np

from oracle.user_map import INVALID_ARG, OK, OUT_OF_SLOTS, UserMapOracle


def test_hand_example():
    m = UserMapOracle(3, [0, 1, 2])                       # top = 2
    assert m.lookup([10**12, 7, 10**12], insert=True) == (OK, [2, 1, 2])
    assert m.lookup([7, 5], insert=False) == (OK, [1, -1])
    assert m.erase([10**12, 999]) == OK                   # unknown id ignored
    assert m.stack == [0, 2]
    assert m.lookup([5, 6, 8], insert=True) == (OUT_OF_SLOTS, [-1, -1, -1])
    assert m.stack == [0, 2] and set(m.slot) == {7}       # unchanged
    assert m.lookup([5, 6], insert=True) == (OK, [2, 0])
    assert m.lookup([-1], insert=False)[0] == INVALID_ARG


def test_random_sequences_keep_slots_unique():
    rng = np.random.default_rng(4)
    m = UserMapOracle(50, rng.permutation(50))
    for _ in range(200):
        ids = rng.integers(0, 2**40, size=int(rng.integers(1, 8))) if rng.random() < 0.5 else \
            rng.choice(list(m.slot) or [1], size=3)
        if rng.random() < 0.3:
            m.erase(ids)
        else:
            m.lookup(ids, insert=True)
        held = list(m.slot.values())
        assert len(set(held)) == len(held) and set(held).isdisjoint(m.stack)
        assert len(held) + len(m.stack) == 50
