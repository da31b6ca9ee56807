"""Pins of the ring-cache oracle: a hand-worked example and collections.deque."""

from collections import deque

import pytest
from hypothesis import given, settings, strategies as st

from oracle import RingRef


def test_hand_example_five_slots():
    r = RingRef(5)
    assert r.insert(["a", "b", "c"]) == 0
    assert (r.head, r.count) == (3, 3)
    assert r.insert(["d", "e", "f"]) == 1          # "a" evicted
    assert (r.head, r.count) == (1, 5)
    assert r.slots == ["f", "b", "c", "d", "e"]
    assert r.logical_frames() == ["b", "c", "d", "e", "f"]
    assert [r.slot_of(j) for j in range(6)] == [1, 2, 3, 4, 0, -1]
    assert r.insert(["g", "h", "i"]) == 3
    assert r.logical_frames() == ["d", "e", "f", "g", "h", "i"][-5:]
    assert r.valid_slots() == [0, 1, 2, 3, 4]


def test_insert_more_than_slots_rejected():
    with pytest.raises(ValueError):
        RingRef(3).insert([1, 2, 3, 4])


@settings(max_examples=200, deadline=None)
@given(W=st.integers(1, 9), sizes=st.lists(st.integers(0, 9), max_size=12))
def test_matches_deque(W, sizes):
    r = RingRef(W)
    d = deque(maxlen=W)
    nxt = 0
    for n in sizes:
        n = min(n, W)
        frames = list(range(nxt, nxt + n))
        nxt += n
        before = len(d)
        ev = r.insert(frames)
        d.extend(frames)
        assert ev == before + n - len(d)
        assert r.logical_frames() == list(d)
        assert r.count == len(d)
        # valid slots are exactly the slots holding the deque's frames
        assert sorted(r.slots[s] for s in r.valid_slots()) == sorted(d)


def test_fill_from_empty_keeps_valid_prefix():
    # started at head 0, the valid slots are [0, count) until the ring is full
    r = RingRef(21)
    r.insert([0])
    for step in range(8):
        r.insert(list(range(1 + 5 * step, 6 + 5 * step)))
        if r.count < 21:
            assert r.valid_slots() == list(range(r.count))
        else:
            assert r.valid_slots() == list(range(21))


# ---- pinned prefix ("attention sink" frames kept out of eviction) -----------

def test_pinned_hand_example():
    # 6 slots, 2 pinned: a, b stay; c.. roll through slots 2..5
    r = RingRef(6, pinned=2)
    assert r.insert(["a", "b", "c"]) == 0
    assert (r.head, r.count) == (3, 3)
    assert r.insert(["d", "e", "f"]) == 0
    assert (r.head, r.count) == (2, 6)
    assert r.slots == ["a", "b", "c", "d", "e", "f"]
    assert r.insert(["g", "h"]) == 2                      # c, d evicted; a, b kept
    assert r.slots == ["a", "b", "g", "h", "e", "f"]
    assert r.logical_frames() == ["a", "b", "e", "f", "g", "h"]
    assert [r.slot_of(j) for j in range(7)] == [0, 1, 4, 5, 2, 3, -1]
    with pytest.raises(ValueError):
        r.insert(list("ijklm"))                            # 5 > 4 rolling slots


def test_pinned_zero_is_the_plain_ring():
    a, b = RingRef(5), RingRef(5, pinned=0)
    for frames in (["x"], list("abc"), list("defg"), list("hi")):
        assert a.insert(frames) == b.insert(frames)
        assert a.slots == b.slots and (a.head, a.count) == (b.head, b.count)


@settings(max_examples=200, deadline=None)
@given(W=st.integers(2, 9), P=st.integers(0, 8), sizes=st.lists(st.integers(0, 9), max_size=12))
def test_pinned_matches_prefix_plus_deque(W, P, sizes):
    # model: the first P frames ever inserted, then a deque(maxlen=W-P) of the rest
    P = min(P, W - 1)
    r = RingRef(W, pinned=P)
    prefix, d = [], deque(maxlen=W - P)
    nxt = 0
    for n in sizes:
        n = min(n, r.capacity_for_insert())
        frames = list(range(nxt, nxt + n))
        nxt += n
        before = len(d)
        ev = r.insert(frames)
        for f in frames:
            if len(prefix) < P:
                prefix.append(f)
            else:
                d.append(f)
        rolled_in = sum(1 for f in frames if f not in prefix)
        assert ev == before + rolled_in - len(d)
        assert r.logical_frames() == prefix + list(d)
        assert r.slots[:len(prefix)] == prefix
        # filled from empty, the valid slots are always the prefix [0, count)
        assert r.valid_slots() == list(range(r.count))
