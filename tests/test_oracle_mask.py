"""Pins of the frame-block-causal mask oracle (hand tables, enumeration, counts)."""

import itertools

import numpy as np
import pytest

from oracle import frame_block_visible, frame_pair_visible, default_q_frame_offset


def test_hand_table_4_query_frames_7_key_frames():
    # Query window = last 4 of 7 key frames -> query frames 3,4,5,6; block 3:
    # frames 3,4,5 form block 1 (see key frames 0..5), frame 6 is block 2 (all 7).
    expected = np.array([
        [1, 1, 1, 1, 1, 1, 0],
        [1, 1, 1, 1, 1, 1, 0],
        [1, 1, 1, 1, 1, 1, 0],
        [1, 1, 1, 1, 1, 1, 1],
    ], dtype=bool)
    assert default_q_frame_offset(4, 7, 1) == 3
    assert np.array_equal(frame_pair_visible(4, 7, 3, 3), expected)


def test_hand_table_block_two_offset_zero():
    # query frames 0..3 anchored at key frame 0, block 2
    expected = np.array([
        [1, 1, 0, 0, 0],
        [1, 1, 0, 0, 0],
        [1, 1, 1, 1, 0],
        [1, 1, 1, 1, 0],
    ], dtype=bool)
    assert np.array_equal(frame_pair_visible(4, 5, 0, 2), expected)


def test_two_pass_counts():
    # denoise pass: 15 query frames in a 21-frame context; cache pass: 5 frames
    d = frame_pair_visible(15, 21, default_q_frame_offset(15 * 1560, 21 * 1560, 1560), 3)
    c = frame_pair_visible(5, 21, default_q_frame_offset(5 * 1560, 21 * 1560, 1560), 3)
    assert int(d.sum()) == 225 and d.size == 315
    assert int(c.sum()) == 99 and c.size == 105


def test_brute_force_enumeration():
    # every small configuration against the definition in words, spelled as loops
    for nq, nk, off, b in itertools.product(range(1, 5), range(1, 7), range(0, 5), range(1, 4)):
        got = frame_pair_visible(nq, nk, off, b)
        for a in range(nq):
            for c in range(nk):
                block_of_query = (off + a) // b
                keys_allowed_below = (block_of_query + 1) * b   # first key frame of the next block
                assert got[a, c] == (c < keys_allowed_below)


def test_token_level_expands_frames():
    F = 3
    tok = frame_block_visible(4 * F, 7 * F, F, 3, 3)
    fr = frame_pair_visible(4, 7, 3, 3)
    for r in range(4 * F):
        for c in range(7 * F):
            assert tok[r, c] == fr[r // F, c // F]


def test_visible_keys_form_a_prefix():
    # every query row sees a prefix of the keys (the kernel relies on this shape)
    tok = frame_block_visible(10, 23, 2, 4, 3)
    for row in tok:
        n = int(row.sum())
        assert row[:n].all() and not row[n:].any()


def test_rows_argument():
    full = frame_block_visible(12, 20, 2, 2, 2)
    rows = np.array([0, 5, 11])
    assert np.array_equal(frame_block_visible(12, 20, 2, 2, 2, rows=rows), full[rows])
