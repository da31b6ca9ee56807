"""Pins of the 3D-RoPE oracle.

None of these re-types the oracle's formula: each checks a value or property
that the mathematics fixes (identity at position 0, textbook cos/sin values,
closed-form frequencies such as 10000^(-11/22) = 0.01, norm preservation, the
relative-position property, a library complex rotation).
"""

import math

import numpy as np
import pytest

from oracle import rope3d_ref, token_positions

PAIRS = (22, 21, 21)
D = 128


def unit_pair_input(L, pair):
    """x with (1, 0) in rotary pair ``pair`` of every row (one head)."""
    x = np.zeros((L, 1, D))
    x[:, 0, 2 * pair] = 1.0
    return x


def recovered_angle(y, pair):
    return np.arctan2(y[:, 0, 2 * pair + 1], y[:, 0, 2 * pair])


def test_positions_row_major():
    # 4x6 grid (24 tokens per frame): token 31 is frame 1, row 1, column 1.
    t, h, w = token_positions(np.array([0, 5, 6, 23, 24, 31, 47]), 2, 4, 6)
    assert t.tolist() == [2, 2, 2, 2, 3, 3, 3]
    assert h.tolist() == [0, 0, 1, 3, 0, 1, 3]
    assert w.tolist() == [0, 5, 0, 5, 0, 1, 5]


def test_identity_at_origin():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((1, 3, D))
    assert np.array_equal(rope3d_ref(x, 0, 4, 6, PAIRS), x)


def test_textbook_rotation_values():
    # token 24 of a 4x6 grid with t0 = 0 has t = 1; pair 0 turns by 1 rad.
    y = rope3d_ref(unit_pair_input(25, 0), 0, 4, 6, PAIRS)
    assert y[24, 0, 0] == pytest.approx(0.5403023058681398, abs=1e-15)   # cos 1
    assert y[24, 0, 1] == pytest.approx(0.8414709848078965, abs=1e-15)   # sin 1
    # other elements untouched (pairs are adjacent elements)
    assert np.count_nonzero(y[24, 0, 2:]) == 0
    # the second element of a pair rotates into -sin, +cos
    x = np.zeros((25, 1, D)); x[:, 0, 1] = 1.0
    y = rope3d_ref(x, 0, 4, 6, PAIRS)
    assert y[24, 0, 0] == pytest.approx(-0.8414709848078965, abs=1e-15)
    assert y[24, 0, 1] == pytest.approx(0.5403023058681398, abs=1e-15)


@pytest.mark.parametrize("pair,expected_per_unit,axis", [
    (0, 1.0, "t"),                         # t axis, i = 0
    (11, 0.01, "t"),                       # t axis, i = 11 of 22: 10000^(-1/2)
    (21, 10.0 ** (-4 * 21 / 22), "t"),     # last t pair
    (22, 1.0, "h"),                        # h axis, i = 0
    (29, 10.0 ** (-4.0 / 3.0), "h"),       # h axis, i = 7 of 21: 10000^(-1/3)
    (43, 1.0, "w"),                        # w axis, i = 0
    (57, 10.0 ** (-8.0 / 3.0), "w"),       # w axis, i = 14 of 21: 10000^(-2/3)
])
def test_axis_split_and_frequencies(pair, expected_per_unit, axis):
    # token 31 of a 4x6 grid, t0 = 2: (t, h, w) = (3, 1, 1); token 47: (3, 3, 5)
    y = rope3d_ref(unit_pair_input(48, pair), 2, 4, 6, PAIRS)
    ang = recovered_angle(y, pair)
    pos31 = {"t": 3, "h": 1, "w": 1}[axis]
    pos47 = {"t": 3, "h": 3, "w": 5}[axis]
    def wrapped(a):   # angle difference folded into (-pi, pi]
        return (a + math.pi) % (2 * math.pi) - math.pi
    assert abs(wrapped(ang[31] - pos31 * expected_per_unit)) < 1e-13
    assert abs(wrapped(ang[47] - pos47 * expected_per_unit)) < 1e-13


def test_norm_preserved_per_pair():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((200, 3, D))
    y = rope3d_ref(x, 5, 4, 6, PAIRS)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.max(np.abs(nx - ny)) < 1e-12


def test_matches_complex_rotation():
    # (x0 + i x1) * exp(i a) with numpy's complex exp, angles from textbook law
    rng = np.random.default_rng(2)
    x = rng.standard_normal((48, 2, D))
    y = rope3d_ref(x, 1, 4, 6, PAIRS)
    t, h, w = token_positions(np.arange(48), 1, 4, 6)
    for pair in range(64):
        if pair < 22:
            pos, i, n = t, pair, 22
        elif pair < 43:
            pos, i, n = h, pair - 22, 21
        else:
            pos, i, n = w, pair - 43, 21
        a = pos * math.pow(10000.0, -i / n)
        z = (x[:, :, 2 * pair] + 1j * x[:, :, 2 * pair + 1]) * np.exp(1j * a)[:, None]
        assert np.max(np.abs(z.real - y[:, :, 2 * pair])) < 1e-12
        assert np.max(np.abs(z.imag - y[:, :, 2 * pair + 1])) < 1e-12


def test_score_depends_only_on_relative_offset():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((48, 1, D))
    k = rng.standard_normal((48, 1, D))
    # shift in t: both sequences start 7 frames later
    s0 = np.einsum("qd,kd->qk", rope3d_ref(q, 0, 4, 6, PAIRS)[:, 0], rope3d_ref(k, 3, 4, 6, PAIRS)[:, 0])
    s1 = np.einsum("qd,kd->qk", rope3d_ref(q, 7, 4, 6, PAIRS)[:, 0], rope3d_ref(k, 10, 4, 6, PAIRS)[:, 0])
    assert np.max(np.abs(s0 - s1)) < 1e-11
    # shift in h and w: move both tokens by (+1 row, +2 columns) inside the grid
    qi, ki = 0, 9          # (h, w) = (0, 0) and (1, 3)
    qj, kj = 8, 17         # (1, 2) and (2, 5)
    yq = rope3d_ref(q, 0, 4, 6, PAIRS)[:, 0]
    yk = rope3d_ref(k, 0, 4, 6, PAIRS)[:, 0]
    yq_shift = rope3d_ref(q[[qi] * 24], 0, 4, 6, PAIRS, token_index=np.full(24, qj))[0, 0]
    yk_shift = rope3d_ref(k[[ki] * 24], 0, 4, 6, PAIRS, token_index=np.full(24, kj))[0, 0]
    assert yq[qi] @ yk[ki] == pytest.approx(yq_shift @ yk_shift, abs=1e-11)
    # the same two vectors at a different relative offset score differently
    yk_other = rope3d_ref(k[[ki]], 0, 4, 6, PAIRS, token_index=np.array([kj]))[0, 0]
    assert abs(yq[qi] @ yk[ki] - yq[qi] @ yk_other) > 1e-3


def test_rows_subset_equals_full():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((72, 2, D))
    rows = np.array([0, 17, 24, 71])
    full = rope3d_ref(x, 2, 4, 6, PAIRS)
    part = rope3d_ref(x[rows], 2, 4, 6, PAIRS, token_index=rows)
    assert np.array_equal(full[rows], part)


# ---- rotate-half layout and per-axis frequency bases -------------------------

def test_rotate_half_is_adjacent_after_interleaving():
    # moving element j to 2j and element j + D/2 to 2j + 1 turns the
    # rotate-half layout into the adjacent one, for any input and position
    rng = np.random.default_rng(11)
    x = rng.standard_normal((50, 3, D))
    perm = np.empty(D, dtype=np.int64)
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2
    half = rope3d_ref(x, 4, 5, 6, PAIRS, layout="half")
    adj = rope3d_ref(x[..., perm], 4, 5, 6, PAIRS, layout="adjacent")
    back = np.empty_like(adj)
    back[..., perm] = adj
    np.testing.assert_allclose(half, back, rtol=0, atol=1e-15)


def test_rotate_half_unit_vector_textbook_values():
    # (1, 0) in pair 30 (an h pair: local index 8 of 21), i.e. element 30 in
    # the rotate-half layout; on a 10x1 grid token 7 is row 7: the pair turns
    # by 7 * 10000^(-8/21) and lands on elements 30 and 30 + 64 only
    x = np.zeros((8, 1, D))
    x[:, 0, 30] = 1.0
    y = rope3d_ref(x, 0, 10, 1, PAIRS, layout="half")
    a = 7 * 10000.0 ** (-8 / 21)
    assert abs(y[7, 0, 30] - math.cos(a)) < 1e-15 and abs(y[7, 0, 30 + 64] - math.sin(a)) < 1e-15
    assert np.count_nonzero(np.abs(y[7, 0]) > 1e-15) == 2


def test_per_axis_theta_closed_form_and_default():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((40, 2, D))
    same = rope3d_ref(x, 2, 4, 6, PAIRS, theta=(10000.0, 10000.0, 10000.0))
    np.testing.assert_array_equal(same, rope3d_ref(x, 2, 4, 6, PAIRS, theta=10000.0))
    # h pair with local index 7 of 21 (global pair 29) under theta_h = 100:
    # frequency 100^(-1/3) = 0.2154...; token 13 on a 4x6 grid is row 2
    u = np.zeros((14, 1, D))
    u[:, 0, 2 * 29] = 1.0
    y = rope3d_ref(u, 0, 4, 6, PAIRS, theta=(10000.0, 100.0, 10000.0))
    ang = math.atan2(y[13, 0, 2 * 29 + 1], y[13, 0, 2 * 29])
    assert abs(ang - 2 * 100.0 ** (-1 / 3)) < 1e-12
    # the t and w pairs do not see theta_h
    z = rope3d_ref(x, 2, 4, 6, PAIRS, theta=(10000.0, 100.0, 10000.0))
    ref = rope3d_ref(x, 2, 4, 6, PAIRS, theta=10000.0)
    t_and_w = np.r_[0:44, 86:128]
    np.testing.assert_array_equal(z[..., t_and_w], ref[..., t_and_w])


@pytest.mark.parametrize("layout,theta", [("half", 10000.0), ("adjacent", (500.0, 2000.0, 30000.0)),
                                          ("half", (500.0, 2000.0, 30000.0))])
def test_variants_keep_norms_and_relative_positions(layout, theta):
    rng = np.random.default_rng(13)
    F = 24
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    nq = np.linalg.norm(rope3d_ref(np.repeat(q, 60, 0), 0, 4, 6, PAIRS, theta, layout=layout), axis=-1)
    np.testing.assert_allclose(nq, np.linalg.norm(q), rtol=1e-12)
    # score between token a and token b depends only on their (t, h, w) offset
    def score(ta, tb):
        xq = rope3d_ref(q, 0, 4, 6, PAIRS, theta, token_index=np.array([ta]), layout=layout)
        xk = rope3d_ref(k, 0, 4, 6, PAIRS, theta, token_index=np.array([tb]), layout=layout)
        return float(np.sum(xq * xk))
    assert abs(score(7, 7 + F + 7) - score(2 * F + 7, 3 * F + 14)) < 1e-9
