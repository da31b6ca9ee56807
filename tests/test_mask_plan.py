"""The attention kernel's mask, bit-exact against the integer oracle, on the CPU.

rkv_attn_mask_rows evaluates, on the host, the very functions the kernel
compiles for its mask (each query row's key limit) and for its work units
(the key tiles a unit processes).  For every row the oracle's visible keys
must be exactly the prefix [0, limit); every unit must process the tiles that
hold its rows' visible keys and no tile past them; every (sequence, head,
query block) must be one unit.  Cases: the small and mid workloads, masked at
several offsets, ragged query and key tails, and the full-size two-pass
launch (denoise 23,400 + cache-update 7,800 queries over 32,760 keys, blocks
of 3 frames), checked frame pair by frame pair."""

import numpy as np
import pytest

from oracle import frame_block_visible, frame_pair_visible
from rolling_kv_cache_rope_b200.synth import MID, TINY, TWO_PASS_CACHE, TWO_PASS_DENOISE


@pytest.fixture(scope="module")
def rkv():
    from rolling_kv_cache_rope_b200 import rkv as m
    return m


def check_units(specs, limits, units, H):
    seen = set()
    for si, head, qb, nkt in units.tolist():
        Lq = specs[si]["Lq"]
        rows = limits[si][qb * 512:min(Lq, (qb + 1) * 512)]
        assert len(rows) > 0 and 0 <= head < H
        top = int(rows.max())
        assert nkt == (top + 127) // 128, (si, head, qb, nkt, top)
        seen.add((si, head, qb))
    want = {(si, h, qb) for si, s in enumerate(specs) for h in range(H) for qb in range((s["Lq"] + 511) // 512)}
    assert seen == want and len(units) == len(want)


def check_dense(rkv, specs, H, grid_h, grid_w):
    F = grid_h * grid_w
    limits, units = rkv.attn_mask_rows(specs, H, rkv.make_rope(grid_h, grid_w))
    for s, lim in zip(specs, limits):
        Lq, Lk = s["Lq"], s["Lk"]
        if s.get("block_frames", 0) > 0:
            vis = frame_block_visible(Lq, Lk, F, s["q_frame_offset"], s["block_frames"])
        else:
            vis = np.ones((Lq, Lk), dtype=bool)
        got = np.arange(Lk)[None, :] < lim[:, None]
        assert np.array_equal(got, vis), s
    check_units(specs, limits, units, H)


@pytest.mark.parametrize("block,offset", [(0, 0), (1, 2), (2, 2), (3, 2), (3, 0), (5, 1)])
def test_tiny_layer(rkv, block, offset):
    specs = [dict(Lq=TINY.Lq, Lk=TINY.Lk, q_frame_offset=offset, block_frames=block)]
    check_dense(rkv, specs, TINY.heads, TINY.grid_h, TINY.grid_w)


@pytest.mark.parametrize("block", [0, 3])
def test_mid_layer(rkv, block):
    off = MID.k_frames - MID.q_frames
    specs = [dict(Lq=MID.Lq, Lk=MID.Lk, q_frame_offset=off, block_frames=block)]
    check_dense(rkv, specs, MID.heads, MID.grid_h, MID.grid_w)


def test_ragged_tails_and_several_sequences(rkv):
    # frame-aligned queries of 7 and 13 frames, key lengths that end inside a
    # 128-key tile and inside a frame, one unmasked sequence in between
    specs = [dict(Lq=7 * 24, Lk=9 * 24 + 5, q_frame_offset=2, block_frames=2),
             dict(Lq=100, Lk=333),
             dict(Lq=13 * 24, Lk=20 * 24, q_frame_offset=7, block_frames=3)]
    check_dense(rkv, specs, 3, 4, 6)


def test_random_shapes(rkv):
    # random grids, lengths (ragged tails included), mask blocks and query
    # offsets, several sequences per launch
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=120, deadline=None)
    @given(st.integers(1, 4), st.integers(1, 5), st.integers(1, 3), st.data())
    def check(gh, gw, H, data):
        F = gh * gw
        specs = []
        for _ in range(data.draw(st.integers(1, 4))):
            kf = data.draw(st.integers(1, 40))
            Lk = kf * F - data.draw(st.integers(0, F - 1))
            block = data.draw(st.sampled_from([0, 1, 2, 3, 5]))
            if block:
                qf = data.draw(st.integers(1, kf))
                specs.append(dict(Lq=qf * F, Lk=Lk, q_frame_offset=data.draw(st.integers(0, kf - qf)),
                                  block_frames=block))
            else:
                specs.append(dict(Lq=data.draw(st.integers(1, 700)), Lk=Lk))
        check_dense(rkv, specs, H, gh, gw)

    check()


def test_full_size_two_pass_launch(rkv):
    F = TWO_PASS_DENOISE.frame_tokens
    specs = []
    for layer in (TWO_PASS_DENOISE, TWO_PASS_CACHE):
        specs.append(dict(Lq=layer.Lq, Lk=layer.Lk, q_frame_offset=layer.k_frames - layer.q_frames,
                          block_frames=layer.block_frames))
    limits, units = rkv.attn_mask_rows(specs, 12, rkv.make_rope(TWO_PASS_DENOISE.grid_h, TWO_PASS_DENOISE.grid_w))
    visible_pairs = 0
    for s, lim in zip(specs, limits):
        nq, nk = s["Lq"] // F, s["Lk"] // F
        pairs = frame_pair_visible(nq, nk, s["q_frame_offset"], s["block_frames"])
        visible_pairs += int(pairs.sum())
        for a in range(nq):
            kf = np.flatnonzero(pairs[a])
            # visible key frames form a prefix, so the row's keys do too
            assert np.array_equal(kf, np.arange(len(kf)))
            assert np.all(lim[a * F:(a + 1) * F] == len(kf) * F), a
    assert visible_pairs == 225 + 99
    check_units(specs, limits, units, 12)


def test_mask_rows_rejects(rkv):
    import ctypes
    lib = rkv.lib()
    r = rkv.make_rope(4, 6)
    out = (ctypes.c_int64 * 100)()
    bad = (rkv.rkv_attn_seq * 1)(rkv.rkv_attn_seq(Lq=72, Lk=120, q_frame_offset=-1, block_frames=3))
    assert lib.rkv_attn_mask_rows(bad, 1, 2, ctypes.byref(r), out, None, None) == rkv.RKV_ERR_INVALID_ARG
    ok = (rkv.rkv_attn_seq * 1)(rkv.rkv_attn_seq(Lq=72, Lk=120))
    assert lib.rkv_attn_mask_rows(ok, 1, 0, ctypes.byref(r), out, None, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.rkv_attn_mask_rows(ok, 1, 2, ctypes.byref(r), None, None, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.rkv_attn_mask_rows(ok, 1, 2, ctypes.byref(r), out, None, None) == rkv.RKV_OK
