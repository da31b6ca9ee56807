"""Attention split over ranks by (head, query frame) units, on the CPU.

The planner is checked for what the split promises (every unit exactly once,
runs balanced to one unit, whole heads when the ranks divide them, no cut
inside a frame), and world_size 2 and 3 gloo process groups check the
exchange: each rank computes only its own units with the oracle, on views
that start at the run's first frame (time index q_t0 + f0, mask offset
q_frame_offset + f0), and all_gather_units reassembles them.  The result must
match the oracle on the whole sequence, which pins those two offsets; a
second exchange moves the bf16 outputs, written through shard_seqs' views,
and every rank must end with the same bits."""

import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from rolling_kv_cache_rope_b200.shard import unit_runs  # noqa: E402


@pytest.mark.parametrize("H,q_frames,world", [(12, 15, 8), (12, 15, 2), (12, 15, 3), (12, 5, 8), (3, 4, 5),
                                              (1, 1, 1), (2, 7, 14)])
def test_runs_partition_the_units(H, q_frames, world):
    runs = unit_runs(H, q_frames, world)
    assert [r.rank for r in runs] == list(range(world))
    seen = []
    for r in runs:
        for h, f0, f1 in r.segments():
            assert 0 <= h < H and 0 <= f0 < f1 <= q_frames
            seen.extend((h, f) for f in range(f0, f1))
        h0, h1 = r.heads()
        assert all(h0 <= h < h1 for h, _, _ in r.segments())
    assert seen == [(h, f) for h in range(H) for f in range(q_frames)]
    sizes = [r.units for r in runs]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == H * q_frames


def test_runs_partition_random_shapes():
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=300, deadline=None)
    @given(st.integers(1, 40), st.integers(1, 30), st.data())
    def check(H, q_frames, data):
        world = data.draw(st.integers(1, min(64, H * q_frames)))
        test_runs_partition_the_units(H, q_frames, world)
        # a rank touches at most ceil(units / q_frames) + 1 heads
        for r in unit_runs(H, q_frames, world):
            h0, h1 = r.heads()
            assert h1 - h0 <= -(-r.units // q_frames) + 1

    check()


def test_whole_heads_when_world_divides_heads():
    for world in (1, 2, 3, 4, 6, 12):
        for r in unit_runs(12, 15, world):
            assert all((f0, f1) == (0, 15) for _, f0, f1 in r.segments())
            assert r.heads()[1] - r.heads()[0] == 12 // world


def test_twelve_heads_on_eight_ranks_needs_no_padding():
    # the split the pages could not do with heads alone: 180 units -> 22 or 23
    # per rank (a head-only split would give 2 or 1 heads, half the ranks idle
    # half the time); each rank touches at most 3 heads
    runs = unit_runs(12, 15, 8)
    assert sorted({r.units for r in runs}) == [22, 23]
    assert all(r.heads()[1] - r.heads()[0] <= 3 for r in runs)


def test_more_ranks_than_units_is_an_error():
    with pytest.raises(ValueError):
        unit_runs(2, 3, 7)
    with pytest.raises(ValueError):
        unit_runs(0, 3, 1)


def test_whole_head_runs_become_one_view_per_sequence():
    import torch
    from rolling_kv_cache_rope_b200.rkv import AttnSeq
    from rolling_kv_cache_rope_b200.shard import shard_seqs
    q = torch.zeros((3 * 6, 4, 128), dtype=torch.bfloat16)
    k = torch.zeros((5 * 6, 4, 128), dtype=torch.bfloat16)
    o = torch.zeros_like(q)
    seq = AttnSeq(q, k, k, o, q_t0=2, k_t0=0, block_frames=1, q_frame_offset=2)
    for rank in range(2):
        (s,) = shard_seqs([seq], 6, rank, 2)
        assert s.q.shape == (18, 2, 128) and s.k.shape == (30, 2, 128)
        assert s.q.data_ptr() == q.data_ptr() + rank * 2 * 128 * 2
        assert s.o.data_ptr() == o.data_ptr() + rank * 2 * 128 * 2
        assert (s.q_t0, s.q_frame_offset, s.block_frames, s.flags) == (2, 2, 1, seq.flags)
    # K/V holding only rank 1's heads
    (s,) = shard_seqs([AttnSeq(q, k[:, 2:], k[:, 2:], o)], 6, 1, 2, kv_head0=2)
    assert s.k.data_ptr() == k.data_ptr() + 2 * 128 * 2
    with pytest.raises(ValueError):
        shard_seqs([AttnSeq(q, k[:, 2:], k[:, 2:], o)], 6, 0, 2, kv_head0=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# a small masked problem: 3 heads, 2x3-token frames, 4 query frames that are
# the last 4 of a 6-frame context, blocks of 2 frames
H, GH, GW, D = 3, 2, 3, 128
F = GH * GW
QF, KF = 4, 6
Q_T0 = KF - QF
BLOCK = 2


def _rank_main(rank, world, port, results):
    import torch
    import torch.distributed as dist
    from oracle import bf16_bits_to_f64, f64_to_bf16_bits, fused_attention_ref
    from rolling_kv_cache_rope_b200.rkv import RKV_ROPE_K, RKV_ROPE_Q, AttnSeq
    from rolling_kv_cache_rope_b200.shard import all_gather_units, shard_seqs
    from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)  # noqa: E731
        to_f64 = lambda t: bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))  # noqa: E731
        q = as_bf16(bf16_normal_bits(3100, (QF * F, H, D)))
        k = as_bf16(bf16_normal_bits(3101, (KF * F, H, D)))
        v = as_bf16(bf16_normal_bits(3102, (KF * F, H, D)))
        o = torch.zeros((QF * F, H, D), dtype=torch.bfloat16)
        o64 = np.full((QF * F, H, D), np.nan)
        whole = AttnSeq(q, k, v, o, q_t0=Q_T0, k_t0=0, block_frames=BLOCK, q_frame_offset=Q_T0)
        pieces = shard_seqs([whole], F, rank, world)
        segs = unit_runs(H, QF, world)[rank].segments()
        if world == H:   # whole heads: one view of the rank's head
            assert len(pieces) == 1 and pieces[0].q.shape == (QF * F, 1, D)
        assert len(pieces) == len(segs)
        for s, (h, f0, f1) in zip(pieces, segs):
            assert s.q.shape == (s.o.shape[0], 1, D) and s.k.shape == (KF * F, 1, D)
            val = fused_attention_ref(
                to_f64(s.q), to_f64(s.k), to_f64(s.v), scale=1.0 / math.sqrt(D), grid_h=GH, grid_w=GW,
                rope_q=bool(s.flags & RKV_ROPE_Q), rope_k=bool(s.flags & RKV_ROPE_K), q_t0=s.q_t0, k_t0=s.k_t0,
                block_frames=s.block_frames, q_frame_offset=s.q_frame_offset)
            o64[f0 * F:f1 * F, h:h + 1] = val
            s.o.copy_(as_bf16(f64_to_bf16_bits(val)))      # writes through the view into o
        got64 = all_gather_units(torch.from_numpy(o64), F, rank, world).numpy()
        got16 = all_gather_units(o, F, rank, world).view(torch.int16).numpy().view(np.uint16).copy()
        results[rank] = (got64, got16)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_sharded_units_reassemble_to_the_whole_sequence(world):
    from oracle import bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, fused_attention_ref
    from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        out = dict(results)
    q = bf16_bits_to_f64(bf16_normal_bits(3100, (QF * F, H, D)))
    k = bf16_bits_to_f64(bf16_normal_bits(3101, (KF * F, H, D)))
    v = bf16_bits_to_f64(bf16_normal_bits(3102, (KF * F, H, D)))
    want = fused_attention_ref(q, k, v, scale=1.0 / math.sqrt(D), grid_h=GH, grid_w=GW, rope_q=True, rope_k=True,
                               q_t0=Q_T0, k_t0=0, block_frames=BLOCK, q_frame_offset=Q_T0)
    for rank in range(world):
        got64, got16 = out[rank]
        assert np.all(np.isfinite(got64)), rank
        assert float(np.abs(got64 - want).max()) <= 1e-12, rank
        assert int(bf16_ulp_distance(got16, f64_to_bf16_bits(want)).max()) <= 1, rank
    # every rank ends with the same bf16 bits
    assert all(np.array_equal(out[0][1], out[r][1]) for r in range(world))
