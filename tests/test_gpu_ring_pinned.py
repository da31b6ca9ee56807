"""Rings with a pinned prefix: the first P slots keep the first P frames ever
inserted, later frames roll through slots P..W-1.  Both insert calls (plain
copy, and K rotated on the way in) against RingRef(W, P): head, count,
eviction and slot map exact; V slots (and K for the plain copy) bit-exact; K
of the rotating insert within one bf16 ulp of the correctly rounded fp64
rotation at the frame's own time index; slots not yet filled and guard frames
around the ring untouched.  Then attention from a query window over such a
ring (keys already rotated, physical slot order) against fp64 attention over
the oracle ring's contents."""

import math

import numpy as np
import pytest
import torch

from oracle import RingRef, bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, fused_attention_ref, rope3d_ref
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1
D = 128


def run_pinned(slots, pinned, grid_h, grid_w, H, inserts, seed, rotate):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    F = grid_h * grid_w
    frame_elems = F * H * D
    rope = rkv.make_rope(grid_h, grid_w)
    kbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    vbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    kview = kbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    vview = vbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    ring = rkv.KVRing(slots, F, H, D, k=kview, v=vview, pinned=pinned)
    assert (ring.head, ring.count, ring.pinned) == (pinned, 0, pinned)
    ref = RingRef(slots, pinned)
    t = 0
    for step, n in enumerate(inserts):
        assert n <= ref.capacity_for_insert()
        kb = bf16_normal_bits(seed + 2 * step, (n * F, H * D))
        vb = bf16_normal_bits(seed + 2 * step + 1, (n * F, H * D))
        if rotate:
            kr = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(kb.reshape(n * F, H, D)), t, grid_h, grid_w))
            kr = kr.reshape(n * F, H * D)
        else:
            kr = kb
        frames = [(kr[i * F:(i + 1) * F], vb[i * F:(i + 1) * F], t + i) for i in range(n)]
        kd = to_dev(kb).view(n * F, H, D)
        vd = to_dev(vb).view(n * F, H, D)
        if rotate:
            ev = rkv.kvcache_ring_update_rope(ring, kd, vd, t, rope, n)
        else:
            ev = rkv.kvcache_ring_update(ring, kd, vd, n)
        rkv.rkv_ring_status()
        t += n
        assert ev == ref.insert(frames), step
        assert (ring.head, ring.count) == (ref.head, ref.count), step
        assert [ring.slot(j) for j in range(-1, slots + 1)] == [ref.slot_of(j) for j in range(-1, slots + 1)]
        torch.cuda.synchronize()
        kh = to_bits(kview).reshape(slots, F, H * D)
        vh = to_bits(vview).reshape(slots, F, H * D)
        for s in range(slots):
            if ref.slots[s] is None:
                assert np.all(kh[s] == SENTINEL) and np.all(vh[s] == SENTINEL), (step, s)
                continue
            if rotate:
                assert int(bf16_ulp_distance(kh[s], ref.slots[s][0]).max()) <= 1, (step, s)
            else:
                assert np.array_equal(kh[s], ref.slots[s][0]), (step, s)
            assert np.array_equal(vh[s], ref.slots[s][1]), (step, s)
        # the pinned slots still hold the first frames ever inserted
        for s in range(min(pinned, ref.count)):
            assert ref.slots[s][2] == s
        kg = kbuf.cpu().numpy().view(np.uint16)
        vg = vbuf.cpu().numpy().view(np.uint16)
        for g in (kg[:frame_elems], kg[(slots + 1) * frame_elems:], vg[:frame_elems], vg[(slots + 1) * frame_elems:]):
            assert np.all(g == SENTINEL)
    return ring, ref


@pytest.mark.parametrize("rotate", [False, True])
def test_pinned_fill_cross_and_roll(rotate):
    # 6 slots, 2 pinned: a partial pinned fill, an insert that finishes the
    # prefix and starts rolling, then inserts that wrap the rolling region
    _, ref = run_pinned(6, 2, 4, 6, 2, [1, 3, 4, 2, 3, 4], seed=1200, rotate=rotate)
    assert ref.count == 6


@pytest.mark.parametrize("rotate", [False, True])
def test_pinned_one_insert_fills_everything(rotate):
    # an empty ring takes its whole capacity in one call: 3 pinned + 4 rolling
    _, ref = run_pinned(7, 3, 5, 7, 3, [7, 4, 1, 4], seed=1210, rotate=rotate)
    assert ref.count == 7


@pytest.mark.parametrize("rotate", [False, True])
def test_pinned_single_rolling_slot(rotate):
    # the largest prefix a ring may have: every later frame lands in the last slot
    run_pinned(4, 3, 4, 6, 2, [2, 2, 1, 1], seed=1220, rotate=rotate)


def test_pinned_ring_full_size_schedule():
    # 21 slots of 30x52-token frames, 12 heads, the first frame pinned: one
    # seed frame, then 8 inserts of 5 frames with K rotated on the way in
    _, ref = run_pinned(21, 1, 30, 52, 12, [1] + [5] * 8, seed=1230, rotate=True)
    assert ref.count == 21 and ref.slots[0][2] == 0


def test_pinned_ring_rejects_over_capacity():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    ring = rkv.KVRing(5, 24, 2, D, pinned=2)
    k = torch.zeros((5 * 24, 2, D), dtype=torch.bfloat16, device="cuda")
    assert rkv.kvcache_ring_update(ring, k, k.clone(), 5) == 0      # 2 pinned + 3 rolling
    with pytest.raises(RuntimeError, match="n_frames"):
        rkv.kvcache_ring_update(ring, k, k.clone(), 4)                # only 3 rolling slots now
    assert (ring.head, ring.count) == (2, 5)


def test_attention_over_pinned_ring():
    # queries of the newest frames attend over every valid frame of a full
    # pinned ring: pinned sink frames first in memory, then the rolling slots
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    W, P, grid_h, grid_w, H = 8, 2, 8, 16, 2
    F = grid_h * grid_w
    ring, ref = run_pinned(W, P, grid_h, grid_w, H, [3, 4, 4, 3], seed=1240, rotate=True)
    assert ring.count == W
    t_new = 14 - 3           # the last insert held frames 11..13
    Lq = 3 * F
    qb = bf16_normal_bits(1250, (Lq, H, D))
    Lk = W * F
    kview = ring.k.view(W * F, H, D)
    vview = ring.v.view(W * F, H, D)
    o = torch.full((Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    seq = rkv.AttnSeq(to_dev(qb), kview, vview, o, q_t0=t_new, rope_q=True, rope_k=False)
    ws = rkv.attn_fwd_varlen([seq], rkv.make_rope(grid_h, grid_w))
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    valid = ref.valid_slots()
    assert valid == list(range(W))
    k_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][0]) for s in valid]).reshape(Lk, H, D)
    v_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][1]) for s in valid]).reshape(Lk, H, D)
    want = fused_attention_ref(bf16_bits_to_f64(qb), k_ref, v_ref, scale=1.0 / math.sqrt(D), grid_h=grid_h,
                               grid_w=grid_w, rope_q=True, rope_k=False, q_t0=t_new, k_t0=0)
    assert_attn_close(to_f64(o), want, "pinned ring")
