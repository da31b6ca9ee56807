"""Ring update with K rotated on the way in (kvcache_ring_update_rope) vs the
oracles: every K slot within one bf16 ulp of the correctly rounded fp64
rotation of the frame it should hold (rotated at that frame's time index);
V slots, head, count, eviction and slot map bit-exact against RingRef; guard
frames around the ring untouched.  A consistency check beside the parity
check: the K slots equal what rope3d_apply writes for the same rows.  Shapes
include a long w axis and a one-row grid of 4,000 columns, where each CTA's
cos/sin table holds only the columns its rows reach."""

import numpy as np
import pytest
import torch

from oracle import RingRef, bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, rope3d_ref
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import need_gpu, to_bits, to_dev

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1


def run_ring_rope(slots, grid_h, grid_w, H, inserts, seed, stride_mult=1, t_start=0, pairs=(22, 21, 21)):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    D = 128
    F = grid_h * grid_w
    frame_elems = F * H * D
    rope = rkv.make_rope(grid_h, grid_w, pairs)
    kbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    vbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    kview = kbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    vview = vbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    ring = rkv.KVRing(slots, F, H, D, k=kview, v=vview)
    ref = RingRef(slots)
    t = t_start
    worst = 0
    for step, n in enumerate(inserts):
        kb = bf16_normal_bits(seed + 2 * step, (n * F, H * D))
        vb = bf16_normal_bits(seed + 2 * step + 1, (n * F, H * D))
        kw = np.full((n * F, stride_mult * H * D), 0x1234, dtype=np.uint16)
        vw = np.full((n * F, stride_mult * H * D), 0x4321, dtype=np.uint16)
        kw[:, :H * D] = kb
        vw[:, :H * D] = vb
        kd = to_dev(kw).view(n * F, stride_mult * H, D)[:, :H, :]
        vd = to_dev(vw).view(n * F, stride_mult * H, D)[:, :H, :]
        kr = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(kb.reshape(n * F, H, D)), t, grid_h, grid_w, pairs))
        kr = kr.reshape(n * F, H * D)
        frames = [(kr[i * F:(i + 1) * F], vb[i * F:(i + 1) * F], t + i) for i in range(n)]
        ev = rkv.kvcache_ring_update_rope(ring, kd, vd, t, rope, n)
        rkv.rkv_ring_status()   # raises if a device-side wait gave up
        ev_ref = ref.insert(frames)
        # consistency: the standalone call on the same rows
        ky = torch.empty((n * F, H, D), dtype=torch.bfloat16, device="cuda")
        rkv.rope3d_apply(kd, ky, t0=t, rope=rope)
        t += n
        assert ev == ev_ref
        assert (ring.head, ring.count) == (ref.head, ref.count)
        assert [ring.slot(j) for j in range(slots + 1)] == [ref.slot_of(j) for j in range(slots + 1)]
        torch.cuda.synchronize()
        kh = to_bits(kview).reshape(slots, F, H * D)
        vh = to_bits(vview).reshape(slots, F, H * D)
        for s in range(slots):
            if ref.slots[s] is None:
                assert np.all(kh[s] == SENTINEL) and np.all(vh[s] == SENTINEL)
            else:
                ulp = bf16_ulp_distance(kh[s], ref.slots[s][0])
                worst = max(worst, int(ulp.max()))
                assert int(ulp.max()) <= 1, (step, s, int(ulp.max()))
                assert np.array_equal(vh[s], ref.slots[s][1]), (step, s)
        ky_bits = to_bits(ky).reshape(n, F, H * D)
        for i in range(n):
            assert np.array_equal(kh[ring.slot(ring.count - n + i)], ky_bits[i]), (step, i)
        kg = kbuf.cpu().numpy().view(np.uint16)
        vg = vbuf.cpu().numpy().view(np.uint16)
        for g in (kg[:frame_elems], kg[(slots + 1) * frame_elems:], vg[:frame_elems], vg[(slots + 1) * frame_elems:]):
            assert np.all(g == SENTINEL)
    return ring, ref, worst


def test_tiny_ring_rope_5_slots():
    ring, ref, worst = run_ring_rope(5, 4, 6, 2, [5, 3, 2], seed=1000)
    assert ref.count == 5 and worst <= 1


def test_mid_ring_rope_7_slots():
    run_ring_rope(7, 15, 26, 12, [7, 5, 5], seed=1001)


def test_sweep_ring_rope_21_slots_full_schedule():
    # 21 slots of 30x52-token frames, 12 heads: 1 seed frame, then 8 x 5
    # frames (the 5th insert wraps around the ring)
    ring, ref, _ = run_ring_rope(21, 30, 52, 12, [1] + [5] * 8, seed=4000)
    assert ref.count == 21


def test_ring_rope_strided_source_and_late_time():
    run_ring_rope(6, 5, 7, 3, [4, 4, 4], seed=77, stride_mult=3, t_start=1000)


def test_ring_rope_wide_grid():
    # a 4x100 grid: 100 w positions against 4 h positions
    run_ring_rope(4, 4, 100, 2, [3, 2, 3], seed=78)


def test_ring_rope_one_row_grid():
    # a 1x4000 grid: a table of every position would need 84,000 entries
    run_ring_rope(3, 1, 4000, 1, [2, 2], seed=79)


def test_ring_rope_chunk_on_three_axes():
    # pairs 21/2/41: rotary pairs 20-23 (one 16-byte chunk) lie on t, h, h, w
    run_ring_rope(5, 3, 4, 2, [2, 3, 1, 2], seed=80, pairs=(21, 2, 41))


def test_ring_rope_rejects_grid_mismatch():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    ring = rkv.KVRing(3, 24, 2, 128)
    k = torch.zeros((24, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rkv.RkvError) as e:
        rkv.kvcache_ring_update_rope(ring, k, k.clone(), 0, rkv.make_rope(5, 5), 1)
    assert e.value.status == 1 and (ring.head, ring.count) == (0, 0)


def test_ring_rope_rows_wider_than_a_piece():
    # 160 heads: 40 KB rows; V moves in 32 KB + 8 KB pieces, K rows are
    # rotated 1,024 chunks at a time by each CTA's threads
    run_ring_rope(4, 2, 3, 160, [3, 2, 4], seed=81)
