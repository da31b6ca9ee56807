"""Ring KV-cache update on the GPU vs the ring oracle: bit-exact indices,
eviction counts and slot contents; guard frames around the ring stay intact;
no bounded device-side wait of the bulk copy gives up.  Shapes cover the
ways an insert is cut into bulk-copy pieces: many rows per piece with a
short last piece, strided source rows (one load per row), and rows wider
than a piece (each row split across pieces)."""

import numpy as np
import pytest
import torch

from oracle import RingRef
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import need_gpu, to_bits, to_dev

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1  # a quiet-NaN bf16 pattern no N(0,1) draw can produce


def run_ring(slots, F, H, inserts, seed, stride_mult=1):
    """Insert frame batches; after every call compare with RingRef."""
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    D = 128
    frame_elems = F * H * D
    # ring with one guard frame before and after each tensor
    kbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    vbuf = torch.full(((slots + 2) * frame_elems,), SENTINEL, dtype=torch.int16, device="cuda")
    kview = kbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    vview = vbuf[frame_elems:(slots + 1) * frame_elems].view(torch.bfloat16).view(slots, F, H, D)
    ring = rkv.KVRing(slots, F, H, D, k=kview, v=vview)
    ref = RingRef(slots)
    frame_no = 0
    for step, n in enumerate(inserts):
        kb = bf16_normal_bits(seed + 2 * step, (n * F, H * D))
        vb = bf16_normal_bits(seed + 2 * step + 1, (n * F, H * D))
        # source rows may live inside a wider buffer (row stride = stride_mult*H*D)
        kw = np.full((n * F, stride_mult * H * D), 0x1234, dtype=np.uint16)
        vw = np.full((n * F, stride_mult * H * D), 0x4321, dtype=np.uint16)
        kw[:, :H * D] = kb
        vw[:, :H * D] = vb
        kd = to_dev(kw).view(n * F, stride_mult * H, D)[:, :H, :]
        vd = to_dev(vw).view(n * F, stride_mult * H, D)[:, :H, :]
        frames = [(kb[i * F:(i + 1) * F], vb[i * F:(i + 1) * F], frame_no + i) for i in range(n)]
        frame_no += n
        ev = rkv.kvcache_ring_update(ring, kd, vd, n)
        rkv.rkv_ring_status()   # raises if a device-side wait gave up
        ev_ref = ref.insert(frames)
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
                assert np.array_equal(kh[s], ref.slots[s][0]), (step, s)
                assert np.array_equal(vh[s], ref.slots[s][1]), (step, s)
        kg = kbuf.cpu().numpy().view(np.uint16)
        vg = vbuf.cpu().numpy().view(np.uint16)
        for g in (kg[:frame_elems], kg[(slots + 1) * frame_elems:], vg[:frame_elems], vg[(slots + 1) * frame_elems:]):
            assert np.all(g == SENTINEL)
    return ring, ref


def test_tiny_ring_5_slots_insert_3_evict_3():
    # 5 slots of 4x6-token frames, 2 heads; fill, then 3 in / 3 out
    ring, ref = run_ring(5, 24, 2, [5, 3], seed=1000)
    assert ref.count == 5 and ref.head == 3


def test_mid_ring_7_slots_insert_5_evict_5():
    run_ring(7, 390, 12, [7, 5, 5], seed=1001)


def test_sweep_ring_21_slots_from_one_frame():
    # 21 slots of 30x52-token frames, 12 heads: 1 seed frame, then 8 x 5 frames
    ring, ref = run_ring(21, 1560, 12, [1] + [5] * 8, seed=4000)
    assert ref.count == 21


def test_strided_source_rows():
    # new K/V rows taken from a fused-projection-like buffer (stride 3*H*D)
    run_ring(5, 24, 2, [2, 4, 5], seed=77, stride_mult=3)


def test_random_insert_sizes():
    rng = np.random.default_rng(5)
    sizes = [int(x) for x in rng.integers(0, 7, 12)]
    run_ring(6, 10, 3, sizes, seed=900)


def test_single_slot_ring():
    run_ring(1, 24, 2, [1, 1, 0, 1], seed=901)


def test_one_head_many_rows_per_piece():
    # 256-byte rows: 128 rows per piece, 300-row frames end in a short piece
    run_ring(4, 300, 1, [3, 2, 4], seed=902)
    run_ring(3, 300, 1, [2, 3], seed=903, stride_mult=2)


def test_rows_wider_than_a_piece():
    # 160 heads: 40 KB rows, each split into a 32 KB and an 8 KB piece
    run_ring(4, 6, 160, [3, 2, 4], seed=904)
    run_ring(3, 5, 160, [2, 3], seed=905, stride_mult=2)
