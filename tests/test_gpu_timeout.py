"""Bounded device-side waits run out, report RKV_ERR_TIMEOUT, and leave the
GPU usable: tested by making a handoff never happen, nothing faults or traps.

Attention: attn_fwd_varlen_debug makes the second CTA of the first CTA pair
withhold one handoff to the pair's MMA issuer ("V tile landed", "K tile
rotated" or "P ready"); every wait of that launch is limited to 50 ms.  The
issuer's wait runs out, the pair stops (its other roles leave through the
same bounded waits), rkv_attn_status reports RKV_ERR_TIMEOUT, and the next
normal launch in the same process matches the oracle.

Ring insert: kvcache_ring_update_debug makes the first CTA declare 16 bytes
more for its first piece than it loads, so that piece's wait runs out;
rkv_ring_status reports RKV_ERR_TIMEOUT, and later inserts match the ring
oracle bit for bit."""

import math

import numpy as np
import pytest
import torch

from oracle import RingRef, bf16_bits_to_f64, fused_attention_ref
from rolling_kv_cache_rope_b200.synth import MID, TINY, bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu
D = 128
LIMIT_US = 50_000


def layer_inputs(layer):
    q = bf16_normal_bits(layer.seed, (layer.Lq, layer.heads, D))
    k = bf16_normal_bits(layer.seed + 100, (layer.Lk, layer.heads, D))
    v = bf16_normal_bits(layer.seed + 200, (layer.Lk, layer.heads, D))
    return q, k, v


def attn_seq(rkv, layer, bits):
    q, k, v = (to_dev(b) for b in bits)
    o = torch.full((layer.Lq, layer.heads, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    return rkv.AttnSeq(q, k, v, o, q_t0=layer.q_t0, k_t0=layer.k_t0)


@pytest.mark.parametrize("stall", ["V_READY", "K_READY", "P_FULL"])
@pytest.mark.parametrize("layer", [TINY, MID], ids=["tiny", "mid"])
def test_attention_wait_runs_out_and_gpu_stays_usable(stall, layer):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    bits = layer_inputs(layer)
    rope = rkv.make_rope(layer.grid_h, layer.grid_w)
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(1, layer.heads, D), dtype=torch.uint8, device="cuda")
    rkv.attn_fwd_varlen_debug([attn_seq(rkv, layer, bits)], rope, stall=getattr(rkv, "RKV_DEBUG_STALL_" + stall),
                              timeout_us=LIMIT_US, workspace=ws)
    with pytest.raises(rkv.RkvError) as e:
        rkv.rkv_attn_status(ws)
    assert e.value.status == rkv.RKV_ERR_TIMEOUT
    rkv.rkv_attn_status(ws)          # read once, then cleared

    # the same process, a normal launch: correct results
    seq = attn_seq(rkv, layer, bits)
    rkv.attn_fwd_varlen([seq], rope, workspace=ws)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    want = fused_attention_ref(*(bf16_bits_to_f64(b) for b in bits), scale=1.0 / math.sqrt(D),
                               grid_h=layer.grid_h, grid_w=layer.grid_w, rope_q=True, rope_k=True,
                               q_t0=layer.q_t0, k_t0=layer.k_t0)
    assert_attn_close(to_f64(seq.o), want, f"after a {stall} timeout")


def test_attention_debug_launch_without_stall_reports_ok():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    bits = layer_inputs(TINY)
    rope = rkv.make_rope(TINY.grid_h, TINY.grid_w)
    seq = attn_seq(rkv, TINY, bits)
    ws = rkv.attn_fwd_varlen_debug([seq], rope, timeout_us=LIMIT_US)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    want = fused_attention_ref(*(bf16_bits_to_f64(b) for b in bits), scale=1.0 / math.sqrt(D),
                               grid_h=TINY.grid_h, grid_w=TINY.grid_w, rope_q=True, rope_k=True,
                               q_t0=TINY.q_t0, k_t0=TINY.k_t0)
    assert_attn_close(to_f64(seq.o), want, "debug launch, no stall")


def test_ring_insert_wait_runs_out_and_gpu_stays_usable():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    slots, F, H = 5, 390, 12
    ring = rkv.KVRing(slots, F, H, D)
    kb = bf16_normal_bits(90, (3 * F, H, D))
    vb = bf16_normal_bits(91, (3 * F, H, D))
    rkv.rkv_ring_status()
    rkv.kvcache_ring_update_debug(ring, to_dev(kb), to_dev(vb), 3, stall=rkv.RKV_DEBUG_STALL_BULK_LOAD,
                                  timeout_us=LIMIT_US)
    with pytest.raises(rkv.RkvError) as e:
        rkv.rkv_ring_status()
    assert e.value.status == rkv.RKV_ERR_TIMEOUT
    rkv.rkv_ring_status()            # read once, then cleared

    # a fresh ring in the same process: every insert bit-exact again
    ring = rkv.KVRing(slots, F, H, D)
    ref = RingRef(slots)
    frame_no = 0
    for step, n in enumerate((3, 4, 5)):
        kb = bf16_normal_bits(100 + step, (n * F, H, D))
        vb = bf16_normal_bits(200 + step, (n * F, H, D))
        frames = [(kb[i * F:(i + 1) * F], vb[i * F:(i + 1) * F], frame_no + i) for i in range(n)]
        frame_no += n
        assert rkv.kvcache_ring_update(ring, to_dev(kb), to_dev(vb), n) == ref.insert(frames)
        rkv.rkv_ring_status()
        torch.cuda.synchronize()
        kh, vh = to_bits(ring.k), to_bits(ring.v)
        for s in ref.valid_slots():
            assert np.array_equal(kh[s], ref.slots[s][0]) and np.array_equal(vh[s], ref.slots[s][1]), (step, s)
