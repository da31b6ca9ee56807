"""The rotate-half pair layout and per-axis frequency bases (the two RoPE
choices the pages leave open) on every GPU path that rotates: standalone
rope3d_apply (within one bf16 ulp of the oracle's correctly rounded value),
the rotated ring insert (K slots within one ulp, V bit-exact) and the fused
attention (oracle tolerances)."""

import math

import numpy as np
import pytest
import torch

from oracle import RingRef, bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, fused_attention_ref, rope3d_ref
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu
D = 128
VARIANTS = [("half", 10000.0), ("adjacent", (10000.0, 500.0, 64.0)), ("half", (2000.0, 10000.0, 300.0))]


@pytest.mark.parametrize("layout,theta", VARIANTS)
def test_rope3d_apply_variants(layout, theta):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    for L, H, gh, gw, t0, seed in [(72, 2, 4, 6, 2, 1), (1950, 12, 15, 26, 2, 2), (777, 3, 5, 7, 40, 3)]:
        xb = bf16_normal_bits(seed, (L, H, D))
        ref = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(xb), t0, gh, gw, theta=theta, layout=layout))
        y = torch.empty((L, H, D), dtype=torch.bfloat16, device="cuda")
        rkv.rope3d_apply(to_dev(xb), y, t0=t0, rope=rkv.make_rope(gh, gw, theta=theta, layout=layout))
        torch.cuda.synchronize()
        ulp = bf16_ulp_distance(to_bits(y), ref)
        assert int(ulp.max()) <= 1, (L, int(ulp.max()))
        assert float((ulp == 0).mean()) > 0.999


@pytest.mark.parametrize("layout,theta", VARIANTS)
def test_ring_insert_variants(layout, theta):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    slots, gh, gw, H = 5, 4, 6, 2
    F = gh * gw
    rope = rkv.make_rope(gh, gw, theta=theta, layout=layout)
    ring = rkv.KVRing(slots, F, H, D)
    ref = RingRef(slots)
    t = 3
    for step, n in enumerate([5, 3, 2]):
        kb = bf16_normal_bits(60 + 2 * step, (n * F, H, D))
        vb = bf16_normal_bits(61 + 2 * step, (n * F, H, D))
        kr = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(kb), t, gh, gw, theta=theta, layout=layout))
        ev = rkv.kvcache_ring_update_rope(ring, to_dev(kb), to_dev(vb), t, rope, n)
        assert ev == ref.insert([(kr[i * F:(i + 1) * F], vb[i * F:(i + 1) * F]) for i in range(n)])
        t += n
        torch.cuda.synchronize()
        kh, vh = to_bits(ring.k), to_bits(ring.v)
        for s in ref.valid_slots():
            assert int(bf16_ulp_distance(kh[s], ref.slots[s][0]).max()) <= 1, (step, s)
            assert np.array_equal(vh[s], ref.slots[s][1]), (step, s)


@pytest.mark.parametrize("layout,theta", VARIANTS)
def test_fused_attention_variants(layout, theta):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    H, gh, gw = 3, 4, 6
    F = gh * gw
    for Lq, Lk, block, seed in [(72, 120, 0, 70), (300, 336, 3, 71)]:
        qb, kb, vb = (bf16_normal_bits(seed + 10 * i, (L, H, D)) for i, L in enumerate((Lq, Lk, Lk)))
        off = Lk // F - Lq // F
        o = torch.full((Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        seq = rkv.AttnSeq(to_dev(qb), to_dev(kb), to_dev(vb), o, q_t0=off, k_t0=0, block_frames=block,
                          q_frame_offset=off)
        ws = rkv.attn_fwd_varlen([seq], rkv.make_rope(gh, gw, theta=theta, layout=layout))
        rkv.rkv_attn_status(ws)
        torch.cuda.synchronize()
        want = fused_attention_ref(bf16_bits_to_f64(qb), bf16_bits_to_f64(kb), bf16_bits_to_f64(vb),
                                   scale=1.0 / math.sqrt(D), grid_h=gh, grid_w=gw, rope_q=True, rope_k=True,
                                   q_t0=off, k_t0=0, theta=theta, layout=layout, block_frames=block,
                                   q_frame_offset=off)
        assert_attn_close(to_f64(o), want, f"{layout} {theta} Lq={Lq}")
